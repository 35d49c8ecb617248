"""The C ABI: every function include/sf.h declares is exported by libsf.so (no GPU needed),
the binding mirrors the header's structs, and the oracle and the CUDA path share no code."""
import ctypes
import os
import re

import pytest

from masked_optimizer_step_b200 import binding
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "sf.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sf_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from masked_optimizer_step_b200 import build
    build.build()
    return ctypes.CDLL(binding.LIB_PATH)


def test_header_declares_the_four_hot_path_calls():
    names = _declared()
    for n in ("sf_mask_update", "sf_masked_dw", "sf_embed_grad", "sf_sparse_update"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_only_entry_points_work_without_a_gpu(lib):
    lib.sf_version.restype = ctypes.c_int
    assert lib.sf_version() >= 10000
    lib.sf_status_string.restype = ctypes.c_char_p
    assert b"argument" in lib.sf_status_string(-1)
    lib.sf_embed_grad_ws_bytes.restype = ctypes.c_size_t
    assert lib.sf_embed_grad_ws_bytes(4096, 1000) >= (4096 + 4 * 1000 + 4) * 4


def test_argument_errors_are_reported_before_any_work(lib):
    # a mask with R not a multiple of 32 must be refused synchronously, no device touched
    m = binding.sf_mask(R=33, slot_cap=0)
    lib.sf_mask_init.restype = ctypes.c_int
    assert lib.sf_mask_init(ctypes.byref(m), None) == -1
    assert lib.sf_mask_update(None, None, -1, ctypes.c_float(0.01), None, None) == -1


def _c_struct_fields(name):
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct %s \{(.*?)\} %s;" % (name, name), src, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        names = decl.split(None, 1)[1] if not decl.startswith("const ") else decl.split(None, 2)[2]
        for part in names.split(","):
            fields.append(part.strip().lstrip("*").strip())
    return fields


@pytest.mark.parametrize("name", ["sf_mask", "sf_mask_src", "sf_dw_problem", "sf_matrix", "sf_adam",
                                  "sf_checkpoint", "sf_fwd_problem"])
def test_binding_structs_follow_the_header(name):
    py = [f[0] for f in getattr(binding, name)._fields_]
    assert py == _c_struct_fields(name)


def test_oracle_and_cuda_path_share_no_code():
    """Neither side imports, includes or builds from the other."""
    pkg = os.path.join(ROOT, "masked_optimizer_step_b200")
    bad_py = re.compile(r"^\s*(import|from)\s+(oracle|tests)\b", re.M)
    bad_c = re.compile(r"#\s*include\s*[<\"][^>\"]*oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert not bad_py.search(open(path).read()), path
            elif f.endswith((".cu", ".cuh", ".h", ".cpp")):
                assert not bad_c.search(open(path).read()), path
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c")):
            text = open(os.path.join(ROOT, "oracle", f)).read()
            assert not re.search(r"^\s*(import|from)\s+masked_optimizer_step_b200", text, re.M), f
            assert "#include" not in text or "csrc" not in text and "sf.h" not in text, f


def test_header_is_plain_c_and_links_against_the_library(tmp_path):
    # A C99 translation unit that takes the address of every declared entry point, compiled
    # with gcc and linked against libsf.so (nothing runs: no GPU needed).
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    names = _declared()
    src = ["#include \"sf.h\"", "#include <stdio.h>", "typedef void (*fn)(void);", "int main(void) {",
           "    fn p[] = {"]
    src += [f"        (fn){n}," for n in names]
    src += ["    };", "    printf(\"%d %d\\n\", (int)(sizeof p / sizeof p[0]), sf_version());", "    return 0;", "}"]
    c = tmp_path / "abi.c"
    c.write_text("\n".join(src) + "\n")
    lib_dir = os.path.dirname(binding.LIB_PATH)
    out = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(c), "-o", str(out), "-L", lib_dir, "-lsf", f"-Wl,-rpath,{lib_dir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(out)], capture_output=True, text=True)
    assert run.returncode == 0, run.stderr
    assert run.stdout.split() == [str(len(names)), str(10000)]
