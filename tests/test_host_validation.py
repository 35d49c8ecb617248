"""Host-side argument checks of every C-ABI entry point (CPU, no GPU).

Each case breaks one documented requirement and must come back as the documented error code
before anything is enqueued. The device pointers are placeholders that are never dereferenced:
every case here is rejected before the library touches CUDA. As a second guard the module is
skipped where a GPU is visible (the parity tests cover that machine).
"""
import ctypes

import pytest
import torch

from masked_optimizer_step_b200 import binding as b

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="placeholder device pointers: host validation only")

ARG, ALIGN, UNSUPPORTED = -1, -2, -3
P = 0x7F0000000000            # 16-byte aligned placeholder address, never dereferenced


@pytest.fixture(scope="module")
def lib():
    return b.load()


def _mask(R=256, cap=32):
    return b.sf_mask(R, cap, P, P, P, P, P, P, P, P, P, P)


def _prob(**kw):
    f = dict(dX=P, ld_dx=256, A=P, ld_a=512, T=128, C=512, mask=_mask(), dW=P, ld_dw=512)
    f.update(kw)
    return b.sf_dw_problem(f["dX"], f["ld_dx"], f["A"], f["ld_a"], f["T"], f["C"], f["mask"], f["dW"], f["ld_dw"])


def _dw(lib, probs, ws=None, ws_bytes=0):
    arr = (b.sf_dw_problem * max(len(probs), 1))(*probs)
    return lib.sf_masked_dw(arr, len(probs), ws, ws_bytes, None, None)


@pytest.mark.parametrize("case,kw,code", [
    ("C not a multiple of 8", dict(C=12, ld_dw=12, ld_a=16), ARG),
    ("negative token count", dict(T=-1), ARG),
    ("dW row stride below C", dict(ld_dw=256), ARG),
    ("dX row stride below R", dict(ld_dx=128), ARG),
    ("misaligned dW", dict(dW=P + 8), ALIGN),
    ("dW stride breaks 16 bytes", dict(ld_dw=514), ALIGN),
    ("A stride breaks 16 bytes", dict(ld_a=516), ALIGN),
    ("misaligned dX", dict(dX=P + 2), ALIGN),
    ("null dX with tokens", dict(dX=None), ARG),
    ("mask R not a multiple of 32", dict(mask=_mask(R=250)), ARG),
    ("slot capacity above R", dict(mask=_mask(R=64, cap=65)), ARG),
])
def test_masked_dw_rejects(lib, case, kw, code):
    assert _dw(lib, [_prob(**kw)]) == code, case


def test_masked_dw_rejects_short_or_misaligned_workspace(lib):
    probs = [_prob()]
    arr = (b.sf_dw_problem * 1)(*probs)
    need = lib.sf_masked_dw_ws_bytes(arr, 1)
    assert need > 0
    assert _dw(lib, probs, ws=P, ws_bytes=need - 1) == ARG
    assert _dw(lib, probs, ws=P + 4, ws_bytes=need) == ALIGN
    assert lib.sf_masked_dw(None, 1, None, 0, None, None) == ARG
    assert lib.sf_masked_dw(arr, -1, None, 0, None, None) == ARG


def _embed(lib, n_tok=64, H=512, ld_dy=512, ld_g=512, G=P, ws=P, ws_bytes=1 << 20, cap=32, tokens=P, dY=P):
    m = _mask(R=1024, cap=cap)
    return lib.sf_embed_grad(tokens, n_tok, dY, H, ld_dy, ctypes.byref(m), G, ld_g, ws, ws_bytes, None, None)


@pytest.mark.parametrize("case,kw,code", [
    ("H not a multiple of 8", dict(H=12, ld_dy=12, ld_g=12), ARG),
    ("dY stride below H", dict(ld_dy=256), ARG),
    ("G stride below H", dict(ld_g=256), ARG),
    ("negative token count", dict(n_tok=-1), ARG),
    ("null tokens", dict(tokens=None), ARG),
    ("misaligned G", dict(G=P + 4), ALIGN),
    ("misaligned workspace", dict(ws=P + 8), ALIGN),
    ("workspace too small", dict(ws_bytes=16), ARG),
    ("too many tokens", dict(n_tok=16385), UNSUPPORTED),
])
def test_embed_grad_rejects(lib, case, kw, code):
    assert _embed(lib, **kw) == code, case


def _mat(C=512, partner=-1, R=256, **ptrs):
    f = dict(q=P, s=P, delta=P, m=P, v=P, grad=P, live=P)
    f.update(ptrs)
    return b.sf_matrix(C, partner, 1.0, 0.0, _mask(R=R), f["q"], f["s"], f["delta"], f["m"], f["v"],
                       f["grad"], f["live"])


def _hp(bc=P, t_max=100):
    return b.sf_adam(1e-4, 0.9, 0.999, 1e-8, 0.1, 0.001, 0.0, 0.0, bc, bc, t_max)


def _upd(lib, mats, hp=None):
    arr = (b.sf_matrix * max(len(mats), 1))(*mats)
    h = hp if hp is not None else _hp()
    return lib.sf_sparse_update(arr, len(mats), ctypes.byref(h), None, None)


@pytest.mark.parametrize("case,mats,code", [
    ("C not a multiple of 8", [_mat(C=12)], ARG),
    ("C above the largest row", [_mat(C=32768 + 8)], UNSUPPORTED),
    ("null moments", [_mat(m=None)], ARG),
    ("misaligned residual", [_mat(delta=P + 4)], ALIGN),
    ("misaligned codes", [_mat(q=P + 4)], ALIGN),
    ("partner is itself", [_mat(partner=0)], ARG),
    ("partner out of range", [_mat(partner=1)], ARG),
    ("partner of another shape", [_mat(partner=1), _mat(C=256)], ARG),
    ("partner with other rows", [_mat(partner=1), _mat(R=512)], ARG),
])
def test_sparse_update_rejects(lib, case, mats, code):
    assert _upd(lib, mats) == code, case


def test_sparse_update_rejects_bad_hyper_parameters(lib):
    assert _upd(lib, [_mat()], hp=_hp(bc=None)) == ARG
    assert _upd(lib, [_mat()], hp=_hp(t_max=0)) == ARG
    arr = (b.sf_matrix * 1)(_mat())
    assert lib.sf_sparse_update(arr, 1, None, None, None) == ARG


def test_adam_tables_and_quantize_init_reject(lib):
    f = ctypes.c_float
    assert lib.sf_adam_tables(f(1.0), f(0.999), 10, P, P, None) == ARG
    assert lib.sf_adam_tables(f(0.9), f(0.999), 0, P, P, None) == ARG
    assert lib.sf_adam_tables(f(0.9), f(0.999), 10, None, P, None) == ARG
    assert lib.sf_quantize_init(P, -1, 8, P, P, P, None, None) == ARG
    assert lib.sf_quantize_init(None, 8, 8, P, P, P, None, None) == ARG


def test_checkpoint_rejects(lib):
    def call(name, C=512, cap=32, count=P):
        mats = (b.sf_matrix * 1)(_mat(C=C))
        ck = (b.sf_checkpoint * 1)(b.sf_checkpoint(cap, count, P, P, P, P, P, P, P))
        return getattr(lib, name)(mats, ck, 1, None, None)
    for name in ("sf_checkpoint_save", "sf_checkpoint_restore"):
        assert call(name, C=24) == ARG           # rows copied in 16-byte vectors: C % 16 == 0
        assert call(name, cap=-1) == ARG
        assert call(name, count=None) == ARG


def _mask_with(accum=P, R=256, cap=32):
    return b.sf_mask(R, cap, P, accum, P, P, P, P, P, P, P, P)


@pytest.mark.parametrize("case,accum,src,code", [
    ("output source: accumulator not 16-byte aligned (bf16 rows, 16-byte reductions)", P + 4,
     (b.SF_SRC_OUTPUT_BF16, 128, 256, P), ALIGN),
    ("output source: Y not 16-byte aligned", P, (b.SF_SRC_OUTPUT_BF16, 128, 256, P + 2), ALIGN),
    ("output source: row stride not a multiple of 8", P, (b.SF_SRC_OUTPUT_BF16, 128, 260, P), ALIGN),
    ("output source: row stride below R", P, (b.SF_SRC_OUTPUT_BF16, 128, 128, P), ARG),
    ("output source: negative token count", P, (b.SF_SRC_OUTPUT_BF16, -1, 256, P), ARG),
    ("unknown source kind", P, (9, 128, 256, P), ARG),
])
def test_mask_update_rejects(lib, case, accum, src, code):
    masks = (b.sf_mask * 1)(_mask_with(accum))
    srcs = (b.sf_mask_src * 1)(b.sf_mask_src(*src))
    assert lib.sf_mask_update(masks, srcs, 1, ctypes.c_float(0.01), None, None) == code, case


def test_forward_tracked_rejects_a_misaligned_accumulator(lib):
    # A [128 x 512], W [256 x 512], Y [128 x 256]; the mask's accumulator 4 bytes off
    p = b.sf_fwd_problem(P, 512, P, 512, P, 256, 128, 512, _mask_with(P + 4))
    assert lib.sf_forward_tracked((b.sf_fwd_problem * 1)(p), 1, None, None) == ALIGN
    p = b.sf_fwd_problem(P, 512, P, 512, P + 8, 256, 128, 512, _mask_with(P))
    assert lib.sf_forward_tracked((b.sf_fwd_problem * 1)(p), 1, None, None) == ALIGN
