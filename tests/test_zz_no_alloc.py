"""sf_embed_grad_noalloc: the embedding-row gradient for callers that must not allocate device
memory. It uses a fixed scratch array inside the library instead of a caller buffer; its results
must match sf_embed_grad's on the same inputs, call after call, even though every call reuses
(and leaves behind) the same scratch contents.

Kept in a file of its own, collected last, so that a failure here cannot hide other tests."""
import ctypes

import numpy as np
import pytest
import torch

from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from tests.gpu_helpers import DEV, bf16_dev, host, i32_dev, mask_host

pytestmark = pytest.mark.gpu


def _conductor_mask(V, cap, windows):
    mk = sf.Mask(V, cap, DEV)
    sf.sf_mask_init(mk)
    for tok in windows:
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(tok), n=len(tok))], 0.01)
    return mk


def test_noalloc_matches_workspace_version_on_two_calls_in_a_row(sf):
    """Both entry points run the same deterministic kernels on the same inputs, so their outputs
    must be equal byte for byte. The first call is the larger one (more tokens, more slots), so
    the second runs over the scratch contents the first left behind."""
    V, H = 32000, 512
    status = sf.status_word()
    for call, (n, cap) in enumerate([(8192, 8192), (2048, 1024)]):
        g = synth.rng(21, "tokens", call)
        windows = [synth.zipf_ids(g, n, V) for _ in range(3)]
        tok = windows[-1]
        mk = _conductor_mask(V, cap, windows)
        dY = bf16_dev(synth.normal_bf16(synth.rng(21, "dy", call), (n, H)))
        tok_d = i32_dev(tok)
        ws = torch.zeros(sf.sf_embed_grad_ws_bytes(n, cap) // 4, dtype=torch.int32, device=DEV)
        G_ref = torch.full((cap, H), float("nan"), device=DEV)
        sf.sf_embed_grad(tok_d, dY, mk, G_ref, ws, status)
        G = torch.full((cap, H), float("nan"), device=DEV)
        sf.sf_embed_grad_noalloc(tok_d, dY, mk, G, status)
        mh = mask_host(mk)
        rows = mh["rows"]
        assert len(rows) > 0
        slots = mh["row_slot"][rows]
        assert np.all(slots >= 0)
        ref, got = host(G_ref)[slots], host(G)[slots]
        assert got.tobytes() == ref.tobytes(), f"call {call}"
        assert np.isfinite(got).all()
        # slots no active row holds stay untouched
        unused = np.setdiff1d(np.arange(cap), slots)
        assert np.isnan(host(G)[unused]).all()
    assert int(host(status)[0]) == 0


def test_noalloc_rejects_sizes_beyond_its_fixed_scratch(sf):
    lib = sf.load()
    V, n = 64, 16384
    mk = sf.Mask(V, V, DEV)            # 4 slot_cap + 4 + n_tok scratch ints fit
    sf.sf_mask_init(mk)
    dY = torch.zeros((n, 8), dtype=torch.bfloat16, device=DEV)
    tok = torch.zeros(n, dtype=torch.int32, device=DEV)
    G = torch.zeros((V, 8), device=DEV)
    sf.sf_embed_grad_noalloc(tok, dY, mk, G)
    big = sf.Mask(49152, 49152, DEV)   # 4 * 49152 + 4 + 16384 > 65536 scratch ints: refused up front
    m = big.struct()
    rc = lib.sf_embed_grad_noalloc(tok.data_ptr(), n, dY.data_ptr(), 8, 8, ctypes.byref(m),
                                   G.data_ptr(), 8, None, None)
    assert rc == -3                    # SF_ERR_UNSUPPORTED
    torch.cuda.synchronize()
