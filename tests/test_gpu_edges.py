"""Degenerate inputs through the C ABI (GPU): no tokens, no active rows, no moment slots, empty
calls. Each must do exactly what the header says and leave every other byte alone."""
import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import synth
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host, i32_dev, mask_host, u32_dev

pytestmark = pytest.mark.gpu

CANARY = np.uint32(0x7FBADBAD)


def _canary(shape):
    return torch.from_numpy(np.full(shape, CANARY, dtype=np.uint32).view(np.int32)).to(DEV).view(torch.float32)


def _words_mask(sf, R, cap, rows):
    mk = sf.Mask(R, cap, DEV)
    sf.sf_mask_init(mk)
    sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(synth.words_from_rows(R, rows)))], 0.01)
    return mk


def test_embed_grad_without_tokens_zeroes_the_active_rows(sf):
    V, H = 1024, 256
    mk = _words_mask(sf, V, 16, [3, 70, 900])
    G = _canary((16, H))
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(0, 16) // 4 + 64, dtype=torch.int32, device=DEV)
    status = sf.status_word()
    tok = torch.zeros(0, dtype=torch.int32, device=DEV)
    dY = torch.zeros((0, H), dtype=torch.bfloat16, device=DEV)
    sf.sf_embed_grad(tok, dY, mk, G, ws, status)
    got = host(G)
    mh = mask_host(mk)
    used = {int(mh["row_slot"][r]) for r in mh["rows"]}
    for s in range(16):
        if s in used:
            assert not got[s].any()
        else:
            assert (got[s].view(np.uint32) == CANARY).all()
    assert int(host(status)[0]) == 0


def test_embed_grad_with_no_active_row_writes_nothing(sf):
    V, H, n = 1024, 256, 300
    mk = _words_mask(sf, V, 16, [])
    tok = synth.zipf_ids(synth.rng(5, "tokens"), n, V)
    dY = synth.normal_bf16(synth.rng(5, "dy"), (n, H))
    G = _canary((16, H))
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(n, 16) // 4 + 64, dtype=torch.int32, device=DEV)
    sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G, ws)
    assert (host(G).view(np.uint32) == CANARY).all()


@pytest.mark.parametrize("case", ["one row takes every token", "every token its own row"])
def test_embed_grad_segment_extremes(sf, case):
    """The segment sort at its extremes: a single segment of the largest length (16,384
    positions, a 512-word bitmap, in place) and 2,048 segments of one position each."""
    H = 64
    if case == "one row takes every token":
        V, n, rows = 1024, 16384, [517]
        tok = np.full(n, 517, np.int32)
        tok[::7] = 3                              # an inactive row in between
    else:
        V, n = 4096, 2048
        tok = synth.rng(6, "tokens").permutation(V)[:n].astype(np.int32)
        rows = np.sort(tok)
    cap = max(32, len(rows))
    mk = _words_mask(sf, V, cap, rows)
    dY = synth.normal_bf16(synth.rng(6, "dy", n), (n, H))
    G = _canary((cap, H))
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(n, cap) // 4, dtype=torch.int32, device=DEV)
    status = sf.status_word()
    sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G, ws, status)
    mh = mask_host(mk)
    ref = orc.embed_grad(tok, dY, V, mh["words"])
    got = host(G)
    scale = max(np.abs(ref[mh["rows"]]).max(), 1.0)
    for r in mh["rows"]:
        e = np.max(np.abs(got[mh["row_slot"][r]] - ref[r]) / np.maximum(np.abs(ref[r]), 1e-3 * scale))
        assert e <= 2e-3, int(r)
    assert int(host(status)[0]) == 0
    G2 = _canary((cap, H))                        # the same bytes again
    sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G2, ws)
    assert host(G2).tobytes() == got.tobytes()


def _matrix(sf, R, C, cap, seed):
    W = synth.weights_f32(synth.rng(seed, "weights"), R, C)
    mat = sf.Matrix(R, C, cap, DEV)
    sf.sf_mask_init(mat.mask)
    sf.sf_quantize_init(f32_dev(W), mat)
    return mat


def _bytes(mat):
    return {k: host(getattr(mat, k)).tobytes() for k in ("q", "s", "delta", "live", "m", "v")}


def test_update_with_an_empty_mask_changes_nothing(sf):
    mat = _matrix(sf, 128, 256, 16, 1)
    sf.sf_mask_update([mat.mask], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(np.zeros(4, np.uint32)))], 0.01)
    mat.grad.copy_(torch.randn_like(mat.grad))
    before = _bytes(mat)
    status = sf.status_word()
    sf.sf_sparse_update([sf.matrix_struct(mat)], sf.AdamParams(), status)
    assert _bytes(mat) == before
    assert int(host(status)[0]) == 0


def test_matrix_without_moment_slots_overflows_and_is_left_alone(sf):
    # slot_cap = 0: every active row reports SLOT_OVERFLOW at the mask and is skipped by dW and the
    # update; nothing of the matrix changes.
    R, C, T = 128, 256, 64
    mat = _matrix(sf, R, C, 0, 2)
    status = sf.status_word()
    sf.sf_mask_update([mat.mask], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(synth.words_from_rows(R, [1, 40, 77])))],
                      0.01, status)
    assert int(host(status)[0]) & sf.SF_STATUS_SLOT_OVERFLOW
    mh = mask_host(mat.mask)
    assert mh["counts"][0] == 3 and mh["counts"][3] == 3 and (mh["row_slot"] == -1).all()
    before = _bytes(mat)
    dX = synth.normal_bf16(synth.rng(2, "dx"), (T, R))
    A = synth.normal_bf16(synth.rng(2, "act"), (T, C))
    probs = [sf.dw_problem(bf16_dev(dX), bf16_dev(A), mat.mask, mat.grad)]
    sf.sf_masked_dw(probs, status, ws=sf.dw_workspace(probs))
    sf.sf_sparse_update([sf.matrix_struct(mat)], sf.AdamParams(), status)
    assert _bytes(mat) == before


def test_empty_calls_are_no_ops(sf):
    L = sf.load()
    assert L.sf_sparse_update(None, 0, None, None, None) == -1       # hp is required even for n = 0
    hp = sf.AdamParams()
    h = hp.struct()
    import ctypes
    assert L.sf_sparse_update(None, 0, ctypes.byref(h), None, None) == 0
    assert L.sf_masked_dw(None, 0, None, 0, None, None) == 0
    assert L.sf_mask_update(None, None, 0, ctypes.c_float(0.01), None, None) == 0
    assert L.sf_checkpoint_save(None, None, 0, None, None) == 0
    torch.cuda.synchronize()


def test_first_update_of_a_fresh_row_is_the_closed_form_step(sf):
    # First Adam step from zero moments: u = g / (|g| + eps) per element (bias corrections cancel
    # exactly here only up to fp32 rounding), so the weight moves by about -lr * sign(g).
    R, C = 64, 128
    mat = _matrix(sf, R, C, 8, 3)
    rows = [5, 6]
    sf.sf_mask_update([mat.mask], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(synth.words_from_rows(R, rows)))], 0.01)
    g = np.random.default_rng(3).standard_normal((8, C)).astype(np.float32) * 4
    mat.grad.copy_(f32_dev(g))
    W0 = orc.rebuild(host(mat.q), host(mat.s), host(mat.delta))
    lr = 1e-3
    sf.sf_sparse_update([sf.matrix_struct(mat)], sf.AdamParams(lr=lr), None)
    W1 = orc.rebuild(host(mat.q), host(mat.s), host(mat.delta))
    mh = mask_host(mat.mask)
    for r in rows:
        k = mh["row_slot"][r]
        step = W1[r] - W0[r]
        np.testing.assert_allclose(step, -lr * np.sign(g[k]), rtol=2e-3, atol=1e-7)
