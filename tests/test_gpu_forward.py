"""sf_forward_tracked: the forward projection with the row tracker in its epilogue (GPU).

Y = A W^T on the tensor cores, rounded to bf16, against the fp64 oracle product: within the dW
tolerance plus the bf16 output rounding (|Y - ref| <= (2^-8 + 2e-3) * max(|ref|, 1e-3 max|ref|)).
The folded statistic is checked bit for bit: after the call, each mask's accumulator holds the
oracle's row magnitudes of the Y the kernel stored (as bf16, two bytes per row at the start of the
accumulator), and closing the window gives the oracle tracker's charges, mask and lists on that Y.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from tests.gpu_helpers import DEV, bf16_dev, check_slot_invariants, host, mask_host

pytestmark = pytest.mark.gpu

Y_TOL = 2.0 ** -8 + 2e-3


def _accum_matches(mk, h):
    """The mask's output accumulator: row r's magnitude as bf16 at byte 2r, the rest zero; the
    oracle's h holds each magnitude widened to fp32 bits."""
    acc = host(mk.accum).view(np.uint16)
    want = (h.view(np.uint32) >> 16).astype(np.uint16)
    return acc[: mk.R].tobytes() == want.tobytes() and not np.any(acc[mk.R:])


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check_y(Y_gpu_bits, ref, what):
    got = synth.bf16_bits_to_f32(Y_gpu_bits).astype(np.float64)
    floor = 1e-3 * np.abs(ref).max()
    err = np.abs(got - ref) / np.maximum(np.abs(ref), floor)
    assert err.max() <= Y_TOL, (what, float(err.max()))


def _close_window(masks, Ys):
    srcs = [sf.make_src(sf.SF_SRC_OUTPUT_BF16, Y, n=Y.shape[0], ld=Y.stride(0)) for Y in Ys]
    sf.sf_mask_update_phase(masks, srcs, sf.SF_PHASE_SECOND, 0.01)


@pytest.mark.parametrize("shapes", [
    [(200, 200, 320), (200, 136, 64)],          # ragged tokens, columns and rows; two problems
    [(128, 64, 256)],                           # exactly one unit
    [(1, 8, 32), (300, 1000, 96)],              # a single token; C not a multiple of 64
])
def test_forward_tracked_matches_oracle(sf, shapes):
    masks, Ys, probs, inputs = [], [], [], []
    for i, (T, C, R) in enumerate(shapes):
        g = synth.rng(17, "misc", T, C, R, i)
        A = synth.normal_bf16(g, (T, C))
        W = synth.normal_bf16(g, (R, C), std=0.005)
        W[g.choice(R, size=max(1, R // 32), replace=False)] = synth.normal_bf16(g, (max(1, R // 32), C))
        mk = sf.Mask(R, R // 4, DEV)
        sf.sf_mask_init(mk)
        Y = torch.full((T, R), float("nan"), dtype=torch.bfloat16, device=DEV)
        masks.append(mk)
        Ys.append(Y)
        inputs.append((A, W))
        probs.append(sf.fwd_problem(bf16_dev(A), bf16_dev(W), Y, mk))
    status = sf.status_word()
    sf.sf_forward_tracked(probs, status)
    torch.cuda.synchronize()
    for (A, W), Y, mk, shp in zip(inputs, Ys, masks, shapes):
        yb = _bits(Y)
        _check_y(yb, orc.forward_product(A, W), shp)
        h, n_bad = orc.row_magnitudes(yb)
        assert n_bad == 0
        assert (h.view(np.uint32) & 0xFFFF).max() == 0          # magnitudes are bf16 values
        assert _accum_matches(mk, h), shp
    _close_window(masks, Ys)
    for Y, mk, shp in zip(Ys, masks, shapes):
        charge = np.zeros(mk.R, np.float32)
        words = orc.window_outputs(charge, _bits(Y))
        mh = mask_host(mk)
        assert mh["charge"].tobytes() == charge.tobytes() and np.array_equal(mh["words"], words), shp
        rows, tiles = orc.mask_lists(words)
        assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles)
        check_slot_invariants(mh, mk.slot_cap)
        assert not np.any(host(mk.accum))              # the window is closed: accumulator cleared
    assert int(host(status)[0]) == 0


def test_forward_tracked_7b_layer_matches_tracker_on_its_outputs(sf):
    """One 7B-shaped layer at 2,048 tokens: every projection's Y against the oracle on sampled
    tokens; masks bit-exact against the oracle tracker on the full Y the kernel stored."""
    T = 2048
    shapes = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))
    masks, Ys, probs, keep = [], [], [], []
    for i, (name, R, C) in enumerate(shapes):
        A = synth.device_normal_bf16((T, C), 6, "act", i, device=DEV)
        W = synth.device_normal_bf16((R, C), 6, "weights", i, std=0.005, device=DEV)
        rows = torch.from_numpy(synth.scattered_rows(synth.rng(6, "rows", i), R, 0.01)).long().to(DEV)
        W[rows] = synth.device_normal_bf16((len(rows), C), 6, "weights", i, 1, std=1.0, device=DEV)
        mk = sf.Mask(R, max(32, R // 32), DEV)
        sf.sf_mask_init(mk)
        Y = torch.empty((T, R), dtype=torch.bfloat16, device=DEV)
        masks.append(mk)
        Ys.append(Y)
        keep.append((A, W))
        probs.append(sf.fwd_problem(A, W, Y, mk))
    status = sf.status_word()
    sf.sf_forward_tracked(probs, status)
    _close_window(masks, Ys)
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0
    pick = np.sort(synth.rng(6, "misc", 99).choice(T, size=96, replace=False))
    for (A, W), Y, mk, (name, R, C) in zip(keep, Ys, masks, shapes):
        yb = _bits(Y)
        _check_y(yb[pick], orc.forward_product(_bits(A)[pick], _bits(W)), name)
        charge = np.zeros(R, np.float32)
        words = orc.window_outputs(charge, yb)
        mh = mask_host(mk)
        assert mh["charge"].tobytes() == charge.tobytes() and np.array_equal(mh["words"], words), name
        assert 0 < mh["counts"][0] <= mk.slot_cap, name


def test_forward_tracked_non_finite_outputs(sf):
    """Infinities planted in the weights make some outputs infinite or NaN: the folded statistic
    follows the tracker's reading on exactly the Y that was stored, and the status is raised."""
    T, C, R = 256, 128, 256
    g = synth.rng(18, "misc", 1)
    A = synth.normal_bf16(g, (T, C))
    W = synth.normal_bf16(g, (R, C))
    W[5, 7] = 0x7F80                     # +inf: row 5 of Y is +-inf (or NaN where A is 0)
    W[9, :] = 0x7FC0                     # NaN: row 9 of Y is NaN throughout
    mk = sf.Mask(R, 64, DEV)
    sf.sf_mask_init(mk)
    Y = torch.empty((T, R), dtype=torch.bfloat16, device=DEV)
    status = sf.status_word()
    sf.sf_forward_tracked([sf.fwd_problem(bf16_dev(A), bf16_dev(W), Y, mk)], status)
    torch.cuda.synchronize()
    yb = _bits(Y)
    h, n_bad = orc.row_magnitudes(yb)
    assert n_bad > 0
    assert _accum_matches(mk, h)
    assert int(host(status)[0]) & sf.SF_STATUS_NONFINITE
    _close_window([mk], [Y])
    charge = np.zeros(R, np.float32)
    words = orc.window_outputs(charge, yb)
    mh = mask_host(mk)
    assert mh["charge"].tobytes() == charge.tobytes() and np.array_equal(mh["words"], words)
    assert (mh["words"][0] >> 5) & 1 and not (mh["words"][0] >> 9) & 1
