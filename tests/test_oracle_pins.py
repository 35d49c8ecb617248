"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every check is a closed form derived from the
stated rule, an invariant, a library routine (numpy / torch) or a brute-force computation in
exact arithmetic. Sections refer to "Sparse-First Fine-Tuning" (tensorwirelabs.com).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import synth
from tests.conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# =============================================================================================
# Number formats (fp16 moments, bf16 activations and live weights; section 2.3)
# =============================================================================================

def test_f16_decode_every_pattern_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _format_probe_values():
    g = np.random.default_rng(11)
    x = (g.standard_normal(400_000) * np.exp2(g.uniform(-30, 18, 400_000))).astype(np.float32)
    edges = np.array([0.0, -0.0, 65504, 65519.996, 65520, 65536, 6.1035156e-05, 6.097555e-05,
                      5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 8.9406967e-08, 1.0009766,
                      1.0004883, 1.0014648, np.inf, -np.inf, 3.4e38, 1e-45, -2.0000001],
                     dtype=np.float32)
    # exact f16 halfway points (ties) in the normal and subnormal range
    base = np.arange(0, 31744, 97, dtype=np.uint16).view(np.float16).astype(np.float32)
    nxt = (np.arange(0, 31744, 97, dtype=np.uint16) + 1).view(np.float16).astype(np.float32)
    ties = ((base.astype(np.float64) + nxt.astype(np.float64)) / 2).astype(np.float32)
    return np.concatenate([x, -x[:1000], edges, ties, -ties])


def test_f16_encode_matches_numpy_round_to_nearest_even():
    x = _format_probe_values()
    ours = orc.f32_to_f16(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    assert orc.f32_to_f16(np.array([np.nan], np.float32))[0] & 0x7C00 == 0x7C00


def test_bf16_decode_and_encode_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    x = _format_probe_values()
    enc = orc.f32_to_bf16(x)
    ref_enc = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(enc, ref_enc)


# =============================================================================================
# Section 2.1: the charge rule, the threshold and the masks
# =============================================================================================

def test_silent_row_fades_as_printed_rule_implies():
    gd = _golden("charge_fade.json")
    charge = np.zeros(gd["R"], dtype=np.float32)
    for n, window in enumerate(gd["windows"]):
        words, bad = orc.window_tokens(charge, window)
        assert bad == 0
        assert charge[gd["row"]] == np.float32(gd["charge"][n])
        active = bool((words[0] >> gd["row"]) & 1)
        assert active == gd["active"][n], f"window {n + 1}"
        others = np.delete(charge, gd["row"])
        assert not others.any()


def test_constant_share_closed_form():
    # Rows 0..3 receive 8, 4, 2, 1 hits every window: shares 1, 1/2, 1/4, 1/8. By the rule the
    # charge after n windows is share * (1 - 2^-n), exact in fp32 for these dyadic shares.
    R = 64
    tokens = [0] * 8 + [1] * 4 + [2] * 2 + [3]
    charge = np.zeros(R, dtype=np.float32)
    shares = [Fraction(1), Fraction(1, 2), Fraction(1, 4), Fraction(1, 8)]
    for n in range(1, 21):
        orc.window_tokens(charge, tokens)
        for r, s in enumerate(shares):
            assert Fraction(float(charge[r])) == s * (1 - Fraction(1, 2 ** n))
        assert not charge[4:].any()


def test_charge_recurrence_brute_force_in_exact_arithmetic():
    # Random hit counts on 8 rows over 12 windows (some windows empty): the fp32 oracle must
    # follow the exact rational recurrence q <- q/2 + (h/hmax)/2 to within fp32 rounding, and
    # its activity decision must agree wherever the exact charge is not within rounding of 0.01.
    g = np.random.default_rng(5)
    R = 32
    for trial in range(30):
        exact = [Fraction(0)] * 8
        charge = np.zeros(R, dtype=np.float32)
        for w in range(12):
            hits = g.integers(0, 6, size=8) if g.random() > 0.15 else np.zeros(8, int)
            tokens = np.repeat(np.arange(8), hits)
            g.shuffle(tokens)
            words, _ = orc.window_tokens(charge, tokens)
            hmax = int(hits.max())
            for r in range(8):
                share = Fraction(int(hits[r]), hmax) if hmax else Fraction(0)
                exact[r] = exact[r] / 2 + share / 2
                got = Fraction(float(charge[r]))
                assert abs(got - exact[r]) <= Fraction(1, 2 ** 21) * max(exact[r], Fraction(1, 2 ** 100))
                if abs(exact[r] - Fraction(1, 100)) > Fraction(1, 10 ** 6):
                    assert bool((words[0] >> r) & 1) == (exact[r] >= Fraction(1, 100))


def test_threshold_compares_against_fp32_of_one_percent():
    # 0.02f halved is exactly float32(0.01): that row is active. One ulp less is not.
    R = 32
    charge = np.zeros(R, dtype=np.float32)
    charge[0] = np.float32(0.02)
    charge[1] = np.nextafter(np.float32(0.02), np.float32(0))
    words, _ = orc.window_tokens(charge, [])
    assert charge[0] == np.float32(0.01)
    assert words[0] & 1 == 1
    assert (words[0] >> 1) & 1 == 0


def test_out_of_range_token_ids_are_counted_and_ignored():
    charge = np.zeros(32, dtype=np.float32)
    words, bad = orc.window_tokens(charge, [3, -1, 32, 3, 99])
    assert bad == 3
    assert charge[3] == np.float32(0.5) and words[0] == 1 << 3


def test_output_tracker_uses_row_absmax_share():
    # Planted column maxima 4, -2 (magnitude 2), 1, 0.5 over rows 0..3, everything else smaller
    # than 0.01: shares 1, 1/2, 1/4, 1/8 -> charges 1/2, 1/4, 1/8, 1/16 from zero.
    T, R = 16, 64
    Y = np.full((T, R), 0.0, dtype=np.float32)
    g = np.random.default_rng(1)
    Y[:, :4] = g.uniform(-0.4, 0.4, size=(T, 4))
    Y[3, 0], Y[7, 1], Y[0, 2], Y[15, 3] = 4.0, -2.0, 1.0, -0.5
    Y[:, 4:] = g.uniform(-0.01, 0.01, size=(T, R - 4))
    Yb = synth.f32_to_bf16_bits(Y)
    charge = np.zeros(R, dtype=np.float32)
    words = orc.window_outputs(charge, Yb)
    assert list(charge[:4]) == [0.5, 0.25, 0.125, 0.0625]
    assert words[0] == 0b1111 and words[1] == 0
    # every other row: share = max|Y|/4 (|Y| <= 0.01 before bf16 rounding) -> inactive
    amax = np.abs(synth.bf16_bits_to_f32(Yb)[:, 4:]).max(axis=0)
    np.testing.assert_array_equal(charge[4:], np.float32(0.5) * (amax / np.float32(4)))
    assert np.all(charge[4:] < 0.0013)


def test_tracker_non_finite_outputs():
    # A NaN output carries no magnitude; +-inf counts as the largest finite bf16 magnitude
    # (0x7F7F), so charges stay finite: rows holding an infinity get share 1, the rest share
    # h / largest in fp32 (subnormal for h = 2 and h = 1). Every non-finite output is counted.
    T, R = 8, 64
    g = np.random.default_rng(3)
    Yb = synth.f32_to_bf16_bits(g.uniform(-0.01, 0.01, size=(T, R)).astype(np.float32))
    Yb[2, 0] = 0x7F80            # +inf
    Yb[1, 1] = 0x7FC0            # NaN
    Yb[5, 1] = 0xC000            # -2.0
    Yb[4, 2] = 0xFF80            # -inf
    Yb[:, 3] = 0xFFC1            # NaN (negative sign, other payload) everywhere
    Yb[0, 4] = 0x3F80            # 1.0
    charge = np.zeros(R, dtype=np.float32)
    words, n_bad = orc.window_outputs_counted(charge, Yb)
    assert n_bad == 3 + T
    largest = synth.bf16_bits_to_f32(np.array([0x7F7F], np.uint16))[0]
    assert largest == np.float32(3.3895313892515355e38)
    half = np.float32(0.5)
    assert charge[0] == half and charge[2] == half and charge[3] == 0.0
    assert charge[1] == half * (np.float32(2.0) / largest) and charge[1] > 0
    assert charge[4] == half * (np.float32(1.0) / largest)
    assert np.all(np.isfinite(charge))
    assert words[0] == 0b101 and words[1] == 0


def test_masked_dw_rows_matches_the_loop():
    # Integer-valued bf16 inputs keep every fp64 sum exact, so the matrix-product form must equal
    # the plain loop bit for bit; on N(0,1) inputs they agree to fp64 rounding.
    g = np.random.default_rng(11)
    T, R, C = 37, 96, 40
    dX = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(T, R)).astype(np.float32))
    A = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(T, C)).astype(np.float32))
    rows = np.array([0, 5, 31, 32, 64, 95])
    full = orc.masked_dw(dX, A, synth.words_from_rows(R, rows))
    got = orc.masked_dw_rows(dX, A, rows)
    assert got.shape == (len(rows), C)
    assert np.array_equal(got, full[rows])
    dX = synth.normal_bf16(g, (T, R))
    A = synth.normal_bf16(g, (T, C))
    full = orc.masked_dw(dX, A, synth.words_from_rows(R, rows))
    np.testing.assert_allclose(orc.masked_dw_rows(dX, A, rows), full[rows], rtol=1e-12, atol=1e-12)
    # a transposed or shifted operand is caught
    assert not np.allclose(orc.masked_dw_rows(dX, A, rows[::-1]), full[rows])


def test_activity_rule_split_over_token_shares():
    # The rule applied to combined activities equals the windows counted in one piece: hit
    # counts add over disjoint token shares, row magnitudes combine by max (and so does the
    # non-finite handling), for any split of the tokens.
    g = np.random.default_rng(5)
    R, V, T = 256, 256, 96
    tok = synth.zipf_ids(g, T, V)
    c1, c2 = np.zeros(V, np.float32), np.zeros(V, np.float32)
    w1, _ = orc.window_tokens(c1, tok)
    hits = np.bincount(tok[:40], minlength=V) + np.bincount(tok[40:], minlength=V)
    w2 = orc.window_activity(c2, hits.astype(np.float32))
    assert c1.tobytes() == c2.tobytes() and np.array_equal(w1, w2)
    Y = synth.tracker_outputs(g, T, synth.tracker_gains(R, synth.scattered_rows(g, R, 0.03)))
    Y[5, 7], Y[60, 9] = 0x7F80, 0x7FC0
    c1, c2 = np.zeros(R, np.float32), np.zeros(R, np.float32)
    w1, n1 = orc.window_outputs_counted(c1, Y)
    (ha, na), (hb, nb) = orc.row_magnitudes(Y[:33]), orc.row_magnitudes(Y[33:])
    w2 = orc.window_activity(c2, np.maximum(ha, hb))
    assert c1.tobytes() == c2.tobytes() and np.array_equal(w1, w2) and n1 == na + nb == 2
    # an empty window is pure decay
    c3 = c1.copy()
    orc.window_activity(c3, np.zeros(R, np.float32))
    assert c3.tobytes() == (np.float32(0.5) * c1).tobytes()


def test_forward_product_matches_brute_force():
    # integer-valued bf16 inputs keep fp64 sums exact: the product must equal the plain triple
    # loop bit for bit, and a transposed operand must not
    g = np.random.default_rng(13)
    T, C, R = 7, 24, 5
    A = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(T, C)).astype(np.float32))
    W = synth.f32_to_bf16_bits(g.integers(-8, 9, size=(R, C)).astype(np.float32))
    Af, Wf = synth.bf16_bits_to_f32(A), synth.bf16_bits_to_f32(W)
    ref = np.zeros((T, R))
    for t in range(T):
        for r in range(R):
            for c in range(C):
                ref[t, r] += float(Af[t, c]) * float(Wf[r, c])
    got = orc.forward_product(A, W)
    assert got.shape == (T, R) and np.array_equal(got, ref)
    assert not np.array_equal(orc.forward_product(A[:, ::-1], W), ref)


def test_tracker_recipe_turns_exactly_the_chosen_rows_on():
    g = synth.rng(2, "tracker", 0)
    R, T = 1024, 512
    rows = synth.scattered_rows(g, R, 0.01)
    Y = synth.tracker_outputs(g, T, synth.tracker_gains(R, rows))
    charge = np.zeros(R, dtype=np.float32)
    words = orc.window_outputs(charge, Y)
    got_rows, _ = orc.mask_lists(words)
    assert np.array_equal(got_rows, rows)


def test_mask_lists_golden():
    gd = _golden("mask_lists.json")
    words = synth.words_from_rows(gd["R"], gd["active_rows"])
    assert list(words) == gd["words"]
    rows, tiles = orc.mask_lists(words)
    assert list(rows) == gd["active_rows"]
    assert list(tiles) == gd["active_tiles"]


def test_mask_lists_match_brute_force_on_random_masks():
    g = np.random.default_rng(3)
    for R in (32, 96, 1024):
        act = g.random(R) < 0.1
        act[g.integers(0, R // 32) * 32:][:32] = False
        words = synth.words_from_rows(R, np.nonzero(act)[0])
        rows, tiles = orc.mask_lists(words)
        assert list(rows) == [r for r in range(R) if act[r]]
        assert list(tiles) == [w for w in range(R // 32) if act[32 * w:32 * w + 32].any()]


# =============================================================================================
# Section 2.3: moments only for active rows
# =============================================================================================

def test_moments_follow_mask_zero_on_change_keep_otherwise():
    R, C = 64, 5
    m = np.full((R, C), 0x3C00, dtype=np.uint16)
    v = np.full((R, C), 0x3800, dtype=np.uint16)
    step = np.full(R, 7, dtype=np.int32)
    old = synth.words_from_rows(R, [1, 2, 40])
    new = synth.words_from_rows(R, [2, 3, 40])
    orc.moments_follow_mask(old, new, m, v, step)
    changed = {1, 3}
    for r in range(R):
        if r in changed:
            assert not m[r].any() and not v[r].any() and step[r] == 0
        else:
            assert (m[r] == 0x3C00).all() and (v[r] == 0x3800).all() and step[r] == 7


# =============================================================================================
# Section 2.2: masked weight gradient and embedding-row gradient
# =============================================================================================

def _bf16(g, shape, scale=1.0):
    return synth.f32_to_bf16_bits(g.standard_normal(shape).astype(np.float32) * scale)


def test_dw_all_active_equals_fp64_matmul_non_square():
    g = np.random.default_rng(7)
    T, R, C = 37, 64, 24
    dX, A = _bf16(g, (T, R)), _bf16(g, (T, C))
    words = np.full(R // 32, 0xFFFFFFFF, dtype=np.uint32)
    dW = orc.masked_dw(dX, A, words)
    ref = synth.bf16_bits_to_f32(dX).astype(np.float64).T @ synth.bf16_bits_to_f32(A).astype(np.float64)
    np.testing.assert_allclose(dW, ref, rtol=1e-12, atol=1e-12)


def test_dw_small_integer_example():
    # dX[:, 0] = (1, 2), A[:, 0] = (3, 4), A[:, 1] = (5, -6): dW[0] = (1*3+2*4, 1*5-2*6) = (11, -7)
    dX = np.zeros((2, 32), np.float32)
    dX[:, 0] = [1, 2]
    A = np.array([[3, 5], [4, -6]], np.float32)
    dW = orc.masked_dw(synth.f32_to_bf16_bits(dX), synth.f32_to_bf16_bits(A),
                       synth.words_from_rows(32, [0]))
    assert list(dW[0]) == [11.0, -7.0]


def test_dw_skips_empty_tiles_and_inactive_rows_exactly():
    g = np.random.default_rng(8)
    T, R, C = 20, 128, 16
    dX, A = _bf16(g, (T, R)), _bf16(g, (T, C))
    active = [0, 1, 31, 70]                      # tile 0 partial, tile 2 one row, tiles 1, 3 empty
    words = synth.words_from_rows(R, active)
    canary = np.frombuffer(np.uint64(0x7FF4DEADBEEF0001).tobytes(), np.float64)[0]
    out = np.full((R, C), canary)
    orc.masked_dw(dX, A, words, out)
    ref = synth.bf16_bits_to_f32(dX).astype(np.float64).T @ synth.bf16_bits_to_f32(A).astype(np.float64)
    for r in range(R):
        if r in active:
            np.testing.assert_allclose(out[r], ref[r], rtol=1e-12)
        else:
            assert out[r].tobytes() == np.full(C, canary).tobytes()


def test_embed_grad_equals_numpy_add_at_on_active_rows():
    g = np.random.default_rng(9)
    V, H, n = 96, 40, 300
    tok = synth.zipf_ids(g, n, V)
    dY = _bf16(g, (n, H))
    active = [0, 1, 2, 5, 50, 95]                # 95 likely unseen: must come out as zeros
    words = synth.words_from_rows(V, active)
    G = orc.embed_grad(tok, dY, V, words, out=np.full((V, H), 12345.0))
    ref = np.zeros((V, H))
    np.add.at(ref, tok, synth.bf16_bits_to_f32(dY).astype(np.float64))
    for r in range(V):
        if r in active:
            np.testing.assert_allclose(G[r], ref[r], rtol=1e-12, atol=1e-12)
        else:
            assert (G[r] == 12345.0).all()


# =============================================================================================
# Section 2.3: int8 + scale + residual storage
# =============================================================================================

def test_quantize_golden_row_half_even():
    gd = _golden("quant_row.json")
    W = np.array([gd["W"]], dtype=np.float32)
    q, s, d = orc.quantize_rows(W)
    assert s[0] == np.float32(gd["s"])
    assert list(q[0]) == gd["q"]
    assert list(d[0]) == gd["delta"]


def test_quantize_invariants_on_random_rows():
    g = np.random.default_rng(4)
    W = (g.standard_normal((64, 300)) * 0.02).astype(np.float32)
    W[5] = 0.0
    W[6, :] = 0.0
    W[6, 17] = -3e-5
    q, s, d = orc.quantize_rows(W)
    assert np.abs(q.astype(int)).max() <= 127
    for r in range(64):
        amax = np.abs(W[r]).max()
        assert s[r] == np.float32(amax / np.float32(127)) if amax else s[r] == 0
        if amax > 0:
            assert np.abs(q[r].astype(int)).max() == 127
    assert not q[5].any() and s[5] == 0 and np.array_equal(d[5], W[5])
    # W = s*q + delta, one fused rounding, reproduces W (up to an exact tie, absent here)
    assert np.array_equal(orc.rebuild(q, s, d), W)
    # residual stays below half a quantisation step (plus the rounding of delta itself)
    assert np.all(np.abs(d) <= s[:, None] * np.float32(0.5) * (1 + 1e-6) + 1e-30)


# =============================================================================================
# Sections 2.3 / 2.4: the fused sparse update
# =============================================================================================

HP = orc.AdamHP(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8)


def _grad(g, R, C):
    # |g| in [0.5, 2): moments stay in fp16's normal range, so fp16 storage costs at most 2^-11
    return (g.choice([-1, 1], size=(R, C)) * g.uniform(0.5, 2.0, size=(R, C))).astype(np.float32)


def test_bias_correction_against_exact_rational():
    for beta in (0.9, 0.999, 0.5):
        b = Fraction(float(np.float32(beta)))
        for t in (1, 2, 3, 10, 100, 1000):
            exact = 1 / (1 - b ** t)
            got = orc.bias_correction(beta, t)
            assert abs(Fraction(got) - exact) <= exact * Fraction(1, 2 ** 23)


def test_first_step_closed_form():
    # Fresh moments: m-hat = g, v-hat = g^2, so the step is -lr * g / (|g| + eps) (section 2.4:
    # plain Adam with bias correction), before any fp16 rounding of stored moments.
    g = np.random.default_rng(12)
    R, C = 64, 48
    W0 = synth.weights_f32(g, R, C)
    st = orc.MatrixState(W0)
    st.set_mask(synth.words_from_rows(R, [0, 3, 40, 63]))
    Wq = st.weight()
    grad = (g.standard_normal((R, C)) * 3).astype(np.float32)
    # a few entries near eps, where eps visibly shapes the step (1e-8 -> half a step)
    grad[:, :6] = np.array([1e-8, -1e-8, 3e-9, -2e-7, 5e-8, -1e-9], np.float32)
    orc.update(st, grad, HP)
    Wn = st.weight()
    for r in (0, 3, 40, 63):
        expect = Wq[r].astype(np.float64) - HP.lr * grad[r] / (np.abs(grad[r]) + HP.eps)
        ulp = np.spacing(np.abs(expect).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(Wn[r] - expect) <= 2 * ulp + 1e-12)
        m_ref = (np.float32(1 - np.float32(0.9)) * grad[r]).astype(np.float16).view(np.uint16)
        assert np.array_equal(st.m[r], m_ref)
        assert st.step[r] == 1


def _dense_adam_reference(W, grads, hp, steps):
    """torch.optim.Adam in fp64 on a dense parameter (library routine)."""
    p = torch.nn.Parameter(torch.from_numpy(W.astype(np.float64)))
    opt = torch.optim.Adam([p], lr=hp.lr, betas=(float(np.float32(hp.beta1)),
                                                  float(np.float32(hp.beta2))), eps=hp.eps)
    for k in range(steps):
        p.grad = torch.from_numpy(grads[k].astype(np.float64))
        opt.step()
    return p.detach().numpy()


def _textbook_adam(W, grads, hp, steps):
    """Dense Adam in fp64, plus a bound on what fp16 storage of m and v can move the result.

    Storing a moment in fp16 perturbs it by at most 2^-11 of itself (normal range). A perturbation
    of m_k decays by beta1 per later step, so at step t |dm_t| <= sum_k beta1^(t-k) 2^-11 |m_k|, and
    likewise for v. The step -lr * m_hat / (sqrt(v_hat) + eps) then moves by at most
    lr * (bc1 |dm_t| / sqrt(v_hat) + |m_hat| bc2 |dv_t| / (2 v_hat^1.5)) to first order.
    """
    W = W.astype(np.float64).copy()
    m = np.zeros_like(W)
    v = np.zeros_like(W)
    b1, b2 = float(np.float32(hp.beta1)), float(np.float32(hp.beta2))
    dm = np.zeros_like(W)
    dv = np.zeros_like(W)
    bound = np.zeros_like(W)
    u16 = 2.0 ** -11
    for t in range(1, steps + 1):
        gk = grads[t - 1].astype(np.float64)
        m = b1 * m + (1 - b1) * gk
        v = b2 * v + (1 - b2) * gk * gk
        bc1, bc2 = 1 / (1 - b1 ** t), 1 / (1 - b2 ** t)
        mh, vh = m * bc1, v * bc2
        with np.errstate(divide="ignore", invalid="ignore"):
            e = hp.lr * (bc1 * dm / np.sqrt(vh) + np.abs(mh) * bc2 * dv / (2 * vh ** 1.5))
        bound += np.nan_to_num(e)
        W -= hp.lr * mh / (np.sqrt(vh) + hp.eps)
        dm = b1 * dm + b1 * u16 * np.abs(m)         # rounding of this step's stored m, decayed
        dv = b2 * dv + b2 * u16 * np.abs(v)
    return W, bound


def test_sparse_update_matches_dense_adam_on_active_rows_and_leaves_others():
    # With a fixed mask and zero gradient outside it, sparse Adam equals dense Adam on the
    # support (the coordinate-sparse Adam identity of the SparseLeaf page, section 4); inactive
    # rows must not move at all (Sparse-First section 2.3: inactive rows return immediately).
    g = np.random.default_rng(13)
    R, C, steps = 96, 40, 3
    W0 = synth.weights_f32(g, R, C)
    active = [1, 2, 33, 64, 95]
    st = orc.MatrixState(W0)
    st.set_mask(synth.words_from_rows(R, active))
    Wq = st.weight()
    before = {k: getattr(st, k).copy() for k in ("q", "s", "delta", "m", "v", "step", "live")}
    grads = []
    for k in range(steps):
        gr = np.zeros((R, C), np.float32)
        gr[active] = _grad(g, len(active), C)
        grads.append(gr)
        orc.update(st, gr, HP)
    got = st.weight().astype(np.float64)
    ref_torch = _dense_adam_reference(Wq, grads, HP, steps)
    ref_book, bound = _textbook_adam(Wq, grads, HP, steps)
    np.testing.assert_allclose(ref_torch, ref_book, rtol=0, atol=1e-15)
    err = np.abs(got - ref_torch)[active]
    # fp16-moment bound (first order, 10% slack) plus one fp32 rounding of W per step
    ulp = np.spacing(np.abs(ref_torch[active]).astype(np.float32)).astype(np.float64)
    assert np.all(err <= 1.1 * bound[active] + steps * ulp)
    assert bound[active].max() < 1e-2 * HP.lr   # tight enough that a wrong step (~lr) fails
    inactive = [r for r in range(R) if r not in active]
    for k, arr in before.items():
        cur = getattr(st, k)
        if cur.ndim == 1:
            assert np.array_equal(cur[inactive], arr[inactive]), k
        else:
            assert cur[inactive].tobytes() == arr[inactive].tobytes(), k
    # write-back: live = bf16(W'), W' = s'q' + delta'
    assert np.array_equal(st.live[active], synth.f32_to_bf16_bits(st.weight()[active]))
    assert np.abs(st.q.astype(int)).max() <= 127
    assert all(np.abs(st.q[r].astype(int)).max() == 127 for r in active)


def test_pair_partner_gradient_enters_with_its_coefficient_and_sign():
    # g_a = 0 on the row, g_b nonzero, c_partner = 0.6 (gate-up strength): the first step of a
    # is -lr * (0.6 g_b) / (|0.6 g_b| + eps) -- a dropped or sign-flipped partner term fails.
    g = np.random.default_rng(14)
    R, C = 32, 16
    a = orc.MatrixState(synth.weights_f32(g, R, C))
    b = orc.MatrixState(synth.weights_f32(g, R, C))
    a.set_mask(synth.words_from_rows(R, [4]))
    b.set_mask(synth.words_from_rows(R, [4, 9]))
    Wa = a.weight()
    ga = np.zeros((R, C), np.float32)
    gb = _grad(g, R, C)
    orc.update(a, ga, HP, partner=b, pg=gb, c_self=1.0, c_partner=0.6)
    mix = np.float32(0.6) * gb[4]
    expect = Wa[4].astype(np.float64) - HP.lr * mix / (np.abs(mix) + HP.eps)
    assert np.all(np.abs(a.weight()[4] - expect) <= 2 * np.spacing(np.abs(expect).astype(np.float32)))


def test_pair_partner_row_inactive_contributes_nothing():
    g = np.random.default_rng(15)
    R, C = 32, 16
    W = synth.weights_f32(g, R, C)
    a1, a2 = orc.MatrixState(W), orc.MatrixState(W)
    b = orc.MatrixState(synth.weights_f32(g, R, C))
    for st in (a1, a2):
        st.set_mask(synth.words_from_rows(R, [4]))
    b.set_mask(synth.words_from_rows(R, [5]))          # partner's row 4 is inactive
    ga, gb = _grad(g, R, C), _grad(g, R, C)
    orc.update(a1, ga, HP, partner=b, pg=gb, c_self=1.0, c_partner=0.4)
    orc.update(a2, ga, HP)
    assert a1.q.tobytes() == a2.q.tobytes() and a1.delta.tobytes() == a2.delta.tobytes()


def test_pair_update_is_symmetric_under_swap():
    g = np.random.default_rng(16)
    R, C = 64, 24
    Wa, Wb = synth.weights_f32(g, R, C), synth.weights_f32(g, R, C)
    ma, mb = synth.words_from_rows(R, [1, 2, 40]), synth.words_from_rows(R, [2, 40, 41])
    ga, gb = _grad(g, R, C), _grad(g, R, C)
    c = dict(caa=1.0, cab=0.4 * np.cos(np.radians(36)), cba=-0.25, cbb=0.9)

    def run(W1, W2, m1, m2, g1, g2, c11, c12, c21, c22):
        s1, s2 = orc.MatrixState(W1), orc.MatrixState(W2)
        s1.set_mask(m1)
        s2.set_mask(m2)
        orc.update(s1, g1, HP, partner=s2, pg=g2, c_self=c11, c_partner=c12)
        orc.update(s2, g2, HP, partner=s1, pg=g1, c_self=c22, c_partner=c21)
        return s1, s2

    a, b = run(Wa, Wb, ma, mb, ga, gb, c["caa"], c["cab"], c["cba"], c["cbb"])
    b2, a2 = run(Wb, Wa, mb, ma, gb, ga, c["cbb"], c["cba"], c["cab"], c["caa"])
    for x, y in ((a, a2), (b, b2)):
        for k in ("q", "s", "delta", "m", "v", "live", "step"):
            assert getattr(x, k).tobytes() == getattr(y, k).tobytes(), k


def test_weight_decay_closed_form_with_zero_gradient():
    # Zero gradient: u = 0 / (0 + eps) = 0, so W' = W - lr*wd*W (decoupled decay, section 2.4).
    g = np.random.default_rng(17)
    R, C = 32, 20
    st = orc.MatrixState(synth.weights_f32(g, R, C))
    st.set_mask(synth.words_from_rows(R, [7]))
    W = st.weight()
    hp = orc.AdamHP(lr=1e-2, wd=0.5 * np.cos(np.radians(28.4)))
    orc.update(st, np.zeros((R, C), np.float32), hp)
    expect = W[7].astype(np.float64) * (1 - hp.lr * np.float32(hp.wd))
    assert np.all(np.abs(st.weight()[7] - expect) <= 2 * np.spacing(np.abs(expect).astype(np.float32)))


def test_element_clip_bounds_the_gradient():
    g = np.random.default_rng(18)
    R, C = 32, 8
    W = synth.weights_f32(g, R, C)
    a, b = orc.MatrixState(W), orc.MatrixState(W)
    for st in (a, b):
        st.set_mask(synth.words_from_rows(R, [0]))
    big = np.full((R, C), 10.0, np.float32)
    big[0, ::2] = -10.0
    one = np.clip(big, -1, 1).astype(np.float32)
    orc.update(a, big, orc.AdamHP(clip=1.0))
    orc.update(b, one, orc.AdamHP())
    assert a.m.tobytes() == b.m.tobytes() and a.q.tobytes() == b.q.tobytes()


def test_reactivated_row_restarts_from_zero_moments():
    g = np.random.default_rng(19)
    R, C = 32, 16
    st = orc.MatrixState(synth.weights_f32(g, R, C))
    on, off = synth.words_from_rows(R, [3]), synth.words_from_rows(R, [])
    st.set_mask(on)
    orc.update(st, _grad(g, R, C), HP)
    orc.update(st, _grad(g, R, C), HP)
    assert st.step[3] == 2
    st.set_mask(off)
    st.set_mask(on)
    assert st.step[3] == 0 and not st.m[3].any()
    W = st.weight()
    gr = _grad(g, R, C)
    orc.update(st, gr, HP)
    expect = W[3].astype(np.float64) - HP.lr * gr[3] / (np.abs(gr[3]) + HP.eps)
    assert np.all(np.abs(st.weight()[3] - expect) <= 2 * np.spacing(np.abs(expect).astype(np.float32)))


# =============================================================================================
# Section 2.6: checkpoint and rewind of the active rows
# =============================================================================================

def test_checkpoint_round_trip_restores_saved_rows_only():
    # Save after two steps; train on with a changed mask (a saved row turns inactive, a new row
    # turns active); restore. Saved rows get back exactly their saved storage, their live row is
    # bf16 of the restored weight, moments come back only where the row is active now; rows not
    # in the checkpoint keep whatever they had.
    g = np.random.default_rng(21)
    R, C = 64, 48
    st = orc.MatrixState(synth.weights_f32(g, R, C))
    st.set_mask(synth.words_from_rows(R, [2, 9, 40, 41]))
    for _ in range(2):
        orc.update(st, _grad(g, R, C), HP)
    saved = {k: getattr(st, k).copy() for k in ("q", "s", "delta", "m", "v", "step")}
    ck = orc.Checkpoint(st)
    assert ck.n == 4 and list(ck.rows[:4]) == [2, 9, 40, 41]
    st.set_mask(synth.words_from_rows(R, [2, 9, 41, 50]))          # row 40 out, row 50 in
    for _ in range(3):
        orc.update(st, _grad(g, R, C), HP)
    before = {k: getattr(st, k).copy() for k in ("q", "s", "delta", "m", "v", "step", "live")}
    ck.restore(st)
    for r in (2, 9, 40, 41):
        assert st.q[r].tobytes() == saved["q"][r].tobytes()
        assert st.s[r] == saved["s"][r] and st.delta[r].tobytes() == saved["delta"][r].tobytes()
        expect_live = synth.f32_to_bf16_bits(orc.rebuild(saved["q"][r:r + 1], saved["s"][r:r + 1],
                                                         saved["delta"][r:r + 1]))[0]
        assert np.array_equal(st.live[r], expect_live)
    for r in (2, 9, 41):                                              # still active: moments back
        assert st.m[r].tobytes() == saved["m"][r].tobytes() and st.step[r] == saved["step"][r]
    assert not st.m[40].any() and st.step[40] == 0                    # inactive now: stay dropped
    for k in ("q", "s", "delta", "m", "v", "step", "live"):           # row 50 was not saved
        assert getattr(st, k)[50].tobytes() == before[k][50].tobytes()


def test_checkpoint_capacity_keeps_the_first_rows():
    g = np.random.default_rng(22)
    R, C = 64, 16
    st = orc.MatrixState(synth.weights_f32(g, R, C))
    st.set_mask(synth.words_from_rows(R, [1, 5, 33, 60]))
    ck = orc.Checkpoint(st, cap=2)
    assert ck.n == 2 and list(ck.rows[:2]) == [1, 5]
