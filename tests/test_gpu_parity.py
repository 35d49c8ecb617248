"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bars: masks, lists, counts and every untouched byte bit-exact; dW and embedding gradients within
2e-3 of the fp64 oracle (relative, floored at 1e-3 of the matrix's largest entry); the update
bit-exact (same fp32 operation order on both sides, 1e-6 relative allowed on W and delta, q exact
away from rounding ties). Sections refer to "Sparse-First Fine-Tuning" (tensorwirelabs.com).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from tests.gpu_helpers import (DEV, bf16_dev, check_slot_invariants, f32_dev, host, i32_dev,
                               mask_host, rel_err, u32_dev)

pytestmark = pytest.mark.gpu

DW_TOL = 2e-3
CANARY = np.uint32(0x7FBADBAD)          # a NaN pattern no kernel produces


def _canary(shape):
    return torch.from_numpy(np.full(shape, CANARY, dtype=np.uint32).view(np.int32)).to(DEV).view(torch.float32)


# =============================================================================================
# section 2.1: masks
# =============================================================================================

@pytest.mark.parametrize("V,cap", [(1024, 256), (131072, 256)])
def test_conductor_matches_oracle_window_by_window(sf, V, cap):
    # 131,072 rows: the finalize's shared-memory copy of the mask (3 words per 32 rows, 48 KB)
    # needs the opt-in beyond 48 KB
    mk = sf.Mask(V, cap, DEV)
    sf.sf_mask_init(mk)
    status = sf.status_word()
    charge = np.zeros(V, np.float32)
    g = synth.rng(0, "tokens")
    for w in range(10):
        tok = synth.zipf_ids(g, 64, V)
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(tok), n=len(tok))], 0.01, status)
        words, _ = orc.window_tokens(charge, tok)
        rows, tiles = orc.mask_lists(words)
        mh = mask_host(mk)
        assert mh["charge"].tobytes() == charge.tobytes(), f"window {w}"
        assert np.array_equal(mh["words"], words)
        assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles)
        check_slot_invariants(mh, cap)
    assert host(status)[0] == 0
    # the accumulator is left zero for the next window
    assert not host(mk.accum).any()


def test_conductor_empty_window_bad_ids_and_overflow(sf):
    V, cap = 64, 2
    mk = sf.Mask(V, cap, DEV)
    sf.sf_mask_init(mk)
    status = sf.status_word()
    charge = np.zeros(V, np.float32)
    tok = np.array([3, 3, 5, 7, 70, -1], np.int32)        # two ids out of range, 3 rows active
    sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(tok), n=len(tok))], 0.01, status)
    words, bad = orc.window_tokens(charge, tok)
    mh = mask_host(mk)
    assert bad == 2 and np.array_equal(mh["words"], words)
    st = int(host(status)[0])
    assert st & sf.SF_STATUS_BAD_TOKEN and st & sf.SF_STATUS_SLOT_OVERFLOW
    assert mh["counts"][3] == 1                           # 3 active rows, 2 slots
    check_slot_invariants(mh, cap)
    for _ in range(3):                                    # empty windows: pure decay
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, None, n=0)], 0.01, status)
        orc.window_tokens(charge, [])
        assert mask_host(mk)["charge"].tobytes() == charge.tobytes()


@pytest.mark.parametrize("T,R", [(300, 1024), (1, 64), (2048, 4096)])
def test_tracker_matches_oracle(sf, T, R):
    cap = R // 4
    mk = sf.Mask(R, cap, DEV)
    sf.sf_mask_init(mk)
    status = sf.status_word()
    charge = np.zeros(R, np.float32)
    for w in range(3):
        g = synth.rng(2, "tracker", w, R)
        rows = synth.scattered_rows(g, R, 0.01 + 0.02 * w)
        Y = synth.tracker_outputs(g, T, synth.tracker_gains(R, rows))
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_OUTPUT_BF16, bf16_dev(Y), n=T, ld=R)], 0.01, status)
        words = orc.window_outputs(charge, Y)
        mh = mask_host(mk)
        assert mh["charge"].tobytes() == charge.tobytes()
        assert np.array_equal(mh["words"], words)
        r_, t_ = orc.mask_lists(words)
        assert np.array_equal(mh["rows"], r_) and np.array_equal(mh["tiles"], t_)
        check_slot_invariants(mh, cap)
    assert host(status)[0] == 0


def test_tracker_non_finite_outputs_match_oracle(sf):
    """NaN and infinities planted on the host into Y: a NaN carries no magnitude, an infinity
    counts as the largest finite bf16 magnitude. Charges, words and lists stay bit-exact with the
    oracle window after window, and SF_STATUS_NONFINITE is set exactly for the windows that held
    a non-finite output."""
    R, T, cap = 4096, 1000, 512
    mk = sf.Mask(R, cap, DEV)
    sf.sf_mask_init(mk)
    charge = np.zeros(R, np.float32)
    nan_patterns = np.array([0x7FC0, 0xFFC0, 0x7F81, 0xFFFF, 0x7FFF], np.uint16)
    for w, plant in enumerate(["inf+nan", "finite", "nan", "inf+nan"]):
        g = synth.rng(2, "misc", 31, w)
        rows = synth.scattered_rows(g, R, 0.01)
        Y = synth.tracker_outputs(g, T, synth.tracker_gains(R, rows))
        if "nan" in plant:
            ts, rs = g.integers(0, T, 300), g.integers(0, R, 300)
            Y[ts, rs] = nan_patterns[g.integers(0, len(nan_patterns), 300)]
            Y[:, 77] = 0x7FC0                                  # a row with no magnitude at all
            Y[: T // 2, rows[0]] = 0xFFC0                      # NaN over half of an active row
        if "inf" in plant:
            Y[g.integers(0, T, 5), g.integers(0, R, 5)] = 0x7F80
            Y[T - 1, 4095] = 0xFF80                            # last token, last column
            Y[0, 8] = 0x7F80                                   # first token
        status = sf.status_word()
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_OUTPUT_BF16, bf16_dev(Y), n=T, ld=R)], 0.01, status)
        words, n_bad = orc.window_outputs_counted(charge, Y)
        mh = mask_host(mk)
        assert np.all(np.isfinite(mh["charge"]))
        assert mh["charge"].tobytes() == charge.tobytes(), plant
        assert np.array_equal(mh["words"], words), plant
        r_, t_ = orc.mask_lists(words)
        assert np.array_equal(mh["rows"], r_) and np.array_equal(mh["tiles"], t_)
        check_slot_invariants(mh, cap)
        assert (int(host(status)[0]) & sf.SF_STATUS_NONFINITE != 0) == (n_bad > 0), plant
        assert (n_bad > 0) == (plant != "finite")


@pytest.mark.parametrize("specs", [
    [(1024, "tokens"), (4096, "output"), (256, "words"), (512, "hits"), (11008, "output")],
    # a mask of 16,384 rows or more sends the whole batch through the three-launch finalize;
    # the hit counts start 4 bytes past a 16-byte boundary
    [(1024, "tokens"), (4096, "output"), (256, "words"), (32768, "hits+4"), (11008, "output"),
     (16384, "tokens")],
])
def test_many_masks_in_one_call_and_explicit_sources(sf, specs):
    # several masks of different kinds and sizes in one call, each independent
    masks, srcs, keep, ref = [], [], [], []
    for i, (R, kind) in enumerate(specs):
        mk = sf.Mask(R, R // 2, DEV)
        sf.sf_mask_init(mk)
        g = synth.rng(7, "misc", i)
        charge = np.zeros(R, np.float32)
        if kind == "tokens":
            tok = synth.zipf_ids(g, 500, R)
            t = i32_dev(tok)
            srcs.append(sf.make_src(sf.SF_SRC_TOKENS, t, n=len(tok)))
            words, _ = orc.window_tokens(charge, tok)
        elif kind == "output":
            Y = synth.tracker_outputs(g, 77, synth.tracker_gains(R, synth.scattered_rows(g, R, 0.01)))
            t = bf16_dev(Y)
            srcs.append(sf.make_src(sf.SF_SRC_OUTPUT_BF16, t, n=77, ld=R))
            words = orc.window_outputs(charge, Y)
        elif kind == "words":
            words = synth.tiny_projection_mask(0, R)
            t = u32_dev(words)
            srcs.append(sf.make_src(sf.SF_SRC_WORDS, t))
        else:
            tok = synth.zipf_ids(g, 300, R)
            hits = np.bincount(tok, minlength=R).astype(np.uint32)
            if kind == "hits+4":
                t = u32_dev(np.concatenate([np.zeros(1, np.uint32), hits]))[1:]
                assert t.data_ptr() % 16 == 4
            else:
                t = u32_dev(hits)
            srcs.append(sf.make_src(sf.SF_SRC_HITS_U32, t))
            words, _ = orc.window_tokens(charge, tok)      # same counts, folded by the oracle
        keep.append(t)
        masks.append(mk)
        ref.append((charge, words))
    sf.sf_mask_update(masks, srcs, 0.01)
    for mk, (charge, words), (R, kind) in zip(masks, ref, specs):
        mh = mask_host(mk)
        assert np.array_equal(mh["words"], words), kind
        if kind != "words":
            assert mh["charge"].tobytes() == charge.tobytes(), kind
        else:
            assert not mh["charge"].any()
        check_slot_invariants(mh, R // 2)


def test_slot_lifecycle_release_and_reuse(sf):
    R, cap = 128, 8
    mk = sf.Mask(R, cap, DEV)
    sf.sf_mask_init(mk)
    seq = [[0, 1, 2, 40], [1, 2, 3, 99, 100], [], [5, 6, 7, 8, 9, 10, 11, 12, 13], [5]]
    prev = set()
    for rows in seq:
        w = synth.words_from_rows(R, rows)
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(w))], 0.01)
        mh = mask_host(mk)
        assert list(mh["rows"]) == sorted(rows)
        check_slot_invariants(mh, cap)
        for r in set(rows) - prev:                # fresh rows start with zero Adam steps
            if mh["row_slot"][r] >= 0:
                assert mh["slot_step"][mh["row_slot"][r]] == 0
        prev = set(rows)


# =============================================================================================
# section 2.2: masked weight gradient
# =============================================================================================

def _dw_case(sf, T, R, C, active_rows, seed):
    g = synth.rng(seed, "dx", T, R, C)
    dX = synth.normal_bf16(g, (T, R))
    A = synth.normal_bf16(synth.rng(seed, "act", T, R, C), (T, C))
    words = synth.words_from_rows(R, active_rows)
    cap = min(R, max(len(active_rows), 1) + 5)
    mk = sf.Mask(R, cap, DEV)
    sf.sf_mask_init(mk)
    sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(words))], 0.01)
    dW = _canary((cap, C))
    dXd, Ad = bf16_dev(dX), bf16_dev(A)
    return dict(dX=dX, A=A, words=words, mask=mk, dW=dW, dXd=dXd, Ad=Ad, cap=cap, C=C)


def _check_dw(case, ref=None):
    if ref is None:
        ref = orc.masked_dw(case["dX"], case["A"], case["words"])
    mh = mask_host(case["mask"])
    got = host(case["dW"])
    used = set()
    for r in mh["rows"]:
        s = mh["row_slot"][r]
        assert s >= 0
        used.add(s)
        err = rel_err(got[s], ref[r], 1e-3) if np.abs(ref[r]).max() > 0 else np.abs(got[s]).max()
        assert err <= DW_TOL, (r, err)
    for s in range(case["cap"]):
        if s not in used:
            assert got[s].view(np.uint32).tolist() == [int(CANARY)] * case["C"], f"slot {s} written"


def _run_dw(sf, problems, mode, status=None):
    ws = sf.dw_workspace(problems) if mode == "rows" else None
    sf.sf_masked_dw(problems, status, ws=ws)


@pytest.mark.parametrize("mode", ["tiles", "rows"])
def test_masked_dw_tiny_projection(sf, mode):
    # W 256 x 512, T = 128: tile 0 full, tiles 3..7 empty, Bernoulli(0.03) rows elsewhere
    words = synth.tiny_projection_mask(0, 256)
    case = _dw_case(sf, 128, 256, 512, synth.rows_from_words(words), 0)
    status = sf.status_word()
    _run_dw(sf, [sf.dw_problem(case["dXd"], case["Ad"], case["mask"], case["dW"])], mode, status)
    _check_dw(case)
    assert host(status)[0] == 0


@pytest.mark.parametrize("mode", ["tiles", "rows"])
def test_masked_dw_ragged_grouped_and_degenerate(sf, mode):
    # one launch: ragged T (not a multiple of 64), ragged C (last N-tile 8 wide), a ragged last
    # M-tile (7 active tiles), a full matrix, an all-empty mask and a zero-token problem
    g = synth.rng(3, "rows")
    cases = [
        _dw_case(sf, 100, 384, 520, np.sort(g.choice(384, 40, replace=False)), 1),
        _dw_case(sf, 200, 96, 64, np.arange(96), 2),
        _dw_case(sf, 64, 256, 256, [], 3),
        _dw_case(sf, 0, 64, 256, [1, 2, 63], 4),
        _dw_case(sf, 333, 224, 1032, [0, 31, 32, 95, 96, 223], 5),
    ]
    status = sf.status_word()
    _run_dw(sf, [sf.dw_problem(c["dXd"], c["Ad"], c["mask"], c["dW"]) for c in cases], mode, status)
    for c in cases:
        _check_dw(c)
    assert host(status)[0] == 0


@pytest.mark.parametrize("mode", ["tiles", "rows"])
def test_masked_dw_every_tile_position(sf, mode):
    # each of 40 tiles active with one row, in turn spread over M-tiles: catches slot/lane mixups
    R, C, T = 1280, 256, 96
    rows = np.array([32 * w + (w * 7) % 32 for w in range(R // 32)])
    case = _dw_case(sf, T, R, C, rows, 6)
    _run_dw(sf, [sf.dw_problem(case["dXd"], case["Ad"], case["mask"], case["dW"])], mode)
    _check_dw(case)


@pytest.mark.parametrize("mode", ["tiles", "rows"])
def test_masked_dw_deterministic(sf, mode):
    words = synth.tiny_projection_mask(0, 256)
    case = _dw_case(sf, 1000, 256, 512, synth.rows_from_words(words), 8)
    p = [sf.dw_problem(case["dXd"], case["Ad"], case["mask"], case["dW"])]
    _run_dw(sf, p, mode)
    a = host(case["dW"]).copy()
    _run_dw(sf, p, mode)
    assert a.tobytes() == host(case["dW"]).tobytes()


@pytest.mark.parametrize("T,R,C,kind", [
    (4096, 256, 512, "scattered"),    # 2 units of 64 token stages (four accumulation chunks each)
    (130, 1280, 256, "scattered"),    # 3 stages per unit, ragged T
    (1000, 4096, 2048, "clustered"),  # ~80 units of 16 stages in tile mode
    (2048, 11008, 4096, "scattered"),  # 7B gate-like shape at 1%: row mode
])
def test_masked_dw_workspace_calls_are_repeatable(sf, T, R, C, kind):
    # The call with a workspace (the device picks row or tile mode) against the oracle, byte-equal
    # over two calls whatever the scratch held before, and close to the mask-tile launch without
    # a workspace (the same sums).
    g = synth.rng(31, "rows", T, R)
    rows = synth.scattered_rows(g, R, 0.01 if R > 4096 else 0.15) if kind == "scattered" \
        else synth.clustered_rows(g, R, 0.3)
    case = _dw_case(sf, T, R, C, rows, 31)
    p = [sf.dw_problem(case["dXd"], case["Ad"], case["mask"], case["dW"])]
    status = sf.status_word()
    ws = sf.dw_workspace(p)
    sf.sf_masked_dw(p, status, ws=ws)
    _check_dw(case)
    a = host(case["dW"]).copy()
    ws.fill_(0x5A)                          # stale scratch contents do not matter
    sf.sf_masked_dw(p, status, ws=ws)
    assert a.tobytes() == host(case["dW"]).tobytes()
    sf.sf_masked_dw(p, status)              # whole units (mask-tile mode)
    mh = mask_host(case["mask"])
    b = host(case["dW"])
    for r in mh["rows"]:
        s_ = mh["row_slot"][r]
        assert rel_err(a[s_], b[s_], 1e-2) <= 1e-4, r    # the same sums in another order
    assert host(status)[0] == 0


def test_masked_dw_groups_share_inputs_and_pick_their_mode(sf):
    # q/k/v-like problems reading one A (a group: their scattered rows share 128-row tiles), a
    # gate/up-like pair with whole active tiles (2 M-tiles either way, so tile mode is kept), and
    # a problem whose active rows exceed its slots (row mode impossible -> tile mode).
    T, C = 300, 520
    A_bits = synth.normal_bf16(synth.rng(30, "act"), (T, C))
    A = bf16_dev(A_bits)
    cases, probs = [], []
    g = synth.rng(30, "rows")
    specs = [(512, np.sort(g.choice(512, 9, replace=False)), None, A_bits),
             (512, np.sort(g.choice(512, 70, replace=False)), None, A_bits),
             (1024, np.sort(g.choice(1024, 100, replace=False)), None, A_bits),
             (256, np.arange(64, 128), None, None),
             (256, np.arange(0, 128), None, "same"),
             (384, np.sort(g.choice(384, 60, replace=False)), 20, None)]
    shared2 = None
    for i, (R, rows, cap, a_src) in enumerate(specs):
        dX = synth.normal_bf16(synth.rng(30, "dx", i), (T, R))
        if a_src is None:
            a_bits = synth.normal_bf16(synth.rng(30, "act", i), (T, C))
            a_dev = bf16_dev(a_bits)
            shared2 = (a_bits, a_dev)
        elif isinstance(a_src, str):
            a_bits, a_dev = shared2
        else:
            a_bits, a_dev = A_bits, A
        words = synth.words_from_rows(R, rows)
        slot_cap = cap if cap is not None else min(R, len(rows) + 3)
        mk = sf.Mask(R, slot_cap, DEV)
        sf.sf_mask_init(mk)
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(words))], 0.01)
        dW = _canary((slot_cap, C))
        case = dict(dX=dX, A=a_bits, words=words, mask=mk, dW=dW, cap=slot_cap, C=C)
        cases.append(case)
        probs.append(sf.dw_problem(bf16_dev(dX), a_dev, mk, dW))
    status = sf.status_word()
    _run_dw(sf, probs, "rows", status)
    for c in cases:
        ref = orc.masked_dw(c["dX"], c["A"], c["words"])
        mh = mask_host(c["mask"])
        got = host(c["dW"])
        for r in mh["rows"]:
            s = mh["row_slot"][r]
            if s < 0:
                continue                       # no slot: no gradient is kept for this row
            assert rel_err(got[s], ref[r], 1e-3) <= DW_TOL, r
    assert host(status)[0] == 0


# =============================================================================================
# sections 1 / 2.2: embedding-row gradient
# =============================================================================================

@pytest.mark.parametrize("V,H,n", [(1024, 264, 700), (32000, 512, 4096)])
def test_embed_grad_matches_oracle(sf, V, H, n):
    g = synth.rng(1, "tokens", V)
    tok = synth.zipf_ids(g, n, V)
    dY = synth.normal_bf16(synth.rng(1, "dy", V), (n, H))
    cap = min(V, 2048)
    mk = sf.Mask(V, cap, DEV)
    sf.sf_mask_init(mk)
    charge = np.zeros(V, np.float32)
    for w in range(3):                       # prior windows, then the batch itself
        prior = synth.zipf_ids(synth.rng(1, "tokens", V, w), n, V)
        sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(prior), n=n)], 0.01)
        orc.window_tokens(charge, prior)
    sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(tok), n=n)], 0.01)
    words, _ = orc.window_tokens(charge, tok)
    mh = mask_host(mk)
    assert np.array_equal(mh["words"], words)
    G = _canary((cap, H))
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(n, cap) // 4, dtype=torch.int32, device=DEV)
    status = sf.status_word()
    sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G, ws, status)
    ref = orc.embed_grad(tok, dY, V, words)
    got = host(G)
    used = set()
    scale = max(np.abs(ref[mh["rows"]]).max(), 1.0)
    for r in mh["rows"]:
        s = mh["row_slot"][r]
        used.add(s)
        err = np.abs(got[s].astype(np.float64) - ref[r]) / np.maximum(np.abs(ref[r]), 1e-3 * scale)
        assert err.max() <= DW_TOL, r
    for s in range(cap):
        if s not in used:
            assert (got[s].view(np.uint32) == CANARY).all()
    assert host(status)[0] == 0
    # deterministic
    G2 = _canary((cap, H))
    sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G2, ws)
    assert host(G2).tobytes() == got.tobytes()


def test_embed_grad_same_bytes_in_every_index_layout(sf):
    """The index pass keeps each token's slot in shared memory beside the counts when both fit
    and looks the slots up again otherwise; at 16,384 tokens, slot capacities of 4,096 and 32,000
    keep them and 49,152 does not. Each row's positions are sorted before the sum, so its
    gradient has the same bytes at every capacity (slot numbers may differ), and matches the
    oracle."""
    V, H, n = 49152, 64, 16384
    tok = synth.zipf_ids(synth.rng(3, "tokens", V), n, V)
    dY = synth.normal_bf16(synth.rng(3, "dy", V), (n, H))
    priors = [synth.zipf_ids(synth.rng(3, "tokens", V, w), n, V) for w in range(3)]
    charge = np.zeros(V, np.float32)
    for prior in priors:
        orc.window_tokens(charge, prior)
    words, _ = orc.window_tokens(charge, tok)
    ref = orc.embed_grad(tok, dY, V, words)
    by_cap = {}
    for cap in (4096, 32000, 49152):
        mk = sf.Mask(V, cap, DEV)
        sf.sf_mask_init(mk)
        for prior in priors + [tok]:
            sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_TOKENS, i32_dev(prior), n=n)], 0.01)
        mh = mask_host(mk)
        assert np.array_equal(mh["words"], words)
        G = _canary((cap, H))
        ws = torch.zeros(sf.sf_embed_grad_ws_bytes(n, cap) // 4, dtype=torch.int32, device=DEV)
        status = sf.status_word()
        sf.sf_embed_grad(i32_dev(tok), bf16_dev(dY), mk, G, ws, status)
        got = host(G)
        assert host(status)[0] == 0
        rows = mh["rows"]
        assert 0 < len(rows) <= 4096
        by_cap[cap] = {int(r): got[mh["row_slot"][r]].tobytes() for r in rows}
        scale = max(np.abs(ref[rows]).max(), 1.0)
        for r in rows:
            e = np.abs(got[mh["row_slot"][r]].astype(np.float64) - ref[r]) / np.maximum(np.abs(ref[r]), 1e-3 * scale)
            assert e.max() <= DW_TOL, (cap, r)
    assert by_cap[4096] == by_cap[32000] == by_cap[49152]


# =============================================================================================
# sections 2.3 / 2.4: the fused sparse update
# =============================================================================================

def _state_from_oracle(sf, st: orc.MatrixState, cap: int) -> "sf.Matrix":
    mat = sf.Matrix(st.R, st.C, cap, DEV)
    mat.q.copy_(torch.from_numpy(st.q).to(DEV))
    mat.s.copy_(f32_dev(st.s))
    mat.delta.copy_(f32_dev(st.delta))
    sf.sf_mask_init(mat.mask)
    return mat


def _compare_matrix(mat, st: orc.MatrixState, exact=True):
    q, s, d = host(mat.q), host(mat.s), host(mat.delta)
    mh = mask_host(mat.mask)
    if exact:
        assert q.tobytes() == st.q.tobytes()
        assert s.tobytes() == st.s.tobytes()
        assert d.tobytes() == st.delta.tobytes()
    live = host(mat.live).view(np.uint16)
    rows = synth.rows_from_words(st.words)
    assert np.array_equal(live[rows], st.live[rows])
    m, v, step = host(mat.m).view(np.uint16), host(mat.v).view(np.uint16), mh["slot_step"]
    for r in rows:
        sl = mh["row_slot"][r]
        assert sl >= 0
        assert np.array_equal(m[sl], st.m[r]) and np.array_equal(v[sl], st.v[r]), r
        assert step[sl] == st.step[r]


def _grad_rows(seed, step, R, C, scale=8.0):
    g = synth.rng(seed, "grad", step, R, C)
    return (g.standard_normal((R, C), dtype=np.float32) * np.float32(scale)).astype(np.float32)


def _load_grad(mat, dense: np.ndarray):
    """Place a dense R x C gradient into the slot-indexed buffer (rows with a slot only)."""
    mh = mask_host(mat.mask)
    buf = np.zeros((mat.grad.shape[0], mat.C), np.float32)
    for r in mh["rows"]:
        if mh["row_slot"][r] >= 0:
            buf[mh["row_slot"][r]] = dense[r]
    mat.grad.copy_(f32_dev(buf))


def _set_words(sf, mats_words):
    sf.sf_mask_update([m.mask for m, _ in mats_words],
                      [sf.make_src(sf.SF_SRC_WORDS, u32_dev(w)) for _, w in mats_words], 0.01)


def test_quantize_init_matches_oracle(sf):
    W = synth.weights_f32(synth.rng(0, "weights"), 256, 512)
    W[3] = 0.0
    st = orc.MatrixState(W)
    mat = sf.Matrix(256, 512, 4, DEV)
    sf.sf_quantize_init(f32_dev(W), mat)
    assert host(mat.q).tobytes() == st.q.tobytes()
    assert host(mat.s).tobytes() == st.s.tobytes()
    assert host(mat.delta).tobytes() == st.delta.tobytes()
    assert np.array_equal(host(mat.live).view(np.uint16), synth.f32_to_bf16_bits(W))


def test_adam_tables_match_oracle(sf):
    hp = sf.AdamParams(t_max=3000)
    bc1, bc2 = host(hp.bc1), host(hp.bc2)
    for t in list(range(1, 50)) + [100, 999, 3000]:
        assert bc1[t] == np.float32(orc.bias_correction(0.9, t))
        assert bc2[t] == np.float32(orc.bias_correction(0.999, t))


def test_update_tiny_projection_three_steps_bit_exact(sf):
    R, C = 256, 512
    W = synth.weights_f32(synth.rng(0, "weights"), R, C)
    words = synth.tiny_projection_mask(0, R)
    st = orc.MatrixState(W)
    st.set_mask(words)
    mat = _state_from_oracle(sf, st, 64)
    _set_words(sf, [(mat, words)])
    hp = sf.AdamParams()
    ohp = orc.AdamHP()
    status = sf.status_word()
    q0, d0 = st.q.copy(), st.delta.copy()
    for step in range(3):
        grad = _grad_rows(0, step, R, C)
        _load_grad(mat, grad)
        sf.sf_sparse_update([sf.matrix_struct(mat)], hp, status)
        orc.update(st, grad, ohp)
        _compare_matrix(mat, st)
    assert host(status)[0] == 0
    inactive = np.setdiff1d(np.arange(R), synth.rows_from_words(words))
    assert host(mat.q)[inactive].tobytes() == q0[inactive].tobytes()
    assert host(mat.delta)[inactive].tobytes() == d0[inactive].tobytes()


def test_update_coupled_pairs_and_changing_masks(sf):
    # gate/up-like pair (b = 0.6) and a second pair (b = 0.4) with a rotating mix, plus an
    # unpaired matrix; masks change between steps so slots are released and reused.
    R, C = 128, 264
    rng = synth.rng(11, "weights")
    Ws = [synth.weights_f32(rng, R, C) for _ in range(5)]
    pairs = {0: 1, 1: 0, 2: 3, 3: 2, 4: -1}
    strength = {0: 0.6, 1: 0.6, 2: 0.4, 3: 0.4, 4: 0.0}
    ohp = orc.AdamHP(lr=1e-3, wd=0.01 * np.cos(np.radians(28.4)), clip=40.0)
    hp = sf.AdamParams(lr=1e-3, wd=0.01 * np.cos(np.radians(28.4)), clip=40.0)
    sts = [orc.MatrixState(W) for W in Ws]
    mats = [_state_from_oracle(sf, s, 48) for s in sts]
    g = synth.rng(11, "rows")
    status = sf.status_word()
    for step in range(4):
        words = [synth.words_from_rows(R, np.sort(g.choice(R, 20 + 5 * i, replace=False))) for i in range(5)]
        if step == 2:
            words[0] = words[1].copy()            # a and b fully overlapping
        for st_, w in zip(sts, words):
            st_.set_mask(w)
        _set_words(sf, list(zip(mats, words)))
        grads = [_grad_rows(11, 10 * step + i, R, C) for i in range(5)]
        for m_, gr in zip(mats, grads):
            _load_grad(m_, gr)
        k = np.radians(36.0 * step)
        structs = []
        coef = []
        for i in range(5):
            c_self = 1.0
            c_partner = float(np.float32(strength[i] * np.cos(k + i)))
            coef.append((c_self, c_partner))
            structs.append(sf.matrix_struct(mats[i], pairs[i], c_self, c_partner))
        sf.sf_sparse_update(structs, hp, status)
        # oracle: every matrix reads the original gradients, order is irrelevant
        for i in range(5):
            p = pairs[i]
            if p >= 0:
                orc.update(sts[i], grads[i], ohp, partner=sts[p], pg=grads[p],
                           c_self=coef[i][0], c_partner=coef[i][1])
            else:
                orc.update(sts[i], grads[i], ohp)
        for m_, s_ in zip(mats, sts):
            _compare_matrix(m_, s_)
    assert host(status)[0] == 0


@pytest.mark.parametrize("C", [11008, 12000])
def test_update_wide_rows_and_overflowed_rows_untouched(sf, C):
    # C = 11008 (the 7B feed-forward width) exercises several chunks per thread; C = 12,000 puts
    # the row's shared-memory copy (48,000 B) plus the kernel's static shared memory just over
    # the 48 KB that needs no opt-in. Slot capacity smaller than the active set: rows without a
    # slot must not change.
    R = 64
    W = synth.weights_f32(synth.rng(5, "weights"), R, C)
    words = synth.words_from_rows(R, [0, 5, 9, 33, 63])
    st = orc.MatrixState(W)
    mat = _state_from_oracle(sf, st, 3)
    _set_words(sf, [(mat, words)])
    mh = mask_host(mat.mask)
    with_slot = [r for r in mh["rows"] if mh["row_slot"][r] >= 0]
    assert len(with_slot) == 3
    st.set_mask(synth.words_from_rows(R, with_slot))
    hp, ohp = sf.AdamParams(), orc.AdamHP()
    status = sf.status_word()
    for step in range(2):
        grad = _grad_rows(5, step, R, C)
        _load_grad(mat, grad)
        sf.sf_sparse_update([sf.matrix_struct(mat)], hp, status)
        orc.update(st, grad, ohp)
        _compare_matrix(mat, st)
    assert int(host(status)[0]) == 0


# =============================================================================================
# one tiny-projection step end to end: mask -> dW -> update, three steps
# =============================================================================================

def test_tiny_projection_chain_three_steps(sf):
    R, C, T, steps = 256, 512, 128, 3
    W = synth.weights_f32(synth.rng(0, "weights"), R, C)
    words = synth.tiny_projection_mask(0, R)
    st = orc.MatrixState(W)
    st.set_mask(words)
    mat = sf.Matrix(R, C, 64, DEV)
    sf.sf_mask_init(mat.mask)
    sf.sf_quantize_init(f32_dev(W), mat)
    _set_words(sf, [(mat, words)])
    hp, ohp = sf.AdamParams(), orc.AdamHP()
    status = sf.status_word()
    q0 = host(mat.q).copy()
    for step in range(steps):
        dX = synth.normal_bf16(synth.rng(0, "dx", step), (T, R))
        A = synth.normal_bf16(synth.rng(0, "act", step), (T, C))
        probs = [sf.dw_problem(bf16_dev(dX), bf16_dev(A), mat.mask, mat.grad)]
        sf.sf_masked_dw(probs, status, ws=sf.dw_workspace(probs))
        sf.sf_sparse_update([sf.matrix_struct(mat)], hp, status)
        orc.update(st, orc.masked_dw(dX, A, words, np.zeros((R, C))).astype(np.float32), ohp)
    assert host(status)[0] == 0
    rows = synth.rows_from_words(words)
    Wg = orc.rebuild(host(mat.q), host(mat.s), host(mat.delta))
    Wo = st.weight()
    # the two dW differ by at most 2e-3 relative; through Adam (|u| <= ~3) that moves each step
    # by at most lr * 4 * 2e-3
    tol = steps * ohp.lr * 4 * DW_TOL
    assert np.abs(Wg[rows] - Wo[rows]).max() <= tol
    inactive = np.setdiff1d(np.arange(R), rows)
    assert host(mat.q)[inactive].tobytes() == q0[inactive].tobytes()


def test_update_flags_nonfinite_gradients_and_fp16_overflow(sf):
    # Faults are planted on the host: a NaN in one active row's gradient, and in another run a
    # gradient large enough that v = (1 - beta2) g^2 exceeds fp16's range. Both raise
    # SF_STATUS_NONFINITE; a clean run does not.
    R, C = 64, 256
    W = synth.weights_f32(synth.rng(9, "weights"), R, C)
    words = synth.words_from_rows(R, [3, 40])
    hp = sf.AdamParams()
    for case in ("clean", "nan", "overflow"):
        st = orc.MatrixState(W)
        mat = _state_from_oracle(sf, st, 8)
        _set_words(sf, [(mat, words)])
        grad = _grad_rows(9, 0, R, C)
        if case == "nan":
            grad[40, 17] = np.nan
        elif case == "overflow":
            grad[3, 5] = 1.0e4
        _load_grad(mat, grad)
        status = sf.status_word()
        sf.sf_sparse_update([sf.matrix_struct(mat)], hp, status)
        flagged = bool(int(host(status)[0]) & sf.SF_STATUS_NONFINITE)
        assert flagged == (case != "clean"), case


# =============================================================================================
# section 2.6: checkpoint and rewind of the active rows
# =============================================================================================

def _compare_checkpoint(ck, oc: "orc.Checkpoint"):
    n = int(host(ck.count)[0])
    assert n == oc.n
    assert np.array_equal(host(ck.rows)[:n], oc.rows[:n])
    assert host(ck.q)[:n].tobytes() == oc.q[:n].tobytes()
    assert host(ck.s)[:n].tobytes() == oc.s[:n].tobytes()
    assert host(ck.delta)[:n].tobytes() == oc.delta[:n].tobytes()
    assert np.array_equal(host(ck.m).view(np.uint16)[:n], oc.m[:n])
    assert np.array_equal(host(ck.v).view(np.uint16)[:n], oc.v[:n])
    assert np.array_equal(host(ck.step)[:n], oc.step[:n])


def test_checkpoint_save_train_restore_matches_oracle(sf):
    # Three matrices (one 11008 wide, one paired couple): two steps, save, two more steps with
    # changed masks (some saved rows drop out, new rows come in), restore, one more step.
    shapes = [(128, 272), (128, 272), (64, 11008)]
    pairs = {0: 1, 1: 0, 2: -1}
    hp, ohp = sf.AdamParams(lr=2e-3), orc.AdamHP(lr=2e-3)
    sts = [orc.MatrixState(synth.weights_f32(synth.rng(31, "weights", i), R, C))
           for i, (R, C) in enumerate(shapes)]
    mats = [_state_from_oracle(sf, s_, R) for s_, (R, _) in zip(sts, shapes)]
    g = synth.rng(31, "rows")
    status = sf.status_word()
    cks = [sf.Checkpoint(R, C, DEV) for R, C in shapes]
    saved_rows = None

    def step(k):
        grads = [_grad_rows(31, 10 * k + i, R, C) for i, (R, C) in enumerate(shapes)]
        for m_, gr in zip(mats, grads):
            _load_grad(m_, gr)
        sf.sf_sparse_update([sf.matrix_struct(mats[i], pairs[i], 1.0, 0.5 if pairs[i] >= 0 else 0.0)
                             for i in range(3)], hp, status)
        for i in range(3):
            p = pairs[i]
            if p >= 0:
                orc.update(sts[i], grads[i], ohp, partner=sts[p], pg=grads[p], c_self=1.0, c_partner=0.5)
            else:
                orc.update(sts[i], grads[i], ohp)

    for k in range(5):
        if k == 2:
            sf.sf_checkpoint_save([sf.matrix_struct(m_) for m_ in mats], cks, status)
            ocks = [orc.Checkpoint(s_) for s_ in sts]
            for ck, oc in zip(cks, ocks):
                _compare_checkpoint(ck, oc)
            saved_rows = [oc.rows[:oc.n].copy() for oc in ocks]
        if k in (0, 3):
            words = [synth.words_from_rows(R, np.sort(g.choice(R, R // 4, replace=False)))
                     for R, _ in shapes]
            if k == 3:                                   # keep half of the saved rows active
                for i, (R, _) in enumerate(shapes):
                    keep = saved_rows[i][::2]
                    words[i] = synth.words_from_rows(R, np.union1d(keep, synth.rows_from_words(words[i])))
            for st_, w in zip(sts, words):
                st_.set_mask(w)
            _set_words(sf, list(zip(mats, words)))
        if k == 4:
            sf.sf_checkpoint_restore([sf.matrix_struct(m_) for m_ in mats], cks, status)
            for s_, oc in zip(sts, ocks):
                oc.restore(s_)
            for m_, s_, rows in zip(mats, sts, saved_rows):
                _compare_matrix(m_, s_)
                assert np.array_equal(host(m_.live).view(np.uint16)[rows], s_.live[rows])
        step(k)
        for m_, s_ in zip(mats, sts):
            _compare_matrix(m_, s_)
    assert host(status)[0] == 0


def test_checkpoint_capacity_overflow_and_arguments(sf):
    R, C = 64, 32
    st = orc.MatrixState(synth.weights_f32(synth.rng(32, "weights"), R, C))
    words = synth.words_from_rows(R, [3, 7, 40, 41, 60])
    st.set_mask(words)
    mat = _state_from_oracle(sf, st, R)
    _set_words(sf, [(mat, words)])
    status = sf.status_word()
    ck = sf.Checkpoint(3, C, DEV)
    sf.sf_checkpoint_save([sf.matrix_struct(mat)], [ck], status)
    _compare_checkpoint(ck, orc.Checkpoint(st, cap=3))
    assert int(host(status)[0]) == sf.SF_STATUS_SLOT_OVERFLOW
    # an empty checkpoint restores nothing
    q0 = host(mat.q).copy()
    empty = sf.Checkpoint(0, C, DEV)
    sf.sf_checkpoint_save([sf.matrix_struct(mat)], [empty])
    sf.sf_checkpoint_restore([sf.matrix_struct(mat)], [empty])
    assert host(mat.q).tobytes() == q0.tobytes()
    # C not a multiple of 16
    bad = sf.Matrix(64, 24, 8, DEV)
    sf.sf_mask_init(bad.mask)
    with pytest.raises(RuntimeError):
        sf.sf_checkpoint_save([sf.matrix_struct(bad)], [sf.Checkpoint(4, 24, DEV)])


# =============================================================================================
# failure detection: a bounded wait that runs out (no fault, no hang)
# =============================================================================================

def test_masked_dw_wait_timeout_is_reported_and_the_context_survives(sf, monkeypatch):
    # SF_TEST_DW_WITHHOLD makes CTA 0 of the first launch arm one pipeline stage without issuing
    # its loads. The MMA issuer's wait on that stage gives up after its limit (2 s), the CTA
    # drains its own copies, frees its tensor memory and exits; the call reports
    # SF_STATUS_WAIT_TIMEOUT and the next call on the same context is correct again.
    import time
    R, C, T = 256, 512, 512
    words = synth.tiny_projection_mask(0, R)
    dX = synth.normal_bf16(synth.rng(0, "dx", 9), (T, R))
    A = synth.normal_bf16(synth.rng(0, "act", 9), (T, C))
    mk = sf.Mask(R, R, DEV)
    sf.sf_mask_init(mk)
    sf.sf_mask_update([mk], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(words))], 0.01)
    status = sf.status_word()
    dW = _canary((R, C))
    probs = [sf.dw_problem(bf16_dev(dX), bf16_dev(A), mk, dW)]
    monkeypatch.setenv("SF_TEST_DW_WITHHOLD", "1")
    t0 = time.perf_counter()
    sf.sf_masked_dw(probs, status)            # tile mode (no workspace)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert int(host(status)[0]) & sf.SF_STATUS_WAIT_TIMEOUT
    assert 1.5 < took < 30.0
    monkeypatch.delenv("SF_TEST_DW_WITHHOLD")
    status2 = sf.status_word()
    dW2 = _canary((R, C))
    probs2 = [sf.dw_problem(bf16_dev(dX), bf16_dev(A), mk, dW2)]
    sf.sf_masked_dw(probs2, status2)
    assert int(host(status2)[0]) == 0
    ref = orc.masked_dw(dX, A, words)
    got = host(dW2)
    mh = mask_host(mk)
    for r in mh["rows"]:
        s = mh["row_slot"][r]
        assert rel_err(got[s], ref[r]) <= DW_TOL, r


def test_masked_dw_wait_timeout_with_workspace_leaves_the_next_call_correct(sf, monkeypatch):
    # The same bounded-wait path in a call with a workspace (row mode): after the timeout the
    # next call on the same workspace is correct.
    R, C, T = 1280, 512, 1024
    rows = synth.scattered_rows(synth.rng(32, "rows"), R, 0.2)
    case = _dw_case(sf, T, R, C, rows, 32)
    p = [sf.dw_problem(case["dXd"], case["Ad"], case["mask"], case["dW"])]
    ws = sf.dw_workspace(p)
    status = sf.status_word()
    monkeypatch.setenv("SF_TEST_DW_WITHHOLD", "1")
    sf.sf_masked_dw(p, status, ws=ws)
    torch.cuda.synchronize()
    assert int(host(status)[0]) & sf.SF_STATUS_WAIT_TIMEOUT
    monkeypatch.delenv("SF_TEST_DW_WITHHOLD")
    status2 = sf.status_word()
    case["dW"].view(torch.int32).fill_(int(CANARY))
    sf.sf_masked_dw(p, status2, ws=ws)
    assert int(host(status2)[0]) == 0
    _check_dw(case)
