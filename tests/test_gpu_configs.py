"""Parity of the workloads the benchmark's smaller lines time, at their stated shapes (GPU).

  C1  embedding path: 32,000 x 4,096 int8 + residual table, 8 x 512 Zipf(1.1) token ids (seed 1),
      20 prior conductor windows, then the step: conductor, row gradient of every active row,
      fused update of every active row.
  C2  one 7B-shaped layer (q, k, v, o 4096 x 4096; gate, up 11008 x 4096; down 4096 x 11008) at
      4,096 tokens, ~1% tracker masks, once scattered (every dW group in row mode) and once
      clustered into whole tiles (tile mode), coupled pairs.
  C4  one 11008 x 4096 projection at 4,096 tokens, 5% and 50% scattered rows (row mode gathers
      hundreds to thousands of rows) and 50% clustered tiles (tile mode, 43 x 16 units).

Every stage runs through the same calls the benchmark times (StepPlan / the C ABI). The oracle
recomputes: every mask bit-exactly; dW of every active row (C2) or of rows spread over every
128-row tensor-core tile (C4) within the dW tolerance; the embedding gradient of every active
row; the update bit-exactly, on gradients that come from the oracle or from the seeded
generators (never from the CUDA path), with the weights' quantised state checked first.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from masked_optimizer_step_b200.model import INPUT_OF, STRENGTH, SparseModel, StepPlan
from tests.gpu_helpers import DEV, check_slot_invariants, host, mask_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DW_TOL = 2e-3


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _dw_row_errors(got, ref):
    """Per-row largest relative error |got - ref| / max(|ref|, floor), the floor being 1e-3 of the
    largest |entry| of the projection's checked dW (the dW tolerance's definition)."""
    floor = 1e-3 * max(float(np.abs(ref).max()), 1e-30)
    return np.max(np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref), floor), axis=1)


def _check_dw_rows(mat, mh, dX_bits, A_bits, rows, what):
    ref = orc.masked_dw_rows(dX_bits, A_bits, rows)
    slots = mh["row_slot"][rows]
    assert np.all(slots >= 0), what
    got = host(mat.grad)[slots, : mat.C]
    err = _dw_row_errors(got, ref)
    worst = int(np.argmax(err))
    assert err[worst] <= DW_TOL, (what, int(rows[worst]), float(err[worst]))


def _oracle_rows_state(W_rows):
    """Oracle state holding the given weight rows (rows are independent), padded to 32 rows."""
    n, C = W_rows.shape
    Wt = np.zeros((max(32, -(-n // 32) * 32), C), np.float32)
    Wt[:n] = W_rows
    st = orc.MatrixState(Wt)
    st.set_mask(synth.words_from_rows(Wt.shape[0], np.arange(n)))
    return st


def _padded(rows_data, n_pad):
    out = np.zeros((n_pad,) + rows_data.shape[1:], rows_data.dtype)
    out[: len(rows_data)] = rows_data
    return out


def _check_update_rows(mat, rows, W_rows, before, after_mask, st, what):
    """GPU state of `rows` before the update equals the oracle's quantisation of the seeded
    weights; after it, q, s, delta, the live row, the moments and the step count equal the oracle
    state `st` (already stepped) bit for bit."""
    q0, s0, d0 = before
    n = len(rows)
    ref_q, ref_s, ref_d = orc.quantize_rows(W_rows)
    assert q0[rows].tobytes() == ref_q.tobytes(), what
    assert s0[rows].tobytes() == ref_s.tobytes() and d0[rows].tobytes() == ref_d.tobytes(), what
    q, s, d = host(mat.q), host(mat.s), host(mat.delta)
    live = host(mat.live).view(np.uint16)
    m, v = host(mat.m).view(np.uint16), host(mat.v).view(np.uint16)
    slots = after_mask["row_slot"][rows]
    assert q[rows].tobytes() == st.q[:n].tobytes(), what
    assert s[rows].tobytes() == st.s[:n].tobytes(), what
    assert d[rows].tobytes() == st.delta[:n].tobytes(), what
    assert np.array_equal(live[rows], st.live[:n]), what
    assert np.array_equal(m[slots], st.m[:n]) and np.array_equal(v[slots], st.v[:n]), what
    assert np.all(after_mask["slot_step"][slots] == 1) and np.all(st.step[:n] == 1), what


def _snapshot(mat):
    return host(mat.q).copy(), host(mat.s).copy(), host(mat.delta).copy()


# ------------------------------------------------------------------------------------------
# C1: the embedding path at its stated shape
# ------------------------------------------------------------------------------------------

def test_c1_embedding_path_matches_oracle(sf):
    V, H, T, PRIOR, SEED = 32000, 4096, 8 * 512, 20, 1
    torch.cuda.set_device(0)
    model = SparseModel(0, vocab=V, emb_slots=4096, device=DEV)
    model.init(SEED)
    emb = model.emb
    g = synth.rng(SEED, "tokens")
    toks = np.stack([synth.zipf_ids(g, T, V) for _ in range(PRIOR + 1)])
    tok_dev = torch.from_numpy(toks).to(DEV)
    status = sf.status_word(DEV)
    for w in range(PRIOR):
        sf.sf_mask_update([emb.mask], [sf.make_src(sf.SF_SRC_TOKENS, tok_dev[w], n=T)], 0.01, status)
    dY = synth.device_normal_bf16((T, H), SEED, "dy", device=DEV)
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(T, emb.mask.slot_cap) // 4 + 64, dtype=torch.int32, device=DEV)
    plan = StepPlan(model, {"tokens": tok_dev[PRIOR], "dY": dY, "Y": [], "dX": [], "A": []}, ws)
    stream = torch.cuda.current_stream().cuda_stream
    emb.grad.fill_(float("nan"))
    plan.masks(status.data_ptr(), stream)
    plan.embed(status.data_ptr(), stream)
    torch.cuda.synchronize()

    # conductor over all 21 windows, every row
    charge = np.zeros(V, np.float32)
    for w in range(PRIOR + 1):
        words, bad = orc.window_tokens(charge, toks[w])
        assert bad == 0
    mh = mask_host(emb.mask)
    assert mh["charge"].tobytes() == charge.tobytes()
    assert np.array_equal(mh["words"], words)
    rows, tiles = orc.mask_lists(words)
    assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles)
    check_slot_invariants(mh, emb.mask.slot_cap)
    assert 30 <= len(rows) <= 400, len(rows)

    # row gradient of every active row
    G_ref = orc.embed_grad(toks[PRIOR], _bits(dY), V, words)[rows]
    slots = mh["row_slot"][rows]
    assert np.all(slots >= 0)
    got = host(emb.grad)[slots]
    scale = max(np.abs(G_ref).max(), 1.0)
    err = np.max(np.abs(got - G_ref) / np.maximum(np.abs(G_ref), 1e-3 * scale))
    assert err <= DW_TOL, err

    # fused update of every active row, on the oracle's gradient rounded to fp32
    G32 = G_ref.astype(np.float32)
    emb.grad[torch.from_numpy(slots).long().to(DEV)] = torch.from_numpy(G32).to(DEV)
    before = _snapshot(emb)
    plan.update(sf.AdamParams(device=DEV), status.data_ptr(), stream)
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0
    W_rows = synth.device_weights_f32(V, H, SEED, 0, device=DEV)[torch.from_numpy(rows).long().to(DEV)].cpu().numpy()
    st = _oracle_rows_state(W_rows)
    orc.update(st, _padded(G32, st.R), orc.AdamHP())
    _check_update_rows(emb, rows, W_rows, before, mask_host(emb.mask), st, "C1")


# ------------------------------------------------------------------------------------------
# C2: one 7B-shaped layer at 4,096 tokens
# ------------------------------------------------------------------------------------------

@pytest.fixture(scope="module", params=["scattered", "clustered"])
def layer_step(request):
    T, SEED = 4096, 2
    torch.cuda.set_device(0)
    torch.cuda.empty_cache()
    model = SparseModel(1, vocab=0, device=DEV)
    model.init(SEED)
    projs = [(p.layer, p.name, p.mat.R, p.mat.C, INPUT_OF[p.name]) for p in model.projs]
    bank = synth.step_bank(projs, T, request.param, 0, SEED, device=DEV)
    plan = StepPlan(model, bank, None)
    plan.set_coupling(36.0)
    status = sf.status_word(DEV)
    stream = torch.cuda.current_stream().cuda_stream
    for p in model.projs:
        p.mat.grad.fill_(float("nan"))
    plan.masks(status.data_ptr(), stream)
    plan.dw(status.data_ptr(), stream)
    torch.cuda.synchronize()
    snap = {"masks": [mask_host(p.mat.mask) for p in model.projs],
            "status": int(host(status)[0])}
    yield dict(model=model, bank=bank, plan=plan, status=status, stream=stream, snap=snap, T=T,
               seed=SEED, kind=request.param)
    del model, bank, plan
    torch.cuda.empty_cache()


def test_c2_masks_of_every_projection(layer_step):
    model, bank, snap = layer_step["model"], layer_step["bank"], layer_step["snap"]
    assert snap["status"] == 0
    for i, p in enumerate(model.projs):
        charge = np.zeros(p.mat.R, np.float32)
        words = orc.window_outputs(charge, _bits(bank["Y"][i]))
        mh = snap["masks"][i]
        assert mh["charge"].tobytes() == charge.tobytes(), p.name
        assert np.array_equal(mh["words"], words), p.name
        rows, tiles = orc.mask_lists(words)
        assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles), p.name
        check_slot_invariants(mh, p.mat.mask.slot_cap)
        want = synth.chosen_rows(layer_step["seed"], 0, i, p.mat.R, layer_step["kind"], 0)
        assert np.array_equal(rows, want), p.name          # the tracker found exactly the chosen rows


def test_c2_masked_dw_every_active_row(layer_step):
    model, bank, snap = layer_step["model"], layer_step["bank"], layer_step["snap"]
    for i, p in enumerate(model.projs):
        rows = snap["masks"][i]["rows"]
        assert len(rows) > 0
        _check_dw_rows(p.mat, snap["masks"][i], _bits(bank["dX"][i]), _bits(bank["A"][i]), rows,
                       f"C2 {layer_step['kind']} {p.name}")


def test_c2_update_every_active_row(layer_step):
    model, plan, status, stream = layer_step["model"], layer_step["plan"], layer_step["status"], layer_step["stream"]
    seed = layer_step["seed"]
    dense = {}
    for j, p in enumerate(model.projs):               # seeded gradients into the slot rows
        gen = synth.device_generator(seed, "grad", 78, j, device=DEV)
        G = torch.randn((p.mat.R, p.mat.C), generator=gen, device=DEV).mul_(8.0)
        act = p.mat.mask.active_rows[: int(p.mat.mask.counts[0])].long()
        p.mat.grad[p.mat.mask.row_slot[act].long()] = G[act]
        dense[j] = G
    before = {j: _snapshot(p.mat) for j, p in enumerate(model.projs)}
    plan.update(sf.AdamParams(device=DEV), status.data_ptr(), stream)
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0
    masks = [mask_host(p.mat.mask) for p in model.projs]
    for j, p in enumerate(model.projs):
        rows = masks[j]["rows"]
        idx = torch.from_numpy(rows).long().to(DEV)
        W_rows = synth.device_weights_f32(p.mat.R, p.mat.C, seed, j, device=DEV)[idx].cpu().numpy()
        st = _oracle_rows_state(W_rows)
        g = _padded(dense[j][idx].cpu().numpy(), st.R)
        k = plan.upd_arr[j].partner
        if k >= 0:
            pst = orc.MatrixState(np.zeros((st.R, p.mat.C), np.float32))
            pst.set_mask(synth.words_from_rows(st.R, np.nonzero(masks[k]["row_slot"][rows] >= 0)[0]))
            pg = _padded(dense[k][idx].cpu().numpy(), st.R)
            c_self, c_partner = plan.upd_arr[j].c_self, plan.upd_arr[j].c_partner
            assert c_partner == np.float32(STRENGTH[p.name] * math.cos(math.radians(36.0)))
            orc.update(st, g, orc.AdamHP(), partner=pst, pg=pg, c_self=c_self, c_partner=c_partner)
        else:
            orc.update(st, g, orc.AdamHP())
        _check_update_rows(p.mat, rows, W_rows, before[j], masks[j], st, f"C2 {layer_step['kind']} {p.name}")


# ------------------------------------------------------------------------------------------
# C4: one 11008 x 4096 projection at high densities (both dW modes at many tiles)
# ------------------------------------------------------------------------------------------

def _rows_per_tc_tile(rows, tiles, rows_mode):
    """The active rows of each 128-row tensor-core tile: consecutive runs of 128 active rows in
    row mode, runs of four active 32-row tiles in tile mode."""
    if rows_mode:
        return [rows[i:i + 128] for i in range(0, len(rows), 128)]
    out = []
    for i in range(0, len(tiles), 4):
        tset = set(int(t) for t in tiles[i:i + 4])
        out.append(np.array([r for r in rows if int(r) // 32 in tset], np.int64))
    return out


@pytest.mark.parametrize("kind,density", [("scattered", 0.05), ("scattered", 0.5), ("clustered", 0.5)])
def test_c4_density_point_matches_oracle(sf, kind, density):
    R, C, T, SEED = 11008, 4096, 4096, 4
    torch.cuda.set_device(0)
    torch.cuda.empty_cache()
    g = synth.rng(SEED, "rows", int(density * 1e4), int(kind == "clustered"))
    chosen = synth.scattered_rows(g, R, density) if kind == "scattered" else synth.clustered_rows(g, R, density)
    cap = min(R, -(-len(chosen) // 32) * 32 + 32)
    gy = synth.rng(SEED, "tracker", int(density * 1e4), int(kind == "clustered"))
    Y = synth.tracker_outputs(gy, T, synth.tracker_gains(R, chosen))
    A = synth.device_normal_bf16((T, C), SEED, "act", device=DEV)
    dX = synth.device_normal_bf16((T, R), SEED, "dx", device=DEV)
    W = synth.device_weights_f32(R, C, SEED, 0, device=DEV)
    mat = sf.Matrix(R, C, cap, DEV)
    sf.sf_mask_init(mat.mask)
    sf.sf_quantize_init(W, mat)
    status = sf.status_word(DEV)
    Yd = torch.from_numpy(Y.view(np.int16)).view(torch.bfloat16).to(DEV)
    sf.sf_mask_update([mat.mask], [sf.make_src(sf.SF_SRC_OUTPUT_BF16, Yd, n=T, ld=R)], 0.01, status)
    probs = [sf.dw_problem(dX, A, mat.mask, mat.grad)]
    mat.grad.fill_(float("nan"))
    sf.sf_masked_dw(probs, status, ws=sf.dw_workspace(probs, DEV))
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0

    charge = np.zeros(R, np.float32)
    words = orc.window_outputs(charge, Y)
    mh = mask_host(mat.mask)
    assert mh["charge"].tobytes() == charge.tobytes() and np.array_equal(mh["words"], words)
    rows, tiles = orc.mask_lists(words)
    assert np.array_equal(rows, chosen)
    assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles)
    check_slot_invariants(mh, cap)

    # the device picks row mode when the gathered rows need fewer tensor-core tiles
    um = sf.sf_masked_dw_unit_rows()
    rows_mode = -(-len(rows) // um) < -(-len(tiles) // (um // 32)) and len(rows) <= -(-cap // 32) * 32
    assert rows_mode == (kind == "scattered")
    per_tile = _rows_per_tc_tile(rows, tiles, rows_mode)
    assert len(per_tile) >= 5
    pick_g = synth.rng(SEED, "misc", int(density * 1e4), int(kind == "clustered"))
    sample = []
    for tr in per_tile:                      # first, last and two more rows of every tile
        sample += [tr[0], tr[-1]] + list(pick_g.choice(tr, size=min(2, len(tr)), replace=False))
    sample = np.unique(np.array(sample, np.int64))
    if len(sample) < 128:                    # top up with random active rows to at least 128
        rest = np.setdiff1d(rows, sample)
        sample = np.union1d(sample, pick_g.choice(rest, size=min(128 - len(sample), len(rest)), replace=False))
    assert len(sample) >= min(128, len(rows))
    _check_dw_rows(mat, mh, _bits(dX), _bits(A), sample, f"C4 {kind} {density}")

    # update of 64 sampled active rows on seeded gradients
    gen = synth.device_generator(SEED, "grad", 79, int(density * 1e4), device=DEV)
    G = torch.randn((R, C), generator=gen, device=DEV).mul_(8.0)
    act = mat.mask.active_rows[: int(mat.mask.counts[0])].long()
    mat.grad[mat.mask.row_slot[act].long()] = G[act]
    before = _snapshot(mat)
    sf.sf_sparse_update([sf.matrix_struct(mat)], sf.AdamParams(device=DEV), status)
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0
    upd_rows = np.sort(pick_g.choice(rows, size=min(64, len(rows)), replace=False))
    idx = torch.from_numpy(upd_rows).long().to(DEV)
    W_rows = W[idx].cpu().numpy()
    st = _oracle_rows_state(W_rows)
    orc.update(st, _padded(G[idx].cpu().numpy(), st.R), orc.AdamHP())
    _check_update_rows(mat, upd_rows, W_rows, before, mask_host(mat.mask), st, f"C4 {kind} {density}")
