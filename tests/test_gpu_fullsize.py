"""Parity at the full 7B shape, in the launch configuration bench.py times.

One step of the 32-layer model (plus the 32,000-row embedding, 2,048 tokens, ~1% masks, once
scattered and once clustered into whole tiles) runs through the same StepPlan calls as the
benchmark: 225 masks in one call, the masked
dW of all 224 projections in one call, the embedding-row gradient, and one grouped update. The
oracle then recomputes sampled outputs one by one:
  - conductor charges, masks and lists over 21 windows (all 32,000 rows), and the trackers of
    sampled projections (all rows);
  - dW of every active row of every projection of layers 0, 16 and 31 (one layer in each of the
    three main dW launches: every problem of every group, every 128-row tile);
  - the embedding-row gradient of every active row;
  - the fused update of sampled rows, on seeded gradients written into the gradient buffers
    (so no oracle input comes from the CUDA path), with the rotated pair coupling.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from masked_optimizer_step_b200.model import INPUT_OF, STRENGTH, SparseModel, StepPlan
from tests.gpu_helpers import DEV, host, mask_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SEED, T, PRIOR = 3, 2048, 20
DW_TOL = 2e-3
SAMPLED = [(0, "q"), (0, "o"), (0, "gate"), (0, "up"), (0, "down"), (17, "gate"), (31, "k"), (31, "v")]
DW_LAYERS = (0, 16, 31)


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module", params=["scattered", "clustered"])
def step_state(request):
    """Scattered rows put every dW group in row mode; clustered whole tiles put them in tile mode."""
    torch.cuda.set_device(0)
    torch.cuda.empty_cache()
    model = SparseModel(32, device=DEV)
    model.init(SEED)
    projs = [(p.layer, p.name, p.mat.R, p.mat.C, INPUT_OF[p.name]) for p in model.projs]
    bank = synth.step_bank(projs, T, request.param, 0, SEED, device=DEV)
    toks = synth.token_stream(SEED, PRIOR + 1, T)
    tok_dev = torch.from_numpy(toks).to(DEV)
    srcs = [sf.make_src(sf.SF_SRC_TOKENS, tok_dev[w], n=T) for w in range(PRIOR)]
    for w in range(PRIOR):
        sf.sf_mask_update([model.emb.mask], [srcs[w]], 0.01)
    bank["tokens"] = tok_dev[PRIOR]
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(T, model.emb.mask.slot_cap) // 4 + 64,
                     dtype=torch.int32, device=DEV)
    plan = StepPlan(model, bank, ws)
    plan.set_coupling(36.0)
    status = sf.status_word(DEV)
    stream = torch.cuda.current_stream().cuda_stream
    plan.masks(status.data_ptr(), stream)
    plan.dw(status.data_ptr(), stream)
    plan.embed(status.data_ptr(), stream)
    torch.cuda.synchronize()
    snap = {"masks": [mask_host(m.mask) for m in model.all_mats],
            "grad": {}, "status_before_update": int(host(status)[0])}
    for i, p in enumerate(model.projs):
        if (p.layer, p.name) in SAMPLED or p.layer in DW_LAYERS:
            snap["grad"][(p.layer, p.name)] = host(p.mat.grad).copy()
    snap["emb_grad"] = host(model.emb.grad).copy()
    return dict(model=model, bank=bank, toks=toks, plan=plan, status=status, stream=stream, snap=snap)


def test_fullsize_conductor_and_trackers(step_state):
    model, snap, toks, bank = step_state["model"], step_state["snap"], step_state["toks"], step_state["bank"]
    charge = np.zeros(model.emb.R, np.float32)
    for w in range(PRIOR + 1):
        words, bad = orc.window_tokens(charge, toks[w])
        assert bad == 0
    mh = snap["masks"][0]
    assert mh["charge"].tobytes() == charge.tobytes()
    assert np.array_equal(mh["words"], words)
    rows, tiles = orc.mask_lists(words)
    assert np.array_equal(mh["rows"], rows) and np.array_equal(mh["tiles"], tiles)
    for key in SAMPLED:
        i = model.index[key]
        Y = _bits(bank["Y"][i])
        ch = np.zeros(model.projs[i].mat.R, np.float32)
        w_ = orc.window_outputs(ch, Y)
        m = snap["masks"][i + 1]
        assert m["charge"].tobytes() == ch.tobytes(), key
        assert np.array_equal(m["words"], w_), key
    assert step_state["snap"]["status_before_update"] == 0


def test_fullsize_masked_dw_every_row_of_three_layers(step_state):
    model, snap, bank = step_state["model"], step_state["snap"], step_state["bank"]
    checked = 0
    for i, p in enumerate(model.projs):
        if p.layer not in DW_LAYERS:
            continue
        m = snap["masks"][i + 1]
        rows = m["rows"]
        assert len(rows) > 0
        ref = orc.masked_dw_rows(_bits(bank["dX"][i]), _bits(bank["A"][i]), rows)
        slots = m["row_slot"][rows]
        assert np.all(slots >= 0)
        got = snap["grad"][(p.layer, p.name)][slots, : p.mat.C].astype(np.float64)
        floor = 1e-3 * np.abs(ref).max()          # 1e-3 of the projection's largest |dW| entry
        err = np.max(np.abs(got - ref) / np.maximum(np.abs(ref), floor), axis=1)
        worst = int(np.argmax(err))
        assert err[worst] <= DW_TOL, (p.layer, p.name, int(rows[worst]), float(err[worst]))
        checked += len(rows)
    assert checked >= 3 * 400


def test_fullsize_embedding_gradient(step_state):
    model, snap, toks, bank = step_state["model"], step_state["snap"], step_state["toks"], step_state["bank"]
    m = snap["masks"][0]
    dY = _bits(bank["dY"])
    ref = orc.embed_grad(toks[PRIOR], dY, model.emb.R, m["words"])
    got = snap["emb_grad"]
    scale = max(np.abs(ref[m["rows"]]).max(), 1.0)
    for r in m["rows"]:
        s = m["row_slot"][r]
        err = np.max(np.abs(got[s] - ref[r]) / np.maximum(np.abs(ref[r]), 1e-3 * scale))
        assert err <= DW_TOL, r


def _synth_grad(model, mat_index, R, C):
    """Seeded dense gradient of one matrix (device), by row."""
    gen = synth.device_generator(SEED, "grad", 77, mat_index, device=DEV)
    return torch.randn((R, C), generator=gen, device=DEV, dtype=torch.float32).mul_(8.0)


def test_fullsize_update_sampled_rows(step_state):
    model, plan, status, stream = step_state["model"], step_state["plan"], step_state["status"], step_state["stream"]
    off = 1
    sampled_mats = {model.index[k] + off for k in SAMPLED}
    partners = {plan.upd_arr[j].partner for j in sampled_mats if plan.upd_arr[j].partner >= 0}
    involved = sorted(sampled_mats | partners | {0})
    dense = {}
    for j in involved:                       # seeded gradients into the slot rows
        mat = model.all_mats[j]
        G = _synth_grad(model, j, mat.R, mat.C)
        rs = mat.mask.row_slot
        act = mat.mask.active_rows[: int(mat.mask.counts[0])].long()
        sl = rs[act].long()
        keep = sl >= 0
        mat.grad[sl[keep]] = G[act[keep]]
        dense[j] = G
    before = {j: (host(model.all_mats[j].q).copy(), host(model.all_mats[j].s).copy(),
                  host(model.all_mats[j].delta).copy()) for j in sorted(sampled_mats | {0})}
    hp = sf.AdamParams(device=DEV)
    plan.update(hp, status.data_ptr(), stream)
    torch.cuda.synchronize()
    assert int(host(status)[0]) == 0
    ohp = orc.AdamHP()
    for j in sorted(sampled_mats | {0}):
        mat = model.all_mats[j]
        mh = mask_host(mat.mask)
        rows = mh["rows"]
        pick = np.unique(np.concatenate([rows[:3], rows[-3:]]))
        q0, s0, d0 = before[j]
        # oracle state holding just the sampled rows (rows are updated independently)
        W = orc.rebuild(q0[pick], s0[pick], d0[pick])
        Wt = np.zeros((32, mat.C), np.float32)
        Wt[:len(pick)] = W
        st = orc.MatrixState(Wt)
        assert st.q[:len(pick)].tobytes() == q0[pick].tobytes()   # requantising W gives the same code
        st.set_mask(synth.words_from_rows(32, np.arange(len(pick))))
        g = np.zeros((32, mat.C), np.float32)
        g[:len(pick)] = dense[j][torch.from_numpy(pick).long().to(DEV)].cpu().numpy()
        p = plan.upd_arr[j].partner
        if p >= 0:
            pm = mask_host(model.all_mats[p].mask)
            pst = orc.MatrixState(np.zeros((32, mat.C), np.float32))
            live = [k for k, r in enumerate(pick) if pm["row_slot"][r] >= 0]
            pst.set_mask(synth.words_from_rows(32, live))
            pg = np.zeros((32, mat.C), np.float32)
            pg[:len(pick)] = dense[p][torch.from_numpy(pick).long().to(DEV)].cpu().numpy()
            c_self, c_partner = plan.upd_arr[j].c_self, plan.upd_arr[j].c_partner
            assert c_partner == np.float32(STRENGTH[model.projs[j - off].name] * math.cos(math.radians(36.0)))
            orc.update(st, g, ohp, partner=pst, pg=pg, c_self=c_self, c_partner=c_partner)
        else:
            orc.update(st, g, ohp)
        q, s, d = host(mat.q), host(mat.s), host(mat.delta)
        live_g = host(mat.live).view(np.uint16)
        m_g, v_g = host(mat.m).view(np.uint16), host(mat.v).view(np.uint16)
        for k, r in enumerate(pick):
            assert q[r].tobytes() == st.q[k].tobytes(), (j, r)
            assert s[r] == st.s[k] and d[r].tobytes() == st.delta[k].tobytes(), (j, r)
            assert np.array_equal(live_g[r], st.live[k])
            slot = mh["row_slot"][r]
            assert np.array_equal(m_g[slot], st.m[k]) and np.array_equal(v_g[slot], st.v[k])
            assert mh["slot_step"][slot] == st.step[k] == 1
