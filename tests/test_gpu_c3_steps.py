"""The full 7B-shaped model over 20 steps (the run the throughput figure is quoted on), with
layers 0 and 31 and the embedding checked against the oracle at every step; and the same model
with rows clustered into whole 32-row tiles (the dW in tile mode) over 6 steps.

Each step runs the same StepPlan calls as the benchmark (all 225 masks in one call, the masked
dW of all 224 projections, the embedding-row gradient, one grouped update), alternating the two
input banks (the second drifts ~5% of every projection's chosen rows) over a token stream whose
Zipf rank map drifts 1% per window, so rows activate and deactivate and moment slots are released
and reused at full scale. The oracle follows the run step by step:
  - the conductor's charges, mask, lists and slot bookkeeping, all 32,000 rows, every step;
  - the trackers of all 14 projections of layers 0 and 31, all rows, every step;
  - dW of eight active rows of each of those projections and the embedding-row gradient of
    every active row, at three of the steps;
  - the fused update of 32 fixed rows of each of those projections (rows chosen in either bank,
    so each is active at some steps and not at others), with coupled partners, on seeded
    gradients written into the gradient buffers, carried from step to step on the oracle's own
    state (q, s, delta and the bf16 live row of every sampled row; moments and step counts of the
    active ones).
The checked layers' weights are seeded on the host, so the oracle starts from the same inputs.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from masked_optimizer_step_b200.model import INPUT_OF, SparseModel, StepPlan
from tests.gpu_helpers import DEV, check_slot_invariants, host, mask_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SEED, T, PRIOR = 3, 2048, 20
CHECK_LAYERS = (0, 31)
DW_TOL = 2e-3
K = 32                                    # sampled rows per checked matrix


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _bit(words, r):
    return (int(words[r >> 5]) >> (r & 31)) & 1


def _seeded_grad(step, j, R, C):
    gen = synth.device_generator(SEED, "grad", 300 + step, j, device=DEV)
    return torch.randn((R, C), generator=gen, device=DEV, dtype=torch.float32).mul_(8.0)


@pytest.mark.parametrize("kind,STEPS", [("scattered", 20), ("clustered", 6)])
def test_steps_layers_0_and_31_and_embedding_follow_the_oracle(kind, STEPS):
    DW_STEPS = (0, STEPS // 2 - 1, STEPS - 1)
    torch.cuda.set_device(0)
    torch.cuda.empty_cache()
    model = SparseModel(32, device=DEV)
    model.init(SEED)
    checked = [i for i, p in enumerate(model.projs) if p.layer in CHECK_LAYERS]
    # host-seeded weights for the checked projections; the oracle starts from the same arrays
    picks, subs = {}, {}
    for i in checked:
        p = model.projs[i]
        R, C = p.mat.R, p.mat.C
        W = synth.weights_f32(synth.rng(SEED, "weights", 1000 + i), R, C)
        sf.sf_quantize_init(torch.from_numpy(W).to(DEV), p.mat)
        c0 = synth.chosen_rows(SEED, p.layer, i, R, kind, 0)
        c1 = synth.chosen_rows(SEED, p.layer, i, R, kind, 1)
        pick = np.unique(np.concatenate([c0[:20], np.setdiff1d(c1, c0)[:8],
                                         np.setdiff1d(np.arange(R), np.union1d(c0, c1))[:4]]))
        assert len(pick) <= K
        picks[i] = pick
        Wt = np.zeros((K, C), np.float32)
        Wt[:len(pick)] = W[pick]
        subs[i] = orc.MatrixState(Wt)
        del W
    projs = [(p.layer, p.name, p.mat.R, p.mat.C, INPUT_OF[p.name]) for p in model.projs]
    banks = [synth.step_bank(projs, T, kind, b, SEED, device=DEV) for b in (0, 1)]
    toks = synth.token_stream(SEED, PRIOR + STEPS, T)
    tok_dev = torch.from_numpy(toks).to(DEV)
    emb_charge = np.zeros(model.emb.R, np.float32)
    for w in range(PRIOR):
        sf.sf_mask_update([model.emb.mask], [sf.make_src(sf.SF_SRC_TOKENS, tok_dev[w], n=T)], 0.01)
        orc.window_tokens(emb_charge, toks[w])
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(T, model.emb.mask.slot_cap) // 4 + 64, dtype=torch.int32,
                     device=DEV)
    plans = []
    for b in (0, 1):
        inputs = dict(banks[b])
        inputs["tokens"] = tok_dev[PRIOR]
        plans.append(StepPlan(model, inputs, ws))
    status = sf.status_word(DEV)
    stream = torch.cuda.current_stream().cuda_stream
    hp, ohp = sf.AdamParams(device=DEV), orc.AdamHP()
    charges = {i: np.zeros(model.projs[i].mat.R, np.float32) for i in checked}
    updated = {i: np.zeros(K, bool) for i in checked}
    rows_seen = {i: set() for i in checked}

    for k in range(STEPS):
        plan, bank = plans[k % 2], banks[k % 2]
        plan.set_tokens(tok_dev[PRIOR + k])
        plan.set_coupling(36.0 * k)
        plan.masks(status.data_ptr(), stream)
        plan.dw(status.data_ptr(), stream)
        plan.embed(status.data_ptr(), stream)
        torch.cuda.synchronize()

        # conductor, every row
        words, bad = orc.window_tokens(emb_charge, toks[PRIOR + k])
        assert bad == 0
        me = mask_host(model.emb.mask)
        assert me["charge"].tobytes() == emb_charge.tobytes() and np.array_equal(me["words"], words), k
        rows, tiles = orc.mask_lists(words)
        assert np.array_equal(me["rows"], rows) and np.array_equal(me["tiles"], tiles), k
        check_slot_invariants(me, model.emb.mask.slot_cap)

        # trackers of the checked layers, every row
        mh = {}
        for i in checked:
            w = orc.window_outputs(charges[i], _bits(bank["Y"][i]))
            m = mask_host(model.projs[i].mat.mask)
            assert m["charge"].tobytes() == charges[i].tobytes(), (k, i)
            assert np.array_equal(m["words"], w), (k, i)
            r_, t_ = orc.mask_lists(w)
            assert np.array_equal(m["rows"], r_) and np.array_equal(m["tiles"], t_), (k, i)
            check_slot_invariants(m, model.projs[i].mat.mask.slot_cap)
            assert m["counts"][3] == 0                       # every active row holds a slot
            mh[i] = m
            rows_seen[i].update(int(r) for r in picks[i] if _bit(w, int(r)))

        if k in DW_STEPS:
            for i in checked:
                p = model.projs[i]
                rows = mh[i]["rows"]
                sel = np.unique(rows[np.linspace(0, len(rows) - 1, 8).astype(int)])
                ref = orc.masked_dw_rows(_bits(bank["dX"][i]), _bits(bank["A"][i]), sel)
                got = host(p.mat.grad)[mh[i]["row_slot"][sel], : p.mat.C].astype(np.float64)
                floor = 1e-3 * np.abs(ref).max()
                err = float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), floor)))
                assert err <= DW_TOL, (k, p.layer, p.name, err)
            ref = orc.embed_grad(toks[PRIOR + k], _bits(bank["dY"]), model.emb.R, me["words"])
            got = host(model.emb.grad)
            scale = max(np.abs(ref[me["rows"]]).max(), 1.0)
            for r in me["rows"]:
                e = np.max(np.abs(got[me["row_slot"][r]] - ref[r]) / np.maximum(np.abs(ref[r]), 1e-3 * scale))
                assert e <= DW_TOL, (k, int(r))

        # seeded gradients of the checked projections into their slot rows, then the update
        dense = {}                  # (matrix, rows of matrix) -> seeded gradient rows (host)
        for i in checked:
            mat = model.projs[i].mat
            G = _seeded_grad(k, i, mat.R, mat.C)
            act = torch.from_numpy(mh[i]["rows"].astype(np.int64)).to(DEV)
            sl = torch.from_numpy(mh[i]["row_slot"][mh[i]["rows"]].astype(np.int64)).to(DEV)
            mat.grad[sl] = G[act]
            pj = plan.upd_arr[i + 1].partner
            for owner in {i} | ({pj - 1} if pj >= 0 else set()):
                dense[(i, owner)] = G[torch.from_numpy(picks[owner]).long().to(DEV)].cpu().numpy()
            del G
        plan.update(hp, status.data_ptr(), stream)
        torch.cuda.synchronize()
        assert int(host(status)[0]) == 0, k

        for i in checked:
            mat, pick, st = model.projs[i].mat, picks[i], subs[i]
            n = len(pick)
            active = [kk for kk, r in enumerate(pick) if _bit(mh[i]["words"], int(r))]
            st.set_mask(synth.words_from_rows(K, active))
            g = np.zeros((K, mat.C), np.float32)
            g[:n] = dense[(i, i)]
            j = i + 1                                       # update-array index (embedding first)
            pj = plan.upd_arr[j].partner
            if pj >= 0:
                pi = pj - 1                                 # the partner: same layer, also checked
                pst = orc.MatrixState(np.zeros((K, mat.C), np.float32))
                pst.set_mask(synth.words_from_rows(K, [kk for kk, r in enumerate(pick)
                                                       if mh[pi]["row_slot"][r] >= 0]))
                pg = np.zeros((K, mat.C), np.float32)
                pg[:n] = dense[(pi, i)]                     # the partner's gradient on this matrix's rows
                orc.update(st, g, ohp, partner=pst, pg=pg, c_self=plan.upd_arr[j].c_self,
                           c_partner=plan.upd_arr[j].c_partner)
            else:
                orc.update(st, g, ohp)
            updated[i][active] = True
            # the sampled rows (and the slots of the active ones), gathered on the device
            rows_d = torch.from_numpy(pick.astype(np.int64)).to(DEV)
            q, s, d = host(mat.q[rows_d]), host(mat.s[rows_d]), host(mat.delta[rows_d])
            live = host(mat.live[rows_d]).view(np.uint16)
            slots = mh[i]["row_slot"][pick]
            step_now = host(mat.mask.slot_step)
            for kk, r in enumerate(pick):
                assert q[kk].tobytes() == st.q[kk].tobytes(), (k, i, int(r))
                assert s[kk] == st.s[kk] and d[kk].tobytes() == st.delta[kk].tobytes(), (k, i, int(r))
                if updated[i][kk]:
                    assert np.array_equal(live[kk], st.live[kk]), (k, i, int(r))
                if kk in active:
                    slot = int(slots[kk])
                    m_g = host(mat.m[slot]).view(np.uint16)
                    v_g = host(mat.v[slot]).view(np.uint16)
                    assert np.array_equal(m_g, st.m[kk]) and np.array_equal(v_g, st.v[kk]), (k, i, int(r))
                    assert step_now[slot] == st.step[kk], (k, i, int(r))

    # the sampled rows did change state over the run: every projection saw rows go active and
    # idle, and moments restart after a row comes back
    for i in checked:
        assert 0 < len(rows_seen[i]) < len(picks[i])
        assert subs[i].step.max() >= 2
