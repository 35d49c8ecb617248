"""Row-sharded split of the step over ranks (masked_optimizer_step_b200.shard), on CPU with gloo.

Two ranks each take half of a step's tokens and own half of every matrix's rows. On each rank
the oracle computes what that rank's GPU would: the activity of its tokens, the charge rule on
the combined activity, partial weight gradients (projections) and row sums (embedding) over its
tokens for every active row, then, after the exchange, the fused update of the rows it owns.
The pieces are gathered and compared with the oracle's single-process step over all tokens:
masks bit for bit, gradients to fp64 rounding (and bit for bit once rounded to fp32), and the
updated q, s, delta, moments and live rows bit for bit.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT

# (name, R, C, partner): q and o coupled, down alone; plus an embedding table
MATS = (("q", 256, 128, "o"), ("o", 256, 128, "q"), ("down", 128, 256, None))
V, H, T, SEED = 512, 64, 64, 9
C_PARTNER = float(np.float32(0.4 * math.cos(math.radians(36.0))))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs():
    from masked_optimizer_step_b200 import synth
    g = synth.rng(SEED, "misc", 1)
    tok = synth.zipf_ids(g, T, V)
    dY = synth.normal_bf16(g, (T, H))
    W_emb = synth.weights_f32(g, V, H)
    mats = {}
    chosen = {}
    for name, R, C, _ in MATS:
        rows = synth.scattered_rows(g, R, 0.05)
        if name == "o":                      # share rows with q, so the coupled mix is exercised
            rows = np.union1d(rows, chosen["q"][:6])
        chosen[name] = rows
        mats[name] = dict(R=R, C=C, Y=synth.tracker_outputs(g, T, synth.tracker_gains(R, rows)),
                      dX=synth.normal_bf16(g, (T, R)), A=synth.normal_bf16(g, (T, C)),
                      W=synth.weights_f32(g, R, C))
    return tok, dY, W_emb, mats


def _update_rows(orc, W, rows, grad_rows, partner_rows=None, partner_grad_rows=None, c_partner=0.0):
    """Oracle update of the given rows of W (rows independent; partner entries by row)."""
    R, C = W.shape
    st = orc.MatrixState(W)
    st.set_mask(_words(R, rows))
    g = np.zeros((R, C), np.float32)
    g[rows] = grad_rows
    if partner_rows is None:
        orc.update(st, g, orc.AdamHP())
    else:
        pst = orc.MatrixState(np.zeros((R, C), np.float32))
        pst.set_mask(_words(R, partner_rows))
        pg = np.zeros((R, C), np.float32)
        pg[partner_rows] = partner_grad_rows
        orc.update(st, g, orc.AdamHP(), partner=pst, pg=pg, c_self=1.0, c_partner=c_partner)
    return st


def _words(R, rows):
    from masked_optimizer_step_b200 import synth
    return synth.words_from_rows(R, rows)


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle as orc
    from masked_optimizer_step_b200 import shard
    tok, dY, W_emb, mats = _inputs()
    lo, hi = (T * rank) // world, (T * (rank + 1)) // world          # this rank's tokens

    # activity of this rank's tokens, combined over ranks, then the charge rule on every rank
    hits = torch.from_numpy(np.bincount(tok[lo:hi], minlength=V).astype(np.int32))
    mags = torch.from_numpy(np.concatenate([orc.row_magnitudes(m["Y"][lo:hi])[0] for m in mats.values()]))
    shard.combine_activity(hits=hits, magnitudes=mags)
    words = {"emb": orc.window_activity(np.zeros(V, np.float32), hits.numpy().astype(np.float32))}
    at = 0
    for name, m in mats.items():
        words[name] = orc.window_activity(np.zeros(m["R"], np.float32), mags.numpy()[at:at + m["R"]])
        at += m["R"]
    rows = {k: orc.mask_lists(w)[0] for k, w in words.items()}

    # partial gradients over this rank's tokens for every active row, then the exchange
    parts = [(rows["emb"], torch.from_numpy(orc.embed_grad(tok[lo:hi], dY[lo:hi], V, words["emb"])[rows["emb"]]),
              shard.RowPartition(V, world))]
    for name, m in mats.items():
        partial = orc.masked_dw_rows(m["dX"][lo:hi], m["A"][lo:hi], rows[name])
        parts.append((rows[name], torch.from_numpy(partial), shard.RowPartition(m["R"], world)))
    owned = dict(zip(["emb"] + list(mats), shard.exchange_rows(parts)))

    # update of the owned rows; a coupled partner's gradient rows are owned by the same rank
    res = {"words": {k: w.tobytes() for k, w in words.items()}, "grad": {}, "state": {}}
    for key, (own_rows, g64) in owned.items():
        res["grad"][key] = (own_rows, g64.numpy())
    st = _update_rows(orc, W_emb, owned["emb"][0], owned["emb"][1].numpy().astype(np.float32))
    res["state"]["emb"] = _rows_of(st, owned["emb"][0])
    for name, R, C, partner in MATS:
        own_rows, g = owned[name]
        if partner:
            p_rows, pg = owned[partner]
            common = np.isin(own_rows, p_rows)
            pgr = np.zeros((len(own_rows), C), np.float32)
            pgr[common] = pg.numpy().astype(np.float32)[np.isin(p_rows, own_rows)]
            st = _update_rows(orc, mats[name]["W"], own_rows, g.numpy().astype(np.float32),
                              partner_rows=own_rows[common], partner_grad_rows=pgr[common], c_partner=C_PARTNER)
        else:
            st = _update_rows(orc, mats[name]["W"], own_rows, g.numpy().astype(np.float32))
        res["state"][name] = _rows_of(st, own_rows)
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


def _rows_of(st, rows):
    return {k: getattr(st, k)[rows].copy() for k in ("q", "s", "delta", "m", "v", "live", "step")}


def test_row_partition_covers_rows_once_at_tile_granularity():
    from masked_optimizer_step_b200 import shard
    for R, world in [(256, 2), (11008, 8), (4096, 3), (32000, 8), (64, 4)]:
        p = shard.RowPartition(R, world)
        assert p.bounds[0] == 0 and p.bounds[-1] == R
        assert all(b % 32 == 0 for b in p.bounds) and all(np.diff(p.bounds) >= 0)
        assert max(np.diff(p.bounds)) - min(np.diff(p.bounds)) <= 32
        r = np.arange(R)
        own = p.owner(r)
        for g in range(world):
            a, b = p.range(g)
            assert np.all(own[a:b] == g)
        rows = np.sort(np.random.default_rng(R).choice(R, size=min(R, 50), replace=False))
        off = p.split(rows)
        for g in range(world):
            assert np.all(p.owner(rows[off[g]:off[g + 1]]) == g)


@pytest.mark.slow
def test_two_rank_row_split_equals_the_single_process_step():
    import oracle as orc
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    tok, dY, W_emb, mats = _inputs()

    # single-process oracle step over all tokens
    words = {"emb": orc.window_tokens(np.zeros(V, np.float32), tok)[0]}
    for name, m in mats.items():
        words[name] = orc.window_outputs(np.zeros(m["R"], np.float32), m["Y"])
    rows = {k: orc.mask_lists(w)[0] for k, w in words.items()}
    grads = {"emb": orc.embed_grad(tok, dY, V, words["emb"])[rows["emb"]]}
    for name, m in mats.items():
        grads[name] = orc.masked_dw_rows(m["dX"], m["A"], rows[name])
    for r in range(world):
        for k, w in words.items():
            assert out[r]["words"][k] == w.tobytes(), (r, k)     # every rank derived the same masks
    for k in rows:
        got_rows = np.concatenate([out[r]["grad"][k][0] for r in range(world)])
        got = np.concatenate([out[r]["grad"][k][1] for r in range(world)])
        assert np.array_equal(got_rows, rows[k]) and len(rows[k]) > 0, k
        np.testing.assert_allclose(got, grads[k], rtol=1e-12, atol=1e-12 * np.abs(grads[k]).max())
        assert got.astype(np.float32).tobytes() == grads[k].astype(np.float32).tobytes(), k
    ref = {"emb": _rows_of(_update_rows(orc, W_emb, rows["emb"], grads["emb"].astype(np.float32)), rows["emb"])}
    assert np.isin(rows["q"], rows["o"]).sum() >= 6
    for name, R, C, partner in MATS:
        g32 = grads[name].astype(np.float32)
        if partner:
            common = np.isin(rows[name], rows[partner])
            pg = np.zeros_like(g32)
            pg[common] = grads[partner].astype(np.float32)[np.isin(rows[partner], rows[name])]
            st = _update_rows(orc, mats[name]["W"], rows[name], g32, partner_rows=rows[name][common],
                              partner_grad_rows=pg[common], c_partner=C_PARTNER)
        else:
            st = _update_rows(orc, mats[name]["W"], rows[name], g32)
        ref[name] = _rows_of(st, rows[name])
    for k in ref:
        for field in ref[k]:
            got = np.concatenate([out[r]["state"][k][field] for r in range(world)])
            assert got.tobytes() == ref[k][field].tobytes(), (k, field)
