"""The chunked two-stream schedule gives the same bits as one call per stage.

Both runs start from the same seeded state and inputs (a 3-layer model with small projections and
an embedding); matrices of different chunks share nothing and each matrix's calls keep their
order, so masks, slots, moments, weights and live rows must match byte for byte."""
import numpy as np
import pytest
import torch

from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import synth
from masked_optimizer_step_b200.model import INPUT_OF, Pipeline, SparseModel
from tests.gpu_helpers import DEV, host

pytestmark = pytest.mark.gpu

SHAPES = (("q", 256, 128), ("k", 256, 128), ("v", 256, 128), ("o", 256, 128),
          ("gate", 320, 128), ("up", 320, 128), ("down", 256, 320))


def _run(chunks, graphs=False, overlap=False):
    torch.manual_seed(0)
    model = SparseModel(3, vocab=1024, hidden=128, ffn=320, emb_slots=256, device=DEV, layer_shapes=SHAPES,
                        slot_frac=0.2)
    model.init(7)
    T = 96
    projs = [(p.layer, p.name, p.mat.R, p.mat.C, INPUT_OF[p.name]) for p in model.projs]
    bank = synth.step_bank(projs, T, "scattered", 0, 7, hidden=128, device=DEV)
    toks = torch.from_numpy(synth.token_stream(7, 3, T, V=1024)).to(DEV)
    bank["tokens"] = toks[0]
    ws = torch.zeros(sf.sf_embed_grad_ws_bytes(T, model.emb.mask.slot_cap) // 4 + 64, dtype=torch.int32,
                     device=DEV)
    pipe = Pipeline(model, bank, ws, chunks=chunks, overlap_embedding=overlap)
    hp = sf.AdamParams(device=DEV)
    status = sf.status_word(DEV)
    stream = torch.cuda.current_stream()
    if graphs:
        # warm the calls up un-captured on copies of nothing: one captured graph per phase,
        # token ids copied into a fixed buffer before each replay
        from masked_optimizer_step_b200.model import capture_step_graphs
        buf = torch.empty_like(toks[0])
        snap = {k: v.clone() for k, v in _state(model).items()}
        pipe.step(hp, status.data_ptr(), stream)          # warm-up (changes state) ...
        torch.cuda.synchronize()
        _restore(model, snap)                              # ... so put the state back
        g = capture_step_graphs(pipe, hp, status.data_ptr(), buf, [0.0, 36.0, 72.0])
        for k in range(3):
            buf.copy_(toks[k])
            g[36.0 * k].replay()
    else:
        for k in range(3):
            pipe.set_tokens(toks[k])
            pipe.set_coupling(36.0 * k)
            pipe.step(hp, status.data_ptr(), stream)
    torch.cuda.synchronize()
    out = []
    for m in model.all_mats:
        out.append({k: host(getattr(m, k)).tobytes() for k in ("q", "s", "delta", "live")})
        out[-1]["words"] = host(m.mask.words).tobytes()
        out[-1]["rows"] = host(m.mask.active_rows)[: int(host(m.mask.counts)[0])].tobytes()
        slots = host(m.mask.row_slot)
        mm, vv = host(m.m), host(m.v)
        rows = np.nonzero(slots >= 0)[0]
        out[-1]["moments"] = b"".join(mm[slots[r]].tobytes() + vv[slots[r]].tobytes() for r in rows)
    return out, int(host(status)[0]), len(pipe.plans)


def _state(model):
    """Every device array a step changes (weights, moments, gradients, mask state)."""
    out = {}
    for i, m in enumerate(model.all_mats):
        for k in ("q", "s", "delta", "live", "m", "v", "grad"):
            out[(i, k)] = getattr(m, k)
        for k in ("charge", "accum", "words", "active_rows", "active_tiles", "tile_rows", "row_slot",
                  "free_slots", "slot_step"):
            out[(i, "mask." + k)] = getattr(m.mask, k)
    out[("counts",)] = model.counts
    return out


def _restore(model, snap):
    for key, t in _state(model).items():
        t.copy_(snap[key])


def test_step_replayed_from_cuda_graphs_matches_direct_calls(sf):
    ref, st_ref, _ = _run(1)
    got, st_got, _ = _run(1, graphs=True)
    assert st_ref == st_got == 0
    for i, (a, b) in enumerate(zip(ref, got)):
        for key in a:
            assert a[key] == b[key], (i, key)


def test_chunked_schedule_matches_one_call_per_stage(sf):
    ref, st_ref, n1 = _run(1)
    got, st_got, n3 = _run(3)
    assert n1 == 1 and n3 == 3
    assert st_ref == st_got == 0
    assert len(ref) == len(got)
    for i, (a, b) in enumerate(zip(ref, got)):
        for key in a:
            assert a[key] == b[key], (i, key)


def test_embedding_on_a_side_stream_matches_one_call_per_stage(sf):
    ref, st_ref, _ = _run(1)
    got, st_got, _ = _run(1, overlap=True)
    assert st_ref == st_got == 0
    for i, (a, b) in enumerate(zip(ref, got)):
        for key in a:
            assert a[key] == b[key], (i, key)


def test_embedding_overlap_replayed_from_graphs_matches(sf):
    ref, _, _ = _run(1)
    got, st_got, _ = _run(1, graphs=True, overlap=True)
    assert st_got == 0
    for i, (a, b) in enumerate(zip(ref, got)):
        for key in a:
            assert a[key] == b[key], (i, key)
