"""The rewind policy driving the device checkpoint ("Sparse-First Fine-Tuning", tensorwirelabs.com,
section 2.6) and the Helix mix reaching the update's argument array (sections 2.4, 2.5)."""
import numpy as np
import pytest
import torch

from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200 import helix as hx
from masked_optimizer_step_b200 import synth
from masked_optimizer_step_b200.model import SparseModel, StepPlan
from tests.gpu_helpers import DEV, f32_dev, host, u32_dev

pytestmark = pytest.mark.gpu


def _snapshot(mat):
    return {k: host(getattr(mat, k)).copy() for k in ("q", "s", "delta", "live")}


def test_rewinder_restores_the_state_of_the_last_save(sf):
    R, C = 128, 256
    mats = []
    for i in range(2):
        m = sf.Matrix(R, C, 48, DEV)
        sf.sf_mask_init(m.mask)
        sf.sf_quantize_init(f32_dev(synth.weights_f32(synth.rng(40, "weights", i), R, C)), m)
        words = synth.words_from_rows(R, np.sort(synth.rng(40, "rows", i).choice(R, 30, replace=False)))
        sf.sf_mask_update([m.mask], [sf.make_src(sf.SF_SRC_WORDS, u32_dev(words))], 0.01)
        mats.append(m)
    hp = sf.AdamParams(lr=5e-3)
    status = sf.status_word()
    rw = hx.Rewinder(mats, helix=hx.Helix(), device=DEV)

    def train(k):
        for i, m in enumerate(mats):
            g = synth.rng(40, "grad", k, i).standard_normal((48, C), dtype=np.float32)
            m.grad.copy_(f32_dev(g))
        sf.sf_sparse_update([sf.matrix_struct(m) for m in mats], hp, status)

    losses = [3.0, 2.9, 2.8] + [3.3] * 10
    snap = None
    for k, L in enumerate(losses):
        act = rw.before_step(L, status)
        if act.save:
            snap = [_snapshot(m) for m in mats]
        if act.restore:
            torch.cuda.synchronize()
            for m, sn in zip(mats, snap):
                now = _snapshot(m)
                for key in ("q", "s", "delta", "live"):
                    assert now[key].tobytes() == sn[key].tobytes(), key
            assert act.skip and rw.helix.stride.value == 1
            break
        train(k)
    else:
        pytest.fail("the policy never rewound")
    assert int(host(status)[0]) == 0


def test_step_plan_takes_the_helix_mix(sf):
    shapes = (("q", 64, 128), ("k", 64, 128), ("v", 64, 128), ("o", 64, 128),
              ("gate", 96, 128), ("up", 96, 128), ("down", 64, 96))
    model = SparseModel(1, vocab=0, layer_shapes=shapes, device=DEV)
    T = 32
    inputs = {"tokens": None, "dY": None,
              "Y": [torch.zeros((T, R), dtype=torch.bfloat16, device=DEV) for _, R, _ in shapes],
              "dX": [torch.zeros((T, R), dtype=torch.bfloat16, device=DEV) for _, R, _ in shapes],
              "A": [torch.zeros((T, C), dtype=torch.bfloat16, device=DEV) for _, _, C in shapes]}
    plan = StepPlan(model, inputs, None)
    h = hx.Helix()
    for L in (3.0, 2.9, 2.7):
        h.push_loss(L)
    c = h.coefficients()
    plan.set_mix(c.c_self, c.c_partner)
    got = {p.name: plan.upd_arr[i].c_partner for i, p in enumerate(model.projs)}
    f32 = lambda x: float(np.float32(x))
    assert got["q"] == got["o"] == f32(c.c_partner["q-o"])
    assert got["k"] == got["v"] == f32(c.c_partner["k-v"])
    assert got["gate"] == got["up"] == f32(c.c_partner["gate-up"])
    assert got["down"] == 0.0
