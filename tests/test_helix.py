"""Host logic of "Sparse-First Fine-Tuning" (tensorwirelabs.com) sections 2.4-2.6: the rewind policy
and the Helix schedule. Pinned where the pages fix a fact (constants, the Fibonacci stride, the
36-degree rungs, the ten-step watch, the 15% rebound, three recoveries, cos of the 28.4-degree
pitch); the exponentially weighted trend against its definition summed out by brute force; the
curve walk against exact rational arithmetic. The coefficient formula itself is a reading and
its parity is unpinned: its tests check the properties the prose states."""
import math
from fractions import Fraction

import numpy as np
import pytest

from masked_optimizer_step_b200 import helix as hx


# ---- constants and the stride ---------------------------------------------------------------

def test_fibonacci_rungs_capped_at_21():
    assert hx.fibonacci_rungs() == [1, 1, 2, 3, 5, 8, 13, 21]
    assert hx.fibonacci_rungs(4) == [1, 1, 2, 3]


def test_stride_climbs_while_descending_then_caps_resets_and_steps_down():
    h = hx.Helix()
    loss, seen = 10.0, []
    for _ in range(12):                         # steady, clear descent
        loss -= 0.5
        h.push_loss(loss)
        seen.append(h.stride.value)
    # the first push only sets the reference loss; the smoothed trend is positive from the second
    assert seen[0] == 1
    assert seen[1:9] == [1, 2, 3, 5, 8, 13, 21, 21]
    assert seen[-1] == 21
    h.rewind()
    assert h.stride.value == 1
    for _ in range(3):
        h.push_loss(loss)
    k = h.stride.k
    for _ in range(30):                         # a long rise: the smoothed trend turns negative
        loss += 0.5
        h.push_loss(loss)
    assert h.stride.k < k or h.stride.k == 0
    assert h.stride.value == 1


def test_stride_steps_down_one_rung_at_a_time():
    st = hx.Stride()
    for _ in range(7):
        st.step(1.0, 0.1)
    assert st.value == 21
    vals = []
    for _ in range(8):
        st.step(-1.0, 0.1)
        vals.append(st.value)
    assert vals == [13, 8, 5, 3, 2, 1, 1, 1]
    st.step(0.05, 0.1)                           # between 0 and the threshold: held
    assert st.value == 1


def test_phase_advances_36_degrees_per_rung_and_walks_once_per_turn():
    h = hx.Helix()
    for _ in range(10):                          # flat loss: stride stays 1
        h.push_loss(3.0)
    assert h.stride.value == 1
    assert h.phi_deg == pytest.approx(360.0)
    assert h.turns_done == 1
    x1, y1 = h.walk.x, h.walk.y
    assert (x1, y1) != (-2.0, 3.0)
    for _ in range(9):
        h.push_loss(3.0)
    assert h.turns_done == 1 and (h.walk.x, h.walk.y) == (x1, y1)
    h.push_loss(3.0)
    assert h.turns_done == 2


def test_weight_decay_scale_is_cos_pitch():
    c = hx.Helix().coefficients()
    assert c.wd_scale == pytest.approx(math.cos(math.radians(28.4)), abs=0)
    assert 0.879 < c.wd_scale < 0.880


# ---- the loss trend -------------------------------------------------------------------------

def test_trend_is_the_weighted_mean_of_loss_changes():
    rng = np.random.default_rng(5)
    losses = 5.0 + np.cumsum(rng.normal(-0.01, 0.05, 40))
    tr = hx.LossTrend()
    Cs = []
    for k, L in enumerate(losses):
        tr.push(L)
        if k == 0:
            assert tr.value == 0.0
            Cs.append(0.0)
            continue
        d = [losses[k - i - 1] - losses[k - i] for i in range(k)]   # d[i] = change i steps ago
        w = math.exp(-1 / 10)
        ref = sum(w ** i * d[i] for i in range(k)) / sum(w ** i for i in range(k))
        assert tr.value == pytest.approx(ref, rel=1e-12, abs=1e-15)
        Cs.append(ref)
    # the smoothed copy: the same weighted mean taken over the trend values after each change
    c = Cs[1:]
    n = len(c)
    ref_s = sum(math.exp(-i / 10) * c[n - 1 - i] for i in range(n)) / sum(math.exp(-i / 10) for i in range(n))
    assert tr.smoothed == pytest.approx(ref_s, rel=1e-12)


def test_trend_of_a_constant_descent_is_that_descent():
    tr = hx.LossTrend()
    for k in range(25):
        tr.push(10.0 - 0.25 * k)
    assert tr.value == pytest.approx(0.25, rel=1e-12)
    assert tr.smoothed == pytest.approx(0.25, rel=1e-12)


# ---- the curve walk -------------------------------------------------------------------------

def _add_exact(P, Q, b=17):
    (x1, y1), (x2, y2) = P, Q
    lam = (3 * x1 * x1) / (2 * y1) if (x1 == x2 and y1 == y2) else (y2 - y1) / (x2 - x1)
    x3 = lam * lam - x1 - x2
    return (x3, lam * (x1 - x3) - y1)


def test_curve_walk_matches_exact_rational_multiples():
    G = (Fraction(-2), Fraction(3))
    assert G[1] ** 2 == G[0] ** 3 + 17
    w = hx.CurveWalk()
    P = G
    for k in range(2, 7):                      # kG exactly, as rationals
        P = _add_exact(P, G)
        assert P[1] ** 2 == P[0] ** 3 + 17
        w.advance()
        assert w.x == pytest.approx(float(P[0]), rel=1e-9)
        assert w.y == pytest.approx(float(P[1]), rel=1e-9)


def test_curve_walk_stays_on_the_curve_and_never_repeats():
    w = hx.CurveWalk()
    xs = set()
    for _ in range(500):
        w.advance()
        assert abs(w.on_curve_residual()) <= 1e-9 * max(1.0, abs(w.x) ** 3)
        assert abs(w.psi_deg) <= 3.6 + 1e-12
        xs.add(round(w.x, 9))
    assert len(xs) == 500


# ---- the coefficients (reading; parity unpinned) --------------------------------------------

def test_coefficients_bounded_zero_strength_is_plain_adam_and_sweep_a_turn():
    h = hx.Helix()
    vals = []
    for _ in range(10):                         # one turn at stride 1
        h.push_loss(2.0)
        c = h.coefficients({"p": 0.6, "zero": 0.0})
        assert c.c_self == 1.0
        assert c.c_partner["zero"] == 0.0
        assert abs(c.c_partner["p"]) <= 0.6
        assert 0.0 <= c.exposure <= 1.0
        vals.append(c.c_partner["p"])
    assert max(vals) > 0.25 and min(vals) < -0.2     # strongly shared ... leaning away, each turn


def test_channel_weights_ratio_while_descending_and_on_a_plateau():
    h = hx.Helix()
    for k in range(30):
        h.push_loss(10.0 - 0.5 * k)
    h.phi_deg = 90.0 * 41                      # cos(phi) = 0: no one-turn modulation
    wp, wm = h.channel_weights()
    assert wp == pytest.approx(1.833)
    assert wm == pytest.approx(1.0 + 0.05 * math.cos(math.radians(h.phi_deg) / 10))
    flat = hx.Helix()
    for _ in range(30):
        flat.push_loss(4.0)
    flat.phi_deg = 90.0
    wp, wm = flat.channel_weights()
    assert wp == pytest.approx(1.833)
    assert wm == pytest.approx(1.833 * (1 + 0.05 * math.cos(math.radians(9.0))))


def test_modulation_is_ten_and_five_percent():
    h = hx.Helix()
    for k in range(30):
        h.push_loss(10.0 - 0.5 * k)
    for phi, f1 in ((0.0, 1.10), (180.0, 0.90)):
        h.phi_deg = phi
        wp, _ = h.channel_weights()
        assert wp == pytest.approx(1.833 * f1)
    h.phi_deg = 1800.0                          # half of ten turns: cos(pi) = -1 on the slow term
    _, wm = h.channel_weights()
    assert wm == pytest.approx(1.0 * 0.95)


# ---- the rewind policy ----------------------------------------------------------------------

def _events(policy, losses):
    return [policy.observe(L) for L in losses]


def test_steady_descent_saves_every_minimum():
    p = hx.RewindPolicy()
    acts = _events(p, [2.0 - 0.01 * k for k in range(20)])
    assert all(a.save and a.event == "watch" for a in acts)
    assert not any(a.restore for a in acts)


def test_rebound_past_15_percent_rewinds_when_the_watch_runs_out():
    p = hx.RewindPolicy()
    acts = _events(p, [1.0, 0.95] + [1.0] * 9 + [1.1])        # 1.1 > 1.15 * 0.95 = 1.0925
    assert acts[1].save and acts[1].event == "watch"
    assert not any(a.save or a.restore for a in acts[2:11])   # inside the watch: no saves
    assert acts[11].restore and acts[11].skip and acts[11].event == "rewind"
    assert p.recoveries == 1


def test_rise_within_15_percent_is_accepted():
    p = hx.RewindPolicy()
    acts = _events(p, [1.0, 0.8] + [0.85] * 9 + [0.91])        # 0.91 < 1.15 * 0.8 = 0.92
    assert not acts[1].save                                      # a 20% drop is not saved
    assert acts[11].event == "accept" and not acts[11].restore
    assert p.ckpt_loss == 0.8                                   # the minimum is the reference
    a = p.observe(0.87)                                          # within 10% of 0.8: saved
    assert a.save and p.ckpt_loss == 0.87
    assert not p.observe(0.97).save                              # >10% above 0.87


def test_three_recoveries_per_minimum_then_accept():
    p = hx.RewindPolicy()
    _events(p, [1.0, 0.5])
    rewinds = 0
    for _ in range(3):
        acts = _events(p, [0.7] * 10)
        assert acts[-1].event == "rewind"
        rewinds += 1
    acts = _events(p, [0.7] * 10)
    assert acts[-1].event == "exhausted" and acts[-1].save and not acts[-1].restore
    assert rewinds == 3 and p.best == 0.7 and p.ckpt_loss == 0.7


def test_new_minimum_during_watch_restarts_it_and_resets_recoveries():
    p = hx.RewindPolicy()
    _events(p, [1.0, 0.95] + [1.1] * 10)
    assert p.recoveries == 1
    a = p.observe(0.9)
    assert a.event == "watch" and p.recoveries == 0 and p.watch_left == 10
    assert a.save                                                 # 0.9 within 10% of 0.95


def test_jump_of_more_than_ten_percent_is_not_saved():
    p = hx.RewindPolicy(watch_steps=0)
    _events(p, [1.0])
    assert not p.observe(1.2).save
    assert p.observe(1.05).save


def test_nonfinite_loss_rewinds_only_with_a_checkpoint():
    p = hx.RewindPolicy()
    assert not p.observe(float("nan")).restore
    p.observe(1.0)
    a = p.observe(float("inf"))
    assert a.restore and a.skip


class _FakeBinding:
    """Stands in for the binding on the CPU: records the checkpoint calls."""

    def __init__(self):
        self.calls = []

    class Checkpoint:
        def __init__(self, cap, C, device):
            self.cap, self.C = cap, C

    def matrix_struct(self, m):
        return m

    def sf_checkpoint_save(self, mats, ckpts, status, stream):
        self.calls.append(("save", len(mats)))

    def sf_checkpoint_restore(self, mats, ckpts, status, stream):
        self.calls.append(("restore", len(mats)))


class _FakeMat:
    def __init__(self, R, C, cap):
        self.R, self.C = R, C
        self.mask = type("M", (), {"slot_cap": cap})()


def test_rewinder_drives_save_and_restore_and_resets_the_stride():
    fake = _FakeBinding()
    rw = hx.Rewinder.__new__(hx.Rewinder)
    rw.sf, rw.mats = fake, [_FakeMat(64, 32, 8), _FakeMat(64, 32, 0)]
    rw.policy, rw.helix, rw.saved = hx.RewindPolicy(), hx.Helix(), False
    rw.ckpts = [fake.Checkpoint(m.mask.slot_cap or m.R, m.C, "cpu") for m in rw.mats]
    for L in [3.0 - 0.1 * k for k in range(8)]:
        rw.before_step(L)
    assert rw.helix.stride.value > 1
    assert fake.calls == [("save", 2)] * 8
    for L in [2.7] * 9:
        assert not rw.before_step(L).skip
    a = rw.before_step(2.7)                    # 2.7 > 1.15 * 2.3
    assert a.skip and fake.calls[-1] == ("restore", 2)
    assert rw.helix.stride.value == 1


class _FakePipe:
    def __init__(self, log, name):
        self.log, self.name = log, name

    def set_mix(self, c_self, c_partner):
        self.log.append((self.name, "mix", round(c_partner["gate-up"], 6)))

    def set_tokens(self, t):
        self.log.append((self.name, "tokens", t))

    def step(self, hp, status, stream):
        self.log.append((self.name, "step"))


def test_trainer_orders_policy_mix_and_step_and_skips_after_a_rewind():
    from masked_optimizer_step_b200.model import Trainer
    fake = _FakeBinding()
    rw = hx.Rewinder.__new__(hx.Rewinder)
    rw.sf, rw.mats = fake, [_FakeMat(64, 32, 8)]
    rw.policy, rw.helix, rw.saved = hx.RewindPolicy(), hx.Helix(), False
    rw.ckpts = [fake.Checkpoint(8, 32, "cpu")]
    log = []
    tr = Trainer.__new__(Trainer)
    tr.model, tr.pipes, tr.hp, tr.status = None, [_FakePipe(log, "a"), _FakePipe(log, "b")], None, 0
    tr.stream = type("S", (), {"cuda_stream": 0})()
    tr.helix, tr.rewinder, tr.events = rw.helix, rw, {}
    losses = [2.0, 1.95, 1.9] + [2.3] * 10                 # 2.3 > 1.15 * 1.9: the watch ends in a rewind
    acts = [tr.step(k, L, tokens=k) for k, L in enumerate(losses)]
    assert [a.event for a in acts[:3]] == ["watch"] * 3
    assert acts[12].skip and acts[12].event == "rewind" and fake.calls[-1] == ("restore", 1)
    steps = [e for e in log if e[1] == "step"]
    assert len(steps) == 12                                  # every step but the rewound one
    assert steps[0][0] == "a" and steps[1][0] == "b"       # pipes alternate by step index
    # before each step: the mix, then the tokens, then the step, on the same pipe
    for i, e in enumerate(log):
        if e[1] == "step":
            assert log[i - 1][0] == e[0] and log[i - 1][1] == "tokens"
            assert log[i - 2][0] == e[0] and log[i - 2][1] == "mix"
    assert tr.events["rewind"] == 1 and rw.helix.stride.value == 1
