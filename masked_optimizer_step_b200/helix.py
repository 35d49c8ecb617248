"""Host-side decisions of a sparse-first step: the rewind policy and the Helix coupling schedule.

"Sparse-First Fine-Tuning" (tensorwirelabs.com):
  * section 2.6: when to save the active-row snapshot, when a fresh low of the loss starts a
    watch, and whether that watch closes with a rewind (restore, stride back to 1, skip the step)
    or by keeping the low;
  * sections 2.4 / 2.5 (The coupled update; Adapting to the loss trend): the rotating phase, the
    Fibonacci stride driven by the loss trend, the two channel weights and their slow modulation,
    the non-periodic phase read off a point that steps along an elliptic curve, and the weight decay scaled by
    the cosine of the pitch angle.

Everything here is host arithmetic on scalars that the previous step left behind (its loss); it
reads nothing back from the device while a step is running (section 2.6, last paragraph). The
formula that turns phase, exposure and channel weights into the effective gradients is not in
the text the pages give (it is an image that did not survive extraction), so `Helix.coefficients`
is a reading: the kernel takes any per-pair linear mix, and this is one that follows every
property the prose states. Its parity is unpinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

# constants the pages give (section 2.4, 2.5, 2.6, 2.8)
RUNG_DEG = 36.0                      # phase advance per unit of stride: ten rungs a turn
PITCH_DEG = 28.4                     # fixed pitch angle alpha; weight decay scaled by cos(alpha)
CHANNEL_RATIO = 1.833                # primary : secondary channel weight while descending
TREND_DECAY = 10.0                   # decay length (steps) of the loss-trend mean
FIB_CAP = 21                         # the stride walks 1, 1, 2, 3, 5, 8, 13, 21 and stops there
TURN_MOD = 0.10                      # modulation of the channel weights at the scale of one turn
TEN_TURN_MOD = 0.05                  # ... and at the scale of ten turns
STRENGTH = {"gate-up": 0.6, "q-o": 0.4, "k-v": 0.4}

CKPT_GATE = 0.10                     # save while the loss stays inside +-10% of the saved loss
WATCH_STEPS = 10                     # length of the watch that a fresh loss low starts
REBOUND = 0.15                       # rewind when the loss ends the watch >15% above the minimum
MAX_RECOVERIES = 3                   # rewinds allowed per minimum


def fibonacci_rungs(cap: int = FIB_CAP) -> list[int]:
    """1, 1, 2, 3, 5, ... up to and including cap."""
    seq = [1, 1]
    while seq[-1] + seq[-2] <= cap:
        seq.append(seq[-1] + seq[-2])
    return seq


# ---------------------------------------------------------------------------------------------
# section 2.6: checkpoint and rewind
# ---------------------------------------------------------------------------------------------

@dataclass
class Action:
    """What the host does before launching the next step."""
    save: bool = False               # snapshot the active rows now
    restore: bool = False            # restore the checkpoint (then reset the stride)
    skip: bool = False               # skip this step's update
    event: str = ""                  # "", "save", "watch", "rewind", "accept", "exhausted"


@dataclass
class RewindPolicy:
    """Decides save / watch / rewind from the loss of each step.

    Readings (the text leaves these open):
      * The gate: save when |L - L_ck| <= 0.10 * L_ck, where L_ck is the reference loss of the
        checkpoint; the first loss seen always saves. A jump of more than 10% either way is never
        saved, and outside a watch the checkpoint follows the loss.
      * A loss below every loss seen so far is a new minimum: it (re)opens a watch of WATCH_STEPS
        further losses, resets the count of recoveries and is saved if the gate allows.
      * Inside a watch only new minima are saved, so that a rewind goes back to the minimum's
        state and not to a state from the rise that the watch is judging.
      * When the watch runs out, a loss above (1 + REBOUND) x the minimum rewinds: restore, stride
        back to 1, skip the step, count one recovery and watch again for the same minimum.
      * If not, the low stands: the watch closes and the minimum's loss becomes the
        checkpoint's reference loss, so the gate measures later losses from it. After
        MAX_RECOVERIES rewinds the current state is accepted as it is: it is saved and becomes the
        reference minimum.
      * A non-finite loss rewinds at once when a checkpoint exists (not counted as a recovery);
        the text only says that a diverged dense run is lost, which a rewind avoids.
    """
    gate: float = CKPT_GATE
    watch_steps: int = WATCH_STEPS
    rebound: float = REBOUND
    max_recoveries: int = MAX_RECOVERIES
    ckpt_loss: float | None = None
    best: float = math.inf
    watch_left: int = 0
    recoveries: int = 0
    history: list = field(default_factory=list)

    def observe(self, loss: float) -> Action:
        loss = float(loss)
        act = self._decide(loss)
        self.history.append(act.event)
        return act

    def _gate(self, loss: float) -> bool:
        return self.ckpt_loss is None or abs(loss - self.ckpt_loss) <= self.gate * self.ckpt_loss

    def _decide(self, loss: float) -> Action:
        if not math.isfinite(loss):
            return Action(restore=True, skip=True, event="rewind") if self.ckpt_loss is not None else Action()
        if loss < self.best:                                 # a fresh low starts a watch
            self.best = loss
            self.watch_left = self.watch_steps
            self.recoveries = 0
            if self._gate(loss):
                self.ckpt_loss = loss
                return Action(save=True, event="watch")
            return Action(event="watch")
        if self.watch_left > 0:
            self.watch_left -= 1
            if self.watch_left > 0:
                return Action()
            if loss > (1.0 + self.rebound) * self.best:      # watch over: the loss rebounded
                if self.recoveries < self.max_recoveries:
                    self.recoveries += 1
                    self.watch_left = self.watch_steps
                    return Action(restore=True, skip=True, event="rewind")
                self.best = loss                             # recoveries used up: accept as is
                self.ckpt_loss = loss
                return Action(save=True, event="exhausted")
            self.ckpt_loss = self.best
            return Action(event="accept")
        if self._gate(loss):
            self.ckpt_loss = loss
            return Action(save=True, event="save")
        return Action()


# ---------------------------------------------------------------------------------------------
# section 2.5: the loss trend and the Fibonacci stride
# ---------------------------------------------------------------------------------------------

@dataclass
class LossTrend:
    """Exponentially weighted mean C of the loss changes, decay length TREND_DECAY steps.

    dL_i = L(t-i-1) - L(t-i) is the change i steps ago, positive when the loss falls;
    C = sum_i w^i dL_i / sum_i w^i with w = exp(-1 / TREND_DECAY), over every change seen so far
    (the normalisation keeps C an average while the history is short). The smoothed copy S that
    drives the stride is the same kind of mean taken over C (reading: same decay length)."""
    decay: float = TREND_DECAY
    num: float = 0.0
    den: float = 0.0
    s_num: float = 0.0
    s_den: float = 0.0
    last: float | None = None

    @property
    def w(self) -> float:
        return math.exp(-1.0 / self.decay)

    def push(self, loss: float):
        loss = float(loss)
        if self.last is not None and math.isfinite(loss):
            d = self.last - loss
            self.num = self.w * self.num + d
            self.den = self.w * self.den + 1.0
            self.s_num = self.w * self.s_num + self.value
            self.s_den = self.w * self.s_den + 1.0
        if math.isfinite(loss):
            self.last = loss

    @property
    def value(self) -> float:
        return self.num / self.den if self.den else 0.0

    @property
    def smoothed(self) -> float:
        return self.s_num / self.s_den if self.s_den else 0.0


@dataclass
class Stride:
    """Fibonacci stride: up one rung while the smoothed trend is above a small positive threshold,
    down one rung while it is negative, held in between; back to 1 after a rewind."""
    rungs: list = field(default_factory=fibonacci_rungs)
    k: int = 0

    @property
    def value(self) -> int:
        return self.rungs[self.k]

    def step(self, smoothed: float, threshold: float):
        if smoothed > threshold:
            self.k = min(self.k + 1, len(self.rungs) - 1)
        elif smoothed < 0.0:
            self.k = max(self.k - 1, 0)

    def reset(self):
        self.k = 0


# ---------------------------------------------------------------------------------------------
# section 2.4: the slow non-periodic phase psi (a point stepping along an elliptic curve)
# ---------------------------------------------------------------------------------------------

@dataclass
class CurveWalk:
    """Walk P_{k+1} = P_k + G on the real curve y^2 = x^3 + b (chord-and-tangent addition).

    Reading: the curve y^2 = x^3 + 17 with G = (-2, 3), a rational point of infinite order, so
    the walk never returns to a point it visited (over the reals the group of the curve's one
    component is a circle and G turns it by an angle that is not a rational multiple of a turn).
    The walk takes one step per completed turn of the phase (slow), and psi is the direction of
    the point seen from the origin, scaled to a tenth of a rung."""
    b: float = 17.0
    gx: float = -2.0
    gy: float = 3.0
    x: float = -2.0
    y: float = 3.0
    amplitude_deg: float = RUNG_DEG / 10.0

    def on_curve_residual(self) -> float:
        return self.y * self.y - (self.x ** 3 + self.b)

    def advance(self):
        x1, y1, x2, y2 = self.x, self.y, self.gx, self.gy
        if x1 == x2:
            if y1 == -y2:                      # P + (-P): restart from G
                self.x, self.y = self.gx, self.gy
                return
            lam = 3.0 * x1 * x1 / (2.0 * y1)   # tangent (the curve has no x term)
        else:
            lam = (y2 - y1) / (x2 - x1)
        x3 = lam * lam - x1 - x2
        y3 = lam * (x1 - x3) - y1
        # keep the point on the curve against rounding drift: recompute |y| from x
        r = x3 ** 3 + self.b
        if r > 0.0:
            y3 = math.copysign(math.sqrt(r), y3)
        self.x, self.y = x3, y3

    @property
    def psi_deg(self) -> float:
        return self.amplitude_deg * self.y / math.hypot(self.x, self.y)


# ---------------------------------------------------------------------------------------------
# the schedule
# ---------------------------------------------------------------------------------------------

@dataclass
class Coupling:
    phi_deg: float
    psi_deg: float
    exposure: float
    w_plus: float
    w_minus: float
    c_self: float
    c_partner: dict                      # pair name -> coefficient on the partner's gradient
    wd_scale: float                      # cos(pitch): multiplies the weight decay


@dataclass
class Helix:
    """The phase, stride, trend and channel weights of sections 2.4 and 2.5.

    Per step: push the previous step's loss, then read `coefficients()` for the pair mix and
    `wd_scale` for the decay. `rewind()` resets the stride to 1 (section 2.6)."""
    threshold_rel: float = 1e-3          # "small positive threshold", relative to the loss (reading)
    trend: LossTrend = field(default_factory=LossTrend)
    stride: Stride = field(default_factory=Stride)
    walk: CurveWalk = field(default_factory=CurveWalk)
    phi_deg: float = 0.0                 # unwrapped phase
    turns_done: int = 0

    def push_loss(self, loss: float):
        """Take the previous step's loss and advance the phase by 36 degrees x stride."""
        self.trend.push(loss)
        scale = abs(self.trend.last) if self.trend.last else 1.0
        self.stride.step(self.trend.smoothed, self.threshold_rel * scale)
        self.phi_deg += RUNG_DEG * self.stride.value
        while self.phi_deg >= 360.0 * (self.turns_done + 1):
            self.turns_done += 1
            self.walk.advance()

    def rewind(self):
        self.stride.reset()

    def channel_weights(self) -> tuple[float, float]:
        """Primary and secondary channel weights (reading).

        Descent confidence kappa = clamp(C / threshold, 0, 1): 1 while the trend is clearly
        falling (weights 1.833 : 1), 0 on a plateau or a rise, where the secondary weight grows to
        match the primary. The slow counters modulate the primary by +-10% over one turn and the
        secondary by +-5% over ten turns."""
        scale = abs(self.trend.last) if self.trend.last else 1.0
        thr = self.threshold_rel * scale
        kappa = min(max(self.trend.value / thr, 0.0), 1.0) if thr > 0 else 0.0
        w_plus = CHANNEL_RATIO
        w_minus = 1.0 + (CHANNEL_RATIO - 1.0) * (1.0 - kappa)
        turn = math.radians(self.phi_deg)
        w_plus *= 1.0 + TURN_MOD * math.cos(turn)
        w_minus *= 1.0 + TEN_TURN_MOD * math.cos(turn / 10.0)
        return w_plus, w_minus

    def coefficients(self, strength: dict | None = None) -> Coupling:
        """Mix of each pair (reading; parity unpinned).

        exposure e = cos^2((phi + psi) / 2) sweeps 1 -> 0 -> 1 once a turn; the primary channel
        shares the partner's gradient in proportion to e, the secondary leans against it in
        proportion to 1 - e:
            g~_self = g_self + b * (w+ * e - w- * (1 - e)) / (w+ + w-) * g_partner
        so over each turn a pair goes from strongly shared to mostly its own gradient and past it,
        the primary dominates while the loss falls, and b = 0 is plain Adam."""
        strength = STRENGTH if strength is None else strength
        psi = self.walk.psi_deg
        e = math.cos(math.radians(self.phi_deg + psi) / 2.0) ** 2
        wp, wm = self.channel_weights()
        mix = (wp * e - wm * (1.0 - e)) / (wp + wm)
        return Coupling(phi_deg=self.phi_deg % 360.0, psi_deg=psi, exposure=e, w_plus=wp, w_minus=wm,
                        c_self=1.0, c_partner={k: b * mix for k, b in strength.items()},
                        wd_scale=math.cos(math.radians(PITCH_DEG)))


# ---------------------------------------------------------------------------------------------
# driving the device checkpoint from the policy
# ---------------------------------------------------------------------------------------------

class Rewinder:
    """Binds a RewindPolicy (and optionally a Helix schedule) to device checkpoints of a list of
    matrices: `before_step(loss)` takes the previous step's loss, saves or restores through the
    C ABI as the policy says, and returns the Action (skip means: do not apply this step)."""

    def __init__(self, mats, policy: RewindPolicy | None = None, helix: Helix | None = None,
                 device="cuda"):
        from . import binding as sf
        self.sf = sf
        self.mats = list(mats)
        self.policy = policy or RewindPolicy()
        self.helix = helix
        self.ckpts = [sf.Checkpoint(m.mask.slot_cap if m.mask.slot_cap else m.R, m.C, device)
                      for m in self.mats]
        self.saved = False
        self._args = None                  # ctypes argument arrays, built once (pointers are fixed)

    def structs(self):
        return [self.sf.matrix_struct(m) for m in self.mats]

    def _call(self, name, status, stream):
        sf = self.sf
        if not hasattr(sf, "load"):        # a stand-in binding (host tests): plain calls
            getattr(sf, name)(self.structs(), self.ckpts, status, stream)
            return
        if getattr(self, "_args", None) is None:
            n = len(self.mats)
            self._args = ((sf.sf_matrix * n)(*self.structs()),
                          (sf.sf_checkpoint * n)(*[c.struct() for c in self.ckpts]), n)
        mats, cks, n = self._args
        st = status if status is None or isinstance(status, int) else status.data_ptr()
        sm = stream if stream is None or isinstance(stream, int) else stream.cuda_stream
        sf._check(getattr(sf.load(), name)(mats, cks, n, st, sm), name)

    def save(self, status=None, stream=None):
        self._call("sf_checkpoint_save", status, stream)
        self.saved = True

    def restore(self, status=None, stream=None):
        self._call("sf_checkpoint_restore", status, stream)

    def before_step(self, loss: float, status=None, stream=None) -> Action:
        act = self.policy.observe(loss)
        if act.restore and self.saved:
            self.restore(status, stream)
            if self.helix is not None:
                self.helix.rewind()
        elif act.restore:
            act = Action(event="")
        if act.save:
            self.save(status, stream)
        if self.helix is not None and not act.skip:
            self.helix.push_loss(loss)
        return act
