"""A transformer's worth of sparse-first state and the four calls of one training step.

"Sparse-First Fine-Tuning" (tensorwirelabs.com): a step derives per-row masks (section 2.1),
computes the masked weight gradients (2.2) and the embedding-row gradient, and applies the
fused update with the coupled pairs gate-up, query-output and key-value (2.3, 2.4). The down
projection has no partner in a 7-projection layer and takes the plain (uncoupled) update.

`SparseModel` owns the device state of every matrix (int8 + scale + residual weights, bf16 live
copy, fp16 moments and fp32 gradients for slot rows, masks) and `StepPlan` holds the ABI
argument arrays of one step, built once, so that issuing a step costs four C calls.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import binding as sf

LLAMA_7B_LAYER = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                  ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))
PARTNER = {"q": "o", "o": "q", "k": "v", "v": "k", "gate": "up", "up": "gate"}
PAIR_OF = {"q": "q-o", "o": "q-o", "k": "k-v", "v": "k-v", "gate": "gate-up", "up": "gate-up"}
# coupling strength of each pair (section 2.4): strong for gate-up, weaker for attention pairs
STRENGTH = {"gate": 0.6, "up": 0.6, "q": 0.4, "o": 0.4, "k": 0.4, "v": 0.4}
# which layer input each projection reads: attention input, attention output, FFN input, FFN mid
INPUT_OF = {"q": "x_attn", "k": "x_attn", "v": "x_attn", "o": "attn_out", "gate": "x_ffn",
            "up": "x_ffn", "down": "ffn_mid"}


@dataclass
class Proj:
    layer: int
    name: str
    mat: sf.Matrix


class SparseModel:
    """Device state of an embedding table plus n_layers x 7 projections."""

    def __init__(self, n_layers: int, vocab: int = 32000, hidden: int = 4096, ffn: int = 11008,
                 slot_frac: float = 0.03, emb_slots: int = 4096, device="cuda",
                 layer_shapes=None):
        self.device = device
        shapes = layer_shapes or tuple((n, ffn if R == 11008 else hidden, ffn if C == 11008 else hidden)
                                       for n, R, C in LLAMA_7B_LAYER)
        self.shapes = shapes
        self.emb = sf.Matrix(vocab, hidden, min(vocab, emb_slots), device) if vocab else None
        self.projs: list[Proj] = []
        for layer in range(n_layers):
            for name, R, C in shapes:
                cap = min(R, max(32, int(math.ceil(slot_frac * R))))
                self.projs.append(Proj(layer, name, sf.Matrix(R, C, cap, device)))
        self.index = {(p.layer, p.name): i for i, p in enumerate(self.projs)}
        # all masks' counts in one contiguous block (one copy reads every mask's statistics)
        mats = ([self.emb] if self.emb is not None else []) + [p.mat for p in self.projs]
        self.counts = torch.zeros((len(mats), 8), dtype=torch.int32, device=device)
        for i, m in enumerate(mats):
            m.mask.counts = self.counts[i]
        self.all_mats = mats

    @property
    def n_params(self) -> int:
        return sum(m.R * m.C for m in self.all_mats)

    def state_bytes(self) -> int:
        total = 0
        for m in self.all_mats:
            for t in (m.q, m.s, m.delta, m.m, m.v, m.grad, m.live):
                if t is not None:
                    total += t.numel() * t.element_size()
        return total

    def init(self, seed: int, std: float = 0.02, stream=None):
        """Random-init fp32 weights (seeded, on the device), quantise them, reset every mask."""
        from . import synth
        for i, m in enumerate(self.all_mats):
            W = synth.device_weights_f32(m.R, m.C, seed, i, std=std, device=self.device)
            sf.sf_quantize_init(W, m, stream)
            sf.sf_mask_init(m.mask, stream)
            del W

    def partner_index(self, i: int) -> int:
        """Index (in the update list, embedding first) of projection i's partner, or -1."""
        p = self.projs[i]
        other = PARTNER.get(p.name)
        if other is None:
            return -1
        off = 1 if self.emb is not None else 0
        return self.index[(p.layer, other)] + off


def dw_launch_count(problems, group_bytes=320, prob_bytes=192, payload=32640, max_per_launch=96,
                    max_per_group=8) -> int:
    """Launches sf_masked_dw splits a call into: consecutive problems reading the same input form
    a group, and groups are packed into kernel-parameter payloads of `payload` bytes, evenly.
    problems: [(input identity, C)] in call order."""
    groups = []
    for key in problems:
        if groups and groups[-1][0] == key and groups[-1][1] < max_per_group:
            groups[-1][1] += 1
        else:
            groups.append([key, 1])
    sizes = [group_bytes + n * prob_bytes for _, n in groups]
    n_launch = max(1, -(-sum(sizes) // payload))
    gi, li, launches = 0, 0, 0
    while gi < len(groups):
        left = sum(sizes[gi:])
        target = -(-left // max(1, n_launch - li))
        used, np_, g_end = 0, 0, gi
        while g_end < len(groups):
            add = sizes[g_end]
            if g_end > gi and (used + add > payload or used >= target):
                break
            if g_end - gi + 1 > max_per_launch or np_ + groups[g_end][1] > max_per_launch:
                break
            used += add
            np_ += groups[g_end][1]
            g_end += 1
        if g_end < len(groups) and li + 1 >= n_launch:
            n_launch += 1
        gi, li, launches = g_end, li + 1, launches + 1
    return launches


def dw_gather_launch_count(problems, max_groups=192, max_probs=384, max_per_group=8) -> int:
    """Launches of the row gather that sf_masked_dw issues when given a workspace: the call's
    groups (consecutive problems reading the same input, at most max_per_group) packed in order
    into launches of at most max_groups groups and max_probs problems. problems: [(input, C)]."""
    groups = []
    for key in problems:
        if groups and groups[-1][0] == key and groups[-1][1] < max_per_group:
            groups[-1][1] += 1
        else:
            groups.append([key, 1])
    launches, ng, npb = 0, 0, 0
    for _, cnt in groups:
        if ng == 0 or ng >= max_groups or npb + cnt > max_probs:
            launches += 1
            ng, npb = 0, 0
        ng += 1
        npb += cnt
    return launches


def mask_launch_count(rows) -> int:
    """Launches of one sf_mask_update call over masks of the given row counts (all sources that
    accumulate: tokens or outputs). Per batch of SF_MASKS_PER_LAUNCH masks: the accumulate pass,
    then a one-launch finalize, or a three-launch one (busiest row, charges, lists) when the batch
    holds a mask of SF_MASK_SPLIT_ROWS rows or more."""
    k, n = sf.SF_MASKS_PER_LAUNCH, 0
    for b in range(0, len(rows), k):
        n += 1 + (3 if max(rows[b:b + k]) >= sf.SF_MASK_SPLIT_ROWS else 1)
    return n


class StepPlan:
    """ABI argument arrays of one step over `model` for one set of input buffers.

    inputs: dict with
      tokens  int32 [n] device      (None: no embedding stage)
      dY      bf16 [n x hidden]     upstream gradient of the embedding output
      Y       list per projection: bf16 [T x R] forward outputs (row tracker input)
      dX      list per projection: bf16 [T x R] upstream gradients of the outputs
      A       list per projection: bf16 [T x C] inputs
    """

    def __init__(self, model: SparseModel, inputs: dict, embed_ws: torch.Tensor | None,
                 threshold: float = 0.01, proj_range: tuple[int, int] | None = None,
                 with_embedding: bool = True):
        """proj_range: the projections [i0, i1) this plan covers (default: all); with_embedding:
        whether the embedding matrix's mask, gradient and update belong to this plan."""
        self.model, self.inputs, self.threshold = model, inputs, threshold
        L = sf.load()
        self.lib = L
        i0, i1 = proj_range if proj_range is not None else (0, len(model.projs))
        self.i0, self.i1 = i0, i1
        self.has_emb = with_embedding and model.emb is not None
        projs = list(enumerate(model.projs))[i0:i1]
        mats = ([model.emb] if self.has_emb else []) + [p.mat for _, p in projs]
        n = len(mats)
        self.n_masks = n
        self.mask_arr = (sf.sf_mask * n)(*[m.mask.struct() for m in mats])
        srcs = []
        if self.has_emb:
            tok = inputs["tokens"]
            srcs.append(sf.sf_mask_src(sf.SF_SRC_TOKENS, tok.numel(), 0, tok.data_ptr()))
        for i, p in projs:
            Y = inputs["Y"][i]
            srcs.append(sf.sf_mask_src(sf.SF_SRC_OUTPUT_BF16, Y.shape[0], Y.stride(0), Y.data_ptr()))
        self.src_arr = (sf.sf_mask_src * n)(*srcs)
        off = 1 if self.has_emb else 0             # the trackers alone, for a split masks stage
        self.proj_mask_arr = (sf.sf_mask * max(n - off, 1))(*[m.mask.struct() for m in mats[off:]])
        self.proj_src_arr = (sf.sf_mask_src * max(n - off, 1))(*srcs[off:])
        probs = [sf.dw_problem(inputs["dX"][i], inputs["A"][i], p.mat.mask, p.mat.grad).c for i, p in projs]
        self.n_dw = len(probs)
        self.dw_arr = (sf.sf_dw_problem * max(len(probs), 1))(*probs)
        self.dw_ws = torch.empty(max(L.sf_masked_dw_ws_bytes(self.dw_arr, self.n_dw), 1), dtype=torch.uint8,
                                 device=model.device)
        structs = []
        off = 1 if self.has_emb else 0
        if self.has_emb:
            structs.append(sf.matrix_struct(model.emb))
        for i, p in projs:
            g = model.partner_index(i)             # index in the whole-model list (embedding first)
            if g >= 0:
                g = g - (1 if model.emb is not None else 0) - i0 + off
                assert off <= g < off + len(projs), "pairs must not straddle plans"
            structs.append(sf.matrix_struct(p.mat, g, 1.0, 0.0))
        self.upd_arr = (sf.sf_matrix * len(structs))(*structs)
        self.embed_ws = embed_ws
        keys = [(id(inputs["A"][i]), p.mat.C) for i, p in projs]
        self.dw_launches = dw_launch_count(keys) if projs else 0
        self.gather_launches = dw_gather_launch_count(keys) if projs else 0
        if self.has_emb:
            self.emb_mask = model.emb.mask.struct()

    def set_tokens(self, tokens: torch.Tensor):
        """Point the conductor and the embedding stage at another token batch (same length)."""
        self.inputs["tokens"] = tokens
        if self.has_emb:
            self.src_arr[0].ptr = tokens.data_ptr()

    def set_coupling(self, phase_deg: float):
        """Rotate every pair's mix: c_partner = strength * cos(phase) (section 2.4; the pages'
        exact coefficient formula is not in the extracted text)."""
        off = 1 if self.has_emb else 0
        c = math.cos(math.radians(phase_deg))
        for k, p in enumerate(self.model.projs[self.i0:self.i1]):
            self.upd_arr[k + off].c_partner = STRENGTH.get(p.name, 0.0) * c

    def set_mix(self, c_self: float, c_partner: dict):
        """Per-pair coefficients from a schedule (helix.Helix.coefficients): c_partner maps a
        pair name ("q-o", "k-v", "gate-up") to the weight of the partner's gradient."""
        off = 1 if self.has_emb else 0
        for k, p in enumerate(self.model.projs[self.i0:self.i1]):
            pair = PAIR_OF.get(p.name)
            self.upd_arr[k + off].c_self = c_self
            self.upd_arr[k + off].c_partner = c_partner.get(pair, 0.0) if pair else 0.0

    # the four calls of one step --------------------------------------------------------------
    def masks_embedding(self, status, stream):
        """The conductor alone (the embedding's mask), as its own call."""
        if not self.has_emb:
            return
        sf._check(self.lib.sf_mask_update(self.mask_arr, self.src_arr, 1, self.threshold, status, stream),
                  "sf_mask_update")

    def masks_projections(self, status, stream, phase: int = sf.SF_PHASE_ALL):
        """The row trackers of every projection of the plan, as one call (or one of its passes)."""
        off = 1 if self.has_emb else 0
        n = self.n_masks - off
        if n <= 0:
            return
        sf._check(self.lib.sf_mask_update_phase(self.proj_mask_arr, self.proj_src_arr, n, self.threshold, phase,
                                                status, stream), "sf_mask_update")

    def masks(self, status, stream):
        sf._check(self.lib.sf_mask_update(self.mask_arr, self.src_arr, self.n_masks, self.threshold,
                                          status, stream), "sf_mask_update")

    def dw(self, status, stream, phase: int = sf.SF_PHASE_ALL):
        if self.n_dw == 0:
            return
        sf._check(self.lib.sf_masked_dw_phase(self.dw_arr, self.n_dw, self.dw_ws.data_ptr(), self.dw_ws.numel(),
                                              phase, status, stream), "sf_masked_dw")

    def embed(self, status, stream):
        if not self.has_emb:
            return
        tok, dY, G = self.inputs["tokens"], self.inputs["dY"], self.model.emb.grad
        ws = self.embed_ws
        sf._check(self.lib.sf_embed_grad(tok.data_ptr(), tok.numel(), dY.data_ptr(), dY.shape[1],
                                         dY.stride(0), ctypes.byref(self.emb_mask), G.data_ptr(),
                                         G.stride(0), ws.data_ptr(), ws.numel() * ws.element_size(),
                                         status, stream), "sf_embed_grad")

    def update(self, hp: sf.AdamParams, status, stream):
        h = hp.struct()
        sf._check(self.lib.sf_sparse_update(self.upd_arr, len(self.upd_arr), ctypes.byref(h), status,
                                            stream), "sf_sparse_update")

    def launches(self, split_embedding: bool = False) -> int:
        """Kernel launches one step issues (for the launch count of a timed region)."""
        def chunks(n, k):
            return (n + k - 1) // k

        rows = [m.mask.R for m in ([self.model.emb] if self.has_emb else [])] + \
            [p.mat.mask.R for p in self.model.projs[self.i0:self.i1]]
        if split_embedding and self.has_emb:         # conductor and trackers as two calls
            n = mask_launch_count(rows[:1]) + (mask_launch_count(rows[1:]) if len(rows) > 1 else 0)
        else:
            n = mask_launch_count(rows)
        n += self.gather_launches + self.dw_launches  # row gather, then the main dW launches
        n += 3 if self.has_emb else 0                 # embedding index, sort, sum
        n += chunks(len(self.upd_arr), sf.SF_MATS_PER_LAUNCH)
        return n


class Pipeline:
    """One step issued as one call per stage, or as layer chunks over two CUDA streams.

    The projections are cut into `chunks` runs of whole layers (pairs never straddle a cut). Chunk
    c's masks run on a side stream, back to back; its masked dW, the embedding gradient (chunk 0)
    and its update run on the main stream once that chunk's masks are done. So the tracker pass of
    later chunks (a pure HBM stream) overlaps the dW and update of earlier ones, and the short,
    latency-bound mask finalize hides under them. Every matrix's own calls keep their order and
    matrices of different chunks share no state, so the results are those of one call per stage.
    The side stream starts each step only after everything the main stream issued before it.
    Measured on the 32-layer step, chunking is slower (2 chunks +7%, 4 +8%, 8 +19%): the dW
    kernel's persistent CTAs take their units by index, so CTAs that the concurrent tracker pass
    keeps off the SMs start late and stretch the launch, and both streams draw on the same HBM."""

    def __init__(self, model: SparseModel, inputs: dict, embed_ws, chunks: int = 4, threshold: float = 0.01,
                 overlap_embedding: bool = False):
        layers = sorted({p.layer for p in model.projs})
        chunks = max(1, min(chunks, len(layers))) if layers else 1
        bounds = [0]
        for c in range(1, chunks):
            first_layer = layers[(c * len(layers)) // chunks]
            bounds.append(next(i for i, p in enumerate(model.projs) if p.layer == first_layer))
        bounds.append(len(model.projs))
        self.model = model
        self.plans = [StepPlan(model, inputs, embed_ws if c == 0 else None, threshold,
                               proj_range=(bounds[c], bounds[c + 1]), with_embedding=(c == 0))
                      for c in range(chunks)]
        self.side = torch.cuda.Stream(device=model.device)
        self.start = torch.cuda.Event()
        self.masks_done = [torch.cuda.Event() for _ in self.plans]
        # one call per stage, but the embedding's conductor and row gradient on the side stream,
        # concurrent with the projections' trackers and dW; joined before the update
        self.overlap_embedding = overlap_embedding and len(self.plans) == 1 and self.plans[0].has_emb
        self.emb_done = torch.cuda.Event()

    def set_tokens(self, tokens):
        self.plans[0].set_tokens(tokens)

    def set_coupling(self, phase_deg: float):
        for p in self.plans:
            p.set_coupling(phase_deg)

    def set_mix(self, c_self: float, c_partner: dict):
        for p in self.plans:
            p.set_mix(c_self, c_partner)

    def launches(self) -> int:
        return sum(p.launches(self.overlap_embedding) for p in self.plans)

    def step(self, hp: sf.AdamParams, status, main, timing: list | None = None):
        """Issue one step. main: the torch stream the step belongs to; timing: if a list, gets
        (stage, start event, end event) for every call (events on the call's own stream). With the
        embedding on the side stream, the masks and dW calls are then issued pass by pass, each
        pass on its own events ("masks:accum", "masks:finalize", "masked_dw:gather",
        "masked_dw:main"); the passes are the same launches the full calls make."""
        side = self.side
        sp_main, sp_side = main.cuda_stream, side.cuda_stream

        def timed(stage, stream, fn):
            if timing is None:
                fn()
                return
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            timing.append((stage, e0, e1))

        if self.overlap_embedding:
            plan = self.plans[0]
            self.start.record(main)
            side.wait_event(self.start)
            timed("conductor", side, lambda: plan.masks_embedding(status, sp_side))
            timed("embed_grad", side, lambda: plan.embed(status, sp_side))
            self.emb_done.record(side)
            if timing is None:
                plan.masks_projections(status, sp_main)
                plan.dw(status, sp_main)
            else:                                    # each pass of the two-pass calls on its own events
                timed("masks:accum", main, lambda: plan.masks_projections(status, sp_main, sf.SF_PHASE_FIRST))
                timed("masks:finalize", main, lambda: plan.masks_projections(status, sp_main, sf.SF_PHASE_SECOND))
                timed("masked_dw:gather", main, lambda: plan.dw(status, sp_main, sf.SF_PHASE_FIRST))
                timed("masked_dw:main", main, lambda: plan.dw(status, sp_main, sf.SF_PHASE_SECOND))
            main.wait_event(self.emb_done)
            timed("sparse_update", main, lambda: plan.update(hp, status, sp_main))
            return
        if len(self.plans) == 1:                     # one call per stage, all on the main stream
            plan = self.plans[0]
            timed("masks", main, lambda: plan.masks(status, sp_main))
            timed("masked_dw", main, lambda: plan.dw(status, sp_main))
            timed("embed_grad", main, lambda: plan.embed(status, sp_main))
            timed("sparse_update", main, lambda: plan.update(hp, status, sp_main))
            return
        self.start.record(main)
        side.wait_event(self.start)
        for plan, done in zip(self.plans, self.masks_done):
            timed("masks", side, lambda: plan.masks(status, sp_side))
            done.record(side)
        for plan, done in zip(self.plans, self.masks_done):
            main.wait_event(done)
            timed("masked_dw", main, lambda: plan.dw(status, sp_main))
            if plan.has_emb:
                timed("embed_grad", main, lambda: plan.embed(status, sp_main))
            timed("sparse_update", main, lambda: plan.update(hp, status, sp_main))


def capture_step_graphs(pipe: Pipeline, hp: sf.AdamParams, status, token_buf: torch.Tensor,
                        phases_deg) -> dict:
    """One CUDA graph of `pipe`'s step per coupling phase.

    A step's kernel arguments are fixed except for two things, so a handful of graphs cover every
    step: the token ids, read here from `token_buf` (copy each step's ids into it before replay),
    and the pairs' coupling phase, one graph per value in `phases_deg`. The library's calls only
    enqueue work on the given stream, so they capture as they run. Warm the calls up (run a step
    un-captured) before capturing. Returns {phase: torch.cuda.CUDAGraph}."""
    pipe.set_tokens(token_buf)
    graphs = {}
    for ph in phases_deg:
        pipe.set_coupling(ph)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            pipe.step(hp, status, torch.cuda.current_stream())
        graphs[ph] = g
    return graphs


class Trainer:
    """The host loop around the step ("Sparse-First Fine-Tuning", sections 2.4-2.6).

    Each call to `step` takes the loss of the previous step (read after that step, so nothing is
    read back in the middle of one), lets the rewind policy save or restore the active-row
    checkpoint, sets every pair's mix from the Helix schedule, and issues the step on `stream`,
    or skips it when the policy has just rewound. `pipes` are Pipeline objects over the same
    model (e.g. one per input bank); step k uses pipes[k % len(pipes)]."""

    def __init__(self, model: SparseModel, pipes, hp: sf.AdamParams, status, stream=None,
                 policy=None, helix=None, device=None):
        from . import helix as hx
        self.model, self.pipes, self.hp, self.status = model, list(pipes), hp, status
        self.stream = stream
        self.helix = helix if helix is not None else hx.Helix()
        self.rewinder = hx.Rewinder(model.all_mats, policy or hx.RewindPolicy(), self.helix,
                                    device=device or model.device)
        self.events = {}

    def step(self, k: int, prev_loss: float, tokens: torch.Tensor | None = None):
        stream = self.stream if self.stream is not None else torch.cuda.current_stream()
        st = self.status.data_ptr() if hasattr(self.status, "data_ptr") else self.status
        act = self.rewinder.before_step(prev_loss, st, stream.cuda_stream)
        self.events[act.event or "step"] = self.events.get(act.event or "step", 0) + 1
        if act.skip:
            return act
        pipe = self.pipes[k % len(self.pipes)]
        c = self.helix.coefficients()
        pipe.set_mix(c.c_self, c.c_partner)
        if tokens is not None:
            pipe.set_tokens(tokens)
        pipe.step(self.hp, st, stream)
        return act
