"""Seeded synthetic inputs for the sparse step.

This module only draws numbers: token streams, activations, upstream gradients, weights and
explicit masks. It holds none of the step's arithmetic (no charge rule, no quantisation, no
optimizer), so that both the CUDA path and the CPU oracle can take their inputs from here
without sharing any of the computation they are compared on.

Shapes and distributions follow the workloads of "Sparse-First Fine-Tuning" (tensorwirelabs.com):
7B-shaped projections (4,096 wide, feed-forward 11,008), a 32,000-row embedding, fine-tuning
batches whose active share is near 1% (section 1), token ids with a Zipf(1.1) law. No dataset
is involved; the pages' own fine-tuning samples are not available, and these draws stand in
for them.

Host-side draws use numpy PCG64 streams keyed by (seed, purpose, index). Large device-side
draws use a seeded torch CUDA generator; the oracle reads those back to the host, so an input
always has exactly one source.
"""
from __future__ import annotations

import numpy as np

# Purpose tags keep the independent streams of one seed apart.
_TAG = {
    "weights": 1, "dx": 2, "act": 3, "tokens": 4, "dy": 5, "mask": 6, "tracker": 7,
    "grad": 8, "rows": 9, "misc": 10,
}


def rng(seed: int, purpose: str, *index: int) -> np.random.Generator:
    """Independent PCG64 stream for (seed, purpose, index...)."""
    return np.random.Generator(np.random.PCG64([int(seed), _TAG[purpose], *map(int, index)]))


# ---------------------------------------------------------------------------------------------
# Number-format helpers (data formatting only).
# ---------------------------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), rounded to nearest even by torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) drawn in fp32, stored as bf16 bits."""
    return f32_to_bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(std))


# ---------------------------------------------------------------------------------------------
# Token streams.
# ---------------------------------------------------------------------------------------------

def zipf_cdf(V: int, a: float = 1.1) -> np.ndarray:
    """CDF of the Zipf law truncated to V ids: P(id = k-1) proportional to k^-a."""
    w = np.arange(1, V + 1, dtype=np.float64) ** (-a)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_ids(g: np.random.Generator, n: int, V: int, a: float = 1.1,
             rank_to_id: np.ndarray | None = None) -> np.ndarray:
    """n token ids by inverse CDF. rank_to_id maps Zipf rank -> token id (identity if None)."""
    u = g.random(n)
    ranks = np.minimum(np.searchsorted(zipf_cdf(V, a), u, side="right"), V - 1)
    ids = ranks if rank_to_id is None else rank_to_id[ranks]
    return ids.astype(np.int32)


def drift_rank_map(g: np.random.Generator, rank_to_id: np.ndarray, frac: float) -> np.ndarray:
    """Swap a fraction of ranks pairwise (the drifting token stream of the full-model run)."""
    out = rank_to_id.copy()
    k = max(2, int(round(frac * len(out))) // 2 * 2)
    pick = g.choice(len(out), size=k, replace=False)
    a, b = pick[: k // 2], pick[k // 2:]
    out[a], out[b] = rank_to_id[b], rank_to_id[a]
    return out


# ---------------------------------------------------------------------------------------------
# Masks, rows and weights.
# ---------------------------------------------------------------------------------------------

def words_from_rows(R: int, rows) -> np.ndarray:
    """Pack a set of rows into uint32 words, bit i of word w = row 32w+i."""
    words = np.zeros(R // 32, dtype=np.uint32)
    for r in np.asarray(rows, dtype=np.int64).ravel():
        words[r // 32] |= np.uint32(1) << np.uint32(r % 32)
    return words


def rows_from_words(words: np.ndarray) -> np.ndarray:
    bits = np.unpackbits(np.asarray(words, dtype="<u4").view(np.uint8), bitorder="little")
    return np.nonzero(bits)[0].astype(np.int32)


def tiny_projection_mask(seed: int = 0, R: int = 256, p: float = 0.03) -> np.ndarray:
    """Tiny-projection mask: Bernoulli(p) rows, tile 0 forced full, tiles 3.. forced empty.

    Tiles 1 and 2 keep their draws; if both came out empty, row 40 is forced on so that the
    mask has a partially active tile.
    """
    g = rng(seed, "mask")
    act = g.random(R) < p
    act[0:32] = True
    act[96:] = False
    if not act[32:96].any():
        act[40] = True
    return words_from_rows(R, np.nonzero(act)[0])


def scattered_rows(g: np.random.Generator, R: int, frac: float) -> np.ndarray:
    """round(frac * R) rows (at least one) drawn uniformly without replacement, ascending."""
    k = max(1, int(round(frac * R)))
    return np.sort(g.choice(R, size=k, replace=False)).astype(np.int32)


def clustered_rows(g: np.random.Generator, R: int, frac: float) -> np.ndarray:
    """Whole 32-row tiles drawn at random until at least frac * R rows are chosen."""
    need = max(1, int(np.ceil(frac * R)))
    tiles = g.permutation(R // 32)[: (need + 31) // 32]
    rows = (np.sort(tiles)[:, None] * 32 + np.arange(32)[None, :]).ravel()
    return rows.astype(np.int32)


def weights_f32(g: np.random.Generator, R: int, C: int, std: float = 0.02) -> np.ndarray:
    return g.standard_normal((R, C), dtype=np.float32) * np.float32(std)


def tracker_gains(R: int, rows, hi: float = 1.0, lo: float = 1e-3) -> np.ndarray:
    """Per-row output gain: hi on the chosen rows, lo elsewhere.

    With Y = N(0,1) * gain, an unchosen row's largest |Y| is about lo / hi of the busiest row's,
    far below a 1% share, so the tracker turns exactly the chosen rows on.
    """
    gain = np.full(R, lo, dtype=np.float32)
    gain[np.asarray(rows, dtype=np.int64)] = hi
    return gain


def tracker_outputs(g: np.random.Generator, T: int, gains: np.ndarray) -> np.ndarray:
    """Forward outputs Y[T x R] = N(0,1) * gain[r], as bf16 bits."""
    z = g.standard_normal((T, len(gains)), dtype=np.float32)
    return f32_to_bf16_bits(z * gains[None, :])


# ---------------------------------------------------------------------------------------------
# Device-side draws for the large workloads (torch CUDA generator, seeded).
# ---------------------------------------------------------------------------------------------

def device_generator(seed: int, purpose: str, *index: int, device="cuda"):
    import torch
    key = np.random.SeedSequence([int(seed), _TAG[purpose], *map(int, index)]).generate_state(1)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(key[0]))
    return gen


def device_normal_bf16(shape, seed: int, purpose: str, *index: int, std: float = 1.0,
                       device="cuda", out=None):
    """bf16 N(0, std^2) on the device (drawn in fp32, rounded to bf16)."""
    import torch
    gen = device_generator(seed, purpose, *index, device=device)
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if out is None:
        return x.to(torch.bfloat16)
    out.copy_(x)
    return out


def device_weights_f32(R: int, C: int, seed: int, *index: int, std: float = 0.02, device="cuda"):
    import torch
    gen = device_generator(seed, "weights", *index, device=device)
    return torch.randn((R, C), generator=gen, device=device, dtype=torch.float32).mul_(std)


# ---------------------------------------------------------------------------------------------
# The 7B-shaped step workload: per-projection chosen rows, one bank of step inputs, token stream.
# ---------------------------------------------------------------------------------------------

LAYER_INPUTS = ("x_attn", "attn_out", "x_ffn", "ffn_mid")


def chosen_rows(seed: int, layer: int, idx: int, R: int, kind: str, bank: int) -> np.ndarray:
    """Rows a projection's tracker should find active (~1%): `kind` is "scattered" (single
    rows) or "clustered" (whole 32-row tiles). Bank 1 drifts ~5% of bank 0's choice."""
    g = rng(seed, "rows", layer, idx)
    rows = scattered_rows(g, R, 0.01) if kind == "scattered" else clustered_rows(g, R, 0.01)
    if bank == 1:
        g2 = rng(seed, "rows", layer, idx, 1)
        if kind == "scattered":
            k = max(1, int(round(0.05 * len(rows))))
            keep = np.sort(g2.choice(len(rows), len(rows) - k, replace=False))
            pool = np.setdiff1d(np.arange(R), rows)
            rows = np.sort(np.concatenate([rows[keep], g2.choice(pool, k, replace=False)]))
        else:
            tiles = np.unique(rows // 32)
            k = int(round(0.05 * len(tiles)))
            if k:
                pool = np.setdiff1d(np.arange(R // 32), tiles)
                tiles = np.sort(np.concatenate([g2.choice(tiles, len(tiles) - k, replace=False),
                                                g2.choice(pool, k, replace=False)]))
                rows = (tiles[:, None] * 32 + np.arange(32)[None, :]).ravel()
    return rows.astype(np.int64)


def step_bank(projs, T: int, kind: str, bank: int, seed: int, hidden: int = 4096, device="cuda"):
    """Device-resident inputs of one step for projections [(layer, name, R, C, input_name)]:
    tracker outputs Y [T x R], output gradients dX [T x R], layer inputs A [T x C] (shared by the
    projections that read the same input), and the embedding's upstream gradient dY [T x hidden]."""
    import torch
    Ys, dXs, As = [], [], []
    inputs = {}
    for i, (layer, name, R, C, inp) in enumerate(projs):
        key = (layer, inp)
        if key not in inputs:
            inputs[key] = device_normal_bf16((T, C), seed, "act", bank, layer, LAYER_INPUTS.index(inp),
                                             device=device)
        As.append(inputs[key])
        gain = torch.from_numpy(tracker_gains(R, chosen_rows(seed, layer, i, R, kind, bank))).to(device)
        gen = device_generator(seed, "tracker", bank, i, device=device)
        z = torch.randn((T, R), generator=gen, device=device, dtype=torch.float32)
        Ys.append(z.mul_(gain[None, :]).to(torch.bfloat16))
        del z
        dXs.append(device_normal_bf16((T, R), seed, "dx", bank, i, device=device))
    dY = device_normal_bf16((T, hidden), seed, "dy", bank, device=device)
    return {"Y": Ys, "dX": dXs, "A": As, "dY": dY, "tokens": None, "distinct_A": list(inputs.values())}


def token_stream(seed: int, n_windows: int, T: int, V: int = 32000, drift: float = 0.01) -> np.ndarray:
    """n_windows batches of T token ids, Zipf(1.1) with a rank->id map drifting per window."""
    g = rng(seed, "tokens")
    rank_to_id = np.arange(V)
    out = []
    for _ in range(n_windows):
        rank_to_id = drift_rank_map(g, rank_to_id, drift)
        out.append(zipf_ids(g, T, V, 1.1, rank_to_id))
    return np.stack(out)
