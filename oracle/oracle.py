"""numpy front end of the C oracle (sf_oracle.c) -- TEST INFRASTRUCTURE ONLY.

Marshals numpy arrays into the plain C functions and back. Each function names the section of
"Sparse-First Fine-Tuning" (tensorwirelabs.com) that the C code follows; the arithmetic itself
lives in sf_oracle.c. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
use this module.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sf_oracle.c")
_LIB = os.path.join(_HERE, "libsf_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile sf_oracle.c into libsf_oracle.so (gcc, no fused multiply-add contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float


def _declare(L):
    L.orc_bf16_to_f32.restype = _F
    L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_f32_to_bf16.restype = ctypes.c_uint16
    L.orc_f32_to_bf16.argtypes = [_F]
    L.orc_f16_to_f32.restype = _F
    L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_f32_to_f16.restype = ctypes.c_uint16
    L.orc_f32_to_f16.argtypes = [_F]
    L.orc_convert.restype = None
    L.orc_convert.argtypes = [_I, ctypes.c_long, _P, _P]
    L.orc_window_tokens.restype = _I
    L.orc_window_tokens.argtypes = [_I, _P, _P, _I, _F, _P, _P]
    L.orc_window_outputs.restype = _I
    L.orc_window_outputs.argtypes = [_I, _P, _P, _I, _F, _P, _P]
    L.orc_window_activity.restype = None
    L.orc_window_activity.argtypes = [_I, _P, _P, _F, _P]
    L.orc_row_magnitudes.restype = _I
    L.orc_row_magnitudes.argtypes = [_I, _P, _I, _P]
    L.orc_mask_lists.restype = None
    L.orc_mask_lists.argtypes = [_I, _P, _P, _P, _P, _P]
    L.orc_moments_follow_mask.restype = None
    L.orc_moments_follow_mask.argtypes = [_I, _I, _P, _P, _P, _P, _P]
    L.orc_masked_dw.restype = None
    L.orc_masked_dw.argtypes = [_I, _I, _I, _P, _P, _P, _P]
    L.orc_embed_grad.restype = None
    L.orc_embed_grad.argtypes = [_I, _P, _I, _P, _I, _P, _P]
    L.orc_quantize_rows.restype = None
    L.orc_quantize_rows.argtypes = [_I, _I, _P, _P, _P, _P]
    L.orc_rebuild_rows.restype = None
    L.orc_rebuild_rows.argtypes = [_I, _I, _P, _P, _P, _P]
    L.orc_checkpoint_save.restype = _I
    L.orc_checkpoint_save.argtypes = [_I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P]
    L.orc_checkpoint_restore.restype = None
    L.orc_checkpoint_restore.argtypes = [_I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P]
    L.orc_bias_correction.restype = _F
    L.orc_bias_correction.argtypes = [_F, _I]
    L.orc_update.restype = None
    L.orc_update.argtypes = [_I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _F,
                             _F, _F, _F, _F, _F, _F, _F, _F, _P]


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _arr(a, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


# ---- number formats ------------------------------------------------------------------------

def _convert(kind: int, x, in_dtype, out_dtype) -> np.ndarray:
    src = np.ascontiguousarray(np.asarray(x, dtype=in_dtype))
    out = np.empty(src.shape, dtype=out_dtype)
    lib().orc_convert(kind, src.size, _ptr(src), _ptr(out))
    return out


def bf16_to_f32(bits) -> np.ndarray:
    return _convert(0, bits, np.uint16, np.float32)


def f32_to_bf16(x) -> np.ndarray:
    return _convert(1, x, np.float32, np.uint16)


def f16_to_f32(bits) -> np.ndarray:
    return _convert(2, bits, np.uint16, np.float32)


def f32_to_f16(x) -> np.ndarray:
    return _convert(3, x, np.float32, np.uint16)


# ---- section 2.1: charge rule and masks -----------------------------------------------------

def window_tokens(charge: np.ndarray, tokens, thr: float = 0.01):
    """Fold one window of token ids into the charges (in place); returns (words, n_bad_ids)."""
    R = charge.shape[0]
    assert charge.dtype == np.float32 and R % 32 == 0
    tok = _arr(np.asarray(tokens, dtype=np.int32), np.int32)
    words = np.zeros(R // 32, dtype=np.uint32)
    h = np.zeros(R, dtype=np.float32)
    bad = lib().orc_window_tokens(R, _ptr(charge), _ptr(tok), int(tok.size), float(thr),
                                  _ptr(words), _ptr(h))
    return words, bad


def window_outputs(charge: np.ndarray, Y_bf16: np.ndarray, thr: float = 0.01) -> np.ndarray:
    """Fold one window of forward outputs Y[T x R] (bf16 bits) into the charges (in place)."""
    return window_outputs_counted(charge, Y_bf16, thr)[0]


def window_outputs_counted(charge: np.ndarray, Y_bf16: np.ndarray, thr: float = 0.01):
    """window_outputs, also returning how many outputs were not finite: (words, n_nonfinite).
    A NaN output is skipped; an infinite one counts as the largest finite bf16 magnitude."""
    R = charge.shape[0]
    Y = _arr(Y_bf16, np.uint16)
    assert Y.ndim == 2 and Y.shape[1] == R
    words = np.zeros(R // 32, dtype=np.uint32)
    h = np.zeros(R, dtype=np.float32)
    n = lib().orc_window_outputs(R, _ptr(charge), _ptr(Y), int(Y.shape[0]), float(thr),
                                 _ptr(words), _ptr(h))
    return words, int(n)


def window_activity(charge: np.ndarray, h: np.ndarray, thr: float = 0.01) -> np.ndarray:
    """The charge rule applied to activities h[R] given directly (in place on charge)."""
    R = charge.shape[0]
    h = _arr(np.asarray(h, dtype=np.float32), np.float32)
    assert h.shape == (R,)
    words = np.zeros(R // 32, dtype=np.uint32)
    lib().orc_window_activity(R, _ptr(charge), _ptr(h), float(thr), _ptr(words))
    return words


def row_magnitudes(Y_bf16: np.ndarray):
    """The tracker's activities: (h[R] = largest |Y[t, r]| over tokens, non-finite count)."""
    Y = _arr(Y_bf16, np.uint16)
    T, R = Y.shape
    h = np.zeros(R, dtype=np.float32)
    n = lib().orc_row_magnitudes(R, _ptr(Y), T, _ptr(h))
    return h, int(n)


def mask_lists(words: np.ndarray):
    """(active_rows ascending, active_tiles ascending) of a mask."""
    w = _arr(words, np.uint32)
    R = w.size * 32
    rows = np.zeros(R, dtype=np.int32)
    tiles = np.zeros(w.size, dtype=np.int32)
    nr = np.zeros(1, dtype=np.int32)
    nt = np.zeros(1, dtype=np.int32)
    lib().orc_mask_lists(R, _ptr(w), _ptr(rows), _ptr(nr), _ptr(tiles), _ptr(nt))
    return rows[: nr[0]].copy(), tiles[: nt[0]].copy()


def moments_follow_mask(old_words, new_words, m: np.ndarray, v: np.ndarray, step: np.ndarray):
    """Zero the moments and step count of rows whose activity changed (in place)."""
    R, C = m.shape
    lib().orc_moments_follow_mask(R, C, _ptr(_arr(old_words, np.uint32)),
                                  _ptr(_arr(new_words, np.uint32)), _ptr(m), _ptr(v), _ptr(step))


# ---- section 2.2: masked weight gradient, embedding-row gradient ----------------------------

def masked_dw(dX_bf16: np.ndarray, A_bf16: np.ndarray, words: np.ndarray,
              out: np.ndarray | None = None) -> np.ndarray:
    """dW = dX^T A on active rows only (fp64). out (R x C fp64) keeps its other rows."""
    dX = _arr(dX_bf16, np.uint16)
    A = _arr(A_bf16, np.uint16)
    T, R = dX.shape
    T2, C = A.shape
    assert T == T2 and R % 32 == 0
    if out is None:
        out = np.full((R, C), np.nan, dtype=np.float64)
    assert out.shape == (R, C) and out.dtype == np.float64
    lib().orc_masked_dw(T, R, C, _ptr(dX), _ptr(A), _ptr(_arr(words, np.uint32)), _ptr(out))
    return out


def masked_dw_rows(dX_bf16: np.ndarray, A_bf16: np.ndarray, rows) -> np.ndarray:
    """dW[r, :] = sum_t dX[t, r] * A[t, :] for the given rows, in fp64, one output row per entry
    of `rows` (section 2.2's product restricted to chosen rows). The same definition as
    masked_dw, with the fp64 matrix product of numpy as the summation step: the bf16 inputs
    widen exactly, so the only difference from the loop is the order of fp64 additions."""
    dX = _arr(dX_bf16, np.uint16)
    A = _arr(A_bf16, np.uint16)
    T, R = dX.shape
    assert A.shape[0] == T
    rows = np.asarray(rows, dtype=np.int64)
    assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < R))
    wide = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return wide(dX[:, rows]).T @ wide(A)


def forward_product(A_bf16: np.ndarray, W_bf16: np.ndarray) -> np.ndarray:
    """Y = A W^T in fp64 (A [T x C], W [R x C], bf16 bits), the forward projection whose output
    magnitudes the row tracker observes (section 2.1). The bf16 inputs widen exactly; the fp64
    matrix product of numpy is the summation step."""
    A = _arr(A_bf16, np.uint16)
    W = _arr(W_bf16, np.uint16)
    assert A.shape[1] == W.shape[1]
    wide = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return wide(A) @ wide(W).T


def embed_grad(tokens, dY_bf16: np.ndarray, V: int, words: np.ndarray,
               out: np.ndarray | None = None) -> np.ndarray:
    """G[r] = sum of dY rows of the tokens with id r, active rows only (fp64)."""
    tok = _arr(np.asarray(tokens, dtype=np.int32), np.int32)
    dY = _arr(dY_bf16, np.uint16)
    n, H = dY.shape
    assert tok.size == n
    if out is None:
        out = np.full((V, H), np.nan, dtype=np.float64)
    lib().orc_embed_grad(n, _ptr(tok), H, _ptr(dY), V, _ptr(_arr(words, np.uint32)), _ptr(out))
    return out


# ---- section 2.3 / 2.4: quantised storage and the fused update ------------------------------

def quantize_rows(W: np.ndarray):
    """Per-row absmax int8: returns (q int8, s fp32, delta fp32)."""
    W = _arr(W, np.float32)
    R, C = W.shape
    q = np.zeros((R, C), dtype=np.int8)
    s = np.zeros(R, dtype=np.float32)
    d = np.zeros((R, C), dtype=np.float32)
    lib().orc_quantize_rows(R, C, _ptr(W), _ptr(q), _ptr(s), _ptr(d))
    return q, s, d


def rebuild(q: np.ndarray, s: np.ndarray, delta: np.ndarray) -> np.ndarray:
    """W = fma(s, q, delta) per element, fp32 (section 2.3)."""
    q = _arr(q, np.int8)
    R, C = q.shape
    W = np.empty((R, C), dtype=np.float32)
    lib().orc_rebuild_rows(R, C, _ptr(q), _ptr(_arr(s, np.float32)),
                           _ptr(_arr(delta, np.float32)), _ptr(W))
    return W


def bias_correction(beta: float, t: int) -> float:
    return lib().orc_bias_correction(float(beta), int(t))


class AdamHP:
    """Adam hyper-parameters; one_minus_b* are fp32 (1 - beta) as both sides use them."""

    def __init__(self, lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, clip=0.0):
        self.lr, self.beta1, self.beta2, self.eps = map(float, (lr, beta1, beta2, eps))
        self.wd, self.clip = float(wd), float(clip)
        self.one_minus_b1 = float(np.float32(1.0) - np.float32(beta1))
        self.one_minus_b2 = float(np.float32(1.0) - np.float32(beta2))


class MatrixState:
    """Oracle-side state of one matrix: int8 q, scale s, residual delta, fp16 moments by row,
    per-row step counts and the bf16 live weights."""

    def __init__(self, W: np.ndarray):
        R, C = W.shape
        self.R, self.C = R, C
        self.q, self.s, self.delta = quantize_rows(W)
        self.m = np.zeros((R, C), dtype=np.uint16)
        self.v = np.zeros((R, C), dtype=np.uint16)
        self.step = np.zeros(R, dtype=np.int32)
        self.live = np.zeros((R, C), dtype=np.uint16)
        self.words = np.zeros(R // 32, dtype=np.uint32)

    def set_mask(self, words: np.ndarray):
        """Adopt a new row mask: moments follow it (section 2.3)."""
        words = _arr(words, np.uint32)
        moments_follow_mask(self.words, words, self.m, self.v, self.step)
        self.words = words.copy()

    def weight(self) -> np.ndarray:
        """fp32 weight rebuilt as fma(s, q, delta)."""
        return rebuild(self.q, self.s, self.delta)


def update(a: MatrixState, g: np.ndarray, hp: AdamHP, partner: MatrixState | None = None,
           pg: np.ndarray | None = None, c_self: float = 1.0, c_partner: float = 0.0):
    """One fused sparse update of a's active rows (in place)."""
    g = _arr(g, np.float32)
    assert g.shape == (a.R, a.C)
    if partner is not None:
        pg = _arr(pg, np.float32)
        assert pg.shape == (a.R, a.C)
    scratch = np.zeros(a.C, dtype=np.float32)
    lib().orc_update(a.R, a.C, _ptr(a.q), _ptr(a.s), _ptr(a.delta), _ptr(a.m), _ptr(a.v),
                     _ptr(a.step), _ptr(a.live), _ptr(a.words), _ptr(g),
                     None if partner is None else _ptr(partner.words),
                     None if partner is None else _ptr(pg),
                     float(c_self), float(c_partner), hp.lr, hp.beta1, hp.beta2,
                     hp.one_minus_b1, hp.one_minus_b2, hp.eps, hp.wd, hp.clip, _ptr(scratch))


# ---- section 2.6: checkpoint and rewind of the active rows ----------------------------------

class Checkpoint:
    """Snapshot of a MatrixState's active rows (row ids, q, s, delta, m, v, step)."""

    def __init__(self, st: MatrixState, cap: int | None = None):
        cap = st.R if cap is None else cap
        C = st.C
        self.rows = np.zeros(cap, np.int32)
        self.q = np.zeros((cap, C), np.int8)
        self.s = np.zeros(cap, np.float32)
        self.delta = np.zeros((cap, C), np.float32)
        self.m = np.zeros((cap, C), np.uint16)
        self.v = np.zeros((cap, C), np.uint16)
        self.step = np.zeros(cap, np.int32)
        self.n = lib().orc_checkpoint_save(
            st.R, C, _ptr(st.q), _ptr(st.s), _ptr(st.delta), _ptr(st.m), _ptr(st.v), _ptr(st.step),
            _ptr(st.words), cap, _ptr(self.rows), _ptr(self.q), _ptr(self.s), _ptr(self.delta),
            _ptr(self.m), _ptr(self.v), _ptr(self.step))

    def restore(self, st: MatrixState):
        lib().orc_checkpoint_restore(
            st.R, st.C, _ptr(st.q), _ptr(st.s), _ptr(st.delta), _ptr(st.m), _ptr(st.v), _ptr(st.step),
            _ptr(st.live), _ptr(st.words), self.n, _ptr(self.rows), _ptr(self.q), _ptr(self.s),
            _ptr(self.delta), _ptr(self.m), _ptr(self.v), _ptr(self.step))
