"""Python binding of the C ABI in include/sf.h -- argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but turn torch
tensors into pointers and sizes; all work runs in the CUDA kernels of libsf.so. There is no
fallback: if the library is missing or no B200 is present, calls raise.

State holders (`Mask`, `Matrix`) allocate their device arrays with torch (PyTorch serves as the
device-memory and stream provider) and expose the C structs the ABI takes.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsf.so")

SF_OK = 0
SF_STATUS_SLOT_OVERFLOW = 0x1
SF_STATUS_NONFINITE = 0x2
SF_STATUS_BAD_TOKEN = 0x4
SF_STATUS_WAIT_TIMEOUT = 0x8

SF_SRC_TOKENS = 0
SF_SRC_OUTPUT_BF16 = 1
SF_SRC_HITS_U32 = 2
SF_SRC_WORDS = 3

SF_PHASE_ALL = 0
SF_PHASE_FIRST = 1
SF_PHASE_SECOND = 2

SF_DW_MAX_PER_LAUNCH = 96
SF_MASKS_PER_LAUNCH = 240
SF_MASK_SPLIT_ROWS = 16384
SF_MATS_PER_LAUNCH = 256

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float


class sf_mask(ctypes.Structure):
    _fields_ = [("R", _I32), ("slot_cap", _I32), ("charge", _P), ("accum", _P), ("words", _P),
                ("active_rows", _P), ("active_tiles", _P), ("tile_rows", _P), ("row_slot", _P), ("free_slots", _P),
                ("slot_step", _P), ("counts", _P)]


class sf_mask_src(ctypes.Structure):
    _fields_ = [("kind", _I32), ("n", _I32), ("ld", _I64), ("ptr", _P)]


class sf_dw_problem(ctypes.Structure):
    _fields_ = [("dX", _P), ("ld_dx", _I64), ("A", _P), ("ld_a", _I64), ("T", _I32), ("C", _I32),
                ("mask", sf_mask), ("dW", _P), ("ld_dw", _I64)]


class sf_fwd_problem(ctypes.Structure):
    _fields_ = [("A", _P), ("ld_a", _I64), ("W", _P), ("ld_w", _I64), ("Y", _P), ("ld_y", _I64),
                ("T", _I32), ("C", _I32), ("mask", sf_mask)]


class sf_matrix(ctypes.Structure):
    _fields_ = [("C", _I32), ("partner", _I32), ("c_self", _F), ("c_partner", _F),
                ("mask", sf_mask), ("q", _P), ("s", _P), ("delta", _P), ("m", _P), ("v", _P),
                ("grad", _P), ("live", _P)]


class sf_checkpoint(ctypes.Structure):
    _fields_ = [("cap", _I32), ("count", _P), ("rows", _P), ("q", _P), ("s", _P), ("delta", _P),
                ("m", _P), ("v", _P), ("step", _P)]


class sf_adam(ctypes.Structure):
    _fields_ = [("lr", _F), ("beta1", _F), ("beta2", _F), ("eps", _F), ("one_minus_b1", _F),
                ("one_minus_b2", _F), ("wd", _F), ("clip", _F), ("bc1", _P), ("bc2", _P),
                ("t_max", _I32)]


_lib = None


def load():
    """Load libsf.so (built in-tree by build.py). Raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m masked_optimizer_step_b200.build`;"
                           " there is no CPU fallback")
    L = ctypes.CDLL(LIB_PATH)
    L.sf_status_string.restype = ctypes.c_char_p
    L.sf_status_string.argtypes = [ctypes.c_int]
    L.sf_version.restype = ctypes.c_int
    L.sf_mask_init.argtypes = [ctypes.POINTER(sf_mask), _P]
    L.sf_mask_update.argtypes = [ctypes.POINTER(sf_mask), ctypes.POINTER(sf_mask_src), ctypes.c_int,
                                 _F, _P, _P]
    L.sf_masked_dw.argtypes = [ctypes.POINTER(sf_dw_problem), ctypes.c_int, _P, ctypes.c_size_t, _P, _P]
    L.sf_forward_tracked.argtypes = [ctypes.POINTER(sf_fwd_problem), ctypes.c_int, _P, _P]
    L.sf_mask_update_phase.argtypes = [ctypes.POINTER(sf_mask), ctypes.POINTER(sf_mask_src), ctypes.c_int,
                                       _F, ctypes.c_int, _P, _P]
    L.sf_masked_dw_phase.argtypes = [ctypes.POINTER(sf_dw_problem), ctypes.c_int, _P, ctypes.c_size_t,
                                     ctypes.c_int, _P, _P]
    L.sf_masked_dw_unit_rows.restype = ctypes.c_int
    L.sf_masked_dw_unit_rows.argtypes = []
    L.sf_masked_dw_ws_bytes.restype = ctypes.c_size_t
    L.sf_masked_dw_ws_bytes.argtypes = [ctypes.POINTER(sf_dw_problem), ctypes.c_int]
    L.sf_embed_grad_ws_bytes.restype = ctypes.c_size_t
    L.sf_embed_grad_ws_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
    L.sf_embed_grad.argtypes = [_P, ctypes.c_int, _P, ctypes.c_int, _I64, ctypes.POINTER(sf_mask), _P,
                                _I64, _P, ctypes.c_size_t, _P, _P]
    L.sf_embed_grad_noalloc.argtypes = [_P, ctypes.c_int, _P, ctypes.c_int, _I64, ctypes.POINTER(sf_mask),
                                        _P, _I64, _P, _P]
    L.sf_embed_grad_noalloc.restype = ctypes.c_int
    L.sf_adam_tables.argtypes = [_F, _F, ctypes.c_int, _P, _P, _P]
    L.sf_sparse_update.argtypes = [ctypes.POINTER(sf_matrix), ctypes.c_int, ctypes.POINTER(sf_adam),
                                   _P, _P]
    L.sf_quantize_init.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P]
    for name in ("sf_checkpoint_save", "sf_checkpoint_restore"):
        getattr(L, name).argtypes = [ctypes.POINTER(sf_matrix), ctypes.POINTER(sf_checkpoint), ctypes.c_int, _P, _P]
        getattr(L, name).restype = ctypes.c_int
    for name in ("sf_mask_init", "sf_mask_update", "sf_masked_dw", "sf_embed_grad", "sf_adam_tables",
                 "sf_sparse_update", "sf_quantize_init", "sf_mask_update_phase", "sf_masked_dw_phase",
                 "sf_forward_tracked"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != SF_OK:
        msg = load().sf_status_string(rc).decode()
        raise RuntimeError(f"{what} failed: {msg} ({rc})")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def status_word(device=None) -> torch.Tensor:
    """A zeroed device status word (uint32 bits, held in an int32 tensor)."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


# ---------------------------------------------------------------------------------------------
# State holders
# ---------------------------------------------------------------------------------------------

class Mask:
    """Device arrays of one sf_mask (section 2.1 state: charges, mask, lists, slots)."""

    def __init__(self, R: int, slot_cap: int, device="cuda"):
        if R % 32:
            raise ValueError("R must be a multiple of 32")
        i32 = dict(dtype=torch.int32, device=device)
        self.R, self.slot_cap = R, slot_cap
        self.charge = torch.zeros(R, dtype=torch.float32, device=device)
        self.accum = torch.zeros(R, **i32)
        self.words = torch.zeros(R // 32, **i32)
        self.active_rows = torch.zeros(R, **i32)
        self.active_tiles = torch.zeros(R // 32, **i32)
        self.tile_rows = torch.zeros(R // 32, **i32)
        self.row_slot = torch.full((R,), -1, **i32)
        self.free_slots = torch.zeros(max(slot_cap, 1), **i32)
        self.slot_step = torch.zeros(max(slot_cap, 1), **i32)
        self.counts = torch.zeros(8, **i32)

    def struct(self) -> sf_mask:
        return sf_mask(self.R, self.slot_cap, _ptr(self.charge), _ptr(self.accum), _ptr(self.words),
                       _ptr(self.active_rows), _ptr(self.active_tiles), _ptr(self.tile_rows), _ptr(self.row_slot),
                       _ptr(self.free_slots), _ptr(self.slot_step), _ptr(self.counts))


class Matrix:
    """int8 + scale + residual weights of one matrix with its moments, gradient and live copy."""

    def __init__(self, R: int, C: int, slot_cap: int, device="cuda", live=True):
        self.R, self.C = R, C
        self.mask = Mask(R, slot_cap, device)
        self.q = torch.zeros((R, C), dtype=torch.int8, device=device)
        self.s = torch.zeros(R, dtype=torch.float32, device=device)
        self.delta = torch.zeros((R, C), dtype=torch.float32, device=device)
        n = max(slot_cap, 1)
        self.m = torch.zeros((n, C), dtype=torch.int16, device=device)
        self.v = torch.zeros((n, C), dtype=torch.int16, device=device)
        self.grad = torch.zeros((n, C), dtype=torch.float32, device=device)
        self.live = torch.zeros((R, C), dtype=torch.int16, device=device) if live else None


# ---------------------------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------------------------

def sf_mask_init(mask: Mask, stream=None):
    m = mask.struct()
    _check(load().sf_mask_init(ctypes.byref(m), _stream(stream)), "sf_mask_init")


class Desc:
    """A C descriptor together with the tensors its pointers refer to.

    The tensors stay referenced for as long as the descriptor lives, so that a temporary cannot
    be freed (and its memory handed to the next allocation) before the kernel that reads it has
    been enqueued.
    """

    __slots__ = ("c", "refs")

    def __init__(self, c, *refs):
        self.c = c
        self.refs = refs


def make_src(kind: int, tensor=None, n: int = 0, ld: int = 0) -> Desc:
    return Desc(sf_mask_src(kind, n, ld, _ptr(tensor) if tensor is not None else None), tensor)


def sf_mask_update(masks, srcs, threshold: float = 0.01, status=None, stream=None):
    """masks: list of Mask; srcs: list of make_src() descriptors."""
    n = len(masks)
    arr_m = (sf_mask * n)(*[m.struct() for m in masks])
    arr_s = (sf_mask_src * n)(*[s.c for s in srcs])
    _check(load().sf_mask_update(arr_m, arr_s, n, threshold, _ptr(status), _stream(stream)),
           "sf_mask_update")


def sf_mask_update_phase(masks, srcs, phase: int, threshold: float = 0.01, status=None, stream=None):
    """One pass of sf_mask_update (SF_PHASE_FIRST: activity, SF_PHASE_SECOND: finalize)."""
    n = len(masks)
    arr_m = (sf_mask * n)(*[m.struct() for m in masks])
    arr_s = (sf_mask_src * n)(*[s.c for s in srcs])
    _check(load().sf_mask_update_phase(arr_m, arr_s, n, threshold, phase, _ptr(status), _stream(stream)),
           "sf_mask_update_phase")


def dw_problem(dX, A, mask: Mask, dW) -> Desc:
    """dX [T x R] bf16, A [T x C] bf16, dW [slot_cap x C] fp32 (row = slot)."""
    T, R = dX.shape
    C = A.shape[1]
    assert A.shape[0] == T and R == mask.R and dX.dtype == torch.bfloat16 and A.dtype == torch.bfloat16
    c = sf_dw_problem(_ptr(dX), dX.stride(0), _ptr(A), A.stride(0), T, C, mask.struct(), _ptr(dW),
                      dW.stride(0))
    return Desc(c, dX, A, dW)


def sf_masked_dw_unit_rows() -> int:
    return load().sf_masked_dw_unit_rows()


def sf_masked_dw_ws_bytes(problems) -> int:
    n = len(problems)
    arr = (sf_dw_problem * n)(*[p.c for p in problems])
    return load().sf_masked_dw_ws_bytes(arr, n)


def dw_workspace(problems, device="cuda") -> torch.Tensor:
    """Scratch for sf_masked_dw's row mode (a byte tensor of sf_masked_dw_ws_bytes bytes)."""
    return torch.empty(max(sf_masked_dw_ws_bytes(problems), 1), dtype=torch.uint8, device=device)


def sf_masked_dw(problems, status=None, stream=None, ws=None):
    """problems: list of dw_problem() descriptors; ws: dw_workspace() scratch, or None for the
    mask-tile mode only."""
    n = len(problems)
    arr = (sf_dw_problem * n)(*[p.c for p in problems])
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(load().sf_masked_dw(arr, n, _ptr(ws), nbytes, _ptr(status), _stream(stream)), "sf_masked_dw")


def sf_masked_dw_phase(problems, phase: int, status=None, stream=None, ws=None):
    """One pass of sf_masked_dw (SF_PHASE_FIRST: row gather, SF_PHASE_SECOND: main launches)."""
    n = len(problems)
    arr = (sf_dw_problem * n)(*[p.c for p in problems])
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(load().sf_masked_dw_phase(arr, n, _ptr(ws), nbytes, phase, _ptr(status), _stream(stream)),
           "sf_masked_dw_phase")


def fwd_problem(A, W, Y, mask: Mask) -> Desc:
    """A [T x C] bf16 inputs, W [R x C] bf16 weights, Y [T x R] bf16 outputs (written)."""
    T, C = A.shape
    R = W.shape[0]
    assert W.shape[1] == C and Y.shape == (T, R) and R == mask.R
    assert A.dtype == W.dtype == Y.dtype == torch.bfloat16
    c = sf_fwd_problem(_ptr(A), A.stride(0), _ptr(W), W.stride(0), _ptr(Y), Y.stride(0), T, C, mask.struct())
    return Desc(c, A, W, Y)


def sf_forward_tracked(problems, status=None, stream=None):
    """Forward projections Y = A W^T with each projection's row magnitudes folded into its mask's
    accumulator; close the window with sf_mask_update_phase(..., SF_PHASE_SECOND)."""
    n = len(problems)
    arr = (sf_fwd_problem * max(n, 1))(*[p.c for p in problems])
    _check(load().sf_forward_tracked(arr, n, _ptr(status), _stream(stream)), "sf_forward_tracked")


def sf_embed_grad_ws_bytes(n_tok: int, slot_cap: int) -> int:
    return load().sf_embed_grad_ws_bytes(n_tok, slot_cap)


def sf_embed_grad(tokens, dY, mask: Mask, G, ws, status=None, stream=None):
    n_tok, H = dY.shape
    m = mask.struct()
    _check(load().sf_embed_grad(_ptr(tokens), n_tok, _ptr(dY), H, dY.stride(0), ctypes.byref(m), _ptr(G),
                                G.stride(0), _ptr(ws), ws.numel() * ws.element_size(), _ptr(status),
                                _stream(stream)), "sf_embed_grad")


def sf_embed_grad_noalloc(tokens, dY, mask: Mask, G, status=None, stream=None):
    """sf_embed_grad without a scratch buffer: the library's fixed per-GPU scratch is used, for
    callers that must not allocate device memory. Calls on one GPU must not overlap."""
    n_tok, H = dY.shape
    m = mask.struct()
    _check(load().sf_embed_grad_noalloc(_ptr(tokens), n_tok, _ptr(dY), H, dY.stride(0), ctypes.byref(m),
                                        _ptr(G), G.stride(0), _ptr(status), _stream(stream)),
           "sf_embed_grad_noalloc")


def sf_adam_tables(beta1: float, beta2: float, t_max: int, bc1, bc2, stream=None):
    _check(load().sf_adam_tables(beta1, beta2, t_max, _ptr(bc1), _ptr(bc2), _stream(stream)),
           "sf_adam_tables")


class AdamParams:
    """Adam hyper-parameters plus the device bias-correction tables."""

    def __init__(self, lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, clip=0.0, t_max=20000,
                 device="cuda", stream=None):
        import numpy as np
        self.lr, self.beta1, self.beta2, self.eps, self.wd, self.clip = lr, beta1, beta2, eps, wd, clip
        self.one_minus_b1 = float(np.float32(1.0) - np.float32(beta1))
        self.one_minus_b2 = float(np.float32(1.0) - np.float32(beta2))
        self.t_max = t_max
        self.bc1 = torch.empty(t_max + 1, dtype=torch.float32, device=device)
        self.bc2 = torch.empty(t_max + 1, dtype=torch.float32, device=device)
        sf_adam_tables(beta1, beta2, t_max, self.bc1, self.bc2, stream)

    def struct(self) -> sf_adam:
        return sf_adam(self.lr, self.beta1, self.beta2, self.eps, self.one_minus_b1, self.one_minus_b2,
                       self.wd, self.clip, _ptr(self.bc1), _ptr(self.bc2), self.t_max)


def matrix_struct(mat: Matrix, partner: int = -1, c_self: float = 1.0, c_partner: float = 0.0) -> sf_matrix:
    return sf_matrix(mat.C, partner, c_self, c_partner, mat.mask.struct(), _ptr(mat.q), _ptr(mat.s),
                     _ptr(mat.delta), _ptr(mat.m), _ptr(mat.v), _ptr(mat.grad), _ptr(mat.live))


def sf_sparse_update(mats, hp: AdamParams, status=None, stream=None):
    """mats: list of sf_matrix (see matrix_struct); partner indices refer to this list."""
    n = len(mats)
    arr = (sf_matrix * n)(*mats)
    h = hp.struct()
    _check(load().sf_sparse_update(arr, n, ctypes.byref(h), _ptr(status), _stream(stream)),
           "sf_sparse_update")


def sf_quantize_init(W, mat: Matrix, stream=None):
    R, C = W.shape
    assert W.dtype == torch.float32 and W.is_contiguous() and (R, C) == (mat.R, mat.C)
    _check(load().sf_quantize_init(_ptr(W), R, C, _ptr(mat.q), _ptr(mat.s), _ptr(mat.delta),
                                   _ptr(mat.live), _stream(stream)), "sf_quantize_init")


def sf_version() -> int:
    return load().sf_version()


class Checkpoint:
    """Device buffers of an active-row checkpoint of one matrix (section 2.6)."""

    def __init__(self, cap: int, C: int, device="cuda"):
        self.cap, self.C = cap, C
        n = max(cap, 1)
        self.count = torch.zeros(1, dtype=torch.int32, device=device)
        self.rows = torch.zeros(n, dtype=torch.int32, device=device)
        self.q = torch.zeros((n, C), dtype=torch.int8, device=device)
        self.s = torch.zeros(n, dtype=torch.float32, device=device)
        self.delta = torch.zeros((n, C), dtype=torch.float32, device=device)
        self.m = torch.zeros((n, C), dtype=torch.int16, device=device)
        self.v = torch.zeros((n, C), dtype=torch.int16, device=device)
        self.step = torch.zeros(n, dtype=torch.int32, device=device)

    def struct(self) -> sf_checkpoint:
        return sf_checkpoint(self.cap, _ptr(self.count), _ptr(self.rows), _ptr(self.q), _ptr(self.s),
                             _ptr(self.delta), _ptr(self.m), _ptr(self.v), _ptr(self.step))


def _ckpt_call(name, mats, ckpts, status, stream):
    n = len(mats)
    arr = (sf_matrix * n)(*mats)
    carr = (sf_checkpoint * n)(*[c.struct() for c in ckpts])
    _check(getattr(load(), name)(arr, carr, n, _ptr(status), _stream(stream)), name)


def sf_checkpoint_save(mats, ckpts, status=None, stream=None):
    """mats: list of sf_matrix (matrix_struct); ckpts: list of Checkpoint, same order."""
    _ckpt_call("sf_checkpoint_save", mats, ckpts, status, stream)


def sf_checkpoint_restore(mats, ckpts, status=None, stream=None):
    _ckpt_call("sf_checkpoint_restore", mats, ckpts, status, stream)
