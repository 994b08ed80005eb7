"""Python binding of liblisa (ctypes).

Argument marshalling only: every entry point forwards torch tensors' device
pointers and the current CUDA stream to the C function of the same name in
``liblisa.so``; all arithmetic runs in the library's CUDA kernels.  If the
library is missing this module raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblisa.so")

LISA_OK = 0
LISA_ERR_INVALID_ARG = 1
LISA_ERR_UNSUPPORTED = 2
LISA_ERR_CUDA = 3
LISA_ERR_TIMEOUT = 4
LISA_ERR_DEVICE_BOUNDS = 5
LISA_ERR_WORKSPACE = 6

LISA_F32 = 0
LISA_BF16 = 1
LISA_PHI_IDENTITY = 0
LISA_PHI_ELU1_NORM = 1

LISA_OP_TOPM = 0
LISA_OP_SPARSE_ATTN = 1
LISA_OP_LINEAR_PREFILL = 2
LISA_OP_DECODE_STEP = 3
LISA_OP_DENSE_ATTN = 4
LISA_OP_PREFILL = 5
LISA_OP_GATE_CHANNEL = 6

# Every symbol the header declares.
EXPORTS = (
    "lisa_index_scores", "lisa_topm", "lisa_sparse_attn", "lisa_linear_prefill",
    "lisa_linear_decode", "lisa_gate_fuse", "lisa_decode_step", "lisa_dense_attn",
    "lisa_workspace_size", "lisa_check_status", "lisa_status_string", "lisa_version",
    "lisa_topm_noalloc", "lisa_prefill", "lisa_window_indices", "lisa_decode_step_window",
    "lisa_state_transfer", "lisa_gate_channel",
)


class LisaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class lisa_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "T", "n_past", "N_max", "H_q", "H_kv", "d", "H_I", "H_Ik", "d_I", "M",
                 "chunk", "act_dtype", "phi")] + [("sm_scale", ctypes.c_float)]


class lisa_prefill_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("q_I", ctypes.c_void_p), ("k_I_cache", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("w_tok_stride", ctypes.c_int64), ("q_L", ctypes.c_void_p), ("k_L", ctypes.c_void_p),
        ("v_L", ctypes.c_void_p), ("gate_logit_lin", ctypes.c_void_p), ("S", ctypes.c_void_p),
        ("z", ctypes.c_void_p), ("o", ctypes.c_void_p), ("idx", ctypes.c_void_p),
        ("count", ctypes.c_void_p),
    ]


class lisa_decode_args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p),
        ("q_I", ctypes.c_void_p), ("k_I_new", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("w_tok_stride", ctypes.c_int64), ("q_L", ctypes.c_void_p), ("k_L", ctypes.c_void_p),
        ("v_L", ctypes.c_void_p), ("gate_logit_lin", ctypes.c_void_p),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("k_I_cache", ctypes.c_void_p), ("S", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("count", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load liblisa.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"liblisa.so not found at {LIB_PATH}: build it with "
                           "`python -m hybrid_linear_top_lightning_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    dp = ctypes.POINTER(lisa_dims)
    sigs = {
        "lisa_index_scores": [dp, vp, vp, vp, i64, vp, vp],
        "lisa_topm": [dp, vp, vp, vp, i64, vp, vp, vp, sz, vp],
        "lisa_sparse_attn": [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "lisa_linear_prefill": [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "lisa_linear_decode": [dp, vp, vp, vp, vp, vp, vp, vp],
        "lisa_gate_fuse": [dp, vp, vp, vp, vp, vp],
        "lisa_decode_step": [dp, ctypes.POINTER(lisa_decode_args), vp, sz, vp],
        "lisa_dense_attn": [dp, vp, vp, vp, vp, vp, sz, vp],
        "lisa_workspace_size": [dp, ctypes.c_int, ctypes.POINTER(sz)],
        "lisa_check_status": [vp, vp],
        "lisa_topm_noalloc": [dp, vp, vp, vp, i64, vp, vp, vp],
        "lisa_prefill": [dp, ctypes.POINTER(lisa_prefill_args), vp, sz, vp],
        "lisa_window_indices": [dp, vp, vp, vp],
        "lisa_decode_step_window": [dp, ctypes.POINTER(lisa_decode_args), vp, sz, vp],
        "lisa_state_transfer": [dp, vp, vp, vp, ctypes.c_int32, ctypes.c_float, vp],
        "lisa_gate_channel": [dp, ctypes.c_int32, vp, vp, vp, vp, vp, vp, sz, vp],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.lisa_status_string.argtypes = [ctypes.c_int]
    lib.lisa_status_string.restype = ctypes.c_char_p
    lib.lisa_version.argtypes = []
    lib.lisa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().lisa_status_string(status).decode()


def version() -> str:
    return load().lisa_version().decode()


def make_dims(B, T, n_past, N_max, H_q, H_kv, d, H_I, H_Ik, d_I, M, chunk=64, dtype="bf16",
              phi=LISA_PHI_IDENTITY, sm_scale=0.0) -> lisa_dims:
    act = {"bf16": LISA_BF16, "f32": LISA_F32, torch.bfloat16: LISA_BF16,
           torch.float32: LISA_F32}[dtype]
    return lisa_dims(B, T, n_past, N_max, H_q, H_kv, d, H_I, H_Ik, d_I, M, chunk, act, phi,
                     float(sm_scale))


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("liblisa entry points take device tensors")
    if not t.is_contiguous():
        raise ValueError("liblisa entry points take contiguous tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != LISA_OK:
        raise LisaError(status, where)


def lisa_workspace_size(dims: lisa_dims, op: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().lisa_workspace_size(ctypes.byref(dims), op, ctypes.byref(n)),
           "lisa_workspace_size")
    return int(n.value)


def workspace(dims: lisa_dims, op: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size `op` needs (at least 256 bytes)."""
    n = max(lisa_workspace_size(dims, op), 256)
    ws = torch.zeros(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def lisa_index_scores(dims, q_I, k_I_cache, w, w_tok_stride, scores, stream=None):
    _check(load().lisa_index_scores(ctypes.byref(dims), _ptr(q_I), _ptr(k_I_cache), _ptr(w),
                                    int(w_tok_stride), _ptr(scores), _stream(stream)),
           "lisa_index_scores")


def lisa_topm(dims, q_I, k_I_cache, w, w_tok_stride, idx, count, ws, stream=None):
    _check(load().lisa_topm(ctypes.byref(dims), _ptr(q_I), _ptr(k_I_cache), _ptr(w),
                            int(w_tok_stride), _ptr(idx), _ptr(count), _ptr(ws), ws.numel(),
                            _stream(stream)), "lisa_topm")


def lisa_topm_noalloc(dims, q_I, k_I_cache, w, w_tok_stride, idx, count, stream=None):
    """lisa_topm without a workspace (scores kept in the library's built-in 4 MiB array)."""
    _check(load().lisa_topm_noalloc(ctypes.byref(dims), _ptr(q_I), _ptr(k_I_cache), _ptr(w),
                                    int(w_tok_stride), _ptr(idx), _ptr(count), _stream(stream)),
           "lisa_topm_noalloc")


def lisa_sparse_attn(dims, q, k_cache, v_cache, idx, count, o_sparse, ws, stream=None):
    _check(load().lisa_sparse_attn(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(idx), _ptr(count), _ptr(o_sparse), _ptr(ws), ws.numel(),
                                   _stream(stream)), "lisa_sparse_attn")


def lisa_dense_attn(dims, q, k_cache, v_cache, o, ws, stream=None):
    _check(load().lisa_dense_attn(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(o), _ptr(ws), ws.numel(), _stream(stream)),
           "lisa_dense_attn")


def lisa_linear_prefill(dims, q_L, k_L, v_L, S, z, o_lin, ws, stream=None):
    _check(load().lisa_linear_prefill(ctypes.byref(dims), _ptr(q_L), _ptr(k_L), _ptr(v_L),
                                      _ptr(S), _ptr(z), _ptr(o_lin), _ptr(ws), ws.numel(),
                                      _stream(stream)), "lisa_linear_prefill")


def lisa_linear_decode(dims, q_L, k_L, v_L, S, z, o_lin, stream=None):
    _check(load().lisa_linear_decode(ctypes.byref(dims), _ptr(q_L), _ptr(k_L), _ptr(v_L),
                                     _ptr(S), _ptr(z), _ptr(o_lin), _stream(stream)),
           "lisa_linear_decode")


def lisa_gate_fuse(dims, gate_logit_lin, o_lin, o_sparse, o, stream=None):
    _check(load().lisa_gate_fuse(ctypes.byref(dims), _ptr(gate_logit_lin), _ptr(o_lin),
                                 _ptr(o_sparse), _ptr(o), _stream(stream)), "lisa_gate_fuse")


def decode_args(q, k_new, v_new, q_I, k_I_new, w, w_tok_stride, q_L, k_L, v_L, gate_logit_lin,
                k_cache, v_cache, k_I_cache, S, z, o, idx=None, count=None) -> lisa_decode_args:
    args = lisa_decode_args(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_I), _ptr(k_I_new), _ptr(w),
                            int(w_tok_stride), _ptr(q_L), _ptr(k_L), _ptr(v_L),
                            _ptr(gate_logit_lin), _ptr(k_cache), _ptr(v_cache), _ptr(k_I_cache),
                            _ptr(S), _ptr(z), _ptr(o), _ptr(idx), _ptr(count))
    # the struct holds raw device pointers: keep the tensors alive with it
    args._keep = (q, k_new, v_new, q_I, k_I_new, w, q_L, k_L, v_L, gate_logit_lin, k_cache,
                  v_cache, k_I_cache, S, z, o, idx, count)
    return args


def prefill_args(q, k_cache, v_cache, q_I, k_I_cache, w, w_tok_stride, q_L, k_L, v_L,
                 gate_logit_lin, S, z, o, idx=None, count=None) -> lisa_prefill_args:
    args = lisa_prefill_args(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(q_I), _ptr(k_I_cache),
                             _ptr(w), int(w_tok_stride), _ptr(q_L), _ptr(k_L), _ptr(v_L),
                             _ptr(gate_logit_lin), _ptr(S), _ptr(z), _ptr(o), _ptr(idx),
                             _ptr(count))
    # the struct holds raw device pointers: keep the tensors alive with it
    args._keep = (q, k_cache, v_cache, q_I, k_I_cache, w, q_L, k_L, v_L, gate_logit_lin, S, z,
                  o, idx, count)
    return args


def lisa_prefill(dims, args: lisa_prefill_args, ws, stream=None):
    _check(load().lisa_prefill(ctypes.byref(dims), ctypes.byref(args), _ptr(ws), ws.numel(),
                               _stream(stream)), "lisa_prefill")


def lisa_window_indices(dims, idx, count, stream=None):
    _check(load().lisa_window_indices(ctypes.byref(dims), _ptr(idx), _ptr(count), _stream(stream)),
           "lisa_window_indices")


def lisa_decode_step_window(dims, args: lisa_decode_args, ws, stream=None):
    _check(load().lisa_decode_step_window(ctypes.byref(dims), ctypes.byref(args), _ptr(ws),
                                          ws.numel(), _stream(stream)), "lisa_decode_step_window")


def lisa_state_transfer(dims, S, S_start, grad_sum, t: int, alpha: float, stream=None):
    _check(load().lisa_state_transfer(ctypes.byref(dims), _ptr(S), _ptr(S_start), _ptr(grad_sum),
                                      int(t), float(alpha), _stream(stream)), "lisa_state_transfer")


def lisa_decode_step(dims, args: lisa_decode_args, ws, stream=None):
    _check(load().lisa_decode_step(ctypes.byref(dims), ctypes.byref(args), _ptr(ws), ws.numel(),
                                   _stream(stream)), "lisa_decode_step")


def lisa_check_status(ws, stream=None) -> int:
    """Synchronise and return (and clear) the device status word of `ws`."""
    return load().lisa_check_status(_ptr(ws), _stream(stream))


def default_sm_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def lisa_gate_channel(dims, D_h: int, h, W_g, o_lin, o_sparse, o, ws, stream=None):
    _check(load().lisa_gate_channel(ctypes.byref(dims), int(D_h), _ptr(h), _ptr(W_g), _ptr(o_lin),
                                    _ptr(o_sparse), _ptr(o), _ptr(ws), ws.numel(),
                                    _stream(stream)), "lisa_gate_channel")
