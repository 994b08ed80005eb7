"""ctypes front end of the CPU oracle (test infrastructure only).

Arrays in: float32 numpy arrays holding the exact input values.  Arrays out:
float64 (values) or int32 (positions).  Layouts follow the C library.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

from . import build as _build

_lib = None


class RefDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "T", "n_past", "N_max", "H_q", "H_kv", "d", "H_I", "H_Ik", "d_I", "M",
                 "phi")] + [("sm_scale", ctypes.c_double)]


@dataclasses.dataclass
class Dims:
    B: int
    T: int
    n_past: int
    N_max: int
    H_q: int
    H_kv: int
    d: int
    H_I: int
    H_Ik: int
    d_I: int
    M: int
    phi: int = 0
    sm_scale: float | None = None

    def c(self) -> RefDims:
        sc = self.sm_scale if self.sm_scale is not None else 1.0 / np.sqrt(self.d)
        return RefDims(self.B, self.T, self.n_past, self.N_max, self.H_q, self.H_kv, self.d,
                       self.H_I, self.H_Ik, self.d_I, self.M, self.phi, float(sc))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # LISA_REF_LIB lets the mutation tests load a deliberately broken copy
        path = os.environ.get("LISA_REF_LIB") or _build.build()
        _lib = ctypes.CDLL(path)
        _lib.ref_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return lib().ref_num_threads()


def set_num_threads(n: int) -> None:
    lib().ref_set_num_threads(ctypes.c_int(n))


def _f32(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _rows(D: Dims, rows):
    if rows is None:
        return None, D.T
    r = np.ascontiguousarray(rows, dtype=np.int32)
    assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < D.T))
    return r, int(r.size)


def index_scores(D: Dims, q_I, k_I, w, w_tok_stride: int, rows=None) -> np.ndarray:
    q_I, k_I, w = _f32(q_I), _f32(k_I), _f32(w)
    r, R = _rows(D, rows)
    out = np.empty((D.B, R, D.n_past + D.T), dtype=np.float64)
    lib().ref_index_scores(ctypes.byref(D.c()), _p(q_I), _p(k_I), _p(w),
                           ctypes.c_int64(w_tok_stride), _p(r), ctypes.c_int32(R), _p(out))
    return out


def topm(D: Dims, scores, rows=None):
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    r, R = _rows(D, rows)
    assert scores.shape == (D.B, R, D.n_past + D.T)
    idx = np.empty((D.B, R, D.M), dtype=np.int32)
    cnt = np.empty((D.B, R), dtype=np.int32)
    lib().ref_topm(ctypes.byref(D.c()), _p(scores), _p(r), ctypes.c_int32(R), _p(idx), _p(cnt))
    return idx, cnt


def sparse_attn(D: Dims, q, k_cache, v_cache, idx, count, rows=None) -> np.ndarray:
    q, k_cache, v_cache = _f32(q), _f32(k_cache), _f32(v_cache)
    r, R = _rows(D, rows)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    count = np.ascontiguousarray(count, dtype=np.int32)
    assert idx.shape == (D.B, R, D.M) and count.shape == (D.B, R)
    out = np.empty((D.B, R, D.H_q, D.d), dtype=np.float64)
    lib().ref_sparse_attn(ctypes.byref(D.c()), _p(q), _p(k_cache), _p(v_cache), _p(r),
                          ctypes.c_int32(R), _p(idx), _p(count), _p(out))
    return out


def dense_attn(D: Dims, q, k_cache, v_cache, rows=None) -> np.ndarray:
    q, k_cache, v_cache = _f32(q), _f32(k_cache), _f32(v_cache)
    r, R = _rows(D, rows)
    out = np.empty((D.B, R, D.H_q, D.d), dtype=np.float64)
    lib().ref_dense_attn(ctypes.byref(D.c()), _p(q), _p(k_cache), _p(v_cache), _p(r),
                         ctypes.c_int32(R), _p(out))
    return out


def linear(D: Dims, q_L, k_L, v_L, S0=None, z0=None, rows=None):
    """Returns (o [B,R,H_q,d], S [B,H_kv,d,d], z [B,H_kv,d] or None)."""
    if q_L is None:  # only allowed when no output row is requested
        assert rows is not None and len(rows) == 0
    else:
        q_L = _f32(q_L)
    k_L, v_L = _f32(k_L), _f32(v_L)
    r, R = _rows(D, rows)
    S = np.zeros((D.B, D.H_kv, D.d, D.d)) if S0 is None else np.array(S0, dtype=np.float64)
    z = None
    if D.phi == 1:
        z = np.zeros((D.B, D.H_kv, D.d)) if z0 is None else np.array(z0, dtype=np.float64)
    out = np.empty((D.B, R, D.H_q, D.d), dtype=np.float64)
    lib().ref_linear(ctypes.byref(D.c()), _p(q_L), _p(k_L), _p(v_L), _p(S), _p(z), _p(r),
                     ctypes.c_int32(R), _p(out))
    return out, S, z


def gate(D: Dims, logit, o_lin, o_sp, rows=None) -> np.ndarray:
    logit = _f32(logit)
    r, R = _rows(D, rows)
    o_lin = np.ascontiguousarray(o_lin, dtype=np.float64)
    o_sp = np.ascontiguousarray(o_sp, dtype=np.float64)
    out = np.empty_like(o_lin)
    lib().ref_gate(ctypes.byref(D.c()), _p(logit), _p(r), ctypes.c_int32(R), _p(o_lin),
                   _p(o_sp), _p(out))
    return out


def forward(D: Dims, q, k_cache, v_cache, q_I, k_I, w, w_tok_stride, q_L, k_L, v_L, gate_logit,
            S0=None, z0=None, rows=None):
    """The whole module; returns a dict of idx, count, o_sp, o_lin, o, S, z."""
    arrs = [_f32(a) for a in (q, k_cache, v_cache, q_I, k_I, w, q_L, k_L, v_L, gate_logit)]
    r, R = _rows(D, rows)
    S = np.zeros((D.B, D.H_kv, D.d, D.d)) if S0 is None else np.array(S0, dtype=np.float64)
    z = None
    if D.phi == 1:
        z = np.zeros((D.B, D.H_kv, D.d)) if z0 is None else np.array(z0, dtype=np.float64)
    idx = np.empty((D.B, R, D.M), dtype=np.int32)
    cnt = np.empty((D.B, R), dtype=np.int32)
    o_sp = np.empty((D.B, R, D.H_q, D.d))
    o_lin = np.empty_like(o_sp)
    o = np.empty_like(o_sp)
    q, kc, vc, qI, kI, w_, qL, kL, vL, gl = arrs
    lib().ref_forward(ctypes.byref(D.c()), _p(q), _p(kc), _p(vc), _p(qI), _p(kI), _p(w_),
                      ctypes.c_int64(w_tok_stride), _p(qL), _p(kL), _p(vL), _p(gl), _p(S), _p(z),
                      _p(r), ctypes.c_int32(R), _p(idx), _p(cnt), _p(o_sp), _p(o_lin), _p(o))
    return dict(idx=idx, count=cnt, o_sp=o_sp, o_lin=o_lin, o=o, S=S, z=z)


def window_indices(D: Dims, rows=None):
    """Sliding-window index rows (Stage 1): (idx [B,R,M] int32, count [B,R])."""
    r, R = _rows(D, rows)
    idx = np.empty((D.B, R, D.M), dtype=np.int32)
    cnt = np.empty((D.B, R), dtype=np.int32)
    lib().ref_window_indices(ctypes.byref(D.c()), _p(r), ctypes.c_int32(R), _p(idx), _p(cnt))
    return idx, cnt


def state_transfer(D: Dims, S_end, S_start, grad_sum, t: int, alpha: float):
    """Segment state correction at the end of segment t (Eq. 6-9).
    Returns (S_t, new S_start, new grad_sum), all fp64 copies."""
    S = np.array(S_end, dtype=np.float64)
    S0 = np.array(S_start, dtype=np.float64)
    G = np.array(grad_sum, dtype=np.float64)
    lib().ref_state_transfer(ctypes.byref(D.c()), _p(S), _p(S0), _p(G), ctypes.c_int(t),
                             ctypes.c_double(alpha))
    return S, S0, G


def gate_channel(D: Dims, D_h: int, h, W_g, o_lin, o_sp, rows=None) -> np.ndarray:
    """Per-channel gate (Eq. 5) mixing the two branches; o [B,R,H_q,d]."""
    h, W_g = _f32(h), _f32(W_g)
    r, R = _rows(D, rows)
    o_lin = np.ascontiguousarray(o_lin, dtype=np.float64)
    o_sp = np.ascontiguousarray(o_sp, dtype=np.float64)
    out = np.empty_like(o_lin)
    lib().ref_gate_channel(ctypes.byref(D.c()), ctypes.c_int(D_h), _p(h), _p(W_g), _p(r),
                           ctypes.c_int32(R), _p(o_lin), _p(o_sp), _p(out))
    return out
