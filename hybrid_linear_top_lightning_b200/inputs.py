"""Seeded synthetic inputs for the LISA attention module.

This module draws random numbers and nothing else: it holds none of the
module's arithmetic (no scores, no selection, no attention, no state).  The
CUDA library's tests and benchmark and the CPU oracle both take their inputs
from here, so the two sides always see identical values.

Recipe (shapes follow the DeepSeek-distilled Qwen2.5 layers the paper
evaluates; the values are synthetic):

* Every tensor is drawn from its own Philox4x32-10 stream, keyed by
  ``(seed, tensor id, batch element, block of 1024 positions)``.  A value
  therefore does not depend on which other tensors, batch elements or
  positions were requested, so prefill(n) followed by decode steps sees the
  same tokens as one prefill over the longer sequence.
* ``q, k, v, q_I, k_I`` ~ N(0, sigma^2) per coordinate.  ``sigma`` is 1 for
  the tiny fp32 workload and 1/sqrt(128) for the model-shaped workloads.
* ``w`` (indexer head weights) ~ U(0, 1); ``gate`` (gate logits) ~ N(0, 1).
* Per-channel gate inputs: hidden states ``h`` [B, n, D_h] ~ N(0, 1); gate
  weights ``W_g`` [H_q*d, D_h] ~ N(0, 1/D_h), so a gate logit is ~ N(0, 1);
  branch outputs ``o_lin``, ``o_sp`` [B, n, H_q, d] ~ N(0, 1).
* Planted heavy keys: per batch element, floor(0.01 * n) positions drawn
  uniformly without replacement among the n positions of the workload; at
  each, ``3 * sigma * sqrt(dim) * u`` is added to ``k`` (every KV head) and to
  ``k_I``, with ``u`` one seeded unit vector per tensor shared by all planted
  positions and batch elements.  This shifts the per-coordinate RMS by
  3 sigma along one shared direction.
* bf16 workloads round every drawn value to bf16 (round to nearest even)
  once, here; fp32 workloads keep the float32 draw.  Both sides consume the
  identical rounded values.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BLOCK = 1024  # positions per random stream block

_TENSOR_IDS = {
    "q": 1, "k": 2, "v": 3, "q_I": 4, "k_I": 5, "w": 6, "gate": 7,
    "plant": 8, "u_k": 9, "u_kI": 10, "qL": 11, "kL": 12, "vL": 13,
    "h": 14, "W_g": 15, "o_lin": 16, "o_sp": 17,
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic LISA layer invocation."""

    name: str
    B: int
    n: int              # total positions of the workload (context length)
    H_q: int
    H_kv: int
    d: int
    H_I: int
    H_Ik: int
    d_I: int
    M: int
    chunk: int
    dtype: str          # "f32" or "bf16"
    sigma: float
    plant: bool
    seed: int = 0

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny parity check, 1.5B-shape prefill, 7B-shape decode at
# 16K context, 7B-shape prefill and the long-context decode sweep.
TINY = Workload("tiny_f32", B=1, n=272, H_q=2, H_kv=1, d=64, H_I=2, H_Ik=1, d_I=32,
                M=32, chunk=16, dtype="f32", sigma=1.0, plant=False, seed=0)
PREFILL_1P5B = Workload("prefill_1.5b_n4096", B=1, n=4096, H_q=12, H_kv=2, d=128, H_I=4,
                        H_Ik=1, d_I=64, M=512, chunk=64, dtype="bf16",
                        sigma=1.0 / math.sqrt(128), plant=True, seed=0)
DECODE_7B = Workload("decode_7b_ctx16384_b8", B=8, n=16384, H_q=28, H_kv=4, d=128, H_I=8,
                     H_Ik=1, d_I=64, M=2048, chunk=64, dtype="bf16",
                     sigma=1.0 / math.sqrt(128), plant=True, seed=0)
PREFILL_7B = Workload("prefill_7b_n16384", B=1, n=16384, H_q=28, H_kv=4, d=128, H_I=8,
                      H_Ik=1, d_I=64, M=2048, chunk=64, dtype="bf16",
                      sigma=1.0 / math.sqrt(128), plant=True, seed=0)
SWEEP_CTX = (4096, 8192, 16384, 32768, 65536)
SWEEP_M = (512, 2048)


def sweep_workload(n: int, M: int) -> Workload:
    return Workload(f"decode_7b_ctx{n}_b32_M{M}", B=32, n=n, H_q=28, H_kv=4, d=128, H_I=8,
                    H_Ik=1, d_I=64, M=M, chunk=64, dtype="bf16",
                    sigma=1.0 / math.sqrt(128), plant=True, seed=0)


class Generator:
    """Lazily draws the tensors of one workload, one batch element at a time."""

    def __init__(self, wl: Workload):
        self.wl = wl
        self._plant_cache: dict[int, np.ndarray] = {}
        self._u_cache: dict[str, np.ndarray] = {}

    # -- raw streams -----------------------------------------------------
    def _rng(self, name: str, *key: int) -> np.random.Generator:
        ss = np.random.SeedSequence([self.wl.seed, _TENSOR_IDS[name], *key])
        return np.random.Generator(np.random.Philox(ss))

    def _finish(self, x: np.ndarray) -> np.ndarray:
        x = x.astype(np.float32)
        return round_bf16(x) if self.wl.dtype == "bf16" else x

    def _per_position(self, name: str, b: int, p0: int, p1: int, width: int,
                      kind: str, scale: float) -> np.ndarray:
        """Rows [p0, p1) of a [n, width] tensor of batch element b (float32, unrounded)."""
        out = np.empty((p1 - p0, width), dtype=np.float32)
        for blk in range(p0 // BLOCK, (p1 - 1) // BLOCK + 1 if p1 > p0 else p0 // BLOCK):
            rng = self._rng(name, b, blk)
            if kind == "normal":
                vals = rng.standard_normal((BLOCK, width), dtype=np.float32) * np.float32(scale)
            else:
                vals = rng.random((BLOCK, width), dtype=np.float32)
            lo = max(p0, blk * BLOCK)
            hi = min(p1, (blk + 1) * BLOCK)
            out[lo - p0:hi - p0] = vals[lo - blk * BLOCK:hi - blk * BLOCK]
        return out

    def planted_positions(self, b: int) -> np.ndarray:
        wl = self.wl
        if not wl.plant:
            return np.zeros(0, dtype=np.int64)
        if b not in self._plant_cache:
            cnt = (wl.n * 1) // 100
            rng = self._rng("plant", b)
            self._plant_cache[b] = np.sort(rng.choice(wl.n, size=cnt, replace=False))
        return self._plant_cache[b]

    def unit_vector(self, name: str, dim: int) -> np.ndarray:
        if name not in self._u_cache:
            u = self._rng(name).standard_normal(dim)
            self._u_cache[name] = (u / np.linalg.norm(u)).astype(np.float64)
        return self._u_cache[name]

    def _plant(self, x: np.ndarray, b: int, p0: int, p1: int, uname: str, heads: int,
               dim: int) -> np.ndarray:
        pos = self.planted_positions(b)
        pos = pos[(pos >= p0) & (pos < p1)]
        if pos.size:
            u = self.unit_vector(uname, dim)
            shift = (3.0 * self.wl.sigma * math.sqrt(dim) * u).astype(np.float32)
            x = x.reshape(p1 - p0, heads, dim)
            x[pos - p0] += shift[None, :]
            x = x.reshape(p1 - p0, heads * dim)
        return x

    # -- public tensors (float32, rounded to the workload dtype) -----------
    def q(self, b: int, p0: int, p1: int, name: str = "q") -> np.ndarray:
        wl = self.wl
        x = self._per_position(name, b, p0, p1, wl.H_q * wl.d, "normal", wl.sigma)
        return self._finish(x).reshape(p1 - p0, wl.H_q, wl.d)

    def k(self, b: int, p0: int, p1: int) -> np.ndarray:
        wl = self.wl
        x = self._per_position("k", b, p0, p1, wl.H_kv * wl.d, "normal", wl.sigma)
        x = self._plant(x, b, p0, p1, "u_k", wl.H_kv, wl.d)
        return self._finish(x).reshape(p1 - p0, wl.H_kv, wl.d)

    def v(self, b: int, p0: int, p1: int) -> np.ndarray:
        wl = self.wl
        x = self._per_position("v", b, p0, p1, wl.H_kv * wl.d, "normal", wl.sigma)
        return self._finish(x).reshape(p1 - p0, wl.H_kv, wl.d)

    def q_I(self, b: int, p0: int, p1: int) -> np.ndarray:
        wl = self.wl
        x = self._per_position("q_I", b, p0, p1, wl.H_I * wl.d_I, "normal", wl.sigma)
        return self._finish(x).reshape(p1 - p0, wl.H_I, wl.d_I)

    def k_I(self, b: int, p0: int, p1: int) -> np.ndarray:
        wl = self.wl
        x = self._per_position("k_I", b, p0, p1, wl.H_Ik * wl.d_I, "normal", wl.sigma)
        x = self._plant(x, b, p0, p1, "u_kI", wl.H_Ik, wl.d_I)
        return self._finish(x).reshape(p1 - p0, wl.H_Ik, wl.d_I)

    def w(self, b: int, p0: int, p1: int) -> np.ndarray:
        """Indexer head weights, one per (position, indexer head); always float32."""
        return self._per_position("w", b, p0, p1, self.wl.H_I, "uniform", 1.0)

    def gate(self, b: int, p0: int, p1: int) -> np.ndarray:
        """Gate logits of the linear branch, one per (position, query head)."""
        x = self._per_position("gate", b, p0, p1, self.wl.H_q, "normal", 1.0)
        return self._finish(x)

    def hidden(self, b: int, p0: int, p1: int, D_h: int) -> np.ndarray:
        """Hidden states entering the module, one row of D_h per position."""
        return self._finish(self._per_position("h", b, p0, p1, D_h, "normal", 1.0))

    def gate_weight(self, D_h: int) -> np.ndarray:
        """Per-channel gate weights W_g [H_q*d, D_h] (row c feeds channel c)."""
        N = self.wl.H_q * self.wl.d
        rng = self._rng("W_g", D_h)
        x = rng.standard_normal((N, D_h), dtype=np.float32) * np.float32(1.0 / math.sqrt(D_h))
        return self._finish(x)

    def branch(self, name: str, b: int, p0: int, p1: int) -> np.ndarray:
        """A branch output ("o_lin" or "o_sp") [p1-p0, H_q, d] for the gate alone."""
        x = self._per_position(name, b, p0, p1, self.wl.H_q * self.wl.d, "normal", 1.0)
        return self._finish(x).reshape(p1 - p0, self.wl.H_q, self.wl.d)

    # -- whole-batch helpers -------------------------------------------------
    def batch(self, fn: str, p0: int, p1: int) -> np.ndarray:
        return np.stack([getattr(self, fn)(b, p0, p1) for b in range(self.wl.B)])
