"""Pins of the oracle's functions for the rows after the main path (CPU only):
the sliding-window sparse branch of Stage 1, the segment state transfer of
Sec. 3.3 (Eq. 6-9) and the per-channel gate of Eq. 5 (LISA, arXiv
2607.19358v1).  None re-types the oracle's own formula: hand-worked values,
brute force, closed forms and limits.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import ref

HERE = os.path.dirname(os.path.abspath(__file__))


def _dims(**kw):
    base = dict(B=2, T=1, n_past=0, N_max=64, H_q=4, H_kv=2, d=8, H_I=2, H_Ik=1, d_I=8, M=8)
    base.update(kw)
    return ref.Dims(**base)


# ---------------------------------------------------------------- sliding window
@pytest.mark.parametrize("M", [1, 5, 64])
def test_window_indices_brute_force(M):
    T, n_past = 30, 11
    D = _dims(T=T, n_past=n_past, M=M)
    idx, cnt = ref.window_indices(D)
    for b in range(D.B):
        for t in range(T):
            p = n_past + t
            want = list(range(max(0, p - M + 1), p + 1))
            assert cnt[b, t] == len(want)
            assert list(idx[b, t, :len(want)]) == want
            assert np.all(idx[b, t, len(want):] == -1)


def test_window_covering_the_context_is_dense_attention():
    rng = np.random.default_rng(3)
    T = 12
    D = _dims(T=T, n_past=0, N_max=T, M=T)
    q = rng.standard_normal((D.B, T, D.H_q, D.d)).astype(np.float32)
    k = rng.standard_normal((D.B, T, D.H_kv, D.d)).astype(np.float32)
    v = rng.standard_normal((D.B, T, D.H_kv, D.d)).astype(np.float32)
    idx, cnt = ref.window_indices(D)
    sp = ref.sparse_attn(D, q, k, v, idx, cnt)
    dense = ref.dense_attn(D, q, k, v)
    np.testing.assert_allclose(sp, dense, rtol=1e-12, atol=1e-12)


def test_window_of_one_is_the_current_value_row():
    rng = np.random.default_rng(4)
    T = 6
    D = _dims(T=T, n_past=0, N_max=T, M=1)
    q = rng.standard_normal((D.B, T, D.H_q, D.d)).astype(np.float32)
    k = rng.standard_normal((D.B, T, D.H_kv, D.d)).astype(np.float32)
    v = rng.standard_normal((D.B, T, D.H_kv, D.d)).astype(np.float32)
    idx, cnt = ref.window_indices(D)
    sp = ref.sparse_attn(D, q, k, v, idx, cnt)
    group = D.H_q // D.H_kv
    for h in range(D.H_q):
        np.testing.assert_allclose(sp[:, :, h], v[:, :, h // group], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- state transfer
def test_state_transfer_hand_worked_segments():
    case = json.load(open(os.path.join(HERE, "golden", "state_transfer_cases.json")))
    D = _dims(B=1, H_kv=1, d=1)
    G = np.zeros((1, 1, 1, 1))
    for seg in case["segments"]:
        S_end = np.full((1, 1, 1, 1), seg["S_end"])
        S_start = np.full((1, 1, 1, 1), seg["S_start"])
        S_t, S_next, G = ref.state_transfer(D, S_end, S_start, G, seg["t"], case["alpha"])
        assert S_t.item() == pytest.approx(seg["S_t"], abs=1e-15)
        assert S_next.item() == pytest.approx(seg["S_t"], abs=1e-15)
        assert G.item() == pytest.approx(seg["grad_sum"], abs=1e-15)


def test_state_transfer_limits():
    rng = np.random.default_rng(5)
    D = _dims(B=2, H_kv=3, d=4)
    shape = (2, 3, 4, 4)
    S_start = rng.standard_normal(shape)
    S_end = S_start + rng.standard_normal(shape)
    G = rng.standard_normal(shape) * 3
    # alpha = 0: no correction, the tokens' own state stands
    S_t, _, G1 = ref.state_transfer(D, S_end, S_start, G, 4, 0.0)
    np.testing.assert_allclose(S_t, S_end, rtol=0, atol=1e-12)
    np.testing.assert_allclose(G1, G + (S_end - S_start), rtol=0, atol=1e-12)
    # alpha = 1 at the first segment: the (zero) global direction alone
    S_t, _, _ = ref.state_transfer(D, S_end, S_start, np.zeros(shape), 1, 1.0)
    np.testing.assert_allclose(S_t, S_start, rtol=0, atol=1e-12)
    # alpha = 1 later: the mean of the earlier directions alone
    S_t, _, _ = ref.state_transfer(D, S_end, S_start, G, 4, 1.0)
    np.testing.assert_allclose(S_t, S_start + G / 3, rtol=0, atol=1e-12)


def test_state_transfer_segments_compose():
    """Running segments one after another keeps grad_sum = sum of the raw
    directions and each start equal to the previous corrected state."""
    rng = np.random.default_rng(6)
    D = _dims(B=1, H_kv=1, d=3)
    shape = (1, 1, 3, 3)
    start = np.zeros(shape)
    G = np.zeros(shape)
    raws = []
    for t in range(1, 6):
        end = start + rng.standard_normal(shape)
        raws.append(end - start)
        S_t, start, G = ref.state_transfer(D, end, start, G, t, 0.3)
        mean_prev = np.mean(raws[:-1], axis=0) if t > 1 else np.zeros(shape)
        expect = (end - raws[-1]) + 0.7 * raws[-1] + 0.3 * mean_prev
        np.testing.assert_allclose(S_t, expect, rtol=0, atol=1e-12)
        np.testing.assert_allclose(G, np.sum(raws, axis=0), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- per-channel gate
def test_gate_channel_against_a_matmul_and_its_limits():
    rng = np.random.default_rng(7)
    D = _dims(B=2, T=3, H_q=2, d=4)
    D_h = 5
    h = rng.standard_normal((D.B, D.T, D_h)).astype(np.float32)
    W = rng.standard_normal((D.H_q * D.d, D_h)).astype(np.float32)
    o_lin = rng.standard_normal((D.B, D.T, D.H_q, D.d))
    o_sp = rng.standard_normal((D.B, D.T, D.H_q, D.d))
    got = ref.gate_channel(D, D_h, h, W, o_lin, o_sp)
    g = torch.sigmoid(torch.from_numpy(h.astype(np.float64)) @ torch.from_numpy(W.astype(np.float64)).T)
    g = g.numpy().reshape(D.B, D.T, D.H_q, D.d)
    np.testing.assert_allclose(got, g * o_lin + (1 - g) * o_sp, rtol=1e-12, atol=1e-12)
    # W = 0: an even mix
    half = ref.gate_channel(D, D_h, h, np.zeros_like(W), o_lin, o_sp)
    np.testing.assert_allclose(half, 0.5 * (o_lin + o_sp), rtol=0, atol=1e-12)
    # a large positive gate logit keeps the linear branch
    big = ref.gate_channel(D, D_h, np.ones_like(h), np.full_like(W, 50.0), o_lin, o_sp)
    np.testing.assert_allclose(big, o_lin, rtol=0, atol=1e-12)
