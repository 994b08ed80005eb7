"""Pins of the CPU oracle against facts fixed outside it (CPU only).

Each test checks the oracle against something it does not compute itself:
hand-worked fixtures, brute force on tiny inputs, closed forms and library
routines (numpy / torch) that reach the same mathematical result by another
route, limits and invariants of the method.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ref
from hybrid_linear_top_lightning_b200 import inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))


def _dims(**kw):
    base = dict(B=1, T=1, n_past=0, N_max=None, H_q=1, H_kv=1, d=2, H_I=1, H_Ik=1, d_I=2, M=1,
                phi=0, sm_scale=None)
    base.update(kw)
    if base["N_max"] is None:
        base["N_max"] = base["n_past"] + base["T"]
    return ref.Dims(**base)


# ---------------------------------------------------------------- hand-worked fixtures
@pytest.mark.parametrize("case", ["indexer_shared_key", "indexer_per_head_keys"])
def test_golden_indexer_and_topm(case):
    g = GOLD[case]
    q_I = np.array(g["q_I"], np.float32)[None]
    k_I = np.array(g["k_I"], np.float32)[None]
    w = np.array(g["w"], np.float32)[None]
    for M, expect in g["topm"].items():
        D = _dims(T=g["T"], n_past=g["n_past"], H_I=g["H_I"], H_Ik=g["H_Ik"], d_I=g["d_I"],
                  M=int(M))
        sc = ref.index_scores(D, q_I, k_I, w, 0)
        np.testing.assert_allclose(sc[0, 0], g["scores"], rtol=0, atol=1e-12)
        idx, cnt = ref.topm(D, sc)
        assert idx[0, 0].tolist() == expect
        assert cnt[0, 0] == g["count"][M]


def test_golden_sparse_attention():
    g = GOLD["sparse_attention"]
    D = _dims(T=1, n_past=g["n_past"], H_q=2, H_kv=1, d=2, M=2, sm_scale=g["sm_scale"])
    q = np.array(g["q"], np.float32)[None]
    K = np.array(g["K"], np.float32)[None]
    V = np.array(g["V"], np.float32)[None]
    idx = np.array(g["idx"], np.int32).reshape(1, 1, 2)
    o = ref.sparse_attn(D, q, K, V, idx, np.array([[2]], np.int32))
    np.testing.assert_allclose(o[0, 0], g["o"], atol=g["tol"], rtol=0)


@pytest.mark.parametrize("case,phi", [("linear_identity", 0), ("linear_elu1", 1)])
def test_golden_linear(case, phi):
    g = GOLD[case]
    D = _dims(T=g["T"], d=g["d"], phi=phi)
    q = np.array(g["q"], np.float32).reshape(1, 2, 1, 2)
    k = np.array(g["k"], np.float32).reshape(1, 2, 1, 2)
    v = np.array(g["v"], np.float32).reshape(1, 2, 1, 2)
    o, S, z = ref.linear(D, q, k, v)
    np.testing.assert_allclose(o[0, :, 0], g["o"], atol=1e-12, rtol=0)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-12, rtol=0)
    if phi == 1:
        np.testing.assert_allclose(z[0, 0], g["z"], atol=1e-12, rtol=0)


def test_golden_gate():
    g = GOLD["gate"]
    D = _dims(T=2, H_q=1, d=2)
    logit = np.array(g["logits"], np.float32).reshape(1, 2, 1)
    o_lin = np.array(g["o_lin"]).reshape(1, 2, 1, 2)
    o_sp = np.array(g["o_sp"]).reshape(1, 2, 1, 2)
    o = ref.gate(D, logit, o_lin, o_sp)
    np.testing.assert_allclose(o[0, :, 0], g["o"], atol=g["tol"], rtol=0)


# ---------------------------------------------------------------- indexer vs numpy
@pytest.mark.parametrize("H_Ik", [1, 3])
@pytest.mark.parametrize("w_stride", [0, 3])
def test_index_scores_vs_numpy(H_Ik, w_stride):
    rng = np.random.default_rng(1)
    B, T, n_past, H_I, d_I = 2, 5, 7, 3, 8
    N_max = n_past + T + 2
    q_I = rng.standard_normal((B, T, H_I, d_I)).astype(np.float32)
    k_I = rng.standard_normal((B, N_max, H_Ik, d_I)).astype(np.float32)
    w = rng.random((B, T, H_I) if w_stride else (B, H_I)).astype(np.float32)
    D = _dims(B=B, T=T, n_past=n_past, N_max=N_max, H_I=H_I, H_Ik=H_Ik, d_I=d_I, M=4)
    sc = ref.index_scores(D, q_I, k_I, w, w_stride)
    L = n_past + T
    kfull = k_I[:, :L][:, :, [j % H_Ik for j in range(H_I)]]
    dots = np.einsum("btjc,bsjc->btjs", q_I.astype(np.float64), kfull.astype(np.float64))
    ww = (w if w_stride else np.repeat(w[:, None], T, axis=1)).astype(np.float64)
    expect = np.einsum("btj,btjs->bts", ww, np.maximum(dots, 0.0))
    for t in range(T):
        p = n_past + t
        np.testing.assert_allclose(sc[:, t, :p + 1], expect[:, t, :p + 1], rtol=1e-12, atol=1e-12)
        assert np.all(np.isneginf(sc[:, t, p + 1:]))


def test_index_scores_row_sampling():
    rng = np.random.default_rng(2)
    B, T, n_past, H_I, d_I = 1, 6, 3, 2, 4
    q_I = rng.standard_normal((B, T, H_I, d_I)).astype(np.float32)
    k_I = rng.standard_normal((B, n_past + T, 1, d_I)).astype(np.float32)
    w = rng.random((B, H_I)).astype(np.float32)
    D = _dims(B=B, T=T, n_past=n_past, H_I=H_I, d_I=d_I)
    full = ref.index_scores(D, q_I, k_I, w, 0)
    rows = [5, 0, 2]
    part = ref.index_scores(D, q_I, k_I, w, 0, rows=rows)
    np.testing.assert_array_equal(part[0], full[0, rows])


# ---------------------------------------------------------------- top-M brute force
@pytest.mark.parametrize("levels", [3, 1000])
def test_topm_bruteforce(levels):
    rng = np.random.default_rng(3)
    B, T, n_past, M = 2, 9, 20, 6
    L = n_past + T
    sc = np.floor(rng.random((B, T, L)) * levels) / levels  # many exact ties when levels=3
    for t in range(T):
        sc[:, t, n_past + t + 1:] = -np.inf
    D = _dims(B=B, T=T, n_past=n_past, M=M)
    idx, cnt = ref.topm(D, sc)
    for b in range(B):
        for t in range(T):
            p = n_past + t
            order = sorted(range(p + 1), key=lambda s: (-sc[b, t, s], s))
            keep = sorted(order[:min(M, p + 1)])
            assert cnt[b, t] == len(keep)
            assert idx[b, t, :len(keep)].tolist() == keep
            assert np.all(idx[b, t, len(keep):] == -1)


def test_topm_invariants_and_short_rows():
    rng = np.random.default_rng(4)
    B, T, n_past, M = 1, 12, 0, 8
    sc = rng.random((B, T, T))
    for t in range(T):
        sc[:, t, t + 1:] = -np.inf
    D = _dims(B=B, T=T, n_past=n_past, M=M)
    idx, cnt = ref.topm(D, sc)
    for t in range(T):
        c = cnt[0, t]
        assert c == min(M, t + 1)
        sel = idx[0, t, :c]
        assert np.all(np.diff(sel) > 0)
        unsel = np.setdiff1d(np.arange(t + 1), sel)
        if unsel.size:
            assert sc[0, t, sel].min() >= sc[0, t, unsel].max()
        if t + 1 <= M:
            assert sel.tolist() == list(range(t + 1))


def test_topm_all_equal_scores_take_lowest_positions():
    T, M = 1, 5
    D = _dims(T=T, n_past=40, M=M)
    sc = np.zeros((1, 1, 41))
    idx, cnt = ref.topm(D, sc)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------- sparse attention
def _sdpa_gqa(q, K, V, scale, n_past):
    """torch fp64 causal SDPA with query offset n_past. q [T,H_q,d], K/V [L,H_kv,d]."""
    T, H_q, d = q.shape
    L, H_kv, _ = K.shape
    rep = H_q // H_kv
    qt = torch.tensor(q, dtype=torch.float64).permute(1, 0, 2)
    kt = torch.tensor(K, dtype=torch.float64).permute(1, 0, 2).repeat_interleave(rep, 0)
    vt = torch.tensor(V, dtype=torch.float64).permute(1, 0, 2).repeat_interleave(rep, 0)
    mask = torch.arange(L)[None, :] <= (torch.arange(T)[:, None] + n_past)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return out.permute(1, 0, 2).numpy()


def test_sparse_with_full_budget_is_dense_causal_attention():
    rng = np.random.default_rng(5)
    B, T, n_past, H_q, H_kv, d = 2, 7, 5, 4, 2, 16
    L = n_past + T
    q = rng.standard_normal((B, T, H_q, d)).astype(np.float32)
    K = rng.standard_normal((B, L, H_kv, d)).astype(np.float32)
    V = rng.standard_normal((B, L, H_kv, d)).astype(np.float32)
    q_I = rng.standard_normal((B, T, 2, 4)).astype(np.float32)
    k_I = rng.standard_normal((B, L, 1, 4)).astype(np.float32)
    w = rng.random((B, 2)).astype(np.float32)
    D = _dims(B=B, T=T, n_past=n_past, H_q=H_q, H_kv=H_kv, d=d, H_I=2, d_I=4, M=L)
    idx, cnt = ref.topm(D, ref.index_scores(D, q_I, k_I, w, 0))
    o = ref.sparse_attn(D, q, K, V, idx, cnt)
    dense = ref.dense_attn(D, q, K, V)
    for b in range(B):
        expect = _sdpa_gqa(q[b], K[b], V[b], 1.0 / math.sqrt(d), n_past)
        np.testing.assert_allclose(o[b], expect, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dense[b], expect, rtol=1e-10, atol=1e-12)


def test_sparse_budget_one_returns_value_of_top_key():
    rng = np.random.default_rng(6)
    T, n_past, d = 3, 10, 8
    L = n_past + T
    q = rng.standard_normal((1, T, 2, d)).astype(np.float32)
    K = rng.standard_normal((1, L, 1, d)).astype(np.float32)
    V = rng.standard_normal((1, L, 1, d)).astype(np.float32)
    q_I = rng.standard_normal((1, T, 1, 4)).astype(np.float32)
    k_I = rng.standard_normal((1, L, 1, 4)).astype(np.float32)
    D = _dims(T=T, n_past=n_past, H_q=2, H_kv=1, d=d, H_I=1, d_I=4, M=1)
    sc = ref.index_scores(D, q_I, k_I, np.ones((1, 1), np.float32), 0)
    idx, cnt = ref.topm(D, sc)
    o = ref.sparse_attn(D, q, K, V, idx, cnt)
    for t in range(T):
        p = n_past + t
        best = max(range(p + 1), key=lambda s: (sc[0, t, s], -s))
        for h in range(2):
            np.testing.assert_allclose(o[0, t, h], V[0, best, 0], rtol=0, atol=1e-7)


def test_sparse_is_invariant_to_index_order():
    rng = np.random.default_rng(7)
    d, L = 8, 30
    q = rng.standard_normal((1, 1, 2, d)).astype(np.float32)
    K = rng.standard_normal((1, L, 2, d)).astype(np.float32)
    V = rng.standard_normal((1, L, 2, d)).astype(np.float32)
    D = _dims(T=1, n_past=L - 1, H_q=2, H_kv=2, d=d, M=6)
    sel = np.array([1, 4, 9, 17, 22, 29], np.int32)
    o1 = ref.sparse_attn(D, q, K, V, sel.reshape(1, 1, 6), np.array([[6]], np.int32))
    o2 = ref.sparse_attn(D, q, K, V, rng.permutation(sel).reshape(1, 1, 6), np.array([[6]], np.int32))
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- linear attention
def _phi(x, phi):
    return x if phi == 0 else np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


@pytest.mark.parametrize("phi", [0, 1])
def test_linear_state_and_parallel_form(phi):
    rng = np.random.default_rng(8)
    B, T, H_q, H_kv, d = 2, 11, 4, 2, 8
    q = rng.standard_normal((B, T, H_q, d)).astype(np.float32)
    k = rng.standard_normal((B, T, H_kv, d)).astype(np.float32)
    v = rng.standard_normal((B, T, H_kv, d)).astype(np.float32)
    S0 = rng.standard_normal((B, H_kv, d, d))
    z0 = rng.random((B, H_kv, d)) * 3.0 + 1.0
    D = _dims(B=B, T=T, H_q=H_q, H_kv=H_kv, d=d, phi=phi)
    o, S, z = ref.linear(D, q, k, v, S0=S0, z0=z0)
    rep = H_q // H_kv
    for b in range(B):
        for g in range(H_kv):
            fk = _phi(k[b, :, g].astype(np.float64), phi)
            vv = v[b, :, g].astype(np.float64)
            # closed form of the state: S_T = S_0 + phi(K)^T V (one matmul)
            np.testing.assert_allclose(S[b, g], S0[b, g] + fk.T @ vv, rtol=1e-12, atol=1e-12)
            mask = np.tril(np.ones((T, T)))  # inclusive causal mask
            for hh in range(rep):
                h = g * rep + hh
                fq = _phi(q[b, :, h].astype(np.float64), phi)
                num = fq @ S0[b, g] + (fq @ fk.T * mask) @ vv
                if phi == 0:
                    expect = num
                else:
                    np.testing.assert_allclose(z[b, g], z0[b, g] + fk.sum(0), rtol=1e-12)
                    den = fq @ z0[b, g] + (fq @ fk.T * mask).sum(1)
                    expect = num / den[:, None]
                np.testing.assert_allclose(o[b, :, h], expect, rtol=1e-10, atol=1e-10)


def test_linear_split_calls_carry_state():
    rng = np.random.default_rng(9)
    T, d = 10, 4
    q = rng.standard_normal((1, T, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, T, 1, d)).astype(np.float32)
    v = rng.standard_normal((1, T, 1, d)).astype(np.float32)
    o_full, S_full, _ = ref.linear(_dims(T=T, d=d), q, k, v)
    o_a, S_a, _ = ref.linear(_dims(T=6, d=d), q[:, :6], k[:, :6], v[:, :6])
    o_b, S_b, _ = ref.linear(_dims(T=4, d=d), q[:, 6:], k[:, 6:], v[:, 6:], S0=S_a)
    np.testing.assert_allclose(np.concatenate([o_a, o_b], 1), o_full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S_b, S_full, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- gate limits
def test_gate_limits_select_one_branch():
    rng = np.random.default_rng(10)
    D = _dims(T=3, H_q=2, d=5)
    o_lin = rng.standard_normal((1, 3, 2, 5))
    o_sp = rng.standard_normal((1, 3, 2, 5))
    hi = np.full((1, 3, 2), 100.0, np.float32)
    np.testing.assert_array_equal(ref.gate(D, hi, o_lin, o_sp), o_lin)
    np.testing.assert_allclose(ref.gate(D, -hi, o_lin, o_sp), o_sp, atol=1e-30, rtol=0)


# ---------------------------------------------------------------- whole module
def _tiny_tensors(wl, L):
    gen = inputs.Generator(wl)
    q = gen.batch("q", 0, L)
    k = gen.batch("k", 0, L)
    v = gen.batch("v", 0, L)
    q_I = gen.batch("q_I", 0, L)
    k_I = gen.batch("k_I", 0, L)
    w = gen.batch("w", 0, L)
    gl = gen.batch("gate", 0, L)
    return q, k, v, q_I, k_I, w, gl


@pytest.mark.parametrize("M", [32, 272])
def test_prefill_then_decode_equals_longer_prefill(M):
    """prefill(256) + 16 single-token steps == the last 16 rows of prefill(272)."""
    wl = inputs.TINY.with_(M=M)
    L = wl.n
    q, k, v, q_I, k_I, w, gl = _tiny_tensors(wl, L)
    common = dict(B=1, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I, H_Ik=wl.H_Ik,
                  d_I=wl.d_I, M=M)
    full = ref.forward(ref.Dims(T=L, n_past=0, **common), q, k, v, q_I, k_I, w, wl.H_I,
                       q, k, v, gl)
    pre = ref.forward(ref.Dims(T=256, n_past=0, **common), q[:, :256], k, v, q_I[:, :256], k_I,
                      w[:, :256], wl.H_I, q[:, :256], k[:, :256], v[:, :256], gl[:, :256])
    S = pre["S"]
    for t in range(256, L):
        D1 = ref.Dims(T=1, n_past=t, **common)
        step = ref.forward(D1, q[:, t:t + 1], k, v, q_I[:, t:t + 1], k_I, w[:, t:t + 1], wl.H_I,
                           q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], gl[:, t:t + 1], S0=S)
        S = step["S"]
        np.testing.assert_array_equal(step["idx"][0, 0], full["idx"][0, t])
        np.testing.assert_allclose(step["o"][0, 0], full["o"][0, t], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(S, full["S"], rtol=1e-10, atol=1e-9)
    if M >= L:
        # every position is selected: SA_M is dense causal attention
        dense = ref.dense_attn(ref.Dims(T=L, n_past=0, **common), q, k, v)
        np.testing.assert_allclose(full["o_sp"], dense, rtol=1e-10, atol=1e-12)


def test_batch_elements_are_independent():
    wl = inputs.TINY.with_(B=2, n=40, M=8)
    q, k, v, q_I, k_I, w, gl = _tiny_tensors(wl, 40)
    common = dict(T=40, n_past=0, N_max=40, H_q=2, H_kv=1, d=64, H_I=2, H_Ik=1, d_I=32, M=8)
    both = ref.forward(ref.Dims(B=2, **common), q, k, v, q_I, k_I, w, 2, q, k, v, gl)
    one = ref.forward(ref.Dims(B=1, **common), q[1:], k[1:], v[1:], q_I[1:], k_I[1:], w[1:], 2,
                      q[1:], k[1:], v[1:], gl[1:])
    np.testing.assert_array_equal(both["idx"][1], one["idx"][0])
    np.testing.assert_allclose(both["o"][1], one["o"][0], rtol=1e-13, atol=1e-13)


def test_planted_heavy_keys_are_selected_by_aligned_queries():
    """Queries along the planted direction rank every planted key first."""
    wl = inputs.DECODE_7B.with_(B=1, n=2048, M=64)
    gen = inputs.Generator(wl)
    k_I = gen.k_I(0, 0, wl.n)[None]
    u = gen.unit_vector("u_kI", wl.d_I).astype(np.float32)
    q_I = np.tile(u, (1, 1, wl.H_I, 1)).astype(np.float32).reshape(1, 1, wl.H_I, wl.d_I)
    D = ref.Dims(B=1, T=1, n_past=wl.n - 1, N_max=wl.n, H_q=1, H_kv=1, d=2, H_I=wl.H_I, H_Ik=1,
                 d_I=wl.d_I, M=wl.M)
    idx, cnt = ref.topm(D, ref.index_scores(D, q_I, k_I, np.ones((1, wl.H_I), np.float32), 0))
    planted = gen.planted_positions(0)
    assert planted.size == 20
    assert set(planted.tolist()) <= set(idx[0, 0, :cnt[0, 0]].tolist())


def test_sparse_softmax_is_shift_invariant_at_large_logits():
    """Adding the same large constant to every logit leaves softmax unchanged.

    Built from the hand-worked case: an extra coordinate where q holds 2000
    and every key holds 1 shifts all logits by 2000 (far past exp overflow)."""
    g = GOLD["sparse_attention"]
    q = np.array(g["q"], np.float32)
    K = np.array(g["K"], np.float32)
    V = np.array(g["V"], np.float32)
    q3 = np.concatenate([q, np.full(q.shape[:-1] + (1,), 2000.0, np.float32)], -1)[None]
    K3 = np.concatenate([K, np.ones(K.shape[:-1] + (1,), np.float32)], -1)[None]
    V3 = np.concatenate([V, np.zeros(V.shape[:-1] + (1,), np.float32)], -1)[None]
    D = _dims(T=1, n_past=g["n_past"], H_q=2, H_kv=1, d=3, M=2, sm_scale=1.0)
    idx = np.array(g["idx"], np.int32).reshape(1, 1, 2)
    o = ref.sparse_attn(D, q3, K3, V3, idx, np.array([[2]], np.int32))
    np.testing.assert_allclose(o[0, 0, :, :2], g["o"], atol=g["tol"], rtol=0)
