"""GPU parity of the prefill paths (bf16) against the CPU oracle.

Top-M sets: equal up to near-ties (relative score gap <= 1e-3 at the M-th
score).  Outputs: max abs error <= 2e-2.  The full 1.5B-shape prefill is
checked on every row; the 7B shape (n = 16384) on sampled rows, including the
first row past the budget, tile edges and the last row.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, check_topm, max_abs

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _dv(a, dt=BF):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def _topm_case(wl, T, n_past, rows=None, w_tok=True, zero_qI=False):
    gen = inputs.Generator(wl)
    L = n_past + T
    q_I = gen.batch("q_I", n_past, L)
    if zero_qI:
        q_I = np.zeros_like(q_I)
    k_I = gen.batch("k_I", 0, L)
    w = gen.batch("w", n_past, L)
    if not w_tok:
        w = np.ascontiguousarray(w[:, 0])
    D = lisa.make_dims(wl.B, T, n_past, L, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    idx = torch.empty(wl.B, T, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    stride = wl.H_I if w_tok else 0
    lisa.lisa_topm(D, _dv(q_I), _dv(k_I), _dv(w, torch.float32), stride, idx, cnt, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I, k_I, w, stride, rows=rows)
    r_idx, r_cnt = ref.topm(Dr, sc, rows=rows)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    if rows is not None:
        g_idx, g_cnt = g_idx[:, rows], g_cnt[:, rows]
    swaps = 0
    for b in range(wl.B):
        swaps += check_topm(g_idx[b], g_cnt[b], r_idx[b], r_cnt[b], sc[b])
    return g_idx, g_cnt, swaps


def test_topm_prefill_1p5b_every_row():
    _topm_case(inputs.PREFILL_1P5B, T=4096, n_past=0)


def test_topm_prefill_7b_sampled_rows():
    wl = inputs.PREFILL_7B
    rows = np.array([0, 1, 31, 32, 127, 128, 2046, 2047, 2048, 2049, 4095, 5000, 8191, 8192,
                     12345, 16000, 16351, 16352, 16383], np.int32)
    _topm_case(wl, T=wl.n, n_past=0, rows=rows)


@pytest.mark.parametrize("H_I,w_tok", [(8, True), (2, False), (4, True)])
def test_topm_prefill_ragged_batched_continued(H_I, w_tok):
    """Two sequences, 77 new rows after 200 cached ones: partial query and key tiles."""
    wl = inputs.PREFILL_7B.with_(B=2, n=277, H_I=H_I, M=64)
    _topm_case(wl, T=77, n_past=200, w_tok=w_tok)


def test_topm_prefill_all_ties_take_lowest_positions():
    wl = inputs.PREFILL_7B.with_(B=1, n=600, M=50)
    idx, cnt, _ = _topm_case(wl, T=600, n_past=0, zero_qI=True)
    for t in range(600):
        c = min(50, t + 1)
        assert np.array_equal(idx[0, t, :c], np.arange(c))


# ---------------------------------------------------------------- linear attention prefill
def _linear_case(wl, T, phi, rows, S0_scale=0.0):
    gen = inputs.Generator(wl)
    q = gen.batch("q", 0, T)
    k = gen.batch("k", 0, T)
    v = gen.batch("v", 0, T)
    rng = np.random.default_rng(3)
    S0 = (rng.standard_normal((wl.B, wl.H_kv, wl.d, wl.d)) * S0_scale).astype(np.float32)
    z0 = (rng.random((wl.B, wl.H_kv, wl.d)) * 5.0 + 1.0).astype(np.float32) if phi else None
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       chunk=wl.chunk, phi=phi)
    S = torch.from_numpy(S0.copy()).cuda()
    z = torch.from_numpy(z0.copy()).cuda() if phi else None
    o = torch.empty(wl.B, T, wl.H_q, wl.d, dtype=BF, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_LINEAR_PREFILL)
    lisa.lisa_linear_prefill(D, _dv(q), _dv(k), _dv(v), S, z, o, ws)
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
    r_o, r_S, r_z = ref.linear(Dr, q, k, v, S0=S0, z0=z0, rows=rows)
    g_o = o.float().cpu().numpy()[:, rows]
    err = max_abs(g_o, r_o)
    assert err <= TOL["bf16"], err
    # the state is fp32: compare relative to its scale
    assert max_abs(S.cpu().numpy(), r_S) <= 1e-3 * max(1.0, np.abs(r_S).max())
    if phi:
        assert max_abs(z.cpu().numpy(), r_z) <= 1e-3 * max(1.0, np.abs(r_z).max())
    return err


def test_linear_prefill_1p5b_all_rows():
    wl = inputs.PREFILL_1P5B
    _linear_case(wl, wl.n, 0, rows=np.arange(wl.n, dtype=np.int32))


def test_linear_prefill_7b_sampled_rows():
    wl = inputs.PREFILL_7B
    rows = np.array([0, 1, 63, 64, 65, 4095, 8191, 12000, 16383], np.int32)
    _linear_case(wl, wl.n, 0, rows=rows)


@pytest.mark.parametrize("phi", [lisa.LISA_PHI_IDENTITY, lisa.LISA_PHI_ELU1_NORM])
def test_linear_prefill_ragged_batched_with_state(phi):
    wl = inputs.PREFILL_7B.with_(B=2, n=333)
    _linear_case(wl, 333, phi, rows=np.arange(333, dtype=np.int32), S0_scale=0.3)


# ---------------------------------------------------------------- sparse attention, whole module
def _module_case(wl, T, rows):
    """Prefill of T tokens through the four entry points vs the oracle module."""
    gen = inputs.Generator(wl)
    x = {n: gen.batch(n, 0, T) for n in ("q", "k", "v", "q_I", "k_I", "w", "gate")}
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       chunk=wl.chunk)
    q, k, v = _dv(x["q"]), _dv(x["k"]), _dv(x["v"])
    idx = torch.empty(wl.B, T, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    lisa.lisa_topm(D, _dv(x["q_I"]), _dv(x["k_I"]), _dv(x["w"], torch.float32), wl.H_I, idx, cnt, ws)
    o_sp = torch.empty(wl.B, T, wl.H_q, wl.d, dtype=BF, device="cuda")
    ws_a = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, q, k, v, idx, cnt, o_sp, ws_a)
    S = torch.zeros(wl.B, wl.H_kv, wl.d, wl.d, device="cuda")
    o_lin = torch.empty_like(o_sp)
    ws_l = lisa.workspace(D, lisa.LISA_OP_LINEAR_PREFILL)
    lisa.lisa_linear_prefill(D, q, k, v, S, None, o_lin, ws_l)
    o = torch.empty_like(o_sp)
    lisa.lisa_gate_fuse(D, _dv(x["gate"]), o_lin, o_sp, o)
    assert lisa.lisa_check_status(ws_a) == lisa.LISA_OK
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, x["q_I"], x["k_I"], x["w"], wl.H_I, rows=rows)
    r_idx, r_cnt = ref.topm(Dr, sc, rows=rows)
    g_idx, g_cnt = idx.cpu().numpy()[:, rows], cnt.cpu().numpy()[:, rows]
    for b in range(wl.B):
        check_topm(g_idx[b], g_cnt[b], r_idx[b], r_cnt[b], sc[b])
    # attention and gate of the oracle on the GPU's own index sets
    r_sp = ref.sparse_attn(Dr, x["q"], x["k"], x["v"], g_idx, g_cnt, rows=rows)
    r_lin, _, _ = ref.linear(Dr, x["q"], x["k"], x["v"], rows=rows)
    r_o = ref.gate(Dr, x["gate"], r_lin, r_sp, rows=rows)
    for name, g, r in (("o_sparse", o_sp, r_sp), ("o_lin", o_lin, r_lin), ("o", o, r_o)):
        err = max_abs(g.float().cpu().numpy()[:, rows], r)
        assert err <= TOL["bf16"], (name, err)


def _whole_prefill_case(wl, T, rows, elu=False):
    """The single whole-module entry point (lisa_prefill) vs the oracle module."""
    gen = inputs.Generator(wl)
    x = {n: gen.batch(n, 0, T) for n in ("q", "k", "v", "q_I", "k_I", "w", "gate")}
    phi = lisa.LISA_PHI_ELU1_NORM if elu else lisa.LISA_PHI_IDENTITY
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       chunk=wl.chunk, phi=phi)
    q, k, v = _dv(x["q"]), _dv(x["k"]), _dv(x["v"])
    idx = torch.empty(wl.B, T, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    S = torch.zeros(wl.B, wl.H_kv, wl.d, wl.d, device="cuda")
    z = torch.zeros(wl.B, wl.H_kv, wl.d, device="cuda") if elu else None
    o = torch.empty(wl.B, T, wl.H_q, wl.d, dtype=BF, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_PREFILL)
    args = lisa.prefill_args(q, k, v, _dv(x["q_I"]), _dv(x["k_I"]), _dv(x["w"], torch.float32),
                             wl.H_I, q, k, v, _dv(x["gate"]), S, z, o, idx, cnt)
    lisa.lisa_prefill(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
    sc = ref.index_scores(Dr, x["q_I"], x["k_I"], x["w"], wl.H_I, rows=rows)
    r_idx, r_cnt = ref.topm(Dr, sc, rows=rows)
    g_idx, g_cnt = idx.cpu().numpy()[:, rows], cnt.cpu().numpy()[:, rows]
    for b in range(wl.B):
        check_topm(g_idx[b], g_cnt[b], r_idx[b], r_cnt[b], sc[b])
    r_sp = ref.sparse_attn(Dr, x["q"], x["k"], x["v"], g_idx, g_cnt, rows=rows)
    r_lin, r_S, r_z = ref.linear(Dr, x["q"], x["k"], x["v"], rows=rows)
    r_o = ref.gate(Dr, x["gate"], r_lin, r_sp, rows=rows)
    err = max_abs(o.float().cpu().numpy()[:, rows], r_o)
    assert err <= TOL["bf16"], err
    s_err = max_abs(S.cpu().numpy(), r_S)
    assert s_err <= 1e-3 * max(1.0, float(np.abs(r_S).max())), s_err
    if elu:
        z_err = max_abs(z.cpu().numpy(), r_z)
        assert z_err <= 1e-3 * max(1.0, float(np.abs(r_z).max())), z_err


def test_prefill_entry_point_1p5b_every_row():
    wl = inputs.PREFILL_1P5B
    _whole_prefill_case(wl, wl.n, rows=np.arange(wl.n, dtype=np.int32))


def test_prefill_entry_point_ragged_batched_elu():
    wl = inputs.PREFILL_1P5B.with_(B=3, n=777)
    _whole_prefill_case(wl, wl.n, rows=np.array([0, 1, 63, 64, 511, 512, 700, 776], np.int32),
                        elu=True)


def test_prefill_module_1p5b_every_row():
    wl = inputs.PREFILL_1P5B
    _module_case(wl, wl.n, rows=np.arange(wl.n, dtype=np.int32))


def test_prefill_module_7b_sampled_rows():
    wl = inputs.PREFILL_7B
    rows = np.array([0, 5, 2047, 2048, 2049, 7777, 16383], np.int32)
    _module_case(wl, wl.n, rows=rows)


def test_sparse_attention_reports_out_of_range_positions_bf16():
    """The tensor-core path masks and reports an index outside [0, p]."""
    wl = inputs.PREFILL_7B.with_(B=1, n=64, M=8)
    gen = inputs.Generator(wl)
    q, k, v = (_dv(gen.batch(n, 0, 64)) for n in ("q", "k", "v"))
    D = lisa.make_dims(1, 1, 40, 64, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, 8)
    idx = torch.tensor([[[0, 3, 41, 5, -1, 7, 8, 9]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[8]], dtype=torch.int32, device="cuda")
    o = torch.empty(1, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, q[:, 40:41].contiguous(), k, v, idx, cnt, o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_ERR_DEVICE_BOUNDS
    # the valid entries alone give the result
    Dr = ref.Dims(B=1, T=1, n_past=40, N_max=64, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=1, d_I=wl.d_I, M=8)
    good = np.array([[[0, 3, 5, 7, 8, 9, -1, -1]]], np.int32)
    r = ref.sparse_attn(Dr, gen.batch("q", 40, 41), gen.batch("k", 0, 64), gen.batch("v", 0, 64),
                        good, np.array([[6]], np.int32))
    assert max_abs(o.float().cpu().numpy(), r) <= TOL["bf16"]
