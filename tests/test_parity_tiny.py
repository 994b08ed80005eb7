"""GPU parity on the tiny fp32 workload: prefill(256) through the separate
entry points, then 16 fused decode steps, each against the CPU oracle.

Tolerance: max abs error <= 1e-4 (fp32 outputs); top-M sets equal up to
near-ties (relative score gap <= 1e-3 at the M-th largest score).
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, check_topm, dev, max_abs

pytestmark = pytest.mark.gpu

N_PRE = 256


def _tensors(wl):
    gen = inputs.Generator(wl)
    L = wl.n
    return {name: gen.batch(name, 0, L) for name in ("q", "k", "v", "q_I", "k_I", "w", "gate")}


def _ref_dims(wl, T, n_past, phi):
    return ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=wl.n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                    H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)


def _dims(wl, T, n_past, phi):
    return lisa.make_dims(wl.B, T, n_past, wl.n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I,
                          wl.M, chunk=wl.chunk, dtype=wl.dtype, phi=phi)


@pytest.mark.parametrize("phi", [lisa.LISA_PHI_IDENTITY, lisa.LISA_PHI_ELU1_NORM])
@pytest.mark.parametrize("M", [32, 272])
def test_tiny_prefill_then_decode(M, phi):
    wl = inputs.TINY.with_(M=M)
    x = _tensors(wl)
    tol = TOL[wl.dtype]
    L, d = wl.n, wl.d
    f32 = torch.float32

    # ---- prefill over positions [0, 256) with the separate entry points
    Dr = _ref_dims(wl, N_PRE, 0, phi)
    sl = slice(0, N_PRE)
    r_scores = ref.index_scores(Dr, x["q_I"][:, sl], x["k_I"], x["w"][:, sl], wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, r_scores)
    r_lin, r_S, r_z = ref.linear(Dr, x["q"][:, sl], x["k"][:, sl], x["v"][:, sl])

    kc = torch.zeros(1, L, wl.H_kv, d, device="cuda")
    vc = torch.zeros_like(kc)
    kIc = torch.zeros(1, L, wl.H_Ik, wl.d_I, device="cuda")
    kc[:, sl] = dev(x["k"][:, sl])
    vc[:, sl] = dev(x["v"][:, sl])
    kIc[:, sl] = dev(x["k_I"][:, sl])
    D = _dims(wl, N_PRE, 0, phi)
    q = dev(x["q"][:, sl]).contiguous()
    qI = dev(x["q_I"][:, sl]).contiguous()
    w = dev(x["w"][:, sl]).contiguous()
    gl = dev(x["gate"][:, sl]).contiguous()
    idx = torch.empty(1, N_PRE, M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, N_PRE, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    lisa.lisa_topm(D, qI, kIc, w, wl.H_I, idx, cnt, ws)
    o_sp = torch.empty(1, N_PRE, wl.H_q, d, device="cuda")
    ws_a = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, q, kc, vc, idx, cnt, o_sp, ws_a)
    S = torch.zeros(1, wl.H_kv, d, d, device="cuda")
    z = torch.zeros(1, wl.H_kv, d, device="cuda") if phi else None
    o_lin = torch.empty_like(o_sp)
    ws_l = lisa.workspace(D, lisa.LISA_OP_LINEAR_PREFILL)
    k_L = dev(x["k"][:, sl]).contiguous()
    v_L = dev(x["v"][:, sl]).contiguous()
    lisa.lisa_linear_prefill(D, q, k_L, v_L, S, z, o_lin, ws_l)
    o = torch.empty_like(o_sp)
    lisa.lisa_gate_fuse(D, gl, o_lin, o_sp, o)
    assert lisa.lisa_check_status(ws_a) == lisa.LISA_OK

    g_idx = idx.cpu().numpy()
    check_topm(g_idx[0], cnt.cpu().numpy()[0], r_idx[0], r_cnt[0], r_scores[0])
    r_sp = ref.sparse_attn(Dr, x["q"][:, sl], x["k"], x["v"], g_idx, cnt.cpu().numpy())
    r_o = ref.gate(Dr, x["gate"][:, sl], r_lin, r_sp)
    assert max_abs(o_sp.cpu().numpy(), r_sp) <= tol
    assert max_abs(o_lin.cpu().numpy(), r_lin) <= tol
    assert max_abs(o.cpu().numpy(), r_o) <= tol
    assert max_abs(S.cpu().numpy(), r_S) <= tol
    if phi:
        assert max_abs(z.cpu().numpy(), r_z) <= tol

    # ---- 16 fused decode steps, each appending its token
    o1 = torch.empty(1, 1, wl.H_q, d, device="cuda")
    idx1 = torch.empty(1, 1, M, dtype=torch.int32, device="cuda")
    cnt1 = torch.empty(1, 1, dtype=torch.int32, device="cuda")
    for t in range(N_PRE, L):
        D1 = _dims(wl, 1, t, phi)
        Dr1 = _ref_dims(wl, 1, t, phi)
        st = slice(t, t + 1)
        tq, tk, tv = (dev(x[n][:, st]).contiguous() for n in ("q", "k", "v"))
        args = lisa.decode_args(tq, tk, tv, dev(x["q_I"][:, st]).contiguous(),
                                dev(x["k_I"][:, st]).contiguous(), dev(x["w"][:, st]).contiguous(),
                                wl.H_I, tq, tk, tv, dev(x["gate"][:, st]).contiguous(), kc, vc, kIc,
                                S, z, o1, idx1, cnt1)
        ws_d = lisa.workspace(D1, lisa.LISA_OP_DECODE_STEP)
        lisa.lisa_decode_step(D1, args, ws_d)
        assert lisa.lisa_check_status(ws_d) == lisa.LISA_OK

        rs = ref.index_scores(Dr1, x["q_I"][:, st], x["k_I"], x["w"][:, st], wl.H_I)
        ri, rc = ref.topm(Dr1, rs)
        gi, gc = idx1.cpu().numpy(), cnt1.cpu().numpy()
        check_topm(gi[0], gc[0], ri[0], rc[0], rs[0])
        r_lin1, r_S, r_z = ref.linear(Dr1, x["q"][:, st], x["k"][:, st], x["v"][:, st], S0=r_S,
                                      z0=r_z)
        r_sp1 = ref.sparse_attn(Dr1, x["q"][:, st], x["k"], x["v"], gi, gc)
        r_o1 = ref.gate(Dr1, x["gate"][:, st], r_lin1, r_sp1)
        assert max_abs(o1.cpu().numpy(), r_o1) <= tol, t
    assert max_abs(S.cpu().numpy(), r_S) <= tol
    # the cache now holds every token
    np.testing.assert_array_equal(kc.cpu().numpy(), x["k"])
    np.testing.assert_array_equal(kIc.cpu().numpy(), x["k_I"])


def test_tiny_index_scores_and_dense_attention():
    wl = inputs.TINY
    x = _tensors(wl)
    L = wl.n
    D = _dims(wl, L, 0, 0)
    Dr = _ref_dims(wl, L, 0, 0)
    scores = torch.empty(1, L, L, device="cuda")
    lisa.lisa_index_scores(D, dev(x["q_I"]), dev(x["k_I"]), dev(x["w"]), wl.H_I, scores)
    r = ref.index_scores(Dr, x["q_I"], x["k_I"], x["w"], wl.H_I)
    g = scores.cpu().numpy()
    fin = np.isfinite(r)
    assert np.array_equal(fin, np.isfinite(g))
    np.testing.assert_allclose(g[fin], r[fin], rtol=1e-5, atol=1e-5)

    o = torch.empty(1, L, wl.H_q, wl.d, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_DENSE_ATTN)
    lisa.lisa_dense_attn(D, dev(x["q"]), dev(x["k"]), dev(x["v"]), o, ws)
    r_o = ref.dense_attn(Dr, x["q"], x["k"], x["v"])
    assert max_abs(o.cpu().numpy(), r_o) <= TOL["f32"]


def test_out_of_range_index_is_reported_not_faulted():
    """An index outside [0, p] is skipped and reported through the status word."""
    wl = inputs.TINY.with_(M=4)
    x = _tensors(wl)
    D = _dims(wl, 1, 10, 0)
    idx = torch.tensor([[[0, 3, 11, 5]]], dtype=torch.int32, device="cuda")  # 11 > p = 10
    cnt = torch.tensor([[4]], dtype=torch.int32, device="cuda")
    o = torch.empty(1, 1, wl.H_q, wl.d, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, dev(x["q"][:, 10:11]).contiguous(), dev(x["k"]), dev(x["v"]), idx,
                          cnt, o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_ERR_DEVICE_BOUNDS
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK  # cleared on read
