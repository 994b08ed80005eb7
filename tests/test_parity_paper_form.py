"""GPU parity of the paper's own indexer form against the oracle: every indexer
head has its own keys and the head scores are summed without weights
(LISA, arXiv 2607.19358v1, Sec. 3.2: H_Ik = H_I, w = 1), through lisa_topm
(prefill rows: the tcgen05 per-head score kernel at 8 indexer heads of 64
dims in bf16, the generic kernels otherwise) and lisa_decode_step (bf16 and
fp32).
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, check_topm, max_abs

pytestmark = pytest.mark.gpu


def _dv(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def _wl(dtype):
    base = inputs.PREFILL_1P5B if dtype == "bf16" else inputs.TINY
    return base.with_(B=2, n=700, H_Ik=base.H_I, M=128, dtype=dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_paper_form_topm_prefill_rows(dtype):
    wl = _wl(dtype)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = inputs.Generator(wl)
    T = wl.n
    q_I, k_I = gen.batch("q_I", 0, T), gen.batch("k_I", 0, T)
    w = np.ones((wl.B, T, wl.H_I), np.float32)
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype=dtype)
    idx = torch.empty(wl.B, T, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    lisa.lisa_topm(D, _dv(q_I, dt), _dv(k_I, dt), _dv(w, torch.float32), wl.H_I, idx, cnt, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I, k_I, w, wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, sc)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(wl.B):
        check_topm(g_idx[b], g_cnt[b], r_idx[b], r_cnt[b], sc[b])


@pytest.mark.parametrize("n_past,unit_w", [(0, True), (0, False), (300, True)])
def test_paper_form_topm_prefill_tensor_cores(n_past, unit_w):
    """8 indexer heads with a key each, bf16: the per-head tcgen05 score GEMM;
    partial query and key tiles, a call continuing after cached tokens."""
    wl = inputs.PREFILL_7B.with_(B=2, n=n_past + 700, H_Ik=8, M=160)
    gen = inputs.Generator(wl)
    T, L = 700, n_past + 700
    q_I, k_I = gen.batch("q_I", n_past, L), gen.batch("k_I", 0, L)
    w = np.ones((wl.B, T, wl.H_I), np.float32) if unit_w else gen.batch("w", n_past, L)
    D = lisa.make_dims(wl.B, T, n_past, L, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    idx = torch.empty(wl.B, T, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    lisa.lisa_topm(D, _dv(q_I, torch.bfloat16), _dv(k_I, torch.bfloat16), _dv(w, torch.float32),
                   wl.H_I, idx, cnt, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I, k_I, w, wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, sc)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(wl.B):
        check_topm(g_idx[b], g_cnt[b], r_idx[b], r_cnt[b], sc[b])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_paper_form_decode_step(dtype):
    wl = _wl(dtype)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = inputs.Generator(wl)
    n, p, B = wl.n, wl.n - 1, wl.B
    kc_np, vc_np, kI_np = gen.batch("k", 0, n), gen.batch("v", 0, n), gen.batch("k_I", 0, n)
    q, q_I, gl = gen.batch("q", p, n), gen.batch("q_I", p, n), gen.batch("gate", p, n)
    w = np.ones((B, 1, wl.H_I), np.float32)
    rng = np.random.default_rng(11)
    S0 = (rng.standard_normal((B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    kc, vc, kIc = _dv(kc_np, dt), _dv(vc_np, dt), _dv(kI_np, dt)
    k_new, v_new, kI_new = kc[:, p:].clone(), vc[:, p:].clone(), kIc[:, p:].clone()
    tq = _dv(q, dt)
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype=dtype)
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=dt, device="cuda")
    idx = torch.empty(B, 1, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    S = torch.from_numpy(S0).cuda()
    args = lisa.decode_args(tq, k_new, v_new, _dv(q_I, dt), kI_new, _dv(w, torch.float32), wl.H_I,
                            tq, k_new, v_new, _dv(gl, dt), kc, vc, kIc, S, None, o, idx, cnt)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    lisa.lisa_decode_step(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=B, T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I, kI_np, w, wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, sc)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], sc[:, 0])
    r_lin, _, _ = ref.linear(Dr, q, kc_np[:, p:], vc_np[:, p:], S0=S0)
    r_sp = ref.sparse_attn(Dr, q, kc_np, vc_np, g_idx, g_cnt)
    r_o = ref.gate(Dr, gl, r_lin, r_sp)
    err = max_abs(o.float().cpu().numpy(), r_o)
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("B,n,unit_w", [(8, 16384, True), (3, 5000, False), (2, 700, True)])
def test_paper_form_fast_decode_7b(B, n, unit_w):
    """The sm_100a decode path with a key per indexer head (H_Ik = H_I = 8)."""
    wl = inputs.DECODE_7B.with_(B=B, n=n, H_Ik=8)
    dt = torch.bfloat16
    gen = inputs.Generator(wl)
    p = n - 1
    kc = torch.empty(B, n, wl.H_kv, wl.d, dtype=dt, device="cuda")
    vc = torch.empty_like(kc)
    kIc = torch.empty(B, n, 8, wl.d_I, dtype=dt, device="cuda")
    k_I_all = []
    for b in range(B):
        kc[b], vc[b] = _dv(gen.k(b, 0, n), dt), _dv(gen.v(b, 0, n), dt)
        kI_b = gen.k_I(b, 0, n)
        kIc[b] = _dv(kI_b, dt)
        k_I_all.append(kI_b)
    kI_np = np.stack(k_I_all)
    q, q_I, gl = gen.batch("q", p, n), gen.batch("q_I", p, n), gen.batch("gate", p, n)
    w = np.ones((B, 1, 8), np.float32) if unit_w else gen.batch("w", p, n)
    rng = np.random.default_rng(12)
    S0 = (rng.standard_normal((B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    k_new, v_new, kI_new = kc[:, p:].clone(), vc[:, p:].clone(), kIc[:, p:].clone()
    kIc[:, p:] = 7.0  # the append must fill position p of the k_I cache
    tq = _dv(q, dt)
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, 8, 8, wl.d_I, wl.M)
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=dt, device="cuda")
    idx = torch.empty(B, 1, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    S = torch.from_numpy(S0).cuda()
    args = lisa.decode_args(tq, k_new, v_new, _dv(q_I, dt), kI_new, _dv(w, torch.float32), 8, tq,
                            k_new, v_new, _dv(gl, dt), kc, vc, kIc, S, None, o, idx, cnt)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    lisa.lisa_decode_step(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    assert torch.equal(kIc[:, p:], kI_new)
    sample = [0, B - 1]
    kc_np = np.stack([gen.k(b, 0, n) for b in sample])
    vc_np = np.stack([gen.v(b, 0, n) for b in sample])
    Dr = ref.Dims(B=len(sample), T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=8, H_Ik=8, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I[sample], kI_np[sample], w[sample], 8)
    r_idx, r_cnt = ref.topm(Dr, sc)
    g_idx, g_cnt = idx.cpu().numpy()[sample], cnt.cpu().numpy()[sample]
    check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], sc[:, 0])
    r_lin, _, _ = ref.linear(Dr, q[sample], kc_np[:, p:], vc_np[:, p:], S0=S0[sample])
    r_sp = ref.sparse_attn(Dr, q[sample], kc_np, vc_np, g_idx, g_cnt)
    r_o = ref.gate(Dr, gl[sample], r_lin, r_sp)
    err = max_abs(o.float().cpu().numpy()[sample], r_o)
    assert err <= TOL["bf16"], err
