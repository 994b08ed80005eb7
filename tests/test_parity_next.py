"""GPU parity of the rows after the main path against the oracle: the
sliding-window sparse branch of Stage 1 (index rows and the decode step) and
the segment state transfer of Sec. 3.3 Eq. 6-9 (LISA, arXiv 2607.19358v1).
Tolerances as for the main path: 2e-2 (bf16 outputs), 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, max_abs

pytestmark = pytest.mark.gpu


def _dv(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def _window_decode_case(wl, M):
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    gen = inputs.Generator(wl)
    n, p, B = wl.n, wl.n - 1, wl.B
    kc_np, vc_np = gen.batch("k", 0, n), gen.batch("v", 0, n)
    q, gl = gen.batch("q", p, n), gen.batch("gate", p, n)
    rng = np.random.default_rng(21)
    S0 = (rng.standard_normal((B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    kc, vc = _dv(kc_np, dt), _dv(vc_np, dt)
    kc[:, p:] = 7.0  # the append must fill position p
    vc[:, p:] = 7.0
    k_new, v_new = _dv(kc_np[:, p:], dt), _dv(vc_np[:, p:], dt)
    tq = _dv(q, dt)
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, M, dtype=wl.dtype)
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=dt, device="cuda")
    idx = torch.full((B, 1, M), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    S = torch.from_numpy(S0).cuda()
    args = lisa.decode_args(tq, k_new, v_new, None, None, None, 0, tq, k_new, v_new, _dv(gl, dt),
                            kc, vc, None, S, None, o, idx, cnt)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    lisa.lisa_decode_step_window(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=B, T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=M)
    r_idx, r_cnt = ref.window_indices(Dr)
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), r_cnt)
    r_sp = ref.sparse_attn(Dr, q, kc_np, vc_np, r_idx, r_cnt)
    r_lin, r_S, _ = ref.linear(Dr, q, kc_np[:, p:], vc_np[:, p:], S0=S0)
    r_o = ref.gate(Dr, gl, r_lin, r_sp)
    err = max_abs(o.float().cpu().numpy(), r_o)
    assert err <= TOL[wl.dtype], err
    assert max_abs(S.cpu().numpy(), r_S) <= 1e-3 * max(1.0, float(np.abs(r_S).max()))
    assert kc[:, p].float().cpu().numpy() == pytest.approx(
        torch.from_numpy(kc_np[:, p]).to(dt).float().numpy())


def test_window_decode_step_7b_full_size():
    _window_decode_case(inputs.DECODE_7B, 2048)


@pytest.mark.parametrize("n,M", [(1, 2048), (1500, 512), (3001, 2048), (777, 32)])
def test_window_decode_step_ragged(n, M):
    _window_decode_case(inputs.DECODE_7B.with_(B=3, n=n), M)


def test_window_decode_step_generic_fp32():
    wl = inputs.TINY.with_(B=2, n=300)
    _window_decode_case(wl, 32)


def test_window_rows_feed_sparse_attention_prefill():
    wl = inputs.PREFILL_1P5B.with_(B=2, n=1200)
    dt = torch.bfloat16
    gen = inputs.Generator(wl)
    T = wl.n
    q, k, v = gen.batch("q", 0, T), gen.batch("k", 0, T), gen.batch("v", 0, T)
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, 256)
    idx = torch.empty(wl.B, T, 256, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, T, dtype=torch.int32, device="cuda")
    lisa.lisa_window_indices(D, idx, cnt)
    o = torch.empty(wl.B, T, wl.H_q, wl.d, dtype=dt, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, _dv(q, dt), _dv(k, dt), _dv(v, dt), idx, cnt, o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=256)
    r_idx, r_cnt = ref.window_indices(Dr)
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), r_cnt)
    rows = np.array([0, 1, 255, 256, 700, T - 1], np.int32)
    r_sp = ref.sparse_attn(Dr, q, k, v, r_idx[:, rows], r_cnt[:, rows], rows=rows)
    err = max_abs(o.float().cpu().numpy()[:, rows], r_sp)
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("shape", [(8, 4, 128), (3, 2, 63)])
def test_state_transfer_segments(shape):
    B, H_kv, d = shape
    D = lisa.make_dims(B, 1, 0, 1, 4 * H_kv, H_kv, d, 1, 1, 8, 8, dtype="f32")
    Dr = ref.Dims(B=B, T=1, n_past=0, N_max=1, H_q=4 * H_kv, H_kv=H_kv, d=d, H_I=1, H_Ik=1,
                  d_I=8, M=8)
    rng = np.random.default_rng(8)
    start = np.zeros((B, H_kv, d, d), np.float32)
    G = np.zeros_like(start)
    g_start, g_G = torch.from_numpy(start).cuda(), torch.from_numpy(G).cuda()
    r_start, r_G = start.astype(np.float64), G.astype(np.float64)
    for t in range(1, 5):
        end = (r_start + rng.standard_normal(start.shape)).astype(np.float32)
        g_S = torch.from_numpy(end).cuda()
        lisa.lisa_state_transfer(D, g_S, g_start, g_G, t, 0.3)
        r_S, r_start, r_G = ref.state_transfer(Dr, end, r_start, r_G, t, 0.3)
        assert max_abs(g_S.cpu().numpy(), r_S) <= TOL["f32"]
        assert max_abs(g_start.cpu().numpy(), r_start) <= TOL["f32"]
        assert max_abs(g_G.cpu().numpy(), r_G) <= TOL["f32"]
        r_start = g_start.cpu().numpy().astype(np.float64)  # continue from the GPU's own state


def test_state_transfer_rejects_bad_segment_index():
    D = lisa.make_dims(1, 1, 0, 1, 4, 1, 8, 1, 1, 8, 8, dtype="f32")
    S = torch.zeros(1, 1, 8, 8, device="cuda")
    with pytest.raises(lisa.LisaError):
        lisa.lisa_state_transfer(D, S, S.clone(), S.clone(), 0, 0.5)
