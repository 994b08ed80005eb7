"""GPU parity of consecutive decode steps that share one workspace, and of a
decode step replayed from a CUDA graph.

A generation loop calls lisa_decode_step once per token with the same
workspace while the context grows by one each time.  The step keeps state
between calls in that workspace (key histograms and exchange counters that
return to zero at the end of every call), so each step here is checked
against the CPU oracle: output within 2e-2 (bf16), top-M equal up to
near-ties, and the linear state after the last step within 1e-4 relative.
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


def _dims(wl, p, N, phi=0):
    return lisa.make_dims(wl.B, 1, p, N, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                          phi=phi)


def _ref_dims(wl, p, N, phi=0):
    return ref.Dims(B=wl.B, T=1, n_past=p, N_max=N, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                    H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)


@pytest.mark.parametrize("phi", [0, 1])
def test_decode_steps_with_growing_context_share_one_workspace(phi):
    # contexts 1001 .. 1040: crosses 1024, where the per-call scratch of the
    # workspace grows; the budget is exceeded from the first step on
    wl = inputs.DECODE_7B.with_(B=2, n=1040, M=200)
    N, n0, steps = wl.n, 1000, 40
    gen = inputs.Generator(wl)
    kc_np, vc_np, kI_np = gen.batch("k", 0, N), gen.batch("v", 0, N), gen.batch("k_I", 0, N)
    Dp = ref.Dims(B=wl.B, T=n0, n_past=0, N_max=N, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
    _, S0, z0 = ref.linear(Dp, None, kc_np[:, :n0], vc_np[:, :n0], rows=np.zeros(0, np.int32))
    kc, vc, kIc = _dv(kc_np), _dv(vc_np), _dv(kI_np)
    kc[:, n0:] = 7.0  # rows past the cached tokens: poison
    vc[:, n0:] = 7.0
    kIc[:, n0:] = 7.0
    S = torch.from_numpy(S0.astype(np.float32)).cuda()
    z = torch.from_numpy(z0.astype(np.float32)).cuda() if phi else None
    r_S, r_z = S0, z0
    ws = lisa.workspace(_dims(wl, N - 1, N, phi), lisa.LISA_OP_DECODE_STEP)
    o = torch.empty(wl.B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
    idx = torch.empty(wl.B, 1, wl.M, dtype=torch.int32, device="cuda")
    cnt = torch.empty(wl.B, 1, dtype=torch.int32, device="cuda")
    for s in range(steps):
        p = n0 + s
        q, q_I = gen.batch("q", p, p + 1), gen.batch("q_I", p, p + 1)
        w, gl = gen.batch("w", p, p + 1), gen.batch("gate", p, p + 1)
        tq, k_new, v_new = _dv(q), _dv(kc_np[:, p:p + 1]), _dv(vc_np[:, p:p + 1])
        args = lisa.decode_args(tq, k_new, v_new, _dv(q_I), _dv(kI_np[:, p:p + 1]),
                                _dv(w, torch.float32), wl.H_I, tq, k_new, v_new, _dv(gl),
                                kc, vc, kIc, S, z, o, idx, cnt)
        lisa.lisa_decode_step(_dims(wl, p, N, phi), args, ws)
        assert lisa.lisa_check_status(ws) == lisa.LISA_OK
        Dr = _ref_dims(wl, p, N, phi)
        scores = ref.index_scores(Dr, q_I, kI_np, w, wl.H_I)
        r_idx, r_cnt = ref.topm(Dr, scores)
        g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], scores[:, 0])
        r_lin, r_S, r_z = ref.linear(Dr, q, kc_np[:, p:p + 1], vc_np[:, p:p + 1], S0=r_S, z0=r_z)
        r_sp = ref.sparse_attn(Dr, q, kc_np, vc_np, g_idx, g_cnt)
        r_o = ref.gate(Dr, gl, r_lin, r_sp)
        err = max_abs(o.float().cpu().numpy(), r_o)
        assert err <= TOL["bf16"], (s, err)
    assert max_abs(S.cpu().numpy(), r_S) <= 1e-4 * max(1.0, np.abs(r_S).max())
    if phi:
        assert max_abs(z.cpu().numpy(), r_z) <= 1e-4 * max(1.0, np.abs(r_z).max())
    np.testing.assert_array_equal(kc[:, n0:].float().cpu().numpy(), kc_np[:, n0:])
    np.testing.assert_array_equal(kIc[:, n0:].float().cpu().numpy(), kI_np[:, n0:])


def test_decode_step_from_a_cuda_graph_matches_a_direct_call():
    """The step captured in a CUDA graph and replayed gives the same bits as a
    direct call on an identical copy of the state."""
    wl = inputs.DECODE_7B.with_(B=4, n=6000, M=512)
    gen = inputs.Generator(wl)
    n, p = wl.n, wl.n - 1
    host = {k: gen.batch(k, 0, n) for k in ("k", "v", "k_I")}
    step = {k: gen.batch(k, p, n) for k in ("q", "q_I", "w", "gate")}
    rng = np.random.default_rng(5)
    S0 = (rng.standard_normal((wl.B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    D = _dims(wl, p, n)

    def state():
        kc, vc, kIc = _dv(host["k"]), _dv(host["v"]), _dv(host["k_I"])
        S = torch.from_numpy(S0).cuda()
        o = torch.empty(wl.B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
        idx = torch.empty(wl.B, 1, wl.M, dtype=torch.int32, device="cuda")
        cnt = torch.empty(wl.B, 1, dtype=torch.int32, device="cuda")
        tq, k_new, v_new = _dv(step["q"]), _dv(host["k"][:, p:]), _dv(host["v"][:, p:])
        args = lisa.decode_args(tq, k_new, v_new, _dv(step["q_I"]), _dv(host["k_I"][:, p:]),
                                _dv(step["w"], torch.float32), wl.H_I, tq, k_new, v_new,
                                _dv(step["gate"]), kc, vc, kIc, S, None, o, idx, cnt)
        return dict(args=args, S=S, o=o, idx=idx, ws=lisa.workspace(D, lisa.LISA_OP_DECODE_STEP))

    a, b = state(), state()
    lisa.lisa_decode_step(D, a["args"], a["ws"])
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            lisa.lisa_decode_step(D, b["args"], b["ws"])
    g.replay()
    torch.cuda.synchronize()
    assert lisa.lisa_check_status(a["ws"]) == lisa.LISA_OK
    assert lisa.lisa_check_status(b["ws"]) == lisa.LISA_OK
    for k in ("o", "idx", "S"):
        assert torch.equal(a[k], b[k]), k
