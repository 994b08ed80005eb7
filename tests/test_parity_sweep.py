"""GPU parity at the long-context decode sweep sizes (bf16): B=32 sequences,
every context of 4096 .. 65536 with both budgets M in {512, 2048}, through
lisa_decode_step (the cooperative kernel up to 32768, the four-kernel form at
65536), and the dense causal attention line (lisa_dense_attn) on the same
caches at every context.

The whole batch runs on the GPU; the oracle checks sampled sequences (batch
elements are independent).  The linear state is a seeded random input (the
oracle's prefill of 65535 tokens per sequence would take minutes).
Tolerances: top-M equal up to near-ties; outputs max abs <= 2e-2.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, check_topm, max_abs

pytestmark = pytest.mark.gpu
BF = torch.bfloat16
SAMPLE = [0, 13, 31]


def _dv(a, dt=BF):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def _sweep_case(n, M, dense):
    wl = inputs.sweep_workload(n, M)
    gen = inputs.Generator(wl)
    B, p = wl.B, n - 1
    kc = torch.empty(B, n, wl.H_kv, wl.d, dtype=BF, device="cuda")
    vc = torch.empty_like(kc)
    kIc = torch.empty(B, n, wl.H_Ik, wl.d_I, dtype=BF, device="cuda")
    host = {}
    for b in range(B):
        k_b, v_b, kI_b = gen.k(b, 0, n), gen.v(b, 0, n), gen.k_I(b, 0, n)
        kc[b], vc[b], kIc[b] = _dv(k_b), _dv(v_b), _dv(kI_b)
        if b in SAMPLE:
            host[b] = (k_b, v_b, kI_b)
    q = gen.batch("q", p, n)
    q_I = gen.batch("q_I", p, n)
    w = gen.batch("w", p, n)
    gl = gen.batch("gate", p, n)
    rng = np.random.default_rng(5)
    S0 = (rng.standard_normal((B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    k_new, v_new, kI_new = kc[:, p:].clone(), vc[:, p:].clone(), kIc[:, p:].clone()
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, M)
    tq = _dv(q)
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
    idx = torch.full((B, 1, M), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    S = torch.from_numpy(S0).cuda()
    args = lisa.decode_args(tq, k_new, v_new, _dv(q_I), kI_new, _dv(w, torch.float32), wl.H_I, tq,
                            k_new, v_new, _dv(gl), kc, vc, kIc, S, None, o, idx, cnt)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    lisa.lisa_decode_step(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    o_dense = None
    if dense:
        o_dense = torch.empty_like(o)
        ws_d = lisa.workspace(D, lisa.LISA_OP_DENSE_ATTN)
        lisa.lisa_dense_attn(D, tq, kc, vc, o_dense, ws_d)
        assert lisa.lisa_check_status(ws_d) == lisa.LISA_OK

    # the oracle on the sampled sequences
    sb = np.array(SAMPLE)
    kc_s = np.stack([host[b][0] for b in SAMPLE])
    vc_s = np.stack([host[b][1] for b in SAMPLE])
    kI_s = np.stack([host[b][2] for b in SAMPLE])
    Dr = ref.Dims(B=len(SAMPLE), T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=M)
    scores = ref.index_scores(Dr, q_I[sb], kI_s, w[sb], wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, scores)
    g_idx, g_cnt = idx.cpu().numpy()[sb], cnt.cpu().numpy()[sb]
    check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], scores[:, 0])
    r_lin, _, _ = ref.linear(Dr, q[sb], kc_s[:, p:], vc_s[:, p:], S0=S0[sb])
    r_sp = ref.sparse_attn(Dr, q[sb], kc_s, vc_s, g_idx, g_cnt)
    r_o = ref.gate(Dr, gl[sb], r_lin, r_sp)
    err = max_abs(o.float().cpu().numpy()[sb], r_o)
    assert err <= TOL["bf16"], err
    if dense:
        r_d = ref.dense_attn(Dr, q[sb], kc_s, vc_s)
        err_d = max_abs(o_dense.float().cpu().numpy()[sb], r_d)
        assert err_d <= TOL["bf16"], err_d


@pytest.mark.parametrize("M", inputs.SWEEP_M)
@pytest.mark.parametrize("n", inputs.SWEEP_CTX)
def test_decode_sweep_point(n, M):
    """Every (context, budget) point of the sweep; the dense line (which does
    not depend on M) is checked once per context, with the larger budget."""
    _sweep_case(n, M, dense=(M == max(inputs.SWEEP_M)))
