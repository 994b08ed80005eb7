"""One workspace for a prefill and the decode steps that follow it (GPU).

The decode steps keep state between calls in their workspace (key histograms
and exchange counters, zero between calls); every other entry point uses the
same bytes as scratch.  The rule the header states: a workspace that another
entry point has used is zero-filled again before a decode step uses it.  This
test follows that rule with one workspace sized for both operations: a
whole-module prefill over the cached tokens, a zero-fill, then two decode
steps, each checked against the oracle.
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


def test_prefill_then_decode_on_one_workspace():
    wl = inputs.DECODE_7B.with_(B=2, n=3002, M=256)
    gen = inputs.Generator(wl)
    B, n = wl.B, wl.n
    n0 = n - 2  # tokens of the prefill; two decode steps follow
    x = {k: gen.batch(k, 0, n) for k in ("q", "k", "v", "q_I", "k_I", "w", "gate")}
    kc, vc, kIc = _dv(x["k"]), _dv(x["v"]), _dv(x["k_I"])
    S = torch.zeros(B, wl.H_kv, wl.d, wl.d, device="cuda")
    dims = dict(H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    Dp = lisa.make_dims(B, n0, 0, n, chunk=wl.chunk, **dims)
    Dd = [lisa.make_dims(B, 1, n0 + i, n, **dims) for i in range(2)]
    size = max(lisa.lisa_workspace_size(Dp, lisa.LISA_OP_PREFILL),
               *(lisa.lisa_workspace_size(D, lisa.LISA_OP_DECODE_STEP) for D in Dd))
    ws = torch.zeros(size + 256, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + size]

    q0 = _dv(x["q"][:, :n0])
    o0 = torch.empty(B, n0, wl.H_q, wl.d, dtype=BF, device="cuda")
    k0, v0 = kc[:, :n0].contiguous(), vc[:, :n0].contiguous()
    pa = lisa.prefill_args(q0, kc, vc, _dv(x["q_I"][:, :n0]), kIc, _dv(x["w"][:, :n0], torch.float32),
                           wl.H_I, q0, k0, v0, _dv(x["gate"][:, :n0]), S, None, o0)
    lisa.lisa_prefill(Dp, pa, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK

    for i, D in enumerate(Dd):
        ws.zero_()  # the rule: another entry point used these bytes
        p = n0 + i
        sl = slice(p, p + 1)
        S_before = S.cpu().numpy().copy()
        tq = _dv(x["q"][:, sl])
        k_new, v_new = _dv(x["k"][:, sl]), _dv(x["v"][:, sl])
        o = torch.empty(B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
        idx = torch.full((B, 1, wl.M), -7, dtype=torch.int32, device="cuda")
        cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
        args = lisa.decode_args(tq, k_new, v_new, _dv(x["q_I"][:, sl]), _dv(x["k_I"][:, sl]),
                                _dv(x["w"][:, sl], torch.float32), wl.H_I, tq, k_new, v_new,
                                _dv(x["gate"][:, sl]), kc, vc, kIc, S, None, o, idx, cnt)
        lisa.lisa_decode_step(D, args, ws)
        assert lisa.lisa_check_status(ws) == lisa.LISA_OK

        Dr = ref.Dims(B=B, T=1, n_past=p, N_max=n, **dims)
        q_I = x["q_I"][:, sl]
        scores = ref.index_scores(Dr, q_I, x["k_I"], x["w"][:, sl], wl.H_I)
        r_idx, r_cnt = ref.topm(Dr, scores)
        g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], scores[:, 0])
        r_lin, r_S, _ = ref.linear(Dr, x["q"][:, sl], x["k"][:, sl], x["v"][:, sl], S0=S_before)
        r_sp = ref.sparse_attn(Dr, x["q"][:, sl], x["k"], x["v"], g_idx, g_cnt)
        r_o = ref.gate(Dr, x["gate"][:, sl], r_lin, r_sp)
        assert max_abs(o.float().cpu().numpy(), r_o) <= TOL["bf16"]
        assert max_abs(S.cpu().numpy(), r_S) <= 1e-4 * max(1.0, float(np.abs(r_S).max()))
