"""A bounded device wait gives up, reports LISA_ERR_TIMEOUT and leaves the GPU usable.

The CTAs of one sequence in the decode step meet at exchanges through
counters in the workspace, and every poll of such a counter is bounded.  The
workspace header's fault-injection hook (words 2-3, zero in normal use) makes
one CTA of every sequence leave out its arrival at the first exchange and
shortens that exchange's poll limit.  The other CTAs' waits must then give up:
the call returns, lisa_check_status reports LISA_ERR_TIMEOUT, and once the
hook is cleared and the workspace zero-filled again the next step matches the
oracle.  Nothing faults, traps or waits without a bound.
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


def _step_inputs(wl):
    gen = inputs.Generator(wl)
    n, p = wl.n, wl.n - 1
    host = {k: gen.batch(k, 0, n) for k in ("k", "v", "k_I")}
    host.update({k: gen.batch(k, p, n) for k in ("q", "q_I", "w", "gate")})
    return host


def _call(wl, host, ws):
    n, p, B = wl.n, wl.n - 1, wl.B
    kc, vc, kIc = _dv(host["k"]), _dv(host["v"]), _dv(host["k_I"])
    S = torch.zeros(B, wl.H_kv, wl.d, wl.d, device="cuda")
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
    idx = torch.full((B, 1, wl.M), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    tq = _dv(host["q"])
    k_new, v_new = kc[:, p:].clone(), vc[:, p:].clone()
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    args = lisa.decode_args(tq, k_new, v_new, _dv(host["q_I"]), kIc[:, p:].clone(),
                            _dv(host["w"], torch.float32), wl.H_I, tq, k_new, v_new,
                            _dv(host["gate"]), kc, vc, kIc, S, None, o, idx, cnt)
    lisa.lisa_decode_step(D, args, ws)
    return o, idx, cnt


def test_exchange_wait_gives_up_and_reports_timeout():
    # n > M, so the step needs the exchanges of the threshold; 2 sequences over
    # most of the SMs (cooperative kernel)
    wl = inputs.DECODE_7B.with_(B=2, n=3000, M=256)
    host = _step_inputs(wl)
    D = lisa.make_dims(wl.B, 1, wl.n - 1, wl.n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I,
                       wl.M)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    hook = ws[:16].view(torch.int32)
    hook[2] = 1 + 3      # CTA 3 of every sequence leaves out its arrival at exchange 1
    hook[3] = 4096       # and the others poll the counter at most 4096 times
    _call(wl, host, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_ERR_TIMEOUT
    # the device is still usable: a plain copy round-trips
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert torch.equal((x * 2).cpu(), torch.arange(1024, dtype=torch.float32) * 2)

    # hook off and the workspace zero-filled again: the next step is right
    ws.zero_()
    o, idx, cnt = _call(wl, host, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    p = wl.n - 1
    Dr = ref.Dims(B=wl.B, T=1, n_past=p, N_max=wl.n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    scores = ref.index_scores(Dr, host["q_I"], host["k_I"], host["w"], wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, scores)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], scores[:, 0])
    r_lin, _, _ = ref.linear(Dr, host["q"], host["k"][:, p:], host["v"][:, p:])
    r_sp = ref.sparse_attn(Dr, host["q"], host["k"], host["v"], g_idx, g_cnt)
    r_o = ref.gate(Dr, host["gate"], r_lin, r_sp)
    assert max_abs(o.float().cpu().numpy(), r_o) <= TOL["bf16"]
