"""GPU parity of the fused decode step (bf16) against the CPU oracle.

Covers the headline 7B shape at full size (B=8, context 16384, M=2048), the
1.5B head layout, ragged context lengths, a budget larger than the context,
all-equal scores (tie-break by position across the cluster) and the elu+1
feature map.  Tolerances: outputs max abs <= 2e-2 (bf16); top-M equal up to
near-ties (relative gap <= 1e-3 at the M-th score).
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


def run_decode_case(wl, phi=0, zero_qI=False, S0_from_prefill=True, check_state=True,
                    kI_first_half_scale=1.0):
    """One decode step at position n-1 over a cache of n-1 tokens; returns errors."""
    gen = inputs.Generator(wl)
    n, p, B = wl.n, wl.n - 1, wl.B
    kc_np = gen.batch("k", 0, n)
    vc_np = gen.batch("v", 0, n)
    kI_np = gen.batch("k_I", 0, n)
    # a power of two keeps the bf16 values exact on both sides
    kI_np[:, : n // 2] *= kI_first_half_scale
    q = gen.batch("q", p, n)
    q_I = gen.batch("q_I", p, n)
    if zero_qI:
        q_I = np.zeros_like(q_I)
    w = gen.batch("w", p, n)
    gl = gen.batch("gate", p, n)
    Dr = ref.Dims(B=B, T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
    # linear state from the oracle's own prefill over the cached tokens
    S0 = z0 = None
    if S0_from_prefill and p > 0:
        Dp = ref.Dims(B=B, T=p, n_past=0, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                      H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
        _, S0, z0 = ref.linear(Dp, None, kc_np[:, :p], vc_np[:, :p], rows=np.zeros(0, np.int32))
        S0 = S0.astype(np.float32)
        z0 = z0.astype(np.float32) if z0 is not None else None
    if S0 is None:
        S0 = np.zeros((B, wl.H_kv, wl.d, wl.d), np.float32)
        z0 = np.zeros((B, wl.H_kv, wl.d), np.float32) if phi else None

    kc, vc, kIc = _dv(kc_np), _dv(vc_np), _dv(kI_np)
    # the cache holds n-1 tokens before the step: poison row p so a missed append shows
    kc[:, p:] = 7.0
    vc[:, p:] = 7.0
    kIc[:, p:] = 7.0
    S = torch.from_numpy(S0).cuda()
    z = torch.from_numpy(z0).cuda() if phi else None
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M, phi=phi)
    tq = _dv(q)
    k_new, v_new = _dv(kc_np[:, p:]), _dv(vc_np[:, p:])
    o = torch.empty(B, 1, wl.H_q, wl.d, dtype=BF, device="cuda")
    idx = torch.full((B, 1, wl.M), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    args = lisa.decode_args(tq, k_new, v_new, _dv(q_I), _dv(kI_np[:, p:]), _dv(w, torch.float32),
                            wl.H_I, tq, k_new, v_new, _dv(gl), kc, vc, kIc, S, z, o, idx, cnt)
    ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP)
    lisa.lisa_decode_step(D, args, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK

    scores = ref.index_scores(Dr, q_I, kI_np, w, wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, scores)
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    swaps = check_topm(g_idx[:, 0], g_cnt[:, 0], r_idx[:, 0], r_cnt[:, 0], scores[:, 0])
    r_lin, r_S, r_z = ref.linear(Dr, q, kc_np[:, p:], vc_np[:, p:], S0=S0, z0=z0)
    r_sp = ref.sparse_attn(Dr, q, kc_np, vc_np, g_idx, g_cnt)
    r_o = ref.gate(Dr, gl, r_lin, r_sp)
    err_o = max_abs(o.float().cpu().numpy(), r_o)
    assert err_o <= TOL["bf16"], err_o
    if check_state:
        assert max_abs(S.cpu().numpy(), r_S) <= 1e-4 * max(1.0, np.abs(r_S).max())
        if phi:
            assert max_abs(z.cpu().numpy(), r_z) <= 1e-4 * max(1.0, np.abs(r_z).max())
    # the append landed
    np.testing.assert_array_equal(kc[:, p].float().cpu().numpy(), kc_np[:, p])
    np.testing.assert_array_equal(vc[:, p].float().cpu().numpy(), vc_np[:, p])
    np.testing.assert_array_equal(kIc[:, p].float().cpu().numpy(), kI_np[:, p])
    return dict(err_o=err_o, swaps=swaps, idx=g_idx, cnt=g_cnt)


def test_decode_7b_headline_full_size():
    run_decode_case(inputs.DECODE_7B)


@pytest.mark.parametrize("n", [1, 17, 2049, 3001])
def test_decode_7b_ragged_contexts(n):
    run_decode_case(inputs.DECODE_7B.with_(B=3, n=n, M=256))


def test_decode_budget_exceeds_context_selects_all():
    res = run_decode_case(inputs.DECODE_7B.with_(B=2, n=200, M=256))
    assert np.all(res["cnt"] == 200)
    assert np.all(res["idx"][:, 0, :200] == np.arange(200))
    assert np.all(res["idx"][:, 0, 200:] == -1)


def test_decode_all_scores_equal_take_lowest_positions():
    """q_I = 0 makes every score exactly 0: the budget goes to positions 0..M-1."""
    res = run_decode_case(inputs.DECODE_7B.with_(B=2, n=5000, M=300), zero_qI=True)
    assert np.all(res["idx"][:, 0, :300] == np.arange(300))


def test_decode_elu1_feature_map():
    run_decode_case(inputs.DECODE_7B.with_(B=2, n=4000, M=512), phi=lisa.LISA_PHI_ELU1_NORM)


def test_decode_7b_headline_elu1_full_size():
    """The headline shape with the elu+1 feature map and its normaliser."""
    run_decode_case(inputs.DECODE_7B, phi=lisa.LISA_PHI_ELU1_NORM)


def test_decode_1p5b_head_layout():
    run_decode_case(inputs.PREFILL_1P5B.with_(B=4, n=4096, M=512))


def test_decode_one_kv_head():
    """Eight query heads over a single KV head: 256-byte K/V rows, the deepest
    stage ring and no V requests ahead of the current stage."""
    run_decode_case(inputs.DECODE_7B.with_(B=3, n=5000, M=512, H_q=8, H_kv=1))


def test_decode_fused_matches_generic_path_outputs_shape():
    """The fused path and a second identical call agree (the step is deterministic)."""
    wl = inputs.DECODE_7B.with_(B=2, n=3000, M=256)
    a = run_decode_case(wl)
    b = run_decode_case(wl)
    np.testing.assert_array_equal(a["idx"], b["idx"])


def test_decode_scores_skewed_across_the_context():
    """Indexer keys 4x larger in the first half of the context: the top-M comes
    almost entirely from there, so the parts of the context whose own scores
    suggest a lower threshold have to contribute through the exact path too."""
    res = run_decode_case(inputs.DECODE_7B.with_(B=2, n=16384, M=2048), kI_first_half_scale=4.0)
    assert np.all(res["cnt"] == 2048)
