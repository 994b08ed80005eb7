"""lisa_topm_noalloc: the workspace-free variant of lisa_topm.

Some callers cannot allocate device memory for the library (a host framework
whose allocator is off-limits, plugin interfaces that pass only the call's
tensors).  This entry point keeps its scratch in a device array built into the
library.  The test calls it through the C ABI twice in a row (the shared
array keeps the previous call's contents) and checks that each result equals
what lisa_topm, which takes a caller-provided workspace, returns for the same
inputs, and the oracle's selection.  It lives in its own file, collected last.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import check_topm

pytestmark = pytest.mark.gpu


def _case(wl, T, n_past, seed_shift):
    gen = inputs.Generator(wl.with_(seed=wl.seed + seed_shift))
    L = n_past + T
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    q_I = torch.from_numpy(gen.batch("q_I", n_past, L)).to(dt).cuda()
    k_I = torch.from_numpy(gen.batch("k_I", 0, L)).to(dt).cuda()
    w = torch.from_numpy(gen.batch("w", n_past, L)).cuda()
    D = lisa.make_dims(wl.B, T, n_past, L, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype=wl.dtype)
    return D, q_I, k_I, w, gen


def _topm_both(D, q_I, k_I, w, H_I):
    B, T, M = D.B, D.T, D.M
    idx_ws = torch.empty(B, T, M, dtype=torch.int32, device="cuda")
    cnt_ws = torch.empty(B, T, dtype=torch.int32, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_TOPM)
    lisa.lisa_topm(D, q_I, k_I, w, H_I, idx_ws, cnt_ws, ws)
    idx_na = torch.full((B, T, M), -9, dtype=torch.int32, device="cuda")
    cnt_na = torch.full((B, T), -9, dtype=torch.int32, device="cuda")
    lisa.lisa_topm_noalloc(D, q_I, k_I, w, H_I, idx_na, cnt_na)
    torch.cuda.synchronize()
    return idx_ws.cpu().numpy(), cnt_ws.cpu().numpy(), idx_na.cpu().numpy(), cnt_na.cpu().numpy()


def test_noalloc_topm_matches_workspace_topm_twice():
    # first call: a prefill-shaped fp32 call; second: a bf16 decode-shaped call
    # whose scores overwrite part of the first call's scratch contents
    cases = [(inputs.TINY.with_(M=32), 200, 0, 0), (inputs.DECODE_7B.with_(B=4, M=512), 1, 9000, 1)]
    for wl, T, n_past, shift in cases:
        D, q_I, k_I, w, gen = _case(wl, T, n_past, shift)
        a_idx, a_cnt, b_idx, b_cnt = _topm_both(D, q_I, k_I, w, wl.H_I)
        # lisa_topm may score on the tensor cores and the workspace-free call on
        # the CUDA cores: the index sets agree up to the near-tie rule the other
        # top-M tests use (relative score gap <= 1e-3 at the M-th score)
        L = n_past + T
        Dr = ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                      H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
        sc = ref.index_scores(Dr, q_I.float().cpu().numpy(), k_I.float().cpu().numpy(),
                              w.cpu().numpy(), wl.H_I)
        np.testing.assert_array_equal(b_cnt, a_cnt)
        for bb in range(wl.B):
            check_topm(b_idx[bb], b_cnt[bb], a_idx[bb], a_cnt[bb], sc[bb])
        # and both against the oracle's own selection (a full sort of its scores)
        r_idx, r_cnt = ref.topm(Dr, sc)
        for bb in range(wl.B):
            check_topm(b_idx[bb], b_cnt[bb], r_idx[bb], r_cnt[bb], sc[bb])


def test_noalloc_topm_more_rows_than_a_grid_column():
    """70000 single-token sequences over 14 cached keys: more query rows than
    the 65535 a launch grid's y dimension allows, within the 4 MiB array."""
    wl = inputs.TINY.with_(B=70000, M=4)
    T, n_past = 1, 13
    L = n_past + T
    # one seeded draw for the whole batch (the per-sequence streams of the
    # workload generator would take minutes for 70000 sequences)
    rng = np.random.default_rng(7)
    q_I = torch.from_numpy(rng.standard_normal((wl.B, T, wl.H_I, wl.d_I), dtype=np.float32)).cuda()
    k_I = torch.from_numpy(rng.standard_normal((wl.B, L, wl.H_Ik, wl.d_I), dtype=np.float32)).cuda()
    w = torch.from_numpy(rng.random((wl.B, T, wl.H_I), dtype=np.float32)).cuda()
    D = lisa.make_dims(wl.B, T, n_past, L, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype="f32")
    a_idx, a_cnt, b_idx, b_cnt = _topm_both(D, q_I, k_I, w, wl.H_I)
    Dr = ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    sc = ref.index_scores(Dr, q_I.cpu().numpy(), k_I.cpu().numpy(), w.cpu().numpy(), wl.H_I)
    r_idx, r_cnt = ref.topm(Dr, sc)
    for got_idx, got_cnt in ((a_idx, a_cnt), (b_idx, b_cnt)):
        check_topm(got_idx.reshape(-1, wl.M), got_cnt.reshape(-1), r_idx.reshape(-1, wl.M),
                   r_cnt.reshape(-1), sc.reshape(-1, L))


def test_noalloc_rejects_calls_beyond_its_scratch():
    wl = inputs.DECODE_7B.with_(B=8)
    D = lisa.make_dims(8, 1, 200000, 200001, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(lisa.LisaError) as err:
        lisa.lisa_topm_noalloc(D, t, t, t.float(), wl.H_I, i, i)
    assert err.value.status == lisa.LISA_ERR_UNSUPPORTED
