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
