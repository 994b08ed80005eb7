"""GPU parity of lisa_sparse_attn on the tensor-core form for many query rows
(bf16, head dim 128): the selections become a bit mask and the attention runs
over 128-query x 64-key tiles on tcgen05 (LISA Sec. 3.2 Eq. 1, SA_M).

The index rows here are seeded random sets, not top-M rows: any order, a
count per row below the budget (zero included), rows past a partial last
query tile, a call that continues after cached tokens, head groups of 7, 6,
8, 3 and 1 query heads per KV head (a CTA takes two heads of one query tile,
or, for the odd head of a group, that head on two neighbouring query tiles,
or on the first tile alone), and logits large enough that the running
maximum jumps by more than 2^64 between key tiles (the output is then
rescaled in TMEM).  Every row is
compared with the oracle's sparse attention on the same index rows.
Tolerance: max abs <= 2e-2 (bf16 outputs).
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, max_abs

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _dv(a, dt=BF):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def _random_rows(rng, B, T, n_past, M, zero_every=0):
    """Index rows of distinct positions in [0, p], shuffled, -1 padded."""
    idx = np.full((B, T, M), -1, np.int32)
    cnt = np.zeros((B, T), np.int32)
    for b in range(B):
        for t in range(T):
            p = n_past + t
            c = int(min(M, p + 1, rng.integers(M // 2, M + 1)))
            if zero_every and t % zero_every == zero_every - 1:
                c = 0
            sel = rng.choice(p + 1, size=c, replace=False)
            idx[b, t, :c] = sel  # any order
            cnt[b, t] = c
    return idx, cnt


def _case(wl, T, n_past, seed, q_scale=1.0, zero_every=0):
    gen = inputs.Generator(wl)
    L = n_past + T
    q = gen.batch("q", n_past, L) * np.float32(q_scale)  # a power of two stays exact in bf16
    k = gen.batch("k", 0, L)
    v = gen.batch("v", 0, L)
    rng = np.random.default_rng(seed)
    idx, cnt = _random_rows(rng, wl.B, T, n_past, wl.M, zero_every)
    D = lisa.make_dims(wl.B, T, n_past, L, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    o = torch.full((wl.B, T, wl.H_q, wl.d), 5.0, dtype=BF, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, _dv(q), _dv(k), _dv(v), _dv(idx, torch.int32), _dv(cnt, torch.int32),
                          o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    Dr = ref.Dims(B=wl.B, T=T, n_past=n_past, N_max=L, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                  H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    r = ref.sparse_attn(Dr, q, k, v, idx, cnt)
    g = o.float().cpu().numpy()
    # attention over an empty set has no value: the oracle's 0/0 leaves NaN
    # there, the library writes zeros (its documented result for count == 0)
    live = cnt > 0
    err = max_abs(g[live], r[live])
    assert err <= TOL["bf16"], err
    assert np.all(g[~live] == 0.0)
    return err


@pytest.mark.parametrize("H_q,H_kv", [(28, 4), (12, 2), (8, 1), (6, 2), (4, 4)])
def test_mask_path_random_rows_continued_call(H_q, H_kv):
    # 300 rows (a partial third query tile) after 150 cached tokens, 2 sequences
    wl = inputs.PREFILL_7B.with_(B=2, n=450, M=96, H_q=H_q, H_kv=H_kv)
    _case(wl, T=300, n_past=150, seed=H_q, zero_every=37)


def test_mask_path_running_max_jumps():
    """q scaled by 512: logits spread over far more than 2^8 within a row, so
    the running maximum grows past the lazy bound between key tiles."""
    wl = inputs.PREFILL_7B.with_(B=1, n=640, M=400)
    _case(wl, T=640, n_past=0, seed=9, q_scale=512.0)


def test_mask_path_long_rows():
    """Rows of 2048 keys spread over a 6000-token context (many key tiles)."""
    wl = inputs.PREFILL_7B.with_(B=1, n=6000, M=2048)
    _case(wl, T=256, n_past=5744, seed=4)


def test_mask_path_reports_out_of_range_positions():
    wl = inputs.PREFILL_7B.with_(B=1, n=256, M=16)
    gen = inputs.Generator(wl)
    T = 256
    q, k, v = (gen.batch(n, 0, T) for n in ("q", "k", "v"))
    rng = np.random.default_rng(1)
    idx, cnt = _random_rows(rng, 1, T, 0, 16)
    # row 200 keeps at most 14 valid entries and gets a position past itself
    # and a negative one
    t = 200
    c = min(int(cnt[0, t]), 14)
    idx[0, t, c:] = -1
    cnt[0, t] = c
    good_idx, good_cnt = idx.copy(), cnt.copy()
    idx[0, t, c:c + 2] = [t + 5, -3]
    cnt[0, t] = c + 2
    D = lisa.make_dims(1, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, 16)
    o = torch.empty(1, T, wl.H_q, wl.d, dtype=BF, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_SPARSE_ATTN)
    lisa.lisa_sparse_attn(D, _dv(q), _dv(k), _dv(v), _dv(idx, torch.int32), _dv(cnt, torch.int32),
                          o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_ERR_DEVICE_BOUNDS
    Dr = ref.Dims(B=1, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=16)
    r = ref.sparse_attn(Dr, q, k, v, good_idx, good_cnt)
    assert max_abs(o.float().cpu().numpy(), r) <= TOL["bf16"]
