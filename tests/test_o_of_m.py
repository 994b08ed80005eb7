"""Per-token work of the sparse branch is O(M), not O(n) (CPU).

LISA (Abstract and Sec. 5) cuts attention from O(n^2) to O(nM): at a fixed
budget M, each token's softmax attention reads M cached rows however long the
context; only the lightweight indexer scan grows with n.

- The oracle's selection keeps exactly min(M, p + 1) positions at every
  context length, so the sparse attention of a decode step reads the same
  number of K/V rows at n = 256 and at n = 4096.
- The benchmark's algorithmic byte counts (the roofline numerators) follow
  the same rule: the K/V gather and the Stage-1 window step are constant in n
  at fixed M; the indexer scan is linear in n (128 bytes per cached token per
  sequence at d_I = 64); dense attention is linear in n (2 KB per token).
The GPU counterpart is the benchmark's sweep: the window step's time across
contexts 4K-64K at a fixed budget, next to the full step's.
"""
import numpy as np

import bench
from hybrid_linear_top_lightning_b200 import inputs
from oracle import ref


def test_selected_rows_per_token_do_not_grow_with_the_context():
    M = 64
    counts = []
    for n in (256, 512, 1024, 4096):
        wl = inputs.TINY.with_(B=2, n=n, M=M, d=16, d_I=8, H_I=2)
        gen = inputs.Generator(wl)
        p = n - 1
        q_I = gen.batch("q_I", p, n)
        k_I = gen.batch("k_I", 0, n)
        w = gen.batch("w", p, n)
        D = ref.Dims(B=wl.B, T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d,
                     H_I=wl.H_I, H_Ik=wl.H_Ik, d_I=wl.d_I, M=M)
        scores = ref.index_scores(D, q_I, k_I, w, wl.H_I)
        assert np.isfinite(scores).sum() == wl.B * n  # the indexer scans every cached key
        idx, cnt = ref.topm(D, scores)
        assert np.all(cnt == M)
        for b in range(wl.B):
            sel = idx[b, 0, :M]
            assert np.unique(sel).size == M and sel.min() >= 0 and sel.max() <= p
        counts.append(int(cnt.max()))
    assert len(set(counts)) == 1


def test_algorithmic_bytes_of_the_sweep():
    for M in inputs.SWEEP_M:
        gather, window, scan = [], [], []
        for n in inputs.SWEEP_CTX:
            wl = inputs.sweep_workload(n, M)
            db = bench.decode_bytes(wl)
            gather.append(db["gather"])
            scan.append(db["scan"])
            window.append(bench.window_bytes(wl)["total"])
            assert db["gather"] == min(M, n) * wl.H_kv * wl.d * 2 * 2
        assert len(set(gather)) == 1 and len(set(window)) == 1
        ctx = np.array(inputs.SWEEP_CTX, dtype=np.float64)
        assert np.allclose(np.array(scan) / ctx, 128.0)
