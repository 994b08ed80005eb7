"""GPU parity of the per-channel gate (LISA, arXiv 2607.19358v1, Sec. 3.3
Eq. 5, mixing the branches as in Eq. 1) against the oracle: the tensor-core
tiles at sizes that span several tiles, a ragged token tail and a K ring that
wraps; the decode kernel for a few tokens at the 7B width; the 7B prefill at
full size on sampled token rows; the plain kernel for the other sizes and fp32.
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


def _case(wl, T, D_h):
    gen = inputs.Generator(wl)
    h = np.stack([gen.hidden(b, 0, T, D_h) for b in range(wl.B)])
    W = gen.gate_weight(D_h)
    o_lin = np.stack([gen.branch("o_lin", b, 0, T) for b in range(wl.B)])
    o_sp = np.stack([gen.branch("o_sp", b, 0, T) for b in range(wl.B)])
    return h, W, o_lin, o_sp


def _run(wl, T, D_h, h, W, o_lin, o_sp):
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype=wl.dtype)
    o = torch.full((wl.B, T, wl.H_q, wl.d), 99.0, dtype=dt, device="cuda")
    ws = lisa.workspace(D, lisa.LISA_OP_GATE_CHANNEL)
    lisa.lisa_gate_channel(D, D_h, _dv(h, dt), _dv(W, dt), _dv(o_lin, dt), _dv(o_sp, dt), o, ws)
    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
    return o.float().cpu().numpy()


def _ref(wl, T, D_h, h, W, o_lin, o_sp, rows=None):
    Dr = ref.Dims(B=wl.B, T=T, n_past=0, N_max=T, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    if rows is not None:
        o_lin, o_sp = o_lin[:, rows], o_sp[:, rows]
    return ref.gate_channel(Dr, D_h, h, W, o_lin, o_sp, rows=rows)


# (B, T, H_q, D_h): 2 x 150 tokens = 2 full 128-token tiles and a ragged 44;
# D_h 192 fills 3 of the 4 ring stages, 576 wraps the ring twice; H_q 4 is two
# channel tiles; 65 tokens is the fewest the tensor-core tiles take.
@pytest.mark.parametrize("B,T,H_q,D_h", [(2, 150, 2, 192), (2, 150, 4, 576), (1, 65, 2, 64),
                                         (3, 333, 2, 1024)])
def test_gate_channel_tensor_core_tiles(B, T, H_q, D_h):
    wl = inputs.PREFILL_1P5B.with_(B=B, n=T, H_q=H_q)
    h, W, o_lin, o_sp = _case(wl, T, D_h)
    got = _run(wl, T, D_h, h, W, o_lin, o_sp)
    err = max_abs(got, _ref(wl, T, D_h, h, W, o_lin, o_sp))
    assert err <= TOL["bf16"], err


# up to 64 tokens: tiles of 8, 16, 32 and 64 tokens, ragged
@pytest.mark.parametrize("B,T,H_q,D_h", [(1, 64, 2, 64), (1, 20, 4, 256), (1, 40, 2, 128),
                                         (3, 3, 2, 1088)])
def test_gate_channel_streamed_few_tokens(B, T, H_q, D_h):
    wl = inputs.PREFILL_1P5B.with_(B=B, n=T, H_q=H_q)
    h, W, o_lin, o_sp = _case(wl, T, D_h)
    got = _run(wl, T, D_h, h, W, o_lin, o_sp)
    err = max_abs(got, _ref(wl, T, D_h, h, W, o_lin, o_sp))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("B", [1, 8, 16])
def test_gate_channel_decode_7b(B):
    """A few tokens at the 7B width (3584 channels, D_h 3584): W_g streamed once."""
    wl = inputs.DECODE_7B.with_(B=B)
    D_h = wl.H_q * wl.d
    h, W, o_lin, o_sp = _case(wl, 1, D_h)
    got = _run(wl, 1, D_h, h, W, o_lin, o_sp)
    err = max_abs(got, _ref(wl, 1, D_h, h, W, o_lin, o_sp))
    assert err <= TOL["bf16"], err


def test_gate_channel_prefill_7b_sampled_rows():
    """16384 tokens x 3584 channels x D_h 3584 (the 7B prefill); the oracle
    recomputes 40 token rows, first, last and across the tiles."""
    wl = inputs.PREFILL_7B
    T, D_h = wl.n, wl.H_q * wl.d
    h, W, o_lin, o_sp = _case(wl, T, D_h)
    got = _run(wl, T, D_h, h, W, o_lin, o_sp)
    rows = np.unique(np.concatenate([[0, 127, 128, T - 129, T - 1],
                                     np.random.default_rng(3).integers(0, T, 35)])).astype(np.int32)
    want = _ref(wl, T, D_h, h, W, o_lin, o_sp, rows=rows)
    err = max_abs(got[:, rows], want)
    assert err <= TOL["bf16"], err
    assert np.isfinite(got).all()


@pytest.mark.parametrize("dtype,H_q,d,D_h", [("f32", 2, 64, 40), ("bf16", 3, 64, 100),
                                             ("bf16", 2, 128, 70)])
def test_gate_channel_plain_kernel(dtype, H_q, d, D_h):
    """Sizes off the tensor-core tiling (channels not a multiple of 256, D_h not
    of 64) and fp32 take the plain kernel."""
    base = inputs.TINY if dtype == "f32" else inputs.PREFILL_1P5B
    wl = base.with_(B=2, n=70, H_q=H_q, H_kv=1, d=d)
    h, W, o_lin, o_sp = _case(wl, 70, D_h)
    got = _run(wl, 70, D_h, h, W, o_lin, o_sp)
    err = max_abs(got, _ref(wl, 70, D_h, h, W, o_lin, o_sp))
    assert err <= TOL[dtype], err


def test_gate_channel_empty_and_bad_args():
    wl = inputs.PREFILL_1P5B.with_(B=1, n=8, H_q=2)
    D = lisa.make_dims(1, 0, 0, 8, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    ws = lisa.workspace(D, lisa.LISA_OP_GATE_CHANNEL)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lisa.lisa_gate_channel(D, 64, x, x, x, x, x, ws)  # no tokens: nothing to do
    D1 = lisa.make_dims(1, 8, 0, 8, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    with pytest.raises(lisa.LisaError):
        lisa.lisa_gate_channel(D1, 0, x, x, x, x, x, ws)
