"""GPU parity of lisa_linear_decode, one recurrent step of the linear branch
(LISA Sec. 3.1 "Linear Attention"; Sec. 3.3 Eq. 3-4), against the oracle's
recurrent form: S <- S + phi(k)^T v, z <- z + phi(k), o = phi(q) S (divided
by phi(q) . z in the elu+1 mode).

bf16 activations with the 7B head layout and fp32 activations with the tiny
layout, both feature maps, a non-zero starting state.  Tolerances: outputs
max abs <= 2e-2 (bf16) / 1e-4 (fp32) scaled to the output's magnitude for the
identity map (whose outputs grow with the state); the state S (and z) within
1e-4 of its own magnitude.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_top_lightning_b200 import inputs, lisa
from oracle import ref
from lisa_testutil import TOL, max_abs

pytestmark = pytest.mark.gpu


CASES = [
    ("bf16", inputs.DECODE_7B.with_(B=3, n=64)),
    ("f32", inputs.TINY.with_(B=2)),
]


@pytest.mark.parametrize("phi", [lisa.LISA_PHI_IDENTITY, lisa.LISA_PHI_ELU1_NORM])
@pytest.mark.parametrize("dtype,wl", CASES, ids=[c[0] for c in CASES])
def test_linear_decode_one_step(dtype, wl, phi):
    gen = inputs.Generator(wl)
    p, B = wl.n - 1, wl.B
    q = gen.batch("q", p, p + 1)            # [B, 1, H_q, d]
    k = gen.batch("k", p, p + 1)            # [B, 1, H_kv, d]
    v = gen.batch("v", p, p + 1)
    rng = np.random.default_rng(11)
    S0 = (rng.standard_normal((B, wl.H_kv, wl.d, wl.d)) * 0.05).astype(np.float32)
    # a normaliser state as a run of elu+1 features would leave it: positive
    z0 = (rng.random((B, wl.H_kv, wl.d)) * 20.0 + 1.0).astype(np.float32) if phi else None

    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    tq = torch.from_numpy(q).to(dt).cuda()
    tk = torch.from_numpy(k).to(dt).cuda()
    tv = torch.from_numpy(v).to(dt).cuda()
    S = torch.from_numpy(S0).cuda()
    z = torch.from_numpy(z0).cuda() if phi else None
    o = torch.full((B, 1, wl.H_q, wl.d), 9.0, dtype=dt, device="cuda")
    D = lisa.make_dims(B, 1, p, wl.n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype=dtype, phi=phi)
    lisa.lisa_linear_decode(D, tq, tk, tv, S, z, o)
    torch.cuda.synchronize()

    Dr = ref.Dims(B=B, T=1, n_past=p, N_max=wl.n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                  H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M, phi=phi)
    r_o, r_S, r_z = ref.linear(Dr, q, k, v, S0=S0, z0=z0)
    scale = 1.0 if phi else max(1.0, float(np.abs(r_o).max()))
    err = max_abs(o.float().cpu().numpy(), r_o)
    assert err <= TOL[dtype] * scale, (err, scale)
    assert max_abs(S.cpu().numpy(), r_S) <= 1e-4 * max(1.0, float(np.abs(r_S).max()))
    if phi:
        assert max_abs(z.cpu().numpy(), r_z) <= 1e-4 * max(1.0, float(np.abs(r_z).max()))


def test_linear_decode_rejects_more_than_one_token():
    wl = inputs.TINY
    D = lisa.make_dims(1, 2, 0, 4, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       dtype="f32")
    t = torch.zeros(64, device="cuda")
    with pytest.raises(lisa.LisaError) as err:
        lisa.lisa_linear_decode(D, t, t, t, t, None, t)
    assert err.value.status == lisa.LISA_ERR_INVALID_ARG
