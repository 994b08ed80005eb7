"""The seeded input generator: bf16 rounding and stream independence (CPU only)."""
import numpy as np
import torch

from hybrid_linear_top_lightning_b200 import inputs


def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 65504.0], np.float32)])
    mine = inputs.round_bf16(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(mine.view(np.uint32), theirs.view(np.uint32))


def test_values_do_not_depend_on_the_requested_window():
    gen = inputs.Generator(inputs.PREFILL_1P5B)
    whole = gen.k(0, 0, 3000)
    part = gen.k(0, 1500, 2100)
    np.testing.assert_array_equal(whole[1500:2100], part)
    assert np.all(inputs.round_bf16(whole) == whole)


def test_planting_recipe():
    wl = inputs.DECODE_7B.with_(B=2, n=4096)
    gen = inputs.Generator(wl)
    pos = gen.planted_positions(1)
    assert pos.size == 40 and len(set(pos.tolist())) == 40
    assert not np.array_equal(pos, gen.planted_positions(0))
    u = gen.unit_vector("u_kI", wl.d_I)
    assert abs(np.linalg.norm(u) - 1.0) < 1e-12
    k_I = gen.k_I(1, 0, wl.n).reshape(wl.n, -1).astype(np.float64)
    proj = k_I @ u
    # planted rows carry +3 sigma sqrt(d_I) along u; the rest are N(0, sigma^2) along u
    shift = 3 * wl.sigma * np.sqrt(wl.d_I)
    assert np.all(proj[pos] > shift - 5 * wl.sigma)
    others = np.setdiff1d(np.arange(wl.n), pos)
    assert abs(proj[others].std() / wl.sigma - 1.0) < 0.1
