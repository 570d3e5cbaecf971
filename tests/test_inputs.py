"""The seeded input generators (shared by the CUDA path and the oracle): any unit
regenerates alone, bf16 rounding is round-to-nearest-even, draws are
deterministic and in their stated ranges.  No GPU."""
import numpy as np
import pytest
import torch

from test_sequence_modeling_b200 import inputs as I


@pytest.mark.parametrize("name", I.CONFIG_ORDER)
def test_units_regenerate_alone(name):
    cfg = I.CONFIGS[name].replace(B=3, H=2, T=32)
    full = I.make_inputs(cfg, threads=2)
    for bi, hi in ((0, 0), (2, 1), (1, 0)):
        q, k, v, e = I.unit_inputs(cfg, bi, hi)
        for key, x in (("Q", q), ("K", k), ("V", v)):
            got = full[key][bi, hi]
            if full["qkv_bits"]:
                got = I.bits_to_f32(got)
            assert np.array_equal(got, x), (key, bi, hi)
        assert np.array_equal(full["eta"][bi, hi], e)


def test_batch_offset_draws_the_global_rows():
    cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=16)
    shard = I.make_inputs(cfg, threads=1, batch_offset=5)
    q, _, _, e = I.unit_inputs(cfg, 6, 1)
    assert np.array_equal(I.bits_to_f32(shard["Q"][1, 1]), q)
    assert np.array_equal(shard["eta"][1, 1], e)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32),
                        # exact ties between two bf16 values (low 16 bits = 0x8000)
                        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        np.array([0.0, -0.0, 1e-38, 3.4e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(I.round_to_bf16(x), ref)
    # bf16_bits takes bf16-exact values: the encoding round-trips exactly.
    assert np.array_equal(I.bits_to_f32(I.bf16_bits(I.round_to_bf16(x))), ref)


def test_draws_are_deterministic_and_in_range():
    cfg = I.CONFIGS["mlp_B8H32T8192"].replace(B=2, H=2, T=64)
    a, b = I.make_inputs(cfg, threads=1), I.make_inputs(cfg, threads=3)
    for key in ("Q", "K", "V", "eta", "W1", "W2", "gamma", "beta"):
        assert np.array_equal(a[key], b[key]), key
    assert np.all((a["eta"] > 0) & (a["eta"] < cfg.eta_scale))
    const = I.make_inputs(I.CONFIGS["linear_f32_B1H1T256"].replace(T=32))
    assert np.all(const["eta"] == np.float32(0.1))
    alpha, lam = I.momentum_rates(cfg)
    assert alpha.shape == lam.shape == (2, 2, 64) and alpha.dtype == np.float32
    assert np.all((alpha >= 0) & (alpha < 0.9)) and np.all((lam >= 0) & (lam < 0.05))
    dZ, dWT = I.cotangents(cfg)
    assert dZ.shape == (2, 2, 64, 64) and dWT.shape == (2, 2, 64, 64) and dZ.dtype == np.float32
    assert 0.8 / 8 < float(dZ.std()) < 1.2 / 8
