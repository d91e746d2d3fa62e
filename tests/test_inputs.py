"""The seeded input generator: published hash value, distributions, slicing."""
import numpy as np
import pytest

import moe_inputs as mi


def test_splitmix64_published_first_output():
    # SplitMix64 from state 0 returns 0xE220A8397B1DCDAF first (Vigna's
    # splitmix64.c, Steele et al. 2014); seed = tensor id = index = 0 is that state.
    assert mi.hash64(0, 0, 0) == 0xE220A8397B1DCDAF


def test_hash_depends_on_every_field():
    base = mi.hash64(0, 1, 5)
    assert base != mi.hash64(1, 1, 5)
    assert base != mi.hash64(0, 2, 5)
    assert base != mi.hash64(0, 1, 6)


def test_normal_moments_and_range():
    x = mi.fill_host(1 << 20, 0, 1, ("normal", 0.02), "f32").astype(np.float64)
    assert abs(x.mean()) < 3 * 0.02 / np.sqrt(x.size) * 3
    assert abs(x.std() / 0.02 - 1.0) < 5e-3
    assert np.abs(x).max() <= 0.02 * np.sqrt(3) * 2 * 1.0001
    # fourth moment of a 4-term Irwin-Hall sum: kurtosis 3 - 6/(5*4) = 2.7
    kurt = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert abs(kurt - 2.7) < 0.02


def test_uniform_range_and_mean():
    x = mi.fill_host(1 << 18, 0, 3, ("uniform", -0.01, 0.01), "f32").astype(np.float64)
    assert x.min() >= -0.01 and x.max() < 0.01
    assert abs(x.mean()) < 1e-4
    assert abs(x.std() - 0.02 / np.sqrt(12)) < 1e-4


def test_bf16_storage_is_rounded_fp32():
    f = mi.fill_host(4096, 7, 4, ("normal", 1.0), "f32")
    b = mi.fill_host(4096, 7, 4, ("normal", 1.0), "bf16")
    np.testing.assert_array_equal(mi.f32_to_bf16_f32(f), b)
    # bf16 values have at most 8 significant bits
    m, _ = np.frexp(b.astype(np.float64))
    assert np.all(m * 256 == np.rint(m * 256))


def test_slices_regenerate_the_same_elements():
    cfg = mi.CONFIGS["tiny_fp32"]
    full = mi.host_tensor(cfg, "w_gate")
    part = mi.host_tensor(cfg, "w_gate", rows=slice(3, 5))
    np.testing.assert_array_equal(full[3:5], part)


def test_stress_edit_applies_once():
    cfg = mi.CONFIGS["tiny_fp32"].with_(skew=(3, 8.0, 3.0))
    h = mi.host_tensor(cfg, "h")
    h0 = mi.host_tensor(cfg.with_(skew=None), "h")
    np.testing.assert_array_equal(h[:, 1:], h0[:, 1:])
    np.testing.assert_array_equal(h[:, 0], (h0[:, 0] + np.float32(8.0)).astype(np.float32))
    wr = mi.host_tensor(cfg, "w_router")
    wr_part = mi.host_tensor(cfg, "w_router", rows=slice(2, 4))
    np.testing.assert_array_equal(wr[2:4], wr_part)


@pytest.mark.parametrize("name", list(mi.CONFIGS))
def test_config_shapes(name):
    cfg = mi.CONFIGS[name]
    specs = mi.layer_tensor_specs(cfg)
    assert specs["w_gate"].shape == (cfg.n_experts, cfg.d_ff, cfg.d_model)
    assert specs["w_down"].shape == (cfg.n_experts, cfg.d_model, cfg.d_ff)
    assert ("ws_gate" in specs) == (cfg.d_ff_shared > 0)
