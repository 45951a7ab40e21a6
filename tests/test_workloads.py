"""The seeded generators: deterministic, shaped and distributed as stated."""
import numpy as np

import workloads as wl


def test_configs_match_the_stated_shapes():
    assert [(w.T, w.d, w.N_r, w.n_group, w.topk_group, w.k) for w in wl.ALL] == [
        (64, 512, 64, 4, 2, 4), (4096, 7168, 256, 8, 4, 8), (8192, 7168, 384, 1, 1, 8),
        (64, 7168, 256, 8, 4, 8), (16384, 7168, 256, 8, 4, 8)]
    assert wl.K2_PREFILL.mask_mode == wl.MASK_ZERO and wl.K2_PREFILL.route_scale == 2.827
    assert wl.V3_FULL.hot_experts == 32 and wl.V3_FULL.hot_bias == 1.0


def test_generation_is_deterministic_and_bf16_exact():
    w = wl.V3_DECODE
    a, b = wl.gen_router_inputs(w), wl.gen_router_inputs(w)
    for key in ("x_f32", "x_bf16", "W", "b"):
        assert np.array_equal(a[key], b[key])
    assert np.array_equal(wl.bf16_bits_to_f32(a["x_bf16"]), a["x_f32"])
    assert a["W"].dtype == np.float32 and a["W"].shape == (256, 7168)
    assert abs(a["W"].std() * np.sqrt(7168) - 1) < 0.01
    assert a["b"].min() >= -0.1 and a["b"].max() <= 0.1


def test_block_seeding_independent_of_threads():
    w = wl.TINY.replace(T=3000, d=7000, k=1)  # > one 2^24-element block
    e1 = wl._normal_blocks(wl._child(w.seed, "E"), w.T * w.d, wl.F32, threads=1)
    e4 = wl._normal_blocks(wl._child(w.seed, "E"), w.T * w.d, wl.F32, threads=4)
    assert np.array_equal(e1, e4)


def test_skewed_bias():
    b = wl.gen_b(wl.V3_FULL)
    assert (b[:32] > 0.89).all() and (np.abs(b[32:]) <= 0.1).all()


def test_to_bf16_bits_round_to_nearest_even():
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1.0, 0.0], np.float32)
    assert wl.to_bf16_bits(v).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x0000]
