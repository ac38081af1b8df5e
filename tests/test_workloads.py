"""The seeded input generator: published SplitMix64 definition, determinism and
the planted structure (heavy keys, sink, band correlation)."""
import numpy as np

import workloads as W

MASK = (1 << 64) - 1


def _mix_reference(z):
    # SplitMix64 finaliser as published (Steele, Lea, Flood 2014; Vigna).
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def test_splitmix_finaliser_matches_definition():
    lib = W.raw()
    for z in (0, 1, 0x9E3779B97F4A7C15, 123456789, MASK):
        assert lib.tsagen_mix64(z) == _mix_reference(z)
    # sequential SplitMix64 from state 0: out_n = mix(gamma * (n + 1))
    gamma = 0x9E3779B97F4A7C15
    assert lib.tsagen_mix64(gamma) == 0xE220A8397B1DCDAF  # first output of seed 0


def test_bf16_rounding_is_nearest_even():
    lib = W.raw()
    for f, want in [(1.0, 0x3F80), (1.00390625, 0x3F80), (1.01171875, 0x3F82),
                    (-2.5, 0xC020), (65504.0, 0x4780), (1.0 + 2.0 ** -9, 0x3F80), (float("inf"), 0x7F80)]:
        assert lib.tsagen_f32_to_bf16(f) == want
    x = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    assert np.array_equal(W.f32_to_bf16_bits(x),
                          np.array([lib.tsagen_f32_to_bf16(float(t)) for t in x], dtype=np.uint16))


def test_generate_is_deterministic_and_seeded():
    wl = W.WORKLOADS["c1_L1K_mha_d64"].with_(L=256)
    a = W.generate(wl)
    b = W.generate(wl)
    c = W.generate(wl.with_(seed=99))
    for x, y, z in zip(a, b, c):
        assert np.array_equal(x, y)
        assert not np.array_equal(x, z)
    v = W.bf16_bits_to_f64(a[2])
    assert abs(v.mean()) < 0.05 and abs(v.std() - 1) < 0.05


def test_heavy_keys_and_sink():
    wl = W.WORKLOADS["c1_L1K_mha_d64"]
    q, k, v = W.generate(wl)
    plain = W.generate(wl.with_(heavy_count=0, sink=False))[1]
    for g in range(wl.Hkv):
        rows = W.heavy_rows(wl, 0, g)
        assert len(rows) == 16 and len(set(rows.tolist())) == 16
        ratio = np.abs(W.bf16_bits_to_f64(k[0, g])).sum(-1) / np.abs(W.bf16_bits_to_f64(plain[0, g])).sum(-1)
        scaled = set(np.where(ratio > 3.5)[0].tolist())
        assert scaled == set(rows.tolist()) | {0}
    # per-sequence fractions drawn in [lo, hi]
    wl5 = W.WORKLOADS["c5_B4_L64K_gqa"].with_(L=4096)
    counts = [len(W.heavy_rows(wl5, b, g)) for b in range(wl5.B) for g in range(wl5.Hkv)]
    assert all(int(np.ceil(0.001 * 4096)) <= c <= int(np.ceil(0.02 * 4096)) for c in counts)
    assert len(set(counts)) > 3


def test_band_bias_correlates_nearby_q_and_k():
    wl = W.WORKLOADS["c3_L32K_gqa_band"].with_(L=4096, heavy_frac_lo=0, heavy_frac_hi=0)
    q, k, _ = W.generate(wl)
    qf, kf = W.bf16_bits_to_f64(q[0, 0]), W.bf16_bits_to_f64(k[0, 0])
    near = np.mean(np.sum(qf[300:3800] * kf[310:3810], -1)) / wl.d
    far = np.mean(np.sum(qf[300:3500] * kf[600:3800], -1)) / wl.d
    # expected near correlation a^2/(1+a^2) * (1 - 10/257) = 0.192; far = 0
    assert 0.15 < near < 0.24 and abs(far) < 0.03
