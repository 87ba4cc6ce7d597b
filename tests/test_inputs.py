"""The seeded input generator: determinism, distribution and bf16 rounding."""
import numpy as np

from long_context_prefill_trianglemix_b200 import inputs as I


def test_deterministic_and_split_independent():
    a = np.empty(4 * 33 * 3 * 16, np.uint16)
    b = np.empty_like(a)
    I.fill_bf16(a, 4, 33, 3, 16, seed=5, tensor_id=1, nthreads=1)
    I.fill_bf16(b, 4, 33, 3, 16, seed=5, tensor_id=1, nthreads=7)
    np.testing.assert_array_equal(a, b)
    c = np.empty_like(a)
    I.fill_bf16(c, 4, 33, 3, 16, seed=6, tensor_id=1)
    assert (a != c).mean() > 0.9


def test_values_are_rounded_normals():
    n = 2 * 5 * 2 * 8
    a = np.empty(n, np.uint16)
    I.fill_bf16(a, 2, 5, 2, 8, seed=3, tensor_id=2)
    z = np.array([I.normal_at(3, 2, e) for e in range(n)], np.float64)
    np.testing.assert_array_equal(a, I.f32_to_bf16_bits(z.astype(np.float32)))


def test_moments():
    a = np.empty(1 << 20, np.uint16)
    I.fill_bf16(a, 1, 1 << 14, 1, 64, seed=0, tensor_id=0)
    f = I.bf16_bits_to_f32(a).astype(np.float64)
    assert abs(f.mean()) < 5e-3 and abs(f.std() - 1.0) < 5e-3


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 0.0, np.inf], np.float32)
    got = I.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(got, [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000, 0x7F80])


def test_outlier_recipe_scales_same_channels_in_q_and_k():
    wl = I.Workload("t", B=1, Hq=8, Hkv=2, N=16, D=32, S=1, W=2, L=1, recipe="outliers")
    (qh, qc), (kh, kc), _ = I.scales_for(wl)
    qc, kc = qc.reshape(8, 32), kc.reshape(2, 32)
    for g in range(2):
        chans = np.flatnonzero(kc[g] == 8.0)
        assert len(chans) == 4
        for h in range(4 * g, 4 * g + 4):
            np.testing.assert_array_equal(np.flatnonzero(qc[h] == 8.0), chans)


def test_headscale_recipe_range():
    wl = I.WORKLOADS["qwen2.5-7b-128k-28layer"]
    (qh, _), (kh, _), _ = I.scales_for(wl)
    assert qh.shape == (28,) and kh.shape == (4,)
    assert (qh >= 0.5).all() and (qh <= 2.0).all() and len(set(qh.tolist())) == 28


def test_planted_recipe_adds_exactly_its_structure():
    import dataclasses
    base = I.WORKLOADS["llama3-8b-128k-planted"]
    wl = dataclasses.replace(base, N=1000, Hq=4, Hkv=2)
    plain = dataclasses.replace(wl, recipe="plain")
    q, k, v = I.make_qkv(wl)
    q0, k0, v0 = I.make_qkv(plain)
    D, nc = wl.D, 2 * len(I.PLANT_PERIODS) + 1
    assert np.array_equal(v, v0)
    assert np.array_equal(q[..., :D - nc], q0[..., :D - nc])
    assert np.array_equal(k[..., :D - nc], k0[..., :D - nc])
    pos = np.arange(wl.N)
    for c, period in enumerate(I.PLANT_PERIODS):
        w = 2 * np.pi / period
        for ch, val in ((D - 1 - 2 * c, np.cos(w * pos)), (D - 2 - 2 * c, np.sin(w * pos))):
            for a, a0 in ((q, q0), (k, k0)):
                want = I.bf16_bits_to_f32(a0[..., ch]) + np.float32(I.PLANT_AMP) * \
                    val.astype(np.float32)[None, :, None]
                assert np.array_equal(a[..., ch], I.f32_to_bf16_bits(want.astype(np.float32)))
    ch = D - nc
    dq = I.bf16_bits_to_f32(q[..., ch]) - I.bf16_bits_to_f32(q0[..., ch])
    assert np.allclose(dq, I.PLANT_VERTICAL_AMP, atol=0.05)
    blocks = I.planted_vertical_blocks(0, wl.Hkv, (wl.N + 127) // 128)
    dk = I.bf16_bits_to_f32(k[..., ch]) - I.bf16_bits_to_f32(k0[..., ch])
    for g in range(wl.Hkv):
        in_v = np.zeros(wl.N, bool)
        for b in blocks[g]:
            in_v[b * 128:(b + 1) * 128] = True
        assert np.allclose(dk[0, in_v, g], I.PLANT_VERTICAL_AMP, atol=0.05)
        assert np.array_equal(dk[0, ~in_v, g], np.zeros((~in_v).sum(), np.float32))
