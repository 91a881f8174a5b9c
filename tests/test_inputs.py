"""The seeded input generator: Philox known answers, Box-Muller moments, bf16 rounding."""
import numpy as np

from sparse_moe_layer_select_b200 import inputs as I


def test_philox4x32_10_known_answers():
    # Known-answer vectors of Philox4x32-10 published with Random123 (Salmon et al., SC'11)
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for ctr, key, want in cases:
        got = I.philox4x32_10(*[np.array([c], dtype=np.uint64) for c in ctr], *key)
        assert tuple(int(g[0]) for g in got) == want


def test_normal_moments_and_offsets():
    z = I.normal_f64_numpy(400_000, 0, 0)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert abs(np.mean(z ** 4) - 3.0) < 0.05
    a = I.generate_numpy((1000,), 0, 3, 0.02)
    assert np.array_equal(I.generate_numpy((11,), 0, 3, 0.02, start=501), a[501:512])
    assert np.array_equal(I.generate_numpy((10,), 0, 3, 0.02, start=500), a[500:510])
    # distinct tensor ids and seeds give distinct streams
    assert not np.array_equal(I.generate_numpy((64,), 0, 4, 1.0), I.generate_numpy((64,), 0, 3, 1.0))
    assert not np.array_equal(I.generate_numpy((64,), 1, 3, 1.0), I.generate_numpy((64,), 0, 3, 1.0))


def test_bf16_round_to_nearest_even():
    one = 1.0
    ulp = 2.0 ** -7
    vals = np.array([one, one + ulp / 2, one + 3 * ulp / 2, one + ulp / 2 + 2 ** -40, -2.5,
                     0.0, 1e-3, 65504.0])
    got = I.bf16_bits_to_f32(I.f64_to_bf16_bits(vals)).astype(np.float64)
    assert got[0] == 1.0
    assert got[1] == 1.0                     # tie -> even
    assert got[2] == one + 2 * ulp           # tie -> even (upwards)
    assert got[3] == one + ulp               # above the tie -> up
    assert got[4] == -2.5 and got[5] == 0.0
    assert abs(got[6] - 1e-3) <= 1e-3 * 2 ** -8
    # matches float32 rounding followed by round-to-nearest-even where no double rounding occurs
    rng = np.random.default_rng(0)
    v = rng.standard_normal(10000)
    b = I.f64_to_bf16_bits(v)
    back = I.bf16_bits_to_f32(b).astype(np.float64)
    assert np.all(np.abs(back - v) <= np.abs(v) * 2.0 ** -8 + 1e-300)


def test_zipf_rank_is_a_permutation():
    r = I.zipf_rank(256)
    assert sorted(r.tolist()) == list(range(1, 257))
    b = I.zipf_bias(256, 1.1, 1.0)
    assert b.dtype == np.float32 and b.max() == 0.0 and np.argmax(b) == np.argmin(r)


def test_workload_table_shapes():
    w = I.get("c2_xs2_small")
    names = [s[0] for s in I.tensor_specs(w)]
    assert names == ["x", "w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"]
    shapes = {s[0]: s[1] for s in I.tensor_specs(w)}
    assert shapes["w_gate"] == (256, 512, 2048) and shapes["w_down"] == (256, 2048, 512)
    h = I.host_inputs(I.get("c1_tiny"))
    assert h["x"].shape == (64, 256) and h["x"].dtype == np.uint16 and h["router_bias"] is None
