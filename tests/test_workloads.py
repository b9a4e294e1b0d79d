"""The seeded input generator shared by the GPU path and the oracle: bf16
rounding (nearest, ties to even) on hand-worked values, determinism, the
4x4x4 block-major storage order, the workload sizes and the mask recipe."""
import numpy as np

from joint_video_audio_rope_b200 import workloads as WL


def _bits(x):
    return int(WL.f32_to_bf16_bits(np.array([x], np.float32))[0])


def test_bf16_round_to_nearest_even():
    assert _bits(1.0) == 0x3F80
    assert _bits(-2.0) == 0xC000
    # 1 + 2^-8 lies halfway between 1 (mantissa ...0, even) and 1 + 2^-7: down
    assert _bits(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): up
    assert _bits(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above a halfway point rounds up, just below rounds down
    assert _bits(np.nextafter(np.float32(1.0 + 2.0 ** -8), np.float32(2.0))) == 0x3F81
    assert _bits(np.nextafter(np.float32(1.0 + 3 * 2.0 ** -8), np.float32(0.0))) == 0x3F81
    assert _bits(np.inf) == 0x7F80 and _bits(-np.inf) == 0xFF80
    assert (_bits(np.nan) & 0x7F80) == 0x7F80 and (_bits(np.nan) & 0x7F) != 0  # still a NaN


def test_bf16_round_trip_and_error_bound():
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    b = WL.f32_to_bf16_bits(x)
    y = WL.bf16_bits_to_f32(b)
    assert np.array_equal(WL.f32_to_bf16_bits(y), b)                 # representable: exact
    assert np.all(np.abs(y - x) <= 2.0 ** -8 * np.abs(x) + 1e-38)    # half a bf16 ulp


def test_generate_is_deterministic_and_seeded():
    w = WL.WORKLOADS["tiny_f32"]
    a, b = WL.generate(w), WL.generate(w)
    for k in ("q", "k", "v"):
        assert np.array_equal(a[k], b[k])
    w2 = WL.reduced("480p", 2, 4, 6, n_audio=10, n_text=5)
    x = WL.generate(w2)
    assert x["q"].dtype == np.uint16 and x["q"].shape == (1, w2.n_tokens, 2, 128)
    assert not np.array_equal(x["q"], x["k"])


def test_block_major_permutation():
    T, H, W = 5, 6, 7
    p = WL._block_major_permutation(T, H, W)
    assert sorted(p.tolist()) == list(range(T * H * W))
    # the first block is the 4x4x4 corner in (t, h, w) raster order
    corner = [(t * H + h) * W + w for t in range(4) for h in range(4) for w in range(4)]
    assert p[:64].tolist() == corner
    # the short last t-slab (t = 4) holds only its real tokens: the final block
    # is the (1 x 2 x 3) corner at t = 4, h >= 4, w >= 4
    last = [(4 * H + h) * W + w for h in range(4, 6) for w in range(4, 7)]
    assert p[-6:].tolist() == last


def test_workload_sizes_and_ranges():
    want = {"480p": 33490, "720p": 76330, "720p_cond_b2": 83530, "1080p_sparse": 171578}
    for name, n in want.items():
        w = WL.WORKLOADS[name]
        assert w.n_tokens == n
        v0, v1 = w.video_range()
        a0, a1 = w.audio_range()
        assert a1 - a0 == 218 and v1 - v0 == w.n_video and v0 == 0
    assert WL.WORKLOADS["480p"].text_range() == (32978, 33490)
    assert WL.WORKLOADS["1080p_sparse"].text_range() == (0, 0)


def test_mask_recipe_covers_thirty_percent():
    w = WL.reduced("720p_cond_b2", 6, 9, 16, n_audio=20, n_text=8)
    m = WL.generate(w)["mask"]
    frames = sum(s["T"] for s in w.segments if s["kind"] == WL.SEG_VIDEO)
    assert m.shape == (w.batch, frames, 9, 16) and m.dtype == np.uint8
    for b in range(w.batch):
        assert m[b].mean() >= 0.30
        assert set(np.unique(m[b]).tolist()) <= {0, 1}
