"""The seeded input generator (`synth`), checked against facts other than itself: the
published Philox-4x32-10 known-answer vectors, its vectorised path against its scalar
one, and the moments of the normals it draws."""
import os

import numpy as np

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answer_vectors():
    n = 0
    with open(os.path.join(GOLD, "philox4x32_10_kat.txt")) as f:
        for ln in f:
            if not ln.strip() or ln.startswith("#"):
                continue
            w = [int(v, 16) for v in ln.split()]
            got = synth.philox4x32_10(w[0:4], w[4:6])
            assert got.tolist() == w[6:10], ln
            n += 1
    assert n == 3


def test_vectorised_normals_equal_the_scalar_path():
    # offsets and lengths that start and end inside a 16-block group
    for seed, tensor, layer, expert in ((0, 1, 0, 0), (7, 4, 3, 255), (123456789, 8, 15, 17)):
        for off, n in ((0, 64), (0, 1000), (13, 51), (63, 2), (1000003, 777)):
            a = synth.normal_f32(seed, tensor, layer, expert, n, 0.02, off)
            b = synth.normal_f32_scalar(seed, tensor, layer, expert, n, 0.02, off)
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    # a slice of a longer draw is the draw of that slice
    full = synth.normal_f32(3, 2, 1, 5, 4096)
    assert np.array_equal(full[1000:1500], synth.normal_f32(3, 2, 1, 5, 500, offset=1000))


def test_normals_have_standard_moments_and_bounded_tails():
    z = synth.normal_f32(11, 1, 0, 0, 1 << 21).astype(np.float64)
    n = z.size
    assert abs(z.mean()) < 5 / np.sqrt(n)
    assert abs(z.var() - 1) < 5 * np.sqrt(2 / n) + 1e-4      # the table's tails end at 4.42
    assert abs(np.mean(z ** 3)) < 5 * np.sqrt(15 / n)
    assert abs(np.mean(z ** 4) - 3) < 0.02
    assert np.abs(z).max() <= 4.43
    # distinct tensors, layers and experts draw unrelated streams
    w = synth.normal_f32(11, 1, 0, 1, 1 << 21).astype(np.float64)
    assert abs(np.corrcoef(z, w)[0, 1]) < 5 / np.sqrt(n)


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    import torch
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * s for s in (1e-30, 1e-3, 1.0, 1e30)])
    # exact halfway points between two bf16 values, both parities of the kept bit
    halves = (np.arange(0, 1 << 16, 97, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, halves[np.isfinite(halves)], np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38])])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.round_bf16(x), want)


def test_int4_quantiser_follows_the_stated_rule():
    # s = bf16(max|w| / 7) per 128 reduction-axis elements, q = clamp(rint(w / s), -8, 7)
    # with ties to even, element 2b in the low nibble of byte b
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((6, 512)) * 0.02).astype(np.float32)
    w[1, 128:256] = 0.0                                       # an all-zero group: s = 0, q = 0
    q, sbits = synth.quantise_int4(w)
    s = (sbits.astype(np.uint32) << 16).view(np.float32)
    amax = np.abs(w.reshape(6, 4, 128)).max(axis=2)
    assert np.array_equal(sbits, synth.round_bf16((amax / np.float32(7)).astype(np.float32)))
    # exact ties: w = (n + 1/2) s for a group's own s must round to the even neighbour
    w2 = w.copy()
    for g in range(4):
        sg = s[0, g]
        w2[0, 128 * g + 1:128 * g + 9] = (np.arange(-4, 4, dtype=np.float32) + np.float32(0.5)) * sg
    q2, s2 = synth.quantise_int4(w2)
    for ww, qq, ss in ((w, q, sbits), (w2, q2, s2)):
        sv = np.repeat((ss.astype(np.uint32) << 16).view(np.float32), 128, axis=1)
        with np.errstate(divide="ignore", invalid="ignore"):
            want = np.where(sv == 0, 0, np.clip(np.rint(ww / sv), -8, 7)).astype(np.int64)
        lo = (qq & 0x0F).astype(np.int64)
        hi = (qq >> 4).astype(np.int64)
        got = np.empty_like(want)
        got[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
        got[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
        assert np.array_equal(got, want)
    assert np.all(q[1, 64:128] == 0)
