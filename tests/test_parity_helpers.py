"""The comparison helpers of the GPU parity tests, checked on the CPU: the top-k
divergence rule accepts only ties and the float bound rejects an error above it."""
import numpy as np
import pytest

from gpu_util import TIE_GAP, assert_close, first_divergence


def _case():
    # 3 tokens, k = 3; zsel holds the oracle's logits of its own picks, in its order
    ref = np.array([[4, 1, 7], [2, 0, 5], [9, 3, 6]], dtype=np.int32)
    zsel = np.array([[2.0, 1.5, 1.0], [3.0, 2.0, 0.5], [1.0, 0.8, 0.2]])
    gap = np.array([0.3, TIE_GAP / 4, 0.2])
    return ref, zsel, gap


def test_identical_ids_agree():
    ref, zsel, gap = _case()
    assert first_divergence(ref.copy(), ref, gap, zsel) is None


def test_reorder_of_equal_logits_agrees_and_of_distinct_logits_fails():
    ref, zsel, gap = _case()
    zsel[0, 2] = zsel[0, 1] + TIE_GAP / 3
    got = ref.copy()
    got[0, [1, 2]] = got[0, [2, 1]]
    assert first_divergence(got, ref, gap, zsel) is None
    got = ref.copy()
    got[2, [0, 1]] = got[2, [1, 0]]                      # logits 1.0 and 0.8: no tie
    with pytest.raises(AssertionError):
        first_divergence(got, ref, gap, zsel)


def test_tie_at_the_cut_returns_the_token():
    ref, zsel, gap = _case()
    got = ref.copy()
    got[1, 2] = 11                                      # the k-th expert swapped, gap below the bound
    assert first_divergence(got, ref, gap, zsel) == 1
    assert first_divergence(got, ref, gap) == 1         # without zsel: the gap alone decides


def test_other_differences_fail():
    ref, zsel, gap = _case()
    got = ref.copy()
    got[0, 2] = 11                                      # a swap where the gap is large
    with pytest.raises(AssertionError):
        first_divergence(got, ref, gap, zsel)
    got = ref.copy()
    got[1, 0] = 11                                      # small gap, but the top expert dropped
    with pytest.raises(AssertionError):
        first_divergence(got, ref, gap, zsel)
    got = ref.copy()
    got[1, 2] = got[1, 0]                               # a repeated id
    with pytest.raises(AssertionError):
        first_divergence(got, ref, gap, zsel)


def test_float_bound_accepts_rounding_and_rejects_a_planted_error():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((4, 256))
    bf16_like = ref * (1 + rng.uniform(-2 ** -8, 2 ** -8, ref.shape))   # one bf16 rounding
    assert_close(bf16_like, ref, "bf16")
    bad = bf16_like.copy()
    bad[2, 17] += 0.05 * np.sqrt(np.mean(ref * ref))     # one element past 2e-2 * rms
    with pytest.raises(AssertionError):
        assert_close(bad, ref, "bf16")
    with pytest.raises(AssertionError):
        assert_close(ref * 1.01, ref, "bf16")             # a 1% scale error: relative L2 1e-2
    with pytest.raises(AssertionError):
        assert_close(bf16_like, ref, "f32")               # bf16 rounding is far outside the fp32 bound


def test_bf16_storage_allowance():
    # The allowance for bf16-stored outputs is half an ulp of the stored value, checked here
    # against the generator's bf16 rounding (round to nearest even): the exact values stored
    # as bf16 pass the max-abs bound with it even where an outlier's own rounding exceeds
    # 2e-2 * rms, and a real error on top of the rounding still fails.
    import synth
    from gpu_util import bf16_half_ulp
    rng = np.random.default_rng(1)
    ref = rng.standard_normal(20000)
    ref[7] = 9.9                                  # an outlier at ~10 rms: its rounding is ~0.03 rms
    stored = (synth.round_bf16(ref.astype(np.float32)).astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.abs(stored - ref) <= bf16_half_ulp(ref))        # half an ulp bounds RNE
    assert np.abs(stored[7] - ref[7]) > 2e-2 * np.sqrt(np.mean(ref * ref))   # the bound alone fails here
    assert_close(stored, ref, "bf16", stored_bf16=True)
    with pytest.raises(AssertionError):
        assert_close(stored, ref, "bf16")
    bad = stored.astype(np.float64)
    bad[11] += 0.05 * np.sqrt(np.mean(ref * ref))
    with pytest.raises(AssertionError):
        assert_close(bad, ref, "bf16", stored_bf16=True)
    # the half ulp: 2^(e-8) for |v| in [2^e, 2^(e+1))
    assert bf16_half_ulp(1.0) == 2.0 ** -8 and bf16_half_ulp(1.99) == 2.0 ** -8 and bf16_half_ulp(2.0) == 2.0 ** -7
    assert bf16_half_ulp(-0.75) == 2.0 ** -9 and bf16_half_ulp(0.0) == 0.0
