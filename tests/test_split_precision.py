"""The precision argument behind the router backward's tensor-core forms, checked on the
host: an fp32 value v split into hi = bf16(v) and lo = bf16(v - hi) (both rounded to
nearest even) leaves |v - hi - lo| <= 2^-16 |v|, and v - hi is exact in fp32. bf16 rounding
is emulated bit by bit here (no GPU, no library code): the tensor-core kernels form hi and
lo with the same round-to-nearest-even conversion, so this bound is what keeps their fp32
sums, and so the fp32 tolerances of the router-backward parity tests, unchanged."""
import numpy as np


def bf16_rne(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 -> fp32 with round to nearest, ties to even (finite inputs)."""
    b = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return rounded.astype(np.uint32).view(np.float32)


def split(v):
    v = np.asarray(v, np.float32)
    hi = bf16_rne(v)
    r = (v - hi).astype(np.float32)
    lo = bf16_rne(r)
    return hi, r, lo


def test_bf16_rne_emulation_matches_torch():
    import torch
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(100_000) * np.exp2(rng.integers(-60, 60, 100_000))).astype(
        np.float32)
    got = bf16_rne(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(got, ref)


def test_split_residual_is_exact_and_below_2_pow_minus_16():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(400_000) * np.exp2(rng.integers(-100, 100, 400_000))).astype(
        np.float32)
    hi, r, lo = split(v)
    v64, hi64, r64 = v.astype(np.float64), hi.astype(np.float64), r.astype(np.float64)
    assert np.array_equal(v64 - hi64, r64)  # v - hi is exact in fp32
    err = np.abs(v64 - hi64 - lo.astype(np.float64))
    assert np.all(err <= np.abs(v64) * 2.0 ** -16)
    # the bound is tight to a factor of about 2: a single bf16 term leaves up to 2^-8 |v|
    assert err.max() / np.abs(v64[err.argmax()]) > 2.0 ** -18
    single = np.abs(v64 - hi64) / np.abs(v64)
    assert single.max() > 2.0 ** -10


def test_split_at_rounding_ties_and_powers_of_two():
    # values exactly halfway between two bf16 numbers (ties go to even) and next to powers
    # of two, where the spacing changes
    base = np.float32(1.0) + np.arange(0, 256, dtype=np.float32) * np.float32(2.0 ** -7)
    half = (base + np.float32(2.0 ** -8)).astype(np.float32)  # ties
    near = np.concatenate([np.nextafter(np.float32(2.0) ** np.arange(-20, 20), 0).astype(
        np.float32), np.float32(2.0) ** np.arange(-20, 20).astype(np.float32)])
    for v in (half, -half, near, -near):
        hi, r, lo = split(v)
        err = np.abs(v.astype(np.float64) - hi - lo.astype(np.float64))
        assert np.all(err <= np.abs(v.astype(np.float64)) * 2.0 ** -16)


def test_split_products_keep_fp32_accuracy_in_a_sum():
    """sum_t x_t v_t with x bf16 and v fp32: the two-term products summed in fp32 stay
    within fp32 rounding of the fp64 sum; the one-term (bf16 v) sum does not."""
    rng = np.random.default_rng(3)
    T = 4096
    x = bf16_rne(rng.standard_normal(T).astype(np.float32)).astype(np.float64)
    v = (0.1 * rng.standard_normal(T)).astype(np.float32)
    hi, _, lo = split(v)
    exact = float(np.dot(x, v.astype(np.float64)))
    two = float(np.dot(x, hi.astype(np.float64)) + np.dot(x, lo.astype(np.float64)))
    one = float(np.dot(x, hi.astype(np.float64)))
    scale = float(np.sqrt(np.sum((x * v) ** 2)))
    assert abs(two - exact) <= scale * 2.0 ** -16
    assert abs(one - exact) > abs(two - exact) * 16
