"""The three-part bf16 split of an fp32 value that hc_mix's gate kernel feeds
to its tensor-core tiles: hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi
- mid), every rounding to nearest even, every difference in fp32.

Checked here on the host, by the mathematics the kernel relies on, with
numpy's fp32 arithmetic and an exact bf16 rounding of fp32 bit patterns:
  * each difference is exact in fp32 (v and its bf16 rounding share their
    leading bits, so v - hi has at most 16 significant bits);
  * hi + mid + lo equals v to within 2^-24 |v| (three 8-bit pieces carry
    the 24-bit significand; only the last rounding loses anything), for
    every normal fp32 v whose parts stay in range — sampled across the whole
    exponent range, with the binade edges, ties and the largest values that
    bf16 rounds to a finite number;
  * zero, and values so small that their lower parts fall below bf16's
    subnormal range, lose at most what those parts lose (checked as an
    absolute bound there).
No kernel code runs here; this pins the arithmetic claim that the gate
kernel's logits keep fp32 accuracy.
"""
import numpy as np


def bf16_rn(v32):
    """fp32 -> nearest-even bf16, returned as fp32 (bit-exact)."""
    b = np.asarray(v32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def split3(v):
    v = np.asarray(v, dtype=np.float32)
    hi = bf16_rn(v)
    e1 = (v - hi).astype(np.float32)
    mid = bf16_rn(e1)
    e2 = (e1 - mid).astype(np.float32)
    lo = bf16_rn(e2)
    return hi, e1, mid, e2, lo


def samples(rng, n=200_000):
    exps = rng.integers(-100, 120, size=n)
    mant = rng.random(n) + 1.0
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    v = (sign * mant * np.exp2(exps)).astype(np.float32)
    # binade edges, bf16 ties (the 17th bit set alone) and neighbours
    edges = []
    for e in (-100, -20, -1, 0, 1, 20, 100, 126):
        base = np.float32(2.0 ** e)
        bits = np.float32(base).view(np.uint32)
        for d in (0, 1, 2, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x10000):
            edges.append(np.uint32(bits + d).view(np.float32))
            edges.append(np.uint32(bits - 1 - d).view(np.float32) if bits > d + 1 else base)
    # the largest fp32 values that bf16 still rounds to a finite number
    top = np.float32(np.frombuffer(np.uint32(0x7F7F7FFF).tobytes(), dtype=np.float32)[0])
    edges += [top, -top]
    return np.concatenate([v, np.array(edges, dtype=np.float32)])


def test_differences_are_exact_in_fp32():
    v = samples(np.random.default_rng(7))
    hi, e1, mid, e2, lo = split3(v)
    assert np.all(np.isfinite(hi))
    # the fp32 differences equal the exact (float64) ones
    assert np.array_equal(e1.astype(np.float64), v.astype(np.float64) - hi.astype(np.float64))
    assert np.array_equal(e2.astype(np.float64), e1.astype(np.float64) - mid.astype(np.float64))


def test_three_parts_carry_v_to_2_pow_minus_24():
    v = samples(np.random.default_rng(11))
    hi, _, mid, _, lo = split3(v)
    total = hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64)
    err = np.abs(total - v.astype(np.float64))
    av = np.abs(v.astype(np.float64))
    # lower parts below bf16's smallest subnormal (2^-133) are lost outright:
    # there the bound is absolute
    bound = np.maximum(2.0 ** -24 * av, 2.0 ** -133)
    assert np.all(err <= bound), (v[err > bound][:5], err[err > bound][:5])


def test_zero_and_signed_zero_split_to_zero():
    for z in (np.float32(0.0), np.float32(-0.0)):
        hi, _, mid, _, lo = split3(np.array([z]))
        assert hi[0] == 0 and mid[0] == 0 and lo[0] == 0


def test_one_part_is_not_enough_and_two_are_not_either():
    """The split needs all three parts for the 2^-24 bound: with hi alone the
    error reaches 2^-8 relative (half an ulp of 8 significant bits), with
    hi + mid 2^-16 (so a kernel that dropped a part would show in the hc_mix
    criterion's fp32 term)."""
    v = samples(np.random.default_rng(13), n=20_000)
    v = v[np.abs(v) > 2.0 ** -100]
    hi, _, mid, _, _ = split3(v)
    av = np.abs(v.astype(np.float64))
    e1 = np.abs(hi.astype(np.float64) - v) / av
    e2 = np.abs(hi.astype(np.float64) + mid.astype(np.float64) - v) / av
    assert e1.max() > 2.0 ** -10 and e2.max() > 2.0 ** -19
    assert e1.max() <= 2.0 ** -8 and e2.max() <= 2.0 ** -16
