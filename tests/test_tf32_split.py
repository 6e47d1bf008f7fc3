"""Numerics of the tf32 split used by the tensor-core q-bar . k-bar logits.

k_split_tf32 stores every block mean x as x_hi = tf32(x) and x_lo = tf32(x - x_hi)
(round to nearest, ties away from zero, at 10 explicit mantissa bits), and
k_qa_logits accumulates hi.hi + hi.lo + lo.hi per product in fp32.  Here the
split is emulated bit for bit in numpy and checked against exact (fp64)
products: every product within 2^-20 relative (the dropped lo.lo term and the
two roundings are each at most 2^-22), and 128-term dot products at fp32-class
accuracy, against the 1e-4 near-cut tolerance the logits feed."""
import numpy as np


def tf32_rna(x):
    """fp32 -> tf32 (kept in fp32 containers): round half away from zero at bit 13."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x1000)) & np.uint32(0xFFFFE000)).view(np.float32)


def split(x):
    hi = tf32_rna(x)
    lo = tf32_rna(np.asarray(x, dtype=np.float32) - hi)  # the difference is exact in fp32
    return hi, lo


def test_tf32_rounding_keeps_ten_mantissa_bits_and_rounds_half_away():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -10)
    assert tf32_rna(one + ulp * np.float32(0.5)) == one + ulp          # tie: away from zero
    assert tf32_rna(-(one + ulp * np.float32(0.5))) == -(one + ulp)
    assert tf32_rna(one + ulp * np.float32(0.49)) == one
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    assert np.all((tf32_rna(x).view(np.uint32) & np.uint32(0x1FFF)) == 0)
    rel = np.abs(tf32_rna(x).astype(np.float64) - x) / np.abs(x.astype(np.float64))
    assert rel.max() <= 2.0 ** -11


def test_three_product_split_is_within_two_to_the_minus_20_per_product():
    rng = np.random.default_rng(1)
    # block means span several binades (|q-bar| up to ~3, |k-bar| up to ~3, some tiny)
    a = (rng.standard_normal(200000) * np.exp2(rng.integers(-8, 3, 200000))).astype(np.float32)
    b = (rng.standard_normal(200000) * np.exp2(rng.integers(-8, 3, 200000))).astype(np.float32)
    ah, al = split(a)
    bh, bl = split(b)
    exact = a.astype(np.float64) * b.astype(np.float64)
    approx = (ah.astype(np.float64) * bh + ah.astype(np.float64) * bl + al.astype(np.float64) * bh)
    nz = exact != 0
    rel = np.abs(approx[nz] - exact[nz]) / np.abs(exact[nz])
    assert rel.max() <= 2.0 ** -20
    # one product alone (plain tf32) is far coarser: the split is what makes the logits fp32-class
    plain = np.abs(ah.astype(np.float64) * bh - exact)[nz] / np.abs(exact[nz])
    assert plain.max() > 2.0 ** -12


def test_split_dot_products_are_fp32_class():
    """128-term dot products (d = 128) of split operands with fp32 accumulation,
    as the tensor cores form them, against fp64: relative to the sum of |terms|
    the error stays at fp32 rounding level, far inside the logits' 1e-4 near-cut
    tolerance (logits up to ~45)."""
    rng = np.random.default_rng(2)
    q = (rng.standard_normal((256, 128)) * 0.5).astype(np.float32)
    k = (rng.standard_normal((256, 128)) * 0.5).astype(np.float32)
    qh, ql = split(q)
    kh, kl = split(k)
    acc = np.zeros((256, 256), dtype=np.float32)
    for part_q, part_k in ((qh, kh), (qh, kl), (ql, kh)):
        for j in range(128):  # fp32 accumulation, one term at a time
            acc = (acc + np.outer(part_q[:, j], part_k[:, j]).astype(np.float32)).astype(np.float32)
    exact = q.astype(np.float64) @ k.astype(np.float64).T
    scale = np.abs(q.astype(np.float64)) @ np.abs(k.astype(np.float64)).T
    err = np.abs(acc.astype(np.float64) - exact) / scale
    assert err.max() <= 3 * 128 * 2.0 ** -24
