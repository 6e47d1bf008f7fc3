"""The score kernel's per-row reference and the statistics kernel's combination,
modelled in numpy and checked against the exact pooled softmax.

k_score_last takes each 32-column piece's exponentials against the row's
reference m (which persists across parts), moving it to the piece max plus
SCORE_HEADROOM only when the piece's sum exceeds 2^8 or the row has no
reference yet (then rescaling the part's sums so far), and writes per
(row, part) the reference and the sums lo / hi of its two offset halves.
k_head_stats combines the parts by log-sum-exp: M = max_p m_p,
L = sum_p (lo_p + hi_p) 2^(m_p - M), LO_p = lo_p 2^(m_p - M) / L.  The model
checks that this gives the exact row-normalised part masses whatever the
references are, on rows whose maxima rise, jump and start masked."""
import numpy as np

SCORE_HEADROOM, PIECE_SUM = 64.0, 256.0  # k_score_last's kScoreHeadroom and its 2^8 move bound
PIECE, PART = 32, 128


def partials(x, split):
    """x: [L] scores (log2 units, -inf masked); split(c) -> True if column c is on
    the lo side.  Returns per part (m, lo, hi) in fp32 as the kernel keeps them."""
    m = -np.inf
    out = []
    for p0 in range(0, len(x), PART):
        lo = hi = np.float32(0.0)
        for c0 in range(p0, min(p0 + PART, len(x)), PIECE):
            xs = x[c0:c0 + PIECE].astype(np.float32)
            cols = np.arange(c0, c0 + len(xs))
            is_lo = np.array([split(c) for c in cols])

            def piece(ref):
                with np.errstate(over="ignore"):
                    e = np.exp2((xs - np.float32(ref)).astype(np.float32))
                return np.float32(e[is_lo].sum(dtype=np.float32)), np.float32(e[~is_lo].sum(dtype=np.float32))

            move = m == -np.inf
            if not move:
                pl, ph = piece(m)
                move = not (pl + ph) <= PIECE_SUM
            if move:
                pmx = float(xs.max())
                if pmx == -np.inf:
                    continue
                new = max(m, pmx + SCORE_HEADROOM)
                if new > m:
                    f = np.float32(0.0) if m == -np.inf else np.float32(np.exp2(np.float32(m - new)))
                    lo, hi, m = lo * f, hi * f, new
                pl, ph = piece(m)
            lo, hi = np.float32(lo + pl), np.float32(hi + ph)
        out.append((m, lo, hi))
    return out


def combine(parts):
    """The statistics kernel's combination: per-part row-normalised lo / hi masses."""
    ms = np.array([p[0] for p in parts], dtype=np.float64)
    M = ms[np.isfinite(ms)].max()
    w = np.where(np.isfinite(ms), np.exp2(ms - M), 0.0)
    lo = np.array([p[1] for p in parts], dtype=np.float64) * w
    hi = np.array([p[2] for p in parts], dtype=np.float64) * w
    L = (lo + hi).sum()
    return lo / L, hi / L


def exact(x, split):
    xx = x.astype(np.float64)
    w = np.exp2(xx - xx[np.isfinite(xx)].max())
    w[~np.isfinite(xx)] = 0.0
    w /= w.sum()
    nparts = -(-len(x) // PART)
    lo = np.array([sum(w[c] for c in range(p * PART, min((p + 1) * PART, len(x))) if split(c))
                   for p in range(nparts)])
    hi = np.array([w[p * PART:(p + 1) * PART].sum() for p in range(nparts)]) - lo
    return lo, hi


def test_combined_partials_equal_exact_pooled_masses():
    rng = np.random.default_rng(11)
    L = 1024
    base = rng.standard_normal(L) * 2.0
    rows = {
        "normal": base,
        "rising": base + np.linspace(0.0, 300.0, L),
        "jump": np.where(np.arange(L) < 500, base, base + 250.0),
        "masked_prefix": np.where(np.arange(L) < 300, -np.inf, base),
        "falling": base + np.linspace(120.0, 0.0, L),
    }
    split = lambda c: (c % 7) < 4  # an arbitrary lo / hi assignment, as the offset halves give
    for name, x in rows.items():
        x = x.astype(np.float32)
        got_lo, got_hi = combine(partials(x, split))
        ref_lo, ref_hi = exact(x, split)
        assert np.allclose(got_lo, ref_lo, rtol=1e-5, atol=1e-9), name
        assert np.allclose(got_hi, ref_hi, rtol=1e-5, atol=1e-9), name
        assert abs((got_lo + got_hi).sum() - 1.0) < 1e-6, name
