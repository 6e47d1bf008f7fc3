"""The attention softmax's reference rule, modelled in numpy and checked
against exact softmax on adversarial rows.

The attention kernel takes each chunk's exponentials against the row's
current reference m (log2 units), P = bf16(2^(x - m)), and adds the rounded
P into the row sum.  Only when the chunk's row sum exceeds REF_SUM (or the row
has no reference yet) does it move the reference to the chunk's row max plus
REF_HEADROOM, rescale O and the row sum by 2^(m_old - m_new) and recompute
the chunk.  The model below applies the same rule in fp32 with bf16 P and
checks: every P the rule keeps is at most REF_SUM, nothing overflows, and the
output equals exact softmax(x) V in fp64 to bf16-level accuracy.  The rows
are the cases the rule must survive: rising maxima, jumps of hundreds of
log2 units, masked prefixes, a single visible key, flat rows."""
import numpy as np
import torch

REF_SUM, REF_HEADROOM = 256.0, 64.0  # the attention kernel's kRefSum and kRefHeadroom
CHUNK = 128


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def model_row(x, v):
    """x: [L] scores in log2 units (float32, -inf = masked), v: [L, d].
    Returns (output, largest kept P, number of reference moves)."""
    m = -np.inf
    o = np.zeros(v.shape[1], dtype=np.float32)
    l = np.float32(0.0)
    pmax, moves = 0.0, 0
    for c0 in range(0, len(x), CHUNK):
        xs = x[c0:c0 + CHUNK].astype(np.float32)
        vs = v[c0:c0 + CHUNK]

        def chunk_p(ref):
            with np.errstate(over="ignore"):
                p = np.exp2((xs - np.float32(0.0 if ref == -np.inf else ref)).astype(np.float32))
            return bf16(p)

        p = chunk_p(m)
        rs = np.float32(p.astype(np.float32).sum(dtype=np.float32))
        if not rs <= REF_SUM or m == -np.inf:
            mx = float(np.max(xs))
            m_new = max(m, mx + REF_HEADROOM) if mx != -np.inf else m
            if m_new > m:
                alpha = np.float32(0.0) if m == -np.inf else np.float32(np.exp2(np.float32(m - m_new)))
                o *= alpha
                l *= alpha
                m = m_new
                moves += 1
            p = chunk_p(m)
            rs = np.float32(p.astype(np.float32).sum(dtype=np.float32))
        pmax = max(pmax, float(p.max()))
        o = (o + (p[:, None].astype(np.float32) * vs).sum(0, dtype=np.float32)).astype(np.float32)
        l = np.float32(l + rs)
    return o / l, pmax, moves


def exact_row(x, v):
    xx = x.astype(np.float64)
    w = np.exp2(xx - xx[np.isfinite(xx)].max())
    w[~np.isfinite(xx)] = 0.0
    return (w[:, None] * v.astype(np.float64)).sum(0) / w.sum()


def rows():
    rng = np.random.default_rng(7)
    L = 1024
    base = rng.standard_normal(L) * 2.0
    out = {
        "normal": base,
        "rising": base + np.linspace(0.0, 150.0, L),           # the max keeps growing
        "jump_up": np.where(np.arange(L) < 600, base, base + 200.0),  # far past the headroom
        "jump_down": np.where(np.arange(L) < 300, base + 90.0, base),
        "masked_prefix": np.where(np.arange(L) < 400, -np.inf, base),
        "single_key": np.where(np.arange(L) == 777, 3.0, -np.inf),
        "flat": np.zeros(L),
        "spiky": base + (rng.random(L) < 0.01) * 60.0,
    }
    return {k: v.astype(np.float32) for k, v in out.items()}


def test_rule_bounds_p_and_matches_exact_softmax():
    rng = np.random.default_rng(8)
    v = bf16(rng.standard_normal((1024, 16)))
    for name, x in rows().items():
        got, pmax, moves = model_row(x, v)
        ref = exact_row(x, v)
        assert np.all(np.isfinite(got)), name
        assert pmax <= REF_SUM, (name, pmax)
        # bf16 P: each weight within 2^-9 relative, so the output within ~2^-8 of max|v|
        assert np.max(np.abs(got - ref)) <= 2.0 ** -8 * np.abs(v).max(), (name, np.max(np.abs(got - ref)))
        if name in ("rising", "jump_up"):
            assert moves >= 2, (name, moves)


def test_headroom_keeps_ordinary_rows_from_moving_after_the_first_chunk():
    """With the headroom, a row whose later scores stay within ~64 log2 units
    of the first chunk's maximum never moves its reference again."""
    rng = np.random.default_rng(9)
    v = bf16(rng.standard_normal((2048, 8)))
    x = (rng.standard_normal(2048) * 3.0 + np.linspace(0.0, 40.0, 2048)).astype(np.float32)
    _, _, moves = model_row(x, v)
    assert moves == 1
