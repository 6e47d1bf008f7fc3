"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test ties one oracle function to something independent of it: the
exhaustive integer identity of the signed nibble split (maplevalley article,
section 2.3), library routines (numpy integer matmul, scipy's Jensen-Shannon
distance, torch fp64 softmax / scaled_dot_product_attention), closed forms
derived by hand for degenerate inputs, and brute-force subset enumeration
for the gamma-coverage rule (FAST-Prefill article, section 3.1).
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.spatial.distance import jensenshannon
from scipy.special import softmax as sp_softmax

from dynamic_block_sparse_last_b200 import synth
from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(S, Hq, Hkv, d, b, seed, int8=False, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(Hq, S, d, generator=g) * scale).to(torch.bfloat16)
    k = (torch.randn(Hkv, S, d, generator=g) * scale).to(torch.bfloat16)
    v = torch.randn(Hkv, S, d, generator=g).to(torch.bfloat16)
    if not int8:
        return orc.OracleProblem(q, k, v, b), (q, k, v, None, None, None, None)
    q8 = torch.randint(-127, 128, (Hq, S, d), generator=g, dtype=torch.int8)
    k8 = torch.randint(-127, 128, (Hkv, S, d), generator=g, dtype=torch.int8)
    qs = torch.rand(Hq, generator=g) * 0.05 + 0.01
    ks = torch.rand(Hkv, generator=g) * 0.05 + 0.01
    return (orc.OracleProblem(q, k, v, b, q8=q8, k8=k8, q_scale=qs, k_scale=ks),
            (q, k, v, q8, k8, qs, ks))


# ---------------------------------------------------------------- int8 arithmetic

def test_nibble_identity_exhaustive():
    """a*b == aL*bL + (aH*bL + aL*bH)*16 + aH*bH*256 for every signed int8 pair."""
    L = orc.lib()
    for a in range(-128, 128):
        got = [L.orc_nibble_mul(a, bb) for bb in range(-128, 128)]
        assert got == [a * bb for bb in range(-128, 128)], a


def test_int_score_tile_matches_integer_matmul():
    P, (q, k, v, q8, k8, qs, ks) = rand_problem(S=256, Hq=4, Hkv=2, d=128, b=128, seed=3, int8=True)
    for h in (0, 3):
        tile = P.qk_int_tile(h, 128, 64, 64, 96)
        ref = (q8[h, 128:192].to(torch.int64) @ k8[h // 2, 64:160].to(torch.int64).T).numpy()
        assert np.array_equal(tile.astype(np.int64), ref)


def test_int8_logit_bound_fits_int32_and_fp64():
    # |sum| <= 127*128*128 < 2^31 and < 2^53: the oracle's integer sums are exact.
    assert 127 * 128 * 128 < 2 ** 31


# ---------------------------------------------------------------- Jensen-Shannon

def test_jsd_matches_scipy():
    rng = np.random.default_rng(0)
    for n in (2, 7, 64, 1024):
        p = rng.random(n); p /= p.sum()
        q = rng.random(n) ** 3; q /= q.sum()
        ref = jensenshannon(p, q) ** 2          # natural log, squared distance = divergence
        assert abs(orc.jsd(p, q) - ref) < 1e-12
        assert abs(orc.jsd(p, q) - orc.jsd(q, p)) < 1e-15


def test_jsd_special_values():
    p = np.array([0.2, 0.3, 0.5])
    assert orc.jsd(p, p) == 0.0
    assert abs(orc.jsd([1.0, 0.0], [0.0, 1.0]) - math.log(2.0)) < 1e-15
    # Worked by hand: p = (1/2, 1/2), q = (1, 0), m = (3/4, 1/4):
    # JSD = 1/2 [1/2 ln(2/3) + 1/2 ln 2] + 1/2 ln(4/3).
    hand = 0.5 * (0.5 * math.log(0.5 / 0.75) + 0.5 * math.log(0.5 / 0.25)) + 0.5 * math.log(1.0 / 0.75)
    assert abs(orc.jsd([0.5, 0.5], [1.0, 0.0]) - hand) < 1e-15
    rng = np.random.default_rng(1)
    for _ in range(20):
        a = rng.random(16); a /= a.sum()
        b = rng.random(16) ** 4; b /= b.sum()
        assert 0.0 <= orc.jsd(a, b) <= math.log(2.0) + 1e-15


# ---------------------------------------------------------------- selection

def brute_min_cover(w, r, gamma):
    others = [c for c in range(r)]
    for k in range(0, r + 1):
        best = None
        for comb in itertools.combinations(others, k):
            cov = w[r] + sum(w[c] for c in comb)
            if cov >= gamma:
                best = comb if best is None else best
                break
        if best is not None:
            return k + 1
    return r + 1


@pytest.mark.parametrize("seed", range(12))
def test_selection_minimal_by_brute_force(seed):
    rng = np.random.default_rng(seed)
    r = int(rng.integers(0, 11))
    w = rng.random(r + 1) ** float(rng.integers(1, 6))
    w /= w.sum()
    for gamma in (0.3, 0.5, 0.8, 0.9, 0.95, 0.999):
        sel, info = orc.select(w, r, gamma)
        assert r in sel
        assert list(sel) == sorted(set(sel.tolist()))
        cov = w[sel].sum()
        assert cov >= gamma - 1e-12 or len(sel) == r + 1
        assert len(sel) == brute_min_cover(w, r, gamma)
        # The kept non-diagonal blocks are the highest-scoring ones.
        rest = [c for c in range(r) if c not in sel]
        kept = [c for c in sel if c != r]
        if kept and rest:
            assert min(w[kept]) >= max(w[rest])


def test_selection_gamma_one_keeps_every_causal_block():
    w = np.full(9, 1.0 / 9)
    sel, _ = orc.select(w, 8, 1.0)
    assert list(sel) == list(range(9))


def test_selection_diagonal_alone_when_it_covers():
    w = np.array([0.05, 0.05, 0.9])
    sel, info = orc.select(w, 2, 0.9)
    assert list(sel) == [2] and info[0] == -1.0


def test_selection_ties_break_by_lower_index():
    w = np.array([0.2, 0.2, 0.2, 0.2, 0.2])
    sel, _ = orc.select(w, 4, 0.6)
    assert list(sel) == [0, 1, 4]


# ---------------------------------------------------------------- block scores

def test_vs_scores_hand_example():
    ex = json.load(open(os.path.join(GOLDEN, "vs_scores_example.json")))
    w = orc.row_scores(orc.VS, ex["r"], ex["vhat"], ex["shat"], np.zeros(4), np.zeros((len(ex["vhat"]), 4)))
    assert np.allclose(w, ex["expected"], atol=1e-15)


def test_qa_scores_match_scipy_softmax():
    rng = np.random.default_rng(5)
    kbar = rng.normal(size=(12, 16))
    qbar = rng.normal(size=16) * 3
    for r in (0, 5, 11):
        w = orc.row_scores(orc.QA, r, np.zeros(12), np.zeros(12), qbar, kbar)
        ref = sp_softmax(kbar[: r + 1] @ qbar / math.sqrt(16))
        assert np.allclose(w, ref, rtol=1e-13, atol=1e-16)
    pe = orc.pest(qbar, kbar)
    assert np.allclose(pe, sp_softmax(kbar @ qbar / 4.0), rtol=1e-13)


def test_qa_scores_finite_for_large_logits():
    """Block logits near 800 (exp overflows float64 past ~709) that differ by
    a few units: the scores are the softmax of the differences, finite."""
    x = np.array([0.0, 1.0, -2.0, 0.5, 3.0, -1.0])
    kbar = np.zeros((6, 4))
    kbar[:, 0] = 40.0
    kbar[:, 1] = x
    qbar = np.array([40.0, 1.0, 0.0, 0.0])  # logits (1600 + x_c) / 2
    w = orc.row_scores(orc.QA, 5, np.zeros(6), np.zeros(6), qbar, kbar)
    assert np.all(np.isfinite(w))
    assert np.allclose(w, sp_softmax(x / 2.0), rtol=1e-12, atol=0)
    pe = orc.pest(qbar, kbar)
    assert np.all(np.isfinite(pe)) and np.allclose(pe, sp_softmax(x / 2.0), rtol=1e-12, atol=0)


# ---------------------------------------------------------------- last-block statistics

@pytest.mark.parametrize("S,b,d,int8", [(16, 4, 8, False), (24, 8, 16, False), (32, 8, 8, True),
                                         (18, 4, 8, False), (29, 8, 16, True)])
def test_last_block_stats_against_full_attention_matrix(S, b, d, int8):
    """vhat / shat from the full causal softmax matrix (torch fp64), pooled
    by block columns and by torch.diagonal sums; S not a multiple of b gives a
    partial last block whose rows are averaged."""
    P, (q, k, v, q8, k8, qs, ks) = rand_problem(S, 2, 1, d, b, seed=S + b, int8=int8, scale=2.0)
    n = -(-S // b)
    rows_last = S - (n - 1) * b
    for h in range(2):
        if int8:
            logits = (q8[h].double() @ k8[0].double().T) * (float(qs[h]) * float(ks[0])) / math.sqrt(d)
        else:
            logits = (q[h].double() @ k[0].double().T) / math.sqrt(d)
        mask = torch.ones(S, S, dtype=torch.bool).tril()
        A = torch.softmax(logits.masked_fill(~mask, float("-inf")), dim=-1)
        last = A[(n - 1) * b:]
        vref = torch.stack([last[:, c * b:(c + 1) * b].sum() for c in range(n)]) / rows_last
        sref = torch.zeros(n, dtype=torch.float64)
        for delta in range(S):
            diag = torch.diagonal(A, offset=-delta)            # entries (p, p - delta)
            rows = torch.arange(delta, S)
            sref[delta // b] += diag[rows >= (n - 1) * b].sum() / rows_last
        vh, sh, err = P.last_block_stats(h)
        assert err < 1e-12
        assert np.allclose(vh, vref.numpy(), atol=1e-14)
        assert np.allclose(sh, sref.numpy(), atol=1e-14)
        assert abs(vh.sum() - 1) < 1e-13 and abs(sh.sum() - 1) < 1e-13


def test_uniform_attention_closed_form():
    """Q = 0 makes every causal row uniform: A_pj = 1/(p+1).  Then
    vhat[c] = (1/b) sum_i |block c and [0, p_i]| / (p_i + 1) and
    shat[o] = (1/b) sum_i |{delta in [ob, (o+1)b) : delta <= p_i}| / (p_i + 1)."""
    S, b, d = 24, 6, 8
    n = S // b
    q = torch.zeros(1, S, d, dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(9)
    k = torch.randn(1, S, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, S, d, generator=g).to(torch.bfloat16)
    P = orc.OracleProblem(q, k, v, b)
    vh, sh, _ = P.last_block_stats(0)
    vf = [Fraction(0)] * n
    sf = [Fraction(0)] * n
    for i in range(b):
        p = (n - 1) * b + i
        for c in range(n):
            vf[c] += Fraction(max(0, min(p, (c + 1) * b - 1) - c * b + 1), (p + 1) * b)
            sf[c] += Fraction(max(0, min(p, (c + 1) * b - 1) - c * b + 1), (p + 1) * b)
    assert np.allclose(vh, [float(x) for x in vf], atol=1e-15)
    assert np.allclose(sh, [float(x) for x in sf], atol=1e-15)
    out = P.build_index_head(0, 0.9, 0.1)
    assert np.allclose(out["pest"], np.full(n, 1.0 / n), atol=1e-15)   # qbar = 0 -> uniform


def test_single_block_is_query_aware_with_zero_divergence():
    P, _ = rand_problem(S=16, Hq=1, Hkv=1, d=8, b=16, seed=4)
    out = P.build_index_head(0, 0.9, 0.1)
    assert abs(out["jsd"]) < 1e-15 and out["pattern"] == orc.QA
    assert [list(r) for r in out["rows"]] == [[0]]
    out = P.build_index_head(0, 0.9, -1.0)            # jsd < -1 never holds
    assert out["pattern"] == orc.VS


def test_block_means_of_a_partial_last_block():
    P, (q, k, *_r) = rand_problem(S=40, Hq=1, Hkv=1, d=8, b=16, seed=5)
    km = P.block_means("k", 0)
    assert km.shape == (3, 8)
    assert np.allclose(km[2], k[0, 32:40].double().mean(0).numpy(), atol=1e-15)
    assert np.allclose(km[0], k[0, 0:16].double().mean(0).numpy(), atol=1e-15)


def test_block_means_match_torch():
    P, (q, k, v, q8, k8, qs, ks) = rand_problem(S=64, Hq=2, Hkv=1, d=16, b=16, seed=2, int8=True)
    qb = P.block_means("q", 1)
    ref = (q8[1].double().reshape(4, 16, 16).sum(1) * float(qs[1])) / 16
    assert np.allclose(qb, ref.numpy(), rtol=1e-15)
    P2, (q, k, *_r) = rand_problem(S=64, Hq=2, Hkv=1, d=16, b=16, seed=2)
    assert np.allclose(P2.block_means("k", 0), k[0].double().reshape(4, 16, 16).mean(1).numpy(), atol=1e-15)


# ---------------------------------------------------------------- attention

def sdpa_ref(q, k, v, h, g, mask=None, int8=None):
    d = q.shape[-1]
    if int8 is not None:
        q8, k8, qs, ks = int8
        logits = (q8[h].double() @ k8[h // g].double().T) * (float(qs[h]) * float(ks[h // g])) / math.sqrt(d)
    else:
        logits = (q[h].double() @ k[h // g].double().T) / math.sqrt(d)
    S = q.shape[1]
    causal = torch.ones(S, S, dtype=torch.bool).tril()
    m = causal if mask is None else (causal & mask)
    A = torch.softmax(logits.masked_fill(~m, float("-inf")), dim=-1)
    return A @ v[h // g].double()


@pytest.mark.parametrize("int8,S", [(False, 48), (True, 48), (False, 45), (True, 51)])
def test_gamma_one_equals_dense_causal_attention(int8, S):
    b, d = 8, 16
    P, (q, k, v, q8, k8, qs, ks) = rand_problem(S, 4, 2, d, b, seed=11, int8=int8, scale=1.5)
    for h in range(4):
        idx = P.build_index_head(h, 1.0, 0.1)
        assert all(list(r) == list(range(i + 1)) for i, r in enumerate(idx["rows"]))
        nb = -(-S // b)
        got = np.concatenate([P.attn_rows(h, r * b, min((r + 1) * b, S), idx["rows"][r]) for r in range(nb)])
        ref = sdpa_ref(q, k, v, h, 2, int8=(q8, k8, qs, ks) if int8 else None)
        assert np.allclose(got, ref.numpy(), atol=1e-12)
    if not int8:
        sd = torch.nn.functional.scaled_dot_product_attention(
            q.double()[None], k.double().repeat_interleave(2, 0)[None], v.double().repeat_interleave(2, 0)[None],
            is_causal=True)[0]
        nb = -(-S // b)
        got = np.concatenate([P.attn_rows(1, r * b, min((r + 1) * b, S), list(range(r + 1))) for r in range(nb)])
        assert np.allclose(got, sd[1].numpy(), atol=1e-12)


def test_sparse_attention_matches_block_masked_softmax():
    S, b, d = 64, 8, 16
    n = S // b
    P, (q, k, v, *_r) = rand_problem(S, 2, 1, d, b, seed=21)
    rng = np.random.default_rng(2)
    for h in range(2):
        lists = [sorted(set(rng.choice(r + 1, size=int(rng.integers(1, r + 2)), replace=False).tolist()) | {r})
                 for r in range(n)]
        mask = torch.zeros(S, S, dtype=torch.bool)
        for r, blocks in enumerate(lists):
            for c in blocks:
                mask[r * b:(r + 1) * b, c * b:(c + 1) * b] = True
        ref = sdpa_ref(q, k, v, h, 2, mask=mask)
        got = np.concatenate([P.attn_rows(h, r * b, (r + 1) * b, lists[r]) for r in range(n)])
        assert np.allclose(got, ref.numpy(), atol=1e-12)


def test_index_invariants_on_planted_inputs():
    from dynamic_block_sparse_last_b200 import synth
    w = synth.Workload("t", S=1024, Hq=4, Hkv=2, b=128, seed=0, kinds=["vs", "qa", "vs", "qa"])
    x = synth.make_inputs(w)
    P = orc.OracleProblem(x["q"], x["k"], x["v"], w.b)
    for h in range(4):
        out = P.build_index_head(h, w.gamma, w.tau)
        assert out["rowsum_err"] < 1e-12
        assert abs(out["vhat"].sum() - 1) < 1e-12 and abs(out["shat"].sum() - 1) < 1e-12
        assert abs(out["pest"].sum() - 1) < 1e-12
        for r, row in enumerate(out["rows"]):
            assert r in row
            sc = out["scores"][r]
            assert abs(sc.sum() - 1) < 1e-12
            assert sc[row].sum() >= w.gamma - 1e-12
            others = [c for c in row if c != r]
            if others:                                  # minimal: dropping the weakest falls short
                assert sc[row].sum() - sc[others].min() < w.gamma


def test_golden_tiny_index_regression():
    """Regression against the stored output of tests/golden/make_golden.py."""
    from dynamic_block_sparse_last_b200 import synth
    gold = json.load(open(os.path.join(GOLDEN, "tiny_index.json")))
    w = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(w)
    P = orc.OracleProblem(x["q"], x["k"], x["v"], w.b)
    for h, gh in enumerate(gold["heads"]):
        out = P.build_index_head(h, w.gamma, w.tau)
        assert out["pattern"] == gh["pattern"]
        assert abs(out["jsd"] - gh["jsd"]) < 1e-12
        assert np.allclose(out["vhat"], gh["vhat"], atol=1e-14)
        assert [list(map(int, r)) for r in out["rows"]] == gh["rows"]


# ---------------------------------------------------------------------------
# Rotary embedding + block pooling (the projection epilogue, [FP] 1.1 / 2.1)
# ---------------------------------------------------------------------------

def _bf16_grid(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_rope_exact_turns():
    """cos = 0, sin = 1 is a quarter turn (x_i -> -x_{i+d/2}, x_{i+d/2} -> x_i);
    cos = -1, sin = 0 a half turn; both exact in bf16."""
    x = _bf16_grid((2, 5, 128), 1)
    xf = x.double().numpy()
    zero, one = np.zeros((5, 64)), np.ones((5, 64))
    out, _ = orc.rope_pool(x, zero, one, 4)
    assert np.array_equal(out[..., :64], -xf[..., 64:]) and np.array_equal(out[..., 64:], xf[..., :64])
    out, _ = orc.rope_pool(x, -one, zero, 4)
    assert np.array_equal(out, -xf)


def test_rope_equals_complex_rotation():
    """The pair (x_i, x_{i+d/2}) rotates as the complex number x_i + i x_{i+d/2}
    multiplied by cos + i sin (numpy complex128), then rounded to bf16."""
    w = synth.Workload("rope", S=200, Hq=2, Hkv=1, b=64, seed=3)
    x = synth.make_prerope_inputs(w)
    out, _ = orc.rope_pool(x["q_in"], x["cos"], x["sin"], 64)
    xf = x["q_in"].double().numpy()
    z = (xf[..., :64] + 1j * xf[..., 64:]) * (x["cos"].double().numpy() + 1j * x["sin"].double().numpy())[None]
    ref = torch.from_numpy(np.concatenate([z.real, z.imag], -1)).to(torch.bfloat16).double().numpy()
    diff = np.abs(out - ref)
    assert (diff == 0).mean() > 0.999
    assert np.all(diff <= 2.0 ** -7 * np.abs(ref) + 1e-30)


def test_rope_relative_position_property():
    """<R_p q, R_j k> depends on p - j only: the same q, k placed at (p, j) and
    (p + t, j + t) give the same logit up to bf16 rounding of the outputs."""
    S = 256
    cos, sin = synth.rope_tables(S, 128)
    q0 = _bf16_grid((128,), 5).double()
    k0 = _bf16_grid((128,), 6).double()
    x = torch.zeros(2, S, 128, dtype=torch.float64)
    for p in (10, 40, 200):
        x[0, p] = q0
    for j in (3, 33, 193):
        x[1, j] = k0
    out, _ = orc.rope_pool(x, cos, sin, 64)
    dots = [float(out[0, p] @ out[1, j]) for p, j in ((10, 3), (40, 33), (200, 193))]
    scale = float(q0.norm() * k0.norm())
    assert max(dots) - min(dots) <= 2e-2 * scale
    assert abs(float(out[0, 10] @ out[1, 3]) - float(out[0, 10] @ out[1, 33])) > 1e-3 * scale  # not trivially equal


def test_rope_pair_norms_and_block_means():
    """Each rotated pair keeps its length (to bf16 rounding); the means are the
    column means of the rounded rows over each block, the last one partial."""
    w = synth.Workload("rope2", S=300, Hq=3, Hkv=1, b=128, seed=4)
    x = synth.make_prerope_inputs(w)
    out, means = orc.rope_pool(x["q_in"], x["cos"], x["sin"], 128)
    xf = x["q_in"].double().numpy()
    n_in = np.hypot(xf[..., :64], xf[..., 64:])
    n_out = np.hypot(out[..., :64], out[..., 64:])
    assert np.all(np.abs(n_out - n_in) <= 2.0 ** -7 * n_in + 1e-12)
    assert means.shape == (3, 3, 128)
    for c, (lo, hi) in enumerate(((0, 128), (128, 256), (256, 300))):
        assert np.allclose(means[:, c], out[:, lo:hi].mean(1), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- index wiring

def _wiring_problem(seed):
    """S = 48, b = 8, d = 16, Hq = 4, Hkv = 2: Q and K carry a per-block offset
    so the block means q-bar_r, k-bar_c differ from block to block (a q-bar of
    the wrong block, or of the wrong head, changes the result)."""
    S, b, d, Hq, Hkv = 48, 8, 16, 4, 2
    n = S // b
    g = torch.Generator().manual_seed(seed)
    qoff = torch.randn(Hq, n, 1, d, generator=g) * 1.5
    koff = torch.randn(Hkv, n, 1, d, generator=g) * 1.5
    q = (torch.randn(Hq, n, b, d, generator=g) + qoff).reshape(Hq, S, d).to(torch.bfloat16)
    k = (torch.randn(Hkv, n, b, d, generator=g) + koff).reshape(Hkv, S, d).to(torch.bfloat16)
    v = torch.randn(Hkv, S, d, generator=g).to(torch.bfloat16)
    return orc.OracleProblem(q, k, v, b), q, k, S, b, d, Hq, Hkv


def _index_by_hand(q, k, h, S, b, d, g):
    """Every quantity of one head's index, computed here in torch fp64 from the
    definitions (FAST-Prefill article 1.2 and 2.1; maplevalley article 1.1
    steps 1-3) without the oracle."""
    n = S // b
    kv = h // g
    qh, kh = q[h].double(), k[kv].double()
    logits = (qh @ kh.T) / math.sqrt(d)
    mask = torch.ones(S, S, dtype=torch.bool).tril()
    A = torch.softmax(logits.masked_fill(~mask, float("-inf")), dim=-1)
    last = A[(n - 1) * b:]
    vhat = last.reshape(b, n, b).sum(dim=(0, 2)) / b            # column blocks of the last block's rows
    pos = torch.arange(S)
    p = pos[(n - 1) * b:, None]
    off = (p - pos[None, :]).clamp(min=0) // b                  # offset block of (p, j), causal part only
    shat = torch.zeros(n, dtype=torch.float64).index_add_(0, off.flatten(), last.flatten()) / b
    qbar = qh.reshape(n, b, d).mean(1)
    kbar = kh.reshape(n, b, d).mean(1)
    pest = torch.softmax(kbar @ qbar[n - 1] / math.sqrt(d), 0)
    jsd = float(jensenshannon(vhat.numpy(), pest.numpy())) ** 2
    qa = [torch.softmax(kbar[: r + 1] @ qbar[r] / math.sqrt(d), 0).numpy() for r in range(n)]
    vs = []
    for r in range(n):
        wr = torch.stack([vhat[c] + shat[r - c] for c in range(r + 1)])
        vs.append((wr / wr.sum()).numpy())
    return vhat.numpy(), shat.numpy(), pest.numpy(), jsd, qa, vs


@pytest.mark.parametrize("seed", [31, 32])
def test_index_head_wiring_matches_hand_computation(seed):
    """orc_build_index_head feeds the right operands to each step: P_est from
    the LAST block's q-bar, the JSD between v-hat and P_est, query-aware row r
    scored with q-bar_r against k-bar of the head's own KV head, vertical-slash
    row r from v-hat[c] + s-hat[r-c]; then the pattern rule and the selection
    (diagonal forced, score descending, minimal count reaching gamma)."""
    P, q, k, S, b, d, Hq, Hkv = _wiring_problem(seed)
    n, g = S // b, Hq // Hkv
    gamma = 0.8
    for h in range(Hq):
        vhat, shat, pest, jsd, qa, vs = _index_by_hand(q, k, h, S, b, d, g)
        assert not np.allclose(vhat, shat, atol=1e-3)           # the two statistics really differ
        for tau, pat in ((jsd * 1.01, orc.QA), (jsd * 0.99, orc.VS)):
            out = P.build_index_head(h, gamma, tau)
            assert np.allclose(out["vhat"], vhat, atol=1e-14)
            assert np.allclose(out["shat"], shat, atol=1e-14)
            assert np.allclose(out["pest"], pest, rtol=1e-12, atol=1e-15)
            assert abs(out["jsd"] - jsd) < 1e-12
            assert out["pattern"] == pat
            ref = qa if pat == orc.QA else vs
            for r in range(n):
                assert np.allclose(out["scores"][r], ref[r], rtol=1e-12, atol=1e-15), (h, pat, r)
                row = list(out["rows"][r])
                assert r in row
                assert len(row) == brute_min_cover(ref[r], r, gamma)
                rest = [c for c in range(r) if c not in row]
                kept = [c for c in row if c != r]
                if kept and rest:
                    assert min(ref[r][kept]) >= max(ref[r][rest])
        # Forcing a pattern switches only the row scores, not the statistics.
        for force, ref in ((orc.QA, qa), (orc.VS, vs)):
            out = P.build_index_head(h, gamma, 0.1, force_pattern=force)
            assert out["pattern"] == force and abs(out["jsd"] - jsd) < 1e-12
            for r in range(n):
                assert np.allclose(out["scores"][r], ref[r], rtol=1e-12, atol=1e-15)


def test_index_wiring_inputs_distinguish_the_operands():
    """The wiring pin is only meaningful if its inputs separate the operands a
    mistake could swap in: P_est from the first block's q-bar, or JSD against
    s-hat, or a QA row from the last block's q-bar, differ measurably."""
    P, q, k, S, b, d, Hq, Hkv = _wiring_problem(31)
    n, g = S // b, Hq // Hkv
    for h in range(Hq):
        vhat, shat, pest, jsd, qa, vs = _index_by_hand(q, k, h, S, b, d, g)
        qh, kh = q[h].double(), k[h // g].double()
        qbar, kbar = qh.reshape(n, b, d).mean(1), kh.reshape(n, b, d).mean(1)
        first = torch.softmax(kbar @ qbar[0] / math.sqrt(d), 0).numpy()
        assert np.abs(first - pest).max() > 1e-3
        assert abs(float(jensenshannon(shat, pest)) ** 2 - jsd) > 1e-4
        wrong = torch.softmax(kbar[:3] @ qbar[n - 1] / math.sqrt(d), 0).numpy()
        assert np.abs(wrong - qa[2]).max() > 1e-3



# ---------------------------------------------------------------- head-pattern sharing, adaptive block size

def test_share_classes_follow_jsd_between_representatives():
    """Greedy classes in head order: a head joins the earliest earlier
    representative whose vhat is within JSD < eps (scipy's Jensen-Shannon
    distance squared), else it represents its own class."""
    base = np.array([0.4, 0.3, 0.2, 0.1])
    near = np.array([0.38, 0.32, 0.2, 0.1])                  # close to base
    mid = np.array([0.25, 0.25, 0.25, 0.25])
    far = np.array([0.01, 0.01, 0.08, 0.9])
    d_bn = jensenshannon(base, near) ** 2
    d_bm = jensenshannon(base, mid) ** 2
    d_nm = jensenshannon(near, mid) ** 2
    assert d_bn < 1e-3 < d_nm < d_bm
    eps = 0.5 * (d_nm + d_bm) if d_nm < d_bm else None
    # mid is within eps of near (a member, not a representative) but not of base: own class
    cls = orc.share_classes(np.stack([base, near, mid, far]), eps)
    assert list(cls) == [0, 0, 2, 3]
    # a larger eps lets mid join base's class; far still stands alone
    cls = orc.share_classes(np.stack([base, near, mid, far]), d_bm * 1.01)
    assert list(cls) == [0, 0, 0, 3]
    # eps = 0 keeps every head alone (JSD >= 0 is never < 0)
    assert list(orc.share_classes(np.stack([base, base, base]), 0.0)) == [0, 1, 2]
    # identical heads always share for eps > 0 (JSD(P, P) = 0)
    assert list(orc.share_classes(np.stack([far, base, far]), 1e-12)) == [0, 1, 0]


def test_union_lists_is_the_set_union():
    rng = np.random.default_rng(3)
    for r in (0, 5, 40):
        lists = [sorted(set(rng.choice(r + 1, size=int(rng.integers(1, r + 2)), replace=False).tolist()) | {r})
                 for _ in range(3)]
        got = orc.union_lists(lists, r)
        assert list(got) == sorted(set().union(*map(set, lists)))


def test_cover_count_by_sorting():
    rng = np.random.default_rng(4)
    for n in (1, 7, 100, 1024):
        v = rng.random(n) ** 3
        v /= v.sum()
        for gamma in (0.3, 0.8, 0.9, 0.99):
            csum = np.cumsum(np.sort(v)[::-1])
            want = int(np.searchsorted(csum, gamma) + 1)   # first prefix with sum >= gamma
            want = min(want, n)
            assert orc.cover_count(v, gamma) == want, (n, gamma)
    assert orc.cover_count(np.full(4, 0.25), 1.0) == 4


def test_block_size_rule_regimes():
    """rho = mean over heads of (blocks covering gamma of vhat) / n: concentrated
    attention -> 64 (if S/64 <= 1024 blocks), diffuse -> 256, otherwise 128."""
    n = 100
    conc = np.zeros(n); conc[-1] = 0.95; conc[:-1] = 0.05 / (n - 1)        # 1 block covers 0.9
    flat = np.full(n, 1.0 / n)                                            # 90 blocks for 0.9
    assert orc.choose_block_size(np.stack([conc, conc]), 12800, 0.9) == (64, 0.01)
    b, rho = orc.choose_block_size(np.stack([flat, flat]), 12800, 0.9)
    assert b == 256 and abs(rho - 0.90) < 1e-12
    b, rho = orc.choose_block_size(np.stack([conc, flat]), 12800, 0.9)
    assert b == 128 and abs(rho - 0.455) < 1e-12
    # concentrated, but S = 131072 would need 2048 blocks of 64: stays at 128
    assert orc.choose_block_size(np.stack([conc, conc]), 131072, 0.9)[0] == 128
