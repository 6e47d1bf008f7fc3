"""Head-pattern sharing and the adaptive block-size rule (maplevalley
article, section 5) on the GPU, through the C ABI, against the oracle's
written conventions (oracle.share_classes / union_lists / choose_block_size).

Sharing: the classes must equal the oracle's on the oracle's vhat (a
difference is tolerated only for a pair whose JSD lies within 1e-3 relative
of eps), the shared lists must be exactly the union of the GPU's own lists
over each class (the per-head lists themselves are checked against the oracle
by the usual rules), and attention on the shared index must match the oracle
on the same lists.  Block size: rho within one block per head of the
oracle's, and the same b unless rho lies that close to a threshold.
"""
import numpy as np
import pytest
import torch
from scipy.spatial.distance import jensenshannon

from dynamic_block_sparse_last_b200 import synth
from oracle import oracle as orc
from tests import parity
from tests.test_gpu_parity import check_index, check_tiles, nblocks, oracle_problem, sampled_tiles

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import fp as mod
    assert torch.cuda.is_available(), "CUDA device required"
    return mod


def build(fp, w, x):
    dev = torch.device("cuda:0")
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index(q, k, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_BF16, None, None, idx)
    return idx, q, k, v


SHARE = [(synth.Workload("share_g4", S=4096, Hq=8, Hkv=2, b=128, seed=51, n_vertical=64, n_topics=32), 0.05),
         (synth.Workload("share_g3_b256", S=3072, Hq=6, Hkv=2, b=256, gamma=0.95, seed=52,
                         kinds=["vs", "qa", "vs", "qa", "qa", "vs"]), 0.02),
         (synth.Workload("share_g4_b64", S=2048, Hq=8, Hkv=2, b=64, seed=53), 0.05)]


@pytest.mark.parametrize("w,eps", SHARE, ids=[w.name for w, _ in SHARE])
def test_head_sharing_against_oracle(fp, w, eps):
    x = synth.make_inputs(w)
    idx, q, k, v = build(fp, w, x)
    exp0 = fp.fp_index_export(idx)
    P = oracle_problem(x, w)
    heads, _ = check_index(P, exp0, w)                   # the per-head lists, as usual
    fp.fp_index_share(idx, eps)
    out = torch.empty_like(q)
    fp.fp_sparse_attn(q, k, v, None, None, idx, out)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    exp1 = fp.fp_index_export(idx)
    cls = fp.fp_index_classes(idx)
    g, n = w.Hq // w.Hkv, nblocks(w.S, w.b)
    # classes against the oracle's rule on the oracle's vhat
    ocls, _ = orc.share_index(heads, g, eps)
    for h in range(w.Hq):
        if int(cls[h]) != int(ocls[h]):
            a, b2 = h, int(min(cls[h], ocls[h]))
            d = jensenshannon(heads[a]["vhat"], heads[b2]["vhat"]) ** 2
            assert abs(d - eps) <= 1e-3 * eps, (h, int(cls[h]), int(ocls[h]), d)
    # the shared lists are the unions of the GPU's own lists over each class
    rows0 = [parity.gpu_rows(exp0, h, n) for h in range(w.Hq)]
    rows1 = [parity.gpu_rows(exp1, h, n) for h in range(w.Hq)]
    shared_heads = 0
    for h in range(w.Hq):
        members = [m for m in range(w.Hq) if int(cls[m]) == int(cls[h])]
        shared_heads += len(members) > 1
        for r in range(n):
            want = sorted(set().union(*[set(map(int, rows0[m][r])) for m in members]))
            assert list(map(int, rows1[h][r])) == want, (h, r)
    print(f"[{w.name}] eps {eps}: classes {cls.tolist()}, {shared_heads} heads in shared classes; "
          f"density {exp0['nnz'] / (w.Hq * n * (n + 1) / 2):.4f} -> {exp1['nnz'] / (w.Hq * n * (n + 1) / 2):.4f}")
    tiles = [(h, qc) for h in range(w.Hq) for qc in range(nblocks(w.S, 128))]
    check_tiles(P, exp1, out, w, tiles)
    idx.free()


def test_sharing_with_zero_eps_changes_nothing(fp):
    w = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(w)
    idx, q, k, v = build(fp, w, x)
    exp0 = fp.fp_index_export(idx)
    fp.fp_index_share(idx, 0.0)
    exp1 = fp.fp_index_export(idx)
    assert np.array_equal(exp0["row_ptr"], exp1["row_ptr"]) and np.array_equal(exp0["col"], exp1["col"])
    assert list(fp.fp_index_classes(idx)) == list(range(w.Hq))
    idx.free()


BLOCK = [synth.Workload("bs_tiny", S=1024, Hq=4, Hkv=2, b=128, seed=0, kinds=["vs", "qa", "vs", "qa"]),
         synth.Workload("bs_sweep_gen", S=8192, Hq=8, Hkv=2, b=128, n_vertical=64, n_topics=32, seed=2),
         synth.Workload("bs_topics", S=4096, Hq=4, Hkv=2, b=128, seed=61, kinds=["vs", "vs", "vs", "vs"]),
         synth.Workload("bs_uniform", S=4096, Hq=4, Hkv=2, b=128, seed=62, kinds=["qa", "qa", "qa", "qa"])]


@pytest.mark.parametrize("w", BLOCK, ids=[w.name for w in BLOCK])
def test_block_size_rule_against_oracle(fp, w):
    x = synth.make_inputs(w)
    idx, q, k, v = build(fp, w, x)
    b, rho = fp.fp_choose_block_size(idx, w.gamma)
    torch.cuda.synchronize()
    P = oracle_problem(x, w)
    vh = np.stack([P.last_block_stats(h)[0] for h in range(w.Hq)])
    ob, orho = orc.choose_block_size(vh, w.S, w.gamma)
    n = nblocks(w.S, 128)
    assert abs(rho - orho) <= 1.0 / n + 1e-6, (rho, orho)
    if b != ob:
        assert min(abs(orho - 0.1), abs(orho - 0.5)) <= 1.0 / n, (b, ob, orho)
    print(f"[{w.name}] rho {rho:.4f} (oracle {orho:.4f}) -> b = {b} (oracle {ob})")
    idx.free()


def test_block_size_rule_needs_b128(fp):
    w = synth.Workload("bs_b256", S=1024, Hq=2, Hkv=1, b=256, seed=3)
    x = synth.make_inputs(w)
    idx, *_ = build(fp, w, x)
    with pytest.raises(fp.FpError) as e:
        fp.fp_choose_block_size(idx, 0.9)
    assert e.value.code == fp.FP_ERR_STATE
    idx.free()


CSR = [synth.Workload("csr_g4", S=4096, Hq=8, Hkv=2, b=128, seed=71, n_vertical=64, n_topics=32),
       synth.Workload("csr_b64_ragged", S=1000, Hq=6, Hkv=3, b=64, gamma=0.95, seed=72),
       synth.Workload("csr_g1_b256", S=2048, Hq=3, Hkv=3, b=256, seed=73)]


@pytest.mark.parametrize("w", CSR, ids=[w.name for w in CSR])
def test_device_csr_and_group_lists(fp, w):
    """fp_index_csr equals the host export exactly; fp_index_group_lists is,
    per (KV head, query block), the union of the group's lists with the mask
    of the heads that list each block."""
    x = synth.make_inputs(w)
    idx, q, k, v = build(fp, w, x)
    exp = fp.fp_index_export(idx)
    n, g = nblocks(w.S, w.b), w.Hq // w.Hkv
    dev = torch.device("cuda:0")
    rp = torch.full((w.Hq * n + 1,), -1, dtype=torch.int32, device=dev)
    fp.fp_index_csr(idx, rp)                       # offsets only
    torch.cuda.synchronize()
    assert np.array_equal(rp.cpu().numpy(), exp["row_ptr"])
    col = torch.full((int(exp["nnz"]),), -1, dtype=torch.int32, device=dev)
    fp.fp_index_csr(idx, rp, col)
    torch.cuda.synchronize()
    assert np.array_equal(rp.cpu().numpy(), exp["row_ptr"]) and np.array_equal(col.cpu().numpy(), exp["col"])
    gp = torch.zeros(w.Hkv * n + 1, dtype=torch.int32, device=dev)
    fp.fp_index_group_lists(idx, gp)
    torch.cuda.synchronize()
    total = int(gp[-1])
    gc = torch.full((total,), -1, dtype=torch.int32, device=dev)
    gm = torch.zeros(total, dtype=torch.int32, device=dev)
    fp.fp_index_group_lists(idx, gp, gc, gm)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    gp, gc, gm = gp.cpu().numpy(), gc.cpu().numpy(), gm.cpu().numpy().view(np.uint32)
    rows = [parity.gpu_rows(exp, h, n) for h in range(w.Hq)]
    for j in range(w.Hkv):
        for r in range(n):
            want = {}
            for m in range(g):
                for c in rows[j * g + m][r]:
                    want[int(c)] = want.get(int(c), 0) | (1 << m)
            lo, hi = gp[j * n + r], gp[j * n + r + 1]
            assert list(gc[lo:hi]) == sorted(want), (j, r)
            assert [int(x) for x in gm[lo:hi]] == [want[c] for c in sorted(want)], (j, r)
    print(f"[{w.name}] csr nnz {exp['nnz']}, group lists {total} entries "
          f"({total / max(1, exp['nnz']):.3f} per head-list entry)")
    idx.free()
