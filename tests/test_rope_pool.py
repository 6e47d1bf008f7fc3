"""The rotary-embedding epilogue with block pooling (fp_rope_pool) and the
index build that takes its block means (fp_build_index_pooled), on the GPU,
against the oracle.

The oracle rotates its own copy of the inputs exactly; the kernel rotates in
fp32, so their bf16 outputs may differ where the exact value sits within fp32
rounding of a bf16 rounding boundary (or where the two products nearly
cancel): tensors are compared to one bf16 step plus fp32 rounding of the
products (with all but 0.1% equal), and the index and attention on the kernel's tensors are
compared with the usual parity rules against the oracle on its own tensors.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_last_b200 import synth
from oracle import oracle as orc
from tests.test_gpu_parity import check_index, check_tiles, sampled_tiles

pytestmark = pytest.mark.gpu

CASES = [synth.Workload("rp_b128", S=1000, Hq=4, Hkv=2, b=128, seed=90),
         synth.Workload("rp_b256", S=1300, Hq=6, Hkv=2, b=256, seed=91),
         synth.Workload("rp_4k", S=4096, Hq=8, Hkv=2, b=128, gamma=0.95, seed=92)]


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import fp as mod
    assert torch.cuda.is_available(), "CUDA device required"
    return mod


def gpu_rope_pool(fp, x, w, in_place=False):
    n = -(-w.S // w.b)
    q_in, k_in = x["q_in"].cuda(), x["k_in"].cuda()
    cos, sin = x["cos"].cuda(), x["sin"].cuda()
    q_out, k_out = (q_in, k_in) if in_place else (torch.empty_like(q_in), torch.empty_like(k_in))
    qbar = torch.empty(w.Hq, n, 128, device="cuda")
    kbar = torch.empty(w.Hkv, n, 128, device="cuda")
    fp.fp_rope_pool(q_in, k_in, cos, sin, w.S, w.Hq, w.Hkv, 128, w.b, q_out, k_out, qbar, kbar)
    torch.cuda.synchronize()
    return q_out, k_out, qbar, kbar


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_rope_pool_matches_oracle(fp, w):
    x = synth.make_prerope_inputs(w)
    q, k, qbar, kbar = gpu_rope_pool(fp, x, w)
    for got, mean, src in ((q, qbar, "q_in"), (k, kbar, "k_in")):
        ref, ref_mean = orc.rope_pool(x[src], x["cos"], x["sin"], w.b)
        g = got.cpu().double().numpy()
        diff = np.abs(g - ref)
        assert (diff == 0).mean() > 0.999, (src, (diff > 0).mean())
        # one bf16 step of the result, plus fp32 rounding of the two products
        # (which dominates where they nearly cancel)
        xin = x[src].double().numpy()
        terms = np.abs(xin[..., :64]) + np.abs(xin[..., 64:])
        bound = 2.0 ** -7 * np.abs(ref) + 2.0 ** -22 * np.concatenate([terms, terms], -1)
        assert np.all(diff <= bound), (src, float((diff / np.maximum(bound, 1e-30)).max()))
        # the means are those of the stored rows (fp32 sums of the same values)
        m = mean.cpu().double().numpy()
        blocks = [(c * w.b, min((c + 1) * w.b, w.S)) for c in range(m.shape[1])]
        own = np.stack([g[:, lo:hi].mean(1) for lo, hi in blocks], 1)
        assert np.allclose(m, own, rtol=1e-5, atol=1e-6), src
        # and differ from the oracle's only through the differing elements
        slack = np.stack([diff[:, lo:hi].sum(1) / (hi - lo) for lo, hi in blocks], 1)
        assert np.all(np.abs(m - ref_mean) <= slack + 1e-5 * np.abs(ref_mean) + 1e-6), src
    # in place: the same bits
    q2, k2, qbar2, kbar2 = gpu_rope_pool(fp, x, w, in_place=True)
    assert torch.equal(q2, q) and torch.equal(k2, k)
    assert torch.equal(qbar2, qbar) and torch.equal(kbar2, kbar)


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_index_on_pooled_means_matches_oracle(fp, w):
    x = synth.make_prerope_inputs(w)
    q, k, qbar, kbar = gpu_rope_pool(fp, x, w)
    v = x["v"].cuda()
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index_pooled(q, k, qbar, kbar, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, idx)
    out = torch.empty_like(q)
    fp.fp_sparse_attn(q, k, v, None, None, idx, out)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    exp = fp.fp_index_export(idx)
    # the oracle on its own rotated tensors (bf16 values, exactly representable)
    oq, _ = orc.rope_pool(x["q_in"], x["cos"], x["sin"], w.b)
    ok, _ = orc.rope_pool(x["k_in"], x["cos"], x["sin"], w.b)
    P = orc.OracleProblem(torch.from_numpy(oq).to(torch.bfloat16), torch.from_numpy(ok).to(torch.bfloat16),
                          x["v"], w.b)
    check_index(P, exp, w)
    tiles = [(h, qc) for h in range(w.Hq) for qc in range(-(-w.S // 128))]
    check_tiles(P, exp, out, w, tiles)
    idx.free()


def test_index_on_pooled_means_tensor_core_logits(fp):
    """n = 672 >= 640: the query-aware logits of the pooled build run on the
    tensor cores, their operands split from the caller's block means.  Full
    index against the oracle on its own rotated tensors, 24 sampled tiles."""
    w = synth.Workload("rp_n672", S=86016, Hq=4, Hkv=2, b=128, seed=93)
    x = synth.make_prerope_inputs(w)
    q, k, qbar, kbar = gpu_rope_pool(fp, x, w)
    v = x["v"].cuda()
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index_pooled(q, k, qbar, kbar, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, idx)
    out = torch.empty_like(q)
    fp.fp_sparse_attn(q, k, v, None, None, idx, out)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    exp = fp.fp_index_export(idx)
    assert 1 in exp["pattern"].tolist(), "the case needs a query-aware head"
    oq, _ = orc.rope_pool(x["q_in"], x["cos"], x["sin"], w.b)
    ok, _ = orc.rope_pool(x["k_in"], x["cos"], x["sin"], w.b)
    P = orc.OracleProblem(torch.from_numpy(oq).to(torch.bfloat16), torch.from_numpy(ok).to(torch.bfloat16),
                          x["v"], w.b)
    check_index(P, exp, w)
    check_tiles(P, exp, out, w, sampled_tiles(w, 24, seed=w.seed))
    idx.free()
