"""The allocation-free statistics entry point, fp_pattern_stats_noalloc.

Some callers may not allocate device memory (a host framework that owns all
device memory through its own allocator or budget, or a latency-critical loop
that cannot take cudaMalloc's device-wide synchronisation).  For them the
library keeps the statistics kernels' scratch in a fixed device array.  This
file runs last so that a failure here leaves every other test already run;
it passes alone in a fresh process as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_last_b200 import synth

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-3, 2e-6          # the statistics tolerance of the parity tests


def reference_stats(fp, x, w, qq, kk, qs, ks, dt):
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx)
    exp = fp.fp_index_export(idx)
    idx.free()
    return exp


def noalloc_stats(fp, w, qq, kk, qs, ks, dt):
    n = -(-w.S // w.b)
    dev = qq.device
    vhat = torch.full((w.Hq, n), float("nan"), device=dev)
    shat = torch.full((w.Hq, n), float("nan"), device=dev)
    pest = torch.full((w.Hq, n), float("nan"), device=dev)
    jsd = torch.full((w.Hq,), float("nan"), device=dev)
    pattern = torch.full((w.Hq,), -1, dtype=torch.int32, device=dev)
    fp.fp_pattern_stats_noalloc(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.tau, dt, qs, ks, vhat, shat, pest, jsd,
                                pattern)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    return {k: v.cpu().numpy() for k, v in
            dict(vhat=vhat, shat=shat, pest=pest, jsd=jsd, pattern=pattern).items()}


def inputs(fp, w):
    x = synth.make_inputs(w)
    dev = torch.device("cuda:0")
    if w.int8:
        return x, x["q8"].to(dev), x["k8"].to(dev), x["q_scale"].to(dev), x["k_scale"].to(dev), fp.FP_QK_INT8
    return x, x["q"].to(dev), x["k"].to(dev), None, None, fp.FP_QK_BF16


def test_noalloc_statistics_match_build_index_on_consecutive_calls():
    from dynamic_block_sparse_last_b200 import fp
    cases = [synth.WORKLOADS["tiny"],
             synth.Workload("noalloc_b256_int8", S=8192, Hq=8, Hkv=2, b=256, int8=True, seed=21),
             synth.Workload("noalloc_llama3b_shape", S=32768, Hq=32, Hkv=8, b=128, seed=22),
             synth.Workload("noalloc_ragged", S=1500, Hq=4, Hkv=2, b=256, seed=24),
             synth.WORKLOADS["tiny"]]
    for w in cases:      # consecutive calls share (and overwrite) the fixed scratch
        x, qq, kk, qs, ks, dt = inputs(fp, w)
        ref = reference_stats(fp, x, w, qq, kk, qs, ks, dt)
        got = noalloc_stats(fp, w, qq, kk, qs, ks, dt)
        assert np.array_equal(got["pattern"], ref["pattern"].astype(np.int32)), w.name
        for key in ("vhat", "shat", "pest"):
            assert np.allclose(got[key], ref[key], rtol=RTOL, atol=ATOL), (w.name, key)
        assert np.allclose(got["jsd"], ref["jsd"], rtol=RTOL, atol=1e-4), w.name


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    from dynamic_block_sparse_last_b200 import fp
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")      # never read: rejected on the host
    outs = [torch.zeros(4, device="cuda") for _ in range(4)] + [torch.zeros(4, dtype=torch.int32, device="cuda")]
    rc = fp.lib().fp_pattern_stats_noalloc(q.data_ptr(), q.data_ptr(), 131072, 32, 8, 128, 128, 0.1,
                                           fp.FP_QK_BF16, None, None, *[o.data_ptr() for o in outs], None)
    assert rc == fp.FP_ERR_ARG
