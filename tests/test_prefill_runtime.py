"""The host-to-host prefill runtime (include/fp_prefill.h) on the GPU.

The pipeline streams head groups through copy-in, compute and copy-out
streams.  Every head's index and output depend on that head's inputs alone,
so its result must be bit-identical to fp_build_index + fp_sparse_attn over
the whole layer on device buffers (which the oracle parity tests check).
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_last_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import fp as mod
    assert torch.cuda.is_available(), "CUDA device required"
    return mod


def device_path(fp, x, w):
    dev = torch.device("cuda:0")
    if w.int8:
        qq, kk = x["q8"].to(dev), x["k8"].to(dev)
        qs, ks, dt = x["q_scale"].to(dev), x["k_scale"].to(dev), fp.FP_QK_INT8
    else:
        qq, kk, qs, ks, dt = x["q"].to(dev), x["k"].to(dev), None, None, fp.FP_QK_BF16
    v = x["v"].to(dev)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx)
    out = torch.empty(w.Hq, w.S, w.d, dtype=torch.bfloat16, device=dev)
    fp.fp_sparse_attn(qq, kk, v, qs, ks, idx, out)
    torch.cuda.synchronize()
    exp = fp.fp_index_export(idx)
    idx.free()
    return out.cpu(), exp


def host_inputs(x, w):
    q = (x["q8"] if w.int8 else x["q"]).contiguous().pin_memory()
    k = (x["k8"] if w.int8 else x["k"]).contiguous().pin_memory()
    v = x["v"].contiguous().pin_memory()
    qs = x["q_scale"].contiguous() if w.int8 else None
    ks = x["k_scale"].contiguous() if w.int8 else None
    return q, k, v, qs, ks


def check_groups_equal(fp, pipe, exp, w):
    """Each group's index equals the whole-layer index on that group's heads."""
    G = pipe.groups
    hq = w.Hq // G
    n = -(-w.S // w.b)
    for gi in range(G):
        e = fp.fp_index_export(pipe.group_index(gi))
        assert np.array_equal(e["pattern"], exp["pattern"][gi * hq:(gi + 1) * hq])
        for h in range(hq):
            a, c = parity.gpu_rows(e, h, n), parity.gpu_rows(exp, gi * hq + h, n)
            assert all(np.array_equal(r0, r1) for r0, r1 in zip(a, c)), (gi, h)


CASES = [(synth.WORKLOADS["tiny"], 0), (synth.WORKLOADS["tiny"], 1),
         (synth.Workload("pre_g4", S=4096, Hq=8, Hkv=2, b=128, gamma=0.95, seed=41), 2),
         (synth.Workload("pre_ragged_b256", S=1300, Hq=6, Hkv=3, b=256, seed=42), 3),
         (synth.Workload("pre_int8", S=2048, Hq=8, Hkv=4, b=128, int8=True, seed=43), 2),
         # more groups than KV heads: each KV head's query heads in shares
         (synth.WORKLOADS["tiny"], 4),
         (synth.Workload("pre_g4_shares", S=4096, Hq=8, Hkv=2, b=128, gamma=0.95, seed=41), 4),
         (synth.Workload("pre_int8_shares", S=2048, Hq=8, Hkv=4, b=128, int8=True, seed=43), 8),
         (synth.Workload("pre_ragged_shares", S=1300, Hq=6, Hkv=2, b=256, seed=44), 6),
         # n = 700 blocks: the groups' query-aware logits run on the tensor cores
         (synth.Workload("pre_long_tc", S=89550, Hq=4, Hkv=2, b=128, seed=45), 2)]


@pytest.mark.parametrize("w,groups", CASES, ids=[f"{w.name}-G{g}" for w, g in CASES])
def test_prefill_run_equals_device_path(fp, w, groups):
    x = synth.make_inputs(w)
    ref_out, exp = device_path(fp, x, w)
    pipe = fp.Prefill(w.S, w.Hq, w.Hkv, w.d, w.b, fp.FP_QK_INT8 if w.int8 else fp.FP_QK_BF16, groups)
    q, k, v, qs, ks = host_inputs(x, w)
    h_out = torch.empty(w.Hq, w.S, w.d, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.Stream()
    pipe.run(q, k, v, qs, ks, w.gamma, w.tau, h_out, stream)
    stream.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    assert torch.equal(h_out, ref_out)
    check_groups_equal(fp, pipe, exp, w)
    pipe.free()


def test_prefill_consecutive_runs_reuse_the_pipeline(fp):
    """Two runs with different inputs queued back to back on one stream."""
    ws = [synth.Workload(f"pre_seq{i}", S=2048, Hq=4, Hkv=2, b=128, seed=50 + i) for i in range(2)]
    xs = [synth.make_inputs(w) for w in ws]
    refs = [device_path(fp, x, w)[0] for x, w in zip(xs, ws)]
    pipe = fp.Prefill(2048, 4, 2, 128, 128)
    stream = torch.cuda.Stream()
    outs = []
    for x, w in zip(xs, ws):
        q, k, v, _, _ = host_inputs(x, w)
        h_out = torch.empty(4, 2048, 128, dtype=torch.bfloat16).pin_memory()
        pipe.run(q, k, v, None, None, w.gamma, w.tau, h_out, stream)
        outs.append((h_out, q, k, v))
    stream.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    for (h_out, *_), ref in zip(outs, refs):
        assert torch.equal(h_out, ref)
    pipe.free()


@pytest.mark.parametrize("int8,groups", [(False, 0), (False, 4), (True, 2), (True, 8)])
def test_overlapping_runs_keep_their_own_inputs(fp, int8, groups):
    """Three runs queued with fp_prefill_enqueue before one wait: they overlap
    on the device (a run's copies and compute start while the previous run's
    outputs drain), yet each output equals its own device-path result.  The
    int8 runs carry different per-head scales, which exercises the two
    alternating scale slots."""
    ws = [synth.Workload(f"pre_ov{i}", S=2048, Hq=8, Hkv=4, b=128, gamma=0.9, int8=int8, seed=60 + i)
          for i in range(3)]
    xs = [synth.make_inputs(w) for w in ws]
    refs = [device_path(fp, x, w)[0] for x, w in zip(xs, ws)]
    pipe = fp.Prefill(2048, 8, 4, 128, 128, fp.FP_QK_INT8 if int8 else fp.FP_QK_BF16, groups)
    stream = torch.cuda.Stream()
    keep = []
    for x, w in zip(xs, ws):
        q, k, v, qs, ks = host_inputs(x, w)
        h_out = torch.empty(8, 2048, 128, dtype=torch.bfloat16).pin_memory()
        pipe.enqueue(q, k, v, qs, ks, w.gamma, w.tau, h_out, stream)
        keep.append((h_out, q, k, v))
    pipe.wait(stream)
    stream.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    for (h_out, *_), ref in zip(keep, refs):
        assert torch.equal(h_out, ref)
    pipe.free()
