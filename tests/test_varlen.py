"""Packed sequences of different lengths (fp_varlen_*) on the GPU.

Each sequence of a packed [H][T][d] batch is its own problem, so its index
and output must be bit-identical to the single-sequence calls on that
sequence alone (which the oracle parity tests check); one packed case is also
compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_last_b200 import synth
from tests import parity
from tests.test_gpu_parity import check_index, check_tiles, oracle_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import fp as mod
    assert torch.cuda.is_available(), "CUDA device required"
    return mod


def single(fp, x, w):
    dev = torch.device("cuda:0")
    if w.int8:
        qq, kk = x["q8"].to(dev), x["k8"].to(dev)
        qs, ks, dt = x["q_scale"].to(dev), x["k_scale"].to(dev), fp.FP_QK_INT8
    else:
        qq, kk, qs, ks, dt = x["q"].to(dev), x["k"].to(dev), None, None, fp.FP_QK_BF16
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx)
    out = torch.empty(w.Hq, w.S, w.d, dtype=torch.bfloat16, device=dev)
    fp.fp_sparse_attn(qq, kk, x["v"].to(dev), qs, ks, idx, out)
    torch.cuda.synchronize()
    exp = fp.fp_index_export(idx)
    idx.free()
    return out.cpu(), exp


def packed_run(fp, ws, xs, Hq, Hkv, b, gamma, tau, int8):
    dev = torch.device("cuda:0")
    cu = np.concatenate([[0], np.cumsum([w.S for w in ws])]).astype(np.int32)
    key_q, key_k = ("q8", "k8") if int8 else ("q", "k")
    present = [x for x in xs if x is not None]
    q = torch.cat([x[key_q] for x in present], 1).contiguous().to(dev)
    k = torch.cat([x[key_k] for x in present], 1).contiguous().to(dev)
    v = torch.cat([x["v"] for x in present], 1).contiguous().to(dev)
    qs = ks = None
    if int8:
        qs = torch.stack([x["q_scale"] if x is not None else torch.ones(Hq) for x in xs]).contiguous().to(dev)
        ks = torch.stack([x["k_scale"] if x is not None else torch.ones(Hkv) for x in xs]).contiguous().to(dev)
    V = fp.Varlen(cu, Hq, Hkv, 128, b)
    V.build_index(q, k, gamma, tau, fp.FP_QK_INT8 if int8 else fp.FP_QK_BF16, qs, ks)
    out = torch.full((Hq, int(cu[-1]), 128), float("nan"), dtype=torch.bfloat16, device=dev)
    V.sparse_attn(q, k, v, out, qs, ks)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    return V, cu, out.cpu()


CASES = [("b128", [1000, 2048, 0, 77, 1500], 4, 2, 128, False),
         ("b256", [1300, 512, 2000], 6, 2, 256, False),
         ("int8", [2000, 129, 1024], 4, 2, 128, True),
         ("one_seq", [4096], 8, 2, 128, False),
         ("b64", [1000, 333, 2048], 4, 2, 64, False),
         # a sequence with n = 700 blocks: its query-aware logits run on the tensor cores
         ("long_tc", [700, 89550, 1000], 4, 2, 128, False)]


@pytest.mark.parametrize("name,lens,Hq,Hkv,b,int8", CASES, ids=[c[0] for c in CASES])
def test_packed_sequences_equal_single_calls(fp, name, lens, Hq, Hkv, b, int8):
    ws = [synth.Workload(f"vl_{name}_{i}", S=L, Hq=Hq, Hkv=Hkv, b=b, int8=int8, seed=70 + i) if L else None
          for i, L in enumerate(lens)]
    xs = [synth.make_inputs(w) if w is not None else None for w in ws]
    V, cu, out = packed_run(fp, [w if w is not None else synth.Workload("empty", S=0, Hq=Hq, Hkv=Hkv, b=b)
                                 for w in ws], xs, Hq, Hkv, b, 0.9, 0.1, int8)
    for s, (w, x) in enumerate(zip(ws, xs)):
        if w is None:
            assert V.index(s) is None
            continue
        ref_out, ref_exp = single(fp, x, w)
        assert torch.equal(out[:, cu[s]:cu[s + 1]], ref_out), s
        exp = fp.fp_index_export(V.index(s))
        n = -(-w.S // w.b)
        assert np.array_equal(exp["pattern"], ref_exp["pattern"]), s
        for h in range(Hq):
            a, c = parity.gpu_rows(exp, h, n), parity.gpu_rows(ref_exp, h, n)
            assert all(np.array_equal(r0, r1) for r0, r1 in zip(a, c)), (s, h)
    V.free()


def test_packed_sequences_match_the_oracle(fp):
    """Three packed sequences (one of them ragged) checked against the oracle
    per sequence: full index and every output tile."""
    ws = [synth.Workload(f"vl_orc_{i}", S=L, Hq=4, Hkv=2, b=128, seed=80 + i) for i, L in enumerate([1024, 700, 1536])]
    xs = [synth.make_inputs(w) for w in ws]
    V, cu, out = packed_run(fp, ws, xs, 4, 2, 128, 0.9, 0.1, False)
    for s, (w, x) in enumerate(zip(ws, xs)):
        exp = fp.fp_index_export(V.index(s))
        P = oracle_problem(x, w)
        check_index(P, exp, w)
        tiles = [(h, qc) for h in range(w.Hq) for qc in range(-(-w.S // 128))]
        check_tiles(P, exp, out[:, cu[s]:cu[s + 1]], w, tiles)
    V.free()
