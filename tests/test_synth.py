"""The seeded input generator: determinism, rotary-embedding relative-position
property, planted structure bookkeeping and the int8 quantisation bounds."""
import math

import numpy as np

import torch

from dynamic_block_sparse_last_b200 import synth


def small(**kw):
    base = dict(name="t", S=512, Hq=4, Hkv=2, seed=7)
    base.update(kw)
    return synth.Workload(**base)


def test_same_seed_same_tensors():
    a = synth.make_inputs(small())
    b = synth.make_inputs(small())
    c = synth.make_inputs(small(seed=8))
    for key in ("q", "k", "v"):
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])
        assert a[key].dtype == torch.bfloat16 and a[key].is_contiguous()


def test_rope_dot_products_depend_on_offset_only():
    g = torch.Generator().manual_seed(0)
    u = torch.randn(1, 1, 128, generator=g, dtype=torch.float64)
    w = torch.randn(1, 1, 128, generator=g, dtype=torch.float64)
    S = 64
    U = synth.rope_(u.expand(1, S, 128).clone().float()).double()
    W = synth.rope_(w.expand(1, S, 128).clone().float()).double()
    d1 = float(U[0, 40] @ W[0, 30])
    d2 = float(U[0, 20] @ W[0, 10])
    assert abs(d1 - d2) < 1e-3 * max(1.0, abs(d1))
    assert abs(float(U[0, 5].norm()) - float(u.norm())) < 1e-4


def test_head_kinds_split_groups_in_half():
    w = synth.WORKLOADS["llama3b"]
    kinds = w.head_kinds()
    g = w.Hq // w.Hkv
    assert kinds == ["vs"] * (g * w.Hkv // 2) + ["qa"] * (g * w.Hkv // 2)
    assert synth.WORKLOADS["tiny"].head_kinds() == ["vs", "qa", "vs", "qa"]


def test_int8_quantisation_bounds():
    x = synth.make_inputs(small(int8=True))
    for key, skey in (("q8", "q_scale"), ("k8", "k_scale")):
        x8, sc = x[key], x[skey]
        src = x[key[0]].float()
        for h in range(x8.shape[0]):
            assert int(x8[h].abs().max()) == 127
            err = (x8[h].float() * sc[h] - src[h]).abs().max()
            assert float(err) <= float(sc[h]) * 0.5 * (1 + 1e-6)


def test_dense_equivalent_flops():
    assert synth.dense_equiv_flops(131072, 32, 128) == 2.0 * 32 * 128 * 131072 ** 2
    assert math.isclose(synth.dense_equiv_flops(131072, 32, 128), 1.407e14, rel_tol=1e-3)


def test_rope_tables_angles_and_rounding():
    """cos/sin tables: fp64 angles p * theta^(-2i/d) rounded to float32."""
    cos, sin = synth.rope_tables(300, 128)
    assert cos.shape == (300, 64) and cos.dtype == torch.float32 and sin.dtype == torch.float32
    p = np.arange(300)[:, None].astype(np.float64)
    inv = synth.ROPE_THETA ** (-np.arange(64) * 2.0 / 128)
    assert np.array_equal(cos.numpy(), np.cos(p * inv).astype(np.float32))
    assert np.array_equal(sin.numpy(), np.sin(p * inv).astype(np.float32))
    assert np.all(cos[0].numpy() == 1.0) and np.all(sin[0].numpy() == 0.0)


def test_prerope_inputs_are_seeded_and_shaped():
    w = synth.Workload("pr", S=200, Hq=4, Hkv=2, b=64, seed=7)
    a, b = synth.make_prerope_inputs(w), synth.make_prerope_inputs(w)
    assert a["q_in"].shape == (4, 200, 128) and a["k_in"].shape == (2, 200, 128) and a["v"].shape == (2, 200, 128)
    assert a["q_in"].dtype == torch.bfloat16 and a["cos"].shape == (200, 64)
    for key in ("q_in", "k_in", "v", "cos", "sin"):
        assert torch.equal(a[key], b[key]), key
    c = synth.make_prerope_inputs(synth.Workload("pr", S=200, Hq=4, Hkv=2, b=64, seed=8))
    assert not torch.equal(a["q_in"], c["q_in"])


def test_key_ramp_scales_key_rows():
    """key_ramp multiplies key row j by 1 + key_ramp * j / S and touches nothing else."""
    base = synth.Workload("r0", S=256, Hq=2, Hkv=1, seed=5)
    ramp = synth.Workload("r1", S=256, Hq=2, Hkv=1, seed=5, key_ramp=3.0)
    a, b = synth.make_inputs(base), synth.make_inputs(ramp)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["v"], b["v"])
    fac = 1.0 + 3.0 * torch.arange(256, dtype=torch.float32) / 256
    want = (a["k"].float() * fac[None, :, None]).to(torch.bfloat16)
    # both sides round the same fp32 product once; the generator scales before its
    # single bf16 rounding, so allow one bf16 step
    diff = (b["k"].float() - want.float()).abs()
    assert float(diff.max()) <= float(want.float().abs().max()) * 2 ** -7
    norms = b["k"][0].float().norm(dim=1)
    assert float(norms[-32:].mean()) > 3.0 * float(norms[:32].mean())
