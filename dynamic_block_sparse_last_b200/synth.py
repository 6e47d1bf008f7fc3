"""Seeded synthetic inputs for dynamic block-sparse prefill attention.

This module only builds inputs: Gaussian Q/K/V, rotary position embedding, the
planted "vertical-slash" and "query-aware" structure, and the optional
symmetric per-head int8 quantisation of Q and K.  It holds none of the
sparse-attention arithmetic; both the CUDA path and the fp64 oracle consume
what it returns.

Workloads (all batch 1, head-major [H][S][d] layout, bf16 after rounding):

* ``tiny``   S=1024,   Hq=4,  Hkv=2, 16 vertical positions, 8 topics
* ``llama3b`` S=32768, Hq=24, Hkv=8, 16 vertical positions, 8 topics
* ``llama8b`` S=131072, Hq=32, Hkv=8, 64 vertical positions, 32 topics
* ``llama8b_w8a8``  the ``llama8b`` tensors with int8 Q and K

Construction (the workload recipe of the FAST-Prefill article, section 4,
which evaluates 4K-128K contexts; structure planted so both of Flex-Prefill's
head patterns, section 1.2, occur):

1. Q[h], K[j], V[j] ~ N(0, 1) in fp32 from one ``torch.Generator`` seeded
   with ``seed``, drawn in that order.
2. Every query head has a kind, "vs" or "qa".  A KV head whose group holds at
   least one "qa" head gets a topic per token t_p ~ U{0..T-1} and centroids
   c ~ N(0, I); K[j][p] += 2 c[t_p] and, for each "qa" head h of the group,
   Q[h][p] += 2 c[t_p].
3. Rotary embedding (rotate-half convention, theta = 5e5, positions 0..S-1)
   on Q and K.
4. For each "vs" head h: mu_h = unit vector along the mean of Q[h] over all
   positions; K rows of its KV head at positions 0..3 (sinks) and at
   ``n_vertical`` seeded positions drawn from [4, S) get += 3 mu_h.
5. Round to bf16 (round-to-nearest-even).
6. Optional W8A8: per head, scale = max|x| / 127 over the bf16 values,
   x8 = round-half-even(x / scale) clamped to [-127, 127].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

ROPE_THETA = 500000.0


@dataclass
class Workload:
    name: str
    S: int
    Hq: int
    Hkv: int
    d: int = 128
    b: int = 128
    gamma: float = 0.9
    tau: float = 0.1
    n_vertical: int = 16
    n_topics: int = 8
    seed: int = 0
    int8: bool = False
    kinds: list = field(default_factory=list)
    # > 0: key row j is scaled by 1 + key_ramp * j / S after the structure is
    # planted, so the scores (and each row's running maximum) grow along the
    # key axis; 0 leaves the keys as generated
    key_ramp: float = 0.0

    def head_kinds(self):
        if self.kinds:
            return list(self.kinds)
        g = self.Hq // self.Hkv
        half = self.Hkv // 2
        return ["vs" if (h // g) < half else "qa" for h in range(self.Hq)]


WORKLOADS = {
    # Tiny single layer: heads 0 and 2 plant vertical-slash structure,
    # heads 1 and 3 plant query-aware topics.
    "tiny": Workload("tiny", S=1024, Hq=4, Hkv=2, seed=0, kinds=["vs", "qa", "vs", "qa"]),
    # Llama-3.2-3B-shaped attention layer.
    "llama3b": Workload("llama3b", S=32768, Hq=24, Hkv=8, seed=1),
    # Llama-3-8B-shaped attention layer at 128K context.
    "llama8b": Workload("llama8b", S=131072, Hq=32, Hkv=8, n_vertical=64, n_topics=32, seed=2),
    # W8A8 variant of the 128K layer.
    "llama8b_w8a8": Workload("llama8b_w8a8", S=131072, Hq=32, Hkv=8, n_vertical=64, n_topics=32,
                             seed=2, int8=True),
}


def sweep_workloads():
    """The S x b x gamma sweep on the 128K generator (Hq=32, Hkv=8)."""
    out = []
    for S in (4096, 16384, 65536, 131072):
        for b in (128, 256):
            for gamma in (0.8, 0.9, 0.95, 1.0):
                out.append(Workload(f"sweep_S{S}_b{b}_g{gamma}", S=S, Hq=32, Hkv=8, b=b, gamma=gamma,
                                    n_vertical=64, n_topics=32, seed=2))
    return out


def rope_tables(S: int, d: int, theta: float = ROPE_THETA):
    """cos/sin of the rotary angles p * theta^(-2i/d), p in [0, S), i in [0, d/2),
    evaluated in float64 and rounded to float32: two [S][d/2] tensors."""
    half = d // 2
    inv = theta ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / d)
    ang = torch.arange(S, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def rope_(x: torch.Tensor, theta: float = ROPE_THETA) -> torch.Tensor:
    """In-place rotate-half rotary embedding of x[H][S][d] (fp32), positions 0..S-1."""
    H, S, d = x.shape
    half = d // 2
    cos, sin = rope_tables(S, d, theta)
    for h in range(H):
        x1 = x[h, :, :half].clone()
        x2 = x[h, :, half:].clone()
        x[h, :, :half] = x1 * cos - x2 * sin
        x[h, :, half:] = x2 * cos + x1 * sin
    return x


def quantize_per_head(x_bf16: torch.Tensor):
    """Symmetric per-head int8: scale = max|x|/127, round half to even, clamp +-127."""
    H = x_bf16.shape[0]
    scales = torch.empty(H, dtype=torch.float32)
    out = torch.empty(x_bf16.shape, dtype=torch.int8)
    for h in range(H):
        xf = x_bf16[h].to(torch.float32)
        s = xf.abs().max() / 127.0
        if float(s) == 0.0:
            s = torch.tensor(1.0)
        scales[h] = s
        out[h] = torch.clamp(torch.round(xf / s), -127, 127).to(torch.int8)
    return out, scales


def make_inputs(w: Workload):
    """Build the seeded CPU tensors of workload ``w``.

    Returns a dict with q, k, v (bf16, [H][S][d] contiguous), ``kinds`` and,
    when ``w.int8``, q8/k8 (int8) and q_scale/k_scale (fp32 per head).
    """
    S, Hq, Hkv, d = w.S, w.Hq, w.Hkv, w.d
    assert Hq % Hkv == 0
    g = Hq // Hkv
    kinds = w.head_kinds()
    gen = torch.Generator().manual_seed(int(w.seed))
    q = torch.randn((Hq, S, d), generator=gen, dtype=torch.float32)
    k = torch.randn((Hkv, S, d), generator=gen, dtype=torch.float32)
    v = torch.randn((Hkv, S, d), generator=gen, dtype=torch.float32)
    for j in range(Hkv):
        heads = list(range(j * g, (j + 1) * g))
        if any(kinds[h] == "qa" for h in heads):
            topic = torch.randint(0, w.n_topics, (S,), generator=gen)
            cent = torch.randn((w.n_topics, d), generator=gen, dtype=torch.float32)
            tv = 2.0 * cent[topic]
            k[j] += tv
            for h in heads:
                if kinds[h] == "qa":
                    q[h] += tv
            del tv
    rope_(q)
    rope_(k)
    for h in range(Hq):
        if kinds[h] != "vs":
            continue
        mu = q[h].to(torch.float64).mean(dim=0)
        nrm = float(mu.norm())
        mu = (mu / nrm if nrm > 0 else mu).to(torch.float32)
        extra = torch.randperm(max(S - 4, 0), generator=gen)[: min(w.n_vertical, max(S - 4, 0))] + 4
        pos = torch.cat([torch.arange(min(4, S)), extra])
        k[h // g, pos] += 3.0 * mu
    if w.key_ramp:
        k *= (1.0 + w.key_ramp * torch.arange(S, dtype=torch.float32) / S)[None, :, None]
    out = {
        "q": q.to(torch.bfloat16).contiguous(),
        "k": k.to(torch.bfloat16).contiguous(),
        "v": v.to(torch.bfloat16).contiguous(),
        "kinds": kinds,
    }
    del q, k, v
    if w.int8:
        out["q8"], out["q_scale"] = quantize_per_head(out["q"])
        out["k8"], out["k_scale"] = quantize_per_head(out["k"])
    return out


def dense_equiv_flops(S: int, Hq: int, d: int) -> float:
    """Causal dense attention FLOPs, 4*Hq*S^2*d/2 (two GEMMs over the lower triangle)."""
    return 2.0 * Hq * d * float(S) * float(S)


def make_prerope_inputs(w: Workload) -> dict:
    """Q and K before the rotary embedding (as a projection's epilogue sees
    them), V, and the rotary tables: q_in [Hq][S][d], k_in [Hkv][S][d] and v
    bf16 (N(0,1), with the topic structure of the query-aware heads), cos/sin
    [S][d/2] float32.  Seeded like make_inputs."""
    S, Hq, Hkv, d = w.S, w.Hq, w.Hkv, w.d
    g = Hq // Hkv
    gen = torch.Generator().manual_seed(10_000 + w.seed)
    q = torch.randn((Hq, S, d), generator=gen, dtype=torch.float32)
    k = torch.randn((Hkv, S, d), generator=gen, dtype=torch.float32)
    v = torch.randn((Hkv, S, d), generator=gen, dtype=torch.float32)
    for kv in range(Hkv):
        topic = torch.randint(0, w.n_topics, (S,), generator=gen)
        cent = torch.randn((w.n_topics, d), generator=gen, dtype=torch.float32)
        k[kv] += 2.0 * cent[topic]
        for h in range(kv * g, kv * g + g):
            if h % 2:
                q[h] += 2.0 * cent[topic]
    cos, sin = rope_tables(S, d)
    return {"q_in": q.to(torch.bfloat16), "k_in": k.to(torch.bfloat16), "v": v.to(torch.bfloat16),
            "cos": cos, "sin": sin}
