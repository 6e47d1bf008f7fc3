"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Index sets, per-head statistics and patterns are compared in full; attention
outputs on every tile for the small layers and on seeded samples of tiles
(at the launch configuration the benchmark times) for the 32K and 128K
layers.  Tolerances are listed in tests/parity.py.
"""
import math
import random

import numpy as np
import pytest
import torch

from dynamic_block_sparse_last_b200 import synth
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import fp as mod
    assert torch.cuda.is_available(), "CUDA device required"
    return mod


def run_gpu(fp, x, w):
    dev = torch.device("cuda:0")
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    if w.int8:
        qq, kk = x["q8"].to(dev), x["k8"].to(dev)
        qs, ks = x["q_scale"].to(dev), x["k_scale"].to(dev)
        dt = fp.FP_QK_INT8
    else:
        qq, kk, qs, ks, dt = q, k, None, None, fp.FP_QK_BF16
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    fp.fp_build_index(qq, kk, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, dt, qs, ks, idx)
    out = torch.empty_like(q)
    fp.fp_sparse_attn(qq, kk, v, qs, ks, idx, out)
    torch.cuda.synchronize()
    assert fp.fp_get_device_error() == fp.FP_OK
    exp = fp.fp_index_export(idx)
    return exp, out, idx


def oracle_problem(x, w):
    if w.int8:
        return orc.OracleProblem(x["q"], x["k"], x["v"], w.b, q8=x["q8"], k8=x["k8"],
                                 q_scale=x["q_scale"], k_scale=x["k_scale"])
    return orc.OracleProblem(x["q"], x["k"], x["v"], w.b)


def nblocks(S, b):
    return -(-S // b)


def check_index(P, exp, w):
    n = nblocks(w.S, w.b)
    heads = parity.run_parallel(lambda h: P.build_index_head(h, w.gamma, w.tau), range(w.Hq))
    stats = parity.compare_index(exp, heads, n, w.gamma, w.tau,
                                 oracle_forced=lambda h, pat: P.build_index_head(h, w.gamma, w.tau, pat))
    print(f"[{w.name}] index: {stats}; patterns {exp['pattern'].tolist()}; "
          f"density {exp['nnz'] / (w.Hq * n * (n + 1) / 2):.4f}")
    return heads, stats


def check_tiles(P, exp, out, w, tiles):
    """Query tiles (h, qc) of 128 rows; the last one stops at S."""
    n = nblocks(w.S, w.b)

    def one(t):
        # the tile's rows, query block by query block (two blocks per tile when b = 64)
        h, qc = t
        lo, hi = qc * 128, min(qc * 128 + 128, w.S)
        lists = parity.gpu_rows(exp, h, n)
        parts = []
        for r in range(lo // w.b, (hi - 1) // w.b + 1):
            a, z = max(lo, r * w.b), min(hi, (r + 1) * w.b)
            parts.append(P.attn_rows(h, a, z, lists[r]))
        return np.concatenate(parts, 0)

    refs = parity.run_parallel(one, tiles)
    worst_max, sum_mean = 0.0, 0.0
    for (h, qc), ref in zip(tiles, refs):
        got = out[h, qc * 128: min(qc * 128 + 128, w.S)].float().cpu().numpy()
        mx, mean = parity.compare_tile(got, ref)
        assert mx <= parity.OUT_MAX_ABS and mean <= parity.OUT_MEAN_ABS, (h, qc, mx, mean)
        worst_max = max(worst_max, mx)
        sum_mean += mean
    print(f"[{w.name}] {len(tiles)} tiles: worst max-abs {worst_max:.3e}, mean of mean-abs "
          f"{sum_mean / len(tiles):.3e}")


SMALL = [
    synth.WORKLOADS["tiny"],
    synth.Workload("g3_b256", S=2048, Hq=6, Hkv=2, b=256, seed=3),
    synth.Workload("g1_gamma08", S=1536, Hq=4, Hkv=4, b=128, gamma=0.8, seed=4),
    synth.Workload("g4_gamma095", S=4096, Hq=8, Hkv=2, b=128, gamma=0.95, seed=5),
    synth.Workload("gamma1_b256", S=512, Hq=4, Hkv=1, b=256, gamma=1.0, seed=6),
    synth.Workload("one_block", S=128, Hq=2, Hkv=1, b=128, seed=7),
    synth.Workload("one_block_b256", S=256, Hq=2, Hkv=2, b=256, seed=8),
    synth.Workload("two_blocks_tau0", S=256, Hq=2, Hkv=1, b=128, tau=0.0, seed=12),
    synth.Workload("int8_small", S=2048, Hq=4, Hkv=2, b=128, int8=True, seed=9),
    synth.Workload("int8_b256", S=2048, Hq=4, Hkv=1, b=256, gamma=0.95, int8=True, seed=10),
    # lengths that b (and 128) do not divide: a partial last block
    synth.Workload("ragged_b128", S=1000, Hq=4, Hkv=2, b=128, seed=16),
    synth.Workload("ragged_b256_short_tail", S=1300, Hq=6, Hkv=2, b=256, seed=17),
    synth.Workload("ragged_b256_long_tail", S=1500, Hq=4, Hkv=1, b=256, gamma=0.95, seed=18),
    synth.Workload("ragged_one_row_tail", S=129, Hq=2, Hkv=1, b=128, seed=19),
    synth.Workload("ragged_single_block", S=77, Hq=2, Hkv=2, b=256, seed=20),
    synth.Workload("ragged_int8", S=2000, Hq=4, Hkv=2, b=128, int8=True, seed=21),
    synth.Workload("ragged_int8_b256", S=1800, Hq=4, Hkv=2, b=256, gamma=0.95, int8=True, seed=22),
    # block size 64: two query blocks per 128-row tile, two key blocks per chunk
    synth.Workload("b64", S=1024, Hq=4, Hkv=2, b=64, seed=24),
    synth.Workload("b64_ragged", S=1000, Hq=4, Hkv=2, b=64, gamma=0.95, seed=25),
    synth.Workload("b64_odd_blocks", S=1088, Hq=2, Hkv=1, b=64, seed=26),
    synth.Workload("b64_g1", S=1536, Hq=2, Hkv=2, b=64, gamma=0.8, seed=27),
    synth.Workload("b64_int8", S=2048, Hq=4, Hkv=2, b=64, int8=True, seed=28),
    # degenerate lengths: one token, three tokens, exactly one block of 64
    synth.Workload("S1", S=1, Hq=2, Hkv=1, b=128, seed=33),
    synth.Workload("S3_b64", S=3, Hq=2, Hkv=2, b=64, seed=34),
    synth.Workload("S64_b64", S=64, Hq=4, Hkv=2, b=64, seed=35),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_layers_full_parity(fp, w):
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    tiles = [(h, qc) for h in range(w.Hq) for qc in range(nblocks(w.S, 128))]
    check_tiles(P, exp, out, w, tiles)


DENSE = [synth.Workload("dense", S=2048, Hq=8, Hkv=2, b=128, gamma=1.0, seed=13),
         synth.Workload("sweep_gen_b128", S=4096, Hq=32, Hkv=8, b=128, gamma=1.0, n_vertical=64, n_topics=32,
                        seed=2),
         synth.Workload("sweep_gen_b256", S=4096, Hq=32, Hkv=8, b=256, gamma=1.0, n_vertical=64, n_topics=32,
                        seed=2),
         synth.Workload("dense_ragged_b128", S=1234, Hq=8, Hkv=2, b=128, gamma=1.0, seed=23),
         synth.Workload("dense_ragged_b256", S=1234, Hq=8, Hkv=2, b=256, gamma=1.0, seed=23),
         synth.Workload("dense_ragged_b64", S=1234, Hq=8, Hkv=2, b=64, gamma=1.0, seed=23)]


@pytest.mark.parametrize("w", DENSE, ids=[w.name for w in DENSE])
def test_gamma_one_matches_dense_sdpa(fp, w):
    """gamma = 1 keeps every causal block: the output is dense causal attention
    (checked against torch SDPA in fp32 on the GPU)."""
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    n = nblocks(w.S, w.b)
    g = w.Hq // w.Hkv
    assert exp["nnz"] == w.Hq * n * (n + 1) // 2
    q, k, v = (x[t].cuda().float() for t in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None], k.repeat_interleave(g, 0)[None], v.repeat_interleave(g, 0)[None], is_causal=True)[0]
    diff = (out.float() - ref).abs()
    assert float(diff.max()) <= parity.OUT_MAX_ABS and float(diff.mean()) <= parity.OUT_MEAN_ABS


def test_int8_score_tiles_bit_exact(fp):
    w = synth.Workload("i8tiles", S=1024, Hq=4, Hkv=2, b=128, int8=True, seed=14)
    x = synth.make_inputs(w)
    P = oracle_problem(x, w)
    q8, k8 = x["q8"].cuda(), x["k8"].cuda()
    out = torch.empty(128, 128, dtype=torch.int32, device="cuda")
    for h, p0, j0 in [(0, 0, 0), (1, 896, 0), (2, 512, 384), (3, 896, 896)]:
        fp.fp_debug_qk_tile_i8(q8, k8, w.S, w.Hq, w.Hkv, w.d, h, p0, j0, out)
        torch.cuda.synchronize()
        ref = P.qk_int_tile(h, p0, j0, 128, 128)
        assert np.array_equal(out.cpu().numpy(), ref), (h, p0, j0)


def attended_chunks(exp, h, qc, w):
    """128-key chunks the attention kernel computes for query tile qc of head
    h: the chunks of the tile's listed blocks up to the tile itself (with
    b = 64 the tile holds two query blocks and a chunk two key blocks)."""
    n = nblocks(w.S, w.b)
    lists = parity.gpu_rows(exp, h, n)
    if w.b >= 128:
        per, r = w.b // 128, qc * 128 // w.b
        return sorted({int(c) * per + k for c in lists[r] for k in range(per) if int(c) * per + k <= qc})
    return sorted({int(c) // 2 for r in (2 * qc, 2 * qc + 1) if r < n for c in lists[r] if int(c) // 2 <= qc})


def check_production_int8_tiles(fp, w, x, P, idx, score_cases, attn_tiles, dev):
    """Captures raw int32 score tiles from the production int8 kernels (the
    index pass's last-block scores and the attention's score tiles) on their
    normal launch paths and compares each bit for bit with the oracle's exact
    integer products (first article, section 3.3).  Rows past S (a short last
    block) are not compared."""
    q8, k8 = x["q8"].to(dev), x["k8"].to(dev)
    qs, ks, v = x["q_scale"].to(dev), x["k_scale"].to(dev), x["v"].to(dev)
    cap = torch.empty(128, 128, dtype=torch.int32, device=dev)
    n = nblocks(w.S, w.b)
    p_last = (n - 1) * w.b
    checked = 0
    try:
        for h, sl, ch in score_cases:
            cap.fill_(-(2 ** 31))
            fp.fp_debug_capture_i8(0, h, sl, ch, cap)
            fp.fp_build_index(q8, k8, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_INT8, qs, ks, idx)
            torch.cuda.synchronize()
            fp.fp_debug_capture_i8(0, 0, 0, 0, None)
            p0 = p_last + 128 * sl
            rows, cols = min(128, w.S - p0), min(128, w.S - 128 * ch)
            ref = P.qk_int_tile(h, p0, 128 * ch, rows, cols)
            assert np.array_equal(cap[:rows, :cols].cpu().numpy(), ref), ("score", h, sl, ch)
            checked += 1
        fp.fp_build_index(q8, k8, w.S, w.Hq, w.Hkv, w.d, w.b, w.gamma, w.tau, fp.FP_QK_INT8, qs, ks, idx)
        exp = fp.fp_index_export(idx)
        out = torch.empty(w.Hq, w.S, w.d, dtype=torch.bfloat16, device=dev)
        for h, qc in attn_tiles:
            chunks = attended_chunks(exp, h, qc, w)
            for kc in sorted({chunks[0], chunks[len(chunks) // 2], chunks[-1]}):
                cap.fill_(-(2 ** 31))
                fp.fp_debug_capture_i8(1, h, qc, kc, cap)
                fp.fp_sparse_attn(q8, k8, v, qs, ks, idx, out)
                torch.cuda.synchronize()
                fp.fp_debug_capture_i8(1, 0, 0, 0, None)
                rows, cols = min(128, w.S - 128 * qc), min(128, w.S - 128 * kc)
                ref = P.qk_int_tile(h, 128 * qc, 128 * kc, rows, cols)
                assert np.array_equal(cap[:rows, :cols].cpu().numpy(), ref), ("attn", h, qc, kc)
                checked += 1
    finally:
        fp.fp_debug_capture_i8(0, 0, 0, 0, None)
        fp.fp_debug_capture_i8(1, 0, 0, 0, None)
    assert fp.fp_get_device_error() == fp.FP_OK
    print(f"[{w.name}] {checked} production int8 score tiles bit-exact")


INT8_CAPTURE = [synth.Workload("i8cap_b128", S=4096, Hq=8, Hkv=2, b=128, int8=True, seed=41),
                synth.Workload("i8cap_b256", S=4096, Hq=4, Hkv=1, b=256, int8=True, seed=42),
                synth.Workload("i8cap_b64_ragged", S=2000, Hq=4, Hkv=2, b=64, int8=True, seed=43)]


@pytest.mark.parametrize("w", INT8_CAPTURE, ids=[w.name for w in INT8_CAPTURE])
def test_int8_production_score_tiles_bit_exact(fp, w):
    x = synth.make_inputs(w)
    P = oracle_problem(x, w)
    idx = fp.fp_index_create(w.S, w.Hq, w.Hkv, w.d, w.b)
    n, nch = nblocks(w.S, w.b), nblocks(w.S, 128)
    slices = nblocks(w.S - (n - 1) * w.b, 128)
    score_cases = [(0, 0, 0), (w.Hq - 1, slices - 1, nch - 1), (w.Hq // 2, slices - 1, nch // 2), (1, 0, 1)]
    attn_tiles = [(1, nch - 1), (w.Hq - 1, nch // 2), (0, 3)]
    check_production_int8_tiles(fp, w, x, P, idx, score_cases, attn_tiles, torch.device("cuda:0"))
    idx.free()


def test_bounded_wait_reports_timeout_and_context_survives(fp):
    fp.fp_debug_wait_timeout(200000)
    assert fp.fp_get_device_error() == fp.FP_ERR_TIMEOUT
    assert fp.fp_get_device_error() == fp.FP_OK
    w = synth.Workload("after_timeout", S=256, Hq=2, Hkv=1, b=128, seed=15)
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    assert exp["nnz"] >= w.Hq * (w.S // w.b)


def sampled_tiles(w, count, seed):
    rng = random.Random(seed)
    nq = nblocks(w.S, 128)
    tiles = {(h, nq - 1) for h in range(0, w.Hq, max(1, w.Hq // 4))}      # longest rows
    while len(tiles) < count:
        tiles.add((rng.randrange(w.Hq), rng.randrange(nq)))
    return sorted(tiles)


@pytest.mark.parametrize("name,ntiles", [("llama3b", 64), ("llama8b", 64), ("llama8b_w8a8", 64)])
def test_full_size_layers(fp, name, ntiles):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    check_tiles(P, exp, out, w, sampled_tiles(w, ntiles, seed=w.seed))
    if w.int8:
        nch = nblocks(w.S, 128)
        check_production_int8_tiles(fp, w, x, P, idx, [(0, 0, 0), (31, 0, nch - 1), (17, 0, 512)],
                                    [(31, nch - 1), (17, 512), (2, 40)], torch.device("cuda:0"))


LARGE_N = [synth.Workload("b64_n1024", S=65536, Hq=8, Hkv=2, b=64, n_vertical=64, n_topics=32, seed=31),
           synth.Workload("b256_S131072", S=131072, Hq=8, Hkv=2, b=256, n_vertical=64, n_topics=32, seed=32),
           # the q-bar . k-bar logits switch from the FMA form to the tensor cores at n = 640:
           # a ragged n above it (partial last row band of 128 x 128 tiles, partial last block)
           # and n just below
           synth.Workload("logits_tc_n700_ragged", S=89550, Hq=8, Hkv=2, b=128, n_vertical=64, n_topics=32,
                          seed=40),
           synth.Workload("logits_fma_n639", S=81792, Hq=8, Hkv=2, b=128, n_vertical=64, n_topics=32, seed=41)]


@pytest.mark.parametrize("w", LARGE_N, ids=[w.name for w in LARGE_N])
def test_largest_block_counts(fp, w):
    """The largest index a block size allows or the longest layer at b = 256:
    n = 1024 blocks of 64 (every key-block bit of the attention bitmaps in
    use) and S = 131072 at b = 256; and the two sides of the logits kernels'
    switch (n = 700 ragged on the tensor cores, n = 639 on the FMA pipe);
    full index, 32 sampled tiles."""
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    check_tiles(P, exp, out, w, sampled_tiles(w, 32, seed=w.seed))


def test_batched_sequences_equal_separate_calls(fp):
    """B sequences of equal length run as one call with B*Hq / B*Hkv heads
    (stacked sequence-major) and give bit-identical index and output."""
    ws = [synth.Workload(f"seq{i}", S=2048, Hq=4, Hkv=2, b=128, seed=30 + i) for i in range(2)]
    xs = [synth.make_inputs(w) for w in ws]
    single = [run_gpu(fp, x, w) for x, w in zip(xs, ws)]
    xb = {key: torch.cat([x[key] for x in xs], 0) for key in ("q", "k", "v")}
    wb = synth.Workload("batch2", S=2048, Hq=8, Hkv=4, b=128, seed=0)
    exp_b, out_b, _ = run_gpu(fp, xb, wb)
    n = wb.S // wb.b
    for i, (exp, out, _) in enumerate(single):
        assert torch.equal(out_b[4 * i: 4 * i + 4], out)
        assert np.array_equal(exp_b["pattern"][4 * i: 4 * i + 4], exp["pattern"])
        for h in range(4):
            rows_b = parity.gpu_rows(exp_b, 4 * i + h, n)
            rows_s = parity.gpu_rows(exp, h, n)
            assert all(np.array_equal(a, c) for a, c in zip(rows_b, rows_s))


# The S x b x gamma sweep on the 128K generator (Hq=32, Hkv=8): the points the
# other tests do not already cover at this head count.
SWEEP_BY_NAME = {w.name: w for w in synth.sweep_workloads()}
SWEEP_GAMMA1 = ["sweep_S16384_b128_g1.0", "sweep_S65536_b128_g1.0", "sweep_S131072_b128_g1.0",
                "sweep_S131072_b256_g1.0"]
SWEEP_B256 = ["sweep_S16384_b256_g0.8", "sweep_S16384_b256_g0.95", "sweep_S131072_b256_g0.8",
              "sweep_S131072_b256_g0.95"]


@pytest.mark.parametrize("name", SWEEP_GAMMA1)
def test_sweep_gamma_one_is_dense_causal(fp, name):
    """gamma = 1 keeps every causal block, so the layer is dense causal
    attention: the index holds Hq n(n+1)/2 blocks, and 64 seeded query tiles
    (the longest rows of several heads among them) equal the oracle's dense
    causal attention."""
    w = SWEEP_BY_NAME[name]
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    n = nblocks(w.S, w.b)
    assert exp["nnz"] == w.Hq * n * (n + 1) // 2
    for h in range(w.Hq):
        rows = parity.gpu_rows(exp, h, n)
        assert all(len(r) == i + 1 for i, r in enumerate(rows)), h
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    check_tiles(P, exp, out, w, sampled_tiles(w, 64, seed=w.seed + w.S))


@pytest.mark.parametrize("name", SWEEP_B256)
def test_sweep_b256_gammas(fp, name):
    """b = 256 at gamma 0.8 and 0.95 on the 128K generator: the full index
    against the oracle, and query tiles against the oracle on the GPU's index
    (every tile at S = 16K, 64 seeded tiles at S = 128K)."""
    w = SWEEP_BY_NAME[name]
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    nq = nblocks(w.S, 128)
    tiles = [(h, qc) for h in range(w.Hq) for qc in range(nq)] if w.S <= 16384 else \
        sampled_tiles(w, 64, seed=w.seed + w.S)
    check_tiles(P, exp, out, w, tiles)


REF_SUM, REF_HEADROOM = 256.0, 64.0  # the attention kernel's kRefSum and kRefHeadroom


def reference_moves(x, w, heads):
    """How often the softmax's reference max must move after a row's first
    chunk, by the rule the attention kernel applies (the chunk's row sum of
    2^(x - m) above REF_SUM, x = q.k log2(e) / sqrt(d); a moved reference is
    the row max plus REF_HEADROOM), evaluated in fp64 on the bf16 inputs at
    gamma = 1 (every causal key).  Used to show that a case exercises the
    recompute path; the kernel's own sums are of bf16-rounded exponentials,
    so its count can differ slightly."""
    g = w.Hq // w.Hkv
    c = math.log2(math.e) / math.sqrt(w.d)
    moves = 0
    for h in heads:
        q = x["q"][h].double().numpy()
        k = x["k"][h // g].double().numpy()
        sc = (q @ k.T) * c
        for i in range(w.S):
            m = -math.inf
            for c0 in range(0, i + 1, 128):
                xs = sc[i, c0:min(i + 1, c0 + 128)]
                if m == -math.inf:
                    m = float(xs.max()) + REF_HEADROOM
                    continue
                with np.errstate(over="ignore"):
                    total = float(np.exp2(xs - m).sum())
                if not total <= REF_SUM:
                    m = max(m, float(xs.max()) + REF_HEADROOM)
                    moves += 1
    return moves


RAMP = [synth.Workload("ramp_b128", S=2048, Hq=4, Hkv=1, b=128, gamma=1.0, key_ramp=80.0, seed=31),
        synth.Workload("ramp_int8", S=2048, Hq=4, Hkv=1, b=128, gamma=1.0, key_ramp=80.0, int8=True, seed=31),
        synth.Workload("ramp_b64_ragged", S=1500, Hq=4, Hkv=2, b=64, gamma=1.0, key_ramp=80.0, seed=32),
        synth.Workload("ramp_b256", S=2048, Hq=4, Hkv=2, b=256, gamma=1.0, key_ramp=80.0, seed=32),
        # gamma < 1: the selection itself depends on the statistics the moved references produce
        synth.Workload("ramp_b128_gamma09", S=2048, Hq=4, Hkv=2, b=128, gamma=0.9, key_ramp=80.0, seed=33)]


@pytest.mark.parametrize("w", RAMP, ids=[w.name for w in RAMP])
def test_rising_scores_move_the_reference(fp, w):
    """Keys scaled up along the sequence make every row's maximum grow from
    chunk to chunk, so the softmax's reference has to move (and its chunk be
    recomputed, and O rescaled) many times per row, and so does the score
    kernel's per-row reference.  The index (statistics, pattern and block
    sets) is compared with the oracle, and every tile on the GPU's index."""
    x = synth.make_inputs(w)
    exp, out, idx = run_gpu(fp, x, w)
    n = nblocks(w.S, w.b)
    if w.gamma >= 1.0:
        assert exp["nnz"] == w.Hq * n * (n + 1) // 2
    moves = reference_moves(x, w, [0])
    print(f"[{w.name}] reference moves after the first chunk, head 0: {moves} over {w.S} rows")
    assert moves >= w.S  # more than one per row on average
    P = oracle_problem(x, w)
    check_index(P, exp, w)
    tiles = [(h, qc) for h in range(w.Hq) for qc in range(nblocks(w.S, 128))]
    check_tiles(P, exp, out, w, tiles)
