"""Parity at the workloads' full sizes, in the launch configurations the bench uses.

Inputs are drawn on the GPU by the seeded generator (the same module the CPU tests use);
the oracle recomputes what it can afford: every score of a query, full top-k, full
attention outputs of a few queries, and sampled compressed entries.  Tolerances are the
ones of test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import long_context_compressed_csa_b200 as lib
from long_context_compressed_csa_b200.synth import randn, to_f64
from tests.helpers import check_topk_sets, max_rel_rowwise, score_error_bound

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16 = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_compressed_csa_b200 import build
    build.build()


def zeros_ws(nbytes):
    return torch.zeros(nbytes, dtype=torch.uint8, device=DEV)


def check_sampled_csa_entries(S, cache, m, entries, batches):
    for b in batches:
        for i in entries:
            lo = max(0, m * (i - 1))
            rows = [to_f64(x[b, lo:m * (i + 1)]) for x in S]
            ref = oracle.csa_compress(*rows, m, i0=i - lo // m, i1=i - lo // m + 1) if i > 0 else \
                oracle.csa_compress(*rows, m, i0=0, i1=1)
            got = to_f64(cache[b, i:i + 1])
            assert max_rel_rowwise(got, ref).max() <= 2e-2, (b, i)


def run_indexer(qI, wI, KI, t, m, k):
    B, nq = qI.shape[:2]
    idx = torch.empty((B, nq, k), dtype=torch.int32, device=DEV)
    sc = torch.empty((B, nq, k), dtype=torch.float32, device=DEV)
    ws = zeros_ws(lib.csa_indexer_topk_workspace_size(B, nq, KI.shape[1], k))
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    lib.csa_indexer_topk(qI, wI, KI, tt, m, k, idx, ws, scores_out=sc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


def check_indexer(qI, wI, KI, t, m, k, idx, sc, b, q):
    vis = oracle.visible(t, m, KI.shape[1])
    q64, w64 = to_f64(qI[b, q]), to_f64(wI[b, q])
    K64 = to_f64(KI[b, :vis])
    s = oracle.index_scores(q64, w64, K64, vis)
    check_topk_sets(idx[b, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
    got = idx[b, q][idx[b, q] >= 0]
    band = score_error_bound(q64, w64, K64, got) + 1e-6 * np.abs(s[got])
    assert np.all(np.abs(sc[b, q][:len(got)] - s[got]) <= band)


def test_csa_decode_8k_full():
    """B=1, n=8192, m=4 -> 2048 entries, c=512, c^I=128, k=512, n_h=128, n_h^I=64."""
    B, n, m, c, cI, k, n_h, n_hI = 1, 8192, 4, 512, 128, 512, 128, 64
    S = [randn((B, n, c), 1100 + i, BF16, DEV) for i in range(4)]
    SI = [randn((B, n, cI), 1110 + i, BF16, DEV) for i in range(4)]
    N = n // m
    cache = torch.empty((B, N, c), dtype=BF16, device=DEV)
    kI = torch.empty((B, N, cI), dtype=BF16, device=DEV)
    lib.csa_compress(*S, cache, m)
    lib.csa_compress(*SI, kI, m)
    torch.cuda.synchronize()
    ref = oracle.csa_compress(*(to_f64(x[0]) for x in S), m)
    assert max_rel_rowwise(to_f64(cache[0]), ref).max() <= 2e-2
    refI = oracle.csa_compress(*(to_f64(x[0]) for x in SI), m)
    assert max_rel_rowwise(to_f64(kI[0]), refI).max() <= 2e-2
    qI = randn((B, 1, n_hI, cI), 1120, BF16, DEV)
    wI = randn((B, 1, n_hI), 1121, torch.float32, DEV)
    q = randn((B, 1, n_h, c), 1122, BF16, DEV)
    idx, sc = run_indexer(qI, wI, kI, [n], m, k)
    check_indexer(qI, wI, kI, n, m, k, idx, sc, 0, 0)
    o = torch.empty((B, 1, n_h, c), dtype=torch.float32, device=DEV)
    ws = zeros_ws(lib.csa_attn_workspace_size(B, 1, n_h, c, k))
    lib.csa_sparse_attn(q, cache, torch.from_numpy(idx).to(DEV), o, ws)
    torch.cuda.synchronize()
    ref_o, _ = oracle.mqa(to_f64(q[0, 0]), to_f64(cache[0]), idx[0, 0])
    assert max_rel_rowwise(o[0, 0].cpu().numpy(), ref_o).max() <= 2e-2


def test_hca_b16_128k_full():
    """B=16, n=131072, m'=128 -> 1024 entries per sequence; compress + dense decode."""
    B, n, mp, c, n_h = 16, 131072, 128, 512, 128
    C = randn((B, n, c), 1200, BF16, DEV)
    Z = randn((B, n, c), 1201, BF16, DEV)
    N = n // mp
    cache = torch.empty((B, N, c), dtype=BF16, device=DEV)
    lib.hca_compress(C, Z, cache, mp)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1202)
    for b in (0, 7, 15):
        for i in rng.choice(N, 4, replace=False):
            ref = oracle.hca_compress(to_f64(C[b, mp * i:mp * (i + 1)]), to_f64(Z[b, mp * i:mp * (i + 1)]), mp)
            assert max_rel_rowwise(to_f64(cache[b, i:i + 1]), ref).max() <= 2e-2
    del C, Z
    q = randn((B, 1, n_h, c), 1203, BF16, DEV)
    o = torch.empty((B, 1, n_h, c), dtype=torch.float32, device=DEV)
    ws = zeros_ws(lib.csa_attn_workspace_size(B, 1, n_h, c, N))
    t = torch.full((B, 1), n, dtype=torch.int64, device=DEV)
    lib.hca_dense_attn(q, cache, t, mp, o, ws)
    torch.cuda.synchronize()
    for b in (0, 5, 15):
        ref_o, _ = oracle.mqa(to_f64(q[b, 0]), to_f64(cache[b]), np.arange(N, dtype=np.int32))
        assert max_rel_rowwise(o[b, 0].cpu().numpy(), ref_o).max() <= 2e-2


def test_csa_b4_256k_prefill_and_decode():
    """B=4, n=262144 -> 65536 entries, k=1024; then decode steps with incremental
    compression of both caches at the block boundary."""
    B, n, m, c, cI, k, n_h, n_hI = 4, 262144, 4, 512, 128, 1024, 128, 64
    steps = 8
    N = n // m
    N_cap = N + steps // m + 1
    S = [randn((B, n + steps, c), 1300 + i, BF16, DEV) for i in range(4)]
    SI = [randn((B, n + steps, cI), 1310 + i, BF16, DEV) for i in range(4)]
    cache = torch.empty((B, N_cap, c), dtype=BF16, device=DEV)
    kI = torch.empty((B, N_cap, cI), dtype=BF16, device=DEV)
    lib.csa_compress(*(x[:, :n] for x in S), cache, m)
    lib.csa_compress(*(x[:, :n] for x in SI), kI, m)
    torch.cuda.synchronize()
    check_sampled_csa_entries(S, cache, m, [0, 1, 12345, N - 1], [0, 3])
    check_sampled_csa_entries(SI, kI, m, [0, 777, N - 1], [1, 2])
    qI = randn((B, 1, n_hI, cI), 1320, BF16, DEV)
    wI = randn((B, 1, n_hI), 1321, torch.float32, DEV)
    q = randn((B, 1, n_h, c), 1322, BF16, DEV)
    o = torch.empty((B, 1, n_h, c), dtype=torch.float32, device=DEV)
    ws_a = zeros_ws(lib.csa_attn_workspace_size(B, 1, n_h, c, k))
    for step in range(steps):
        t = n + step
        idx, sc = run_indexer(qI, wI, kI, [t] * B, m, k)
        if step in (0, steps - 1):
            for b in (0, 3):
                check_indexer(qI, wI, kI, t, m, k, idx, sc, b, 0)
            lib.csa_sparse_attn(q, cache, torch.from_numpy(idx).to(DEV), o, ws_a)
            torch.cuda.synchronize()
            for b in (0, 2):
                ref_o, _ = oracle.mqa(to_f64(q[b, 0]), to_f64(cache[b]), idx[b, 0])
                assert max_rel_rowwise(o[b, 0].cpu().numpy(), ref_o).max() <= 2e-2
        if (t + 1) % m == 0:  # token t completes block i: append entry i to both caches
            i = (t + 1) // m - 1
            lo = m * (i - 1)
            lib.csa_compress(*(x[:, lo:m * (i + 1)] for x in S), cache, m, i, i + 1, tok0=lo)
            lib.csa_compress(*(x[:, lo:m * (i + 1)] for x in SI), kI, m, i, i + 1, tok0=lo)
            torch.cuda.synchronize()
            check_sampled_csa_entries(S, cache, m, [i], [0, 1, 2, 3])
            check_sampled_csa_entries(SI, kI, m, [i], [0, 3])


def test_hybrid_1m_decode_step():
    """B=1, n=2^20: CSA indexer over 262144 keys, top-1024, sparse MQA; HCA dense MQA over
    8192 entries - the bench's per-token step, checked in full against the oracle."""
    n, m, mp, c, cI, k, n_h, n_hI = 1 << 20, 4, 128, 512, 128, 1024, 128, 64
    N, Nh = n // m, n // mp
    kI = randn((1, N, cI), 1400, BF16, DEV, scale=0.5)
    cache = randn((1, N, c), 1401, BF16, DEV, scale=0.5)
    hcache = randn((1, Nh, c), 1402, BF16, DEV, scale=0.5)
    qI = randn((1, 1, n_hI, cI), 1403, BF16, DEV)
    wI = randn((1, 1, n_hI), 1404, torch.float32, DEV)
    q = randn((1, 1, n_h, c), 1405, BF16, DEV)
    idx, sc = run_indexer(qI, wI, kI, [n], m, k)
    check_indexer(qI, wI, kI, n, m, k, idx, sc, 0, 0)
    o = torch.empty((1, 1, n_h, c), dtype=torch.float32, device=DEV)
    lib.csa_sparse_attn(q, cache, torch.from_numpy(idx).to(DEV), o,
                        zeros_ws(lib.csa_attn_workspace_size(1, 1, n_h, c, k)))
    oh = torch.empty_like(o)
    t = torch.full((1, 1), n, dtype=torch.int64, device=DEV)
    lib.hca_dense_attn(q, hcache, t, mp, oh, zeros_ws(lib.csa_attn_workspace_size(1, 1, n_h, c, Nh)))
    torch.cuda.synchronize()
    sel = idx[0, 0]
    ref_o, _ = oracle.mqa(to_f64(q[0, 0]), to_f64(cache[0, torch.from_numpy(sel).long().to(DEV)]),
                          np.arange(k, dtype=np.int32))
    assert max_rel_rowwise(o[0, 0].cpu().numpy(), ref_o).max() <= 2e-2
    ref_h, _ = oracle.mqa(to_f64(q[0, 0]), to_f64(hcache[0]), np.arange(Nh, dtype=np.int32))
    assert max_rel_rowwise(oh[0, 0].cpu().numpy(), ref_h).max() <= 2e-2


def test_hca_project_compress_b16_128k_sampled():
    """The fused projection + HCA compression at the micro-benchmark's launch: B = 16
    sequences of 131072 tokens, model width d = 4096, c = 512 (1024 entries each).
    Sampled entries are recomputed by the oracle's projections and HCA compressor."""
    B, n, d, c, mp = 16, 131072, 4096, 512, 128
    H = randn((B, n, d), 970, BF16, DEV, scale=d ** -0.25)
    Wc = randn((c, d), 971, BF16, DEV, scale=d ** -0.25)
    Wz = randn((c, d), 972, BF16, DEV, scale=d ** -0.25)
    Bias = randn((mp, c), 973, torch.float32, DEV)
    out = torch.empty((B, n // mp, c), dtype=BF16, device=DEV)
    ws = zeros_ws(256)
    lib.hca_project_compress(H, Wc, Wz, out, mp, ws, Bias=Bias)
    torch.cuda.synchronize()
    assert lib.csa_workspace_status(ws) == 0
    Wc64, Wz64, B64 = to_f64(Wc), to_f64(Wz), to_f64(Bias)
    for b, i in ((0, 0), (3, 511), (7, 1), (15, 1023), (9, 700)):
        rows = to_f64(H[b, mp * i:mp * (i + 1)])
        ref = oracle.hca_compress(oracle.project(rows, Wc64.T), oracle.project(rows, Wz64.T), mp, B64, 0, 1)
        assert max_rel_rowwise(to_f64(out[b, i:i + 1]), ref).max() <= 2e-2, (b, i)


def test_csa_project_compress_b4_256k_sampled():
    """The fused CSA projections + compression at the micro-benchmark's launch: B = 4
    sequences of 262144 tokens, d = 4096, c = 512 (65536 entries each).  Sampled entries,
    the first one (no b-part), tile edges and the split between the two epilogue
    halves of a tile included, are recomputed by the oracle."""
    B, n, d, c, m = 4, 262144, 4096, 512, 4
    H = randn((B, n, d), 980, BF16, DEV, scale=d ** -0.25)
    Ws = [randn((c, d), 981 + w, BF16, DEV, scale=d ** -0.25) for w in range(4)]
    Ba, Bb = randn((m, c), 985, torch.float32, DEV), randn((m, c), 986, torch.float32, DEV)
    out = torch.empty((B, n // m, c), dtype=BF16, device=DEV)
    ws = zeros_ws(256)
    lib.csa_project_compress(H, *Ws, out, m, ws, Ba=Ba, Bb=Bb)
    torch.cuda.synchronize()
    assert lib.csa_workspace_status(ws) == 0
    W64 = [to_f64(W).T for W in Ws]
    Ba64, Bb64 = to_f64(Ba), to_f64(Bb)
    for b, i in ((0, 0), (0, 30), (1, 31), (2, 62), (3, 63), (1, 125), (1, 126), (3, 65535), (2, 40000)):
        lo = max(0, m * (i - 1))
        rows = to_f64(H[b, lo:m * (i + 1)])
        streams = [oracle.project(rows, W) for W in W64]
        i0 = i - lo // m
        ref = oracle.csa_compress(*streams, m, Ba64, Bb64, i0, i0 + 1)
        assert max_rel_rowwise(to_f64(out[b, i:i + 1]), ref).max() <= 2e-2, (b, i)
