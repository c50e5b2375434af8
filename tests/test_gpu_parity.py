"""GPU parity: every C-ABI entry point against the fp64 CPU oracle on seeded inputs.

Tolerances (stated by the workload's target): attention outputs within 2e-2 max
relative error per (query, head) row for bf16 inputs with fp32 accumulation, 1e-5 for
the fp32 path; compressed entries by the same metric per entry; top-k index sets
identical except for near-ties (tests/helpers.check_topk_sets).  Integer-valued inputs
make every score exact in fp32 and fp64 alike, so there the top-k sets, tie order
included, must match exactly.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_csa_b200 import (csa_attn_workspace_size, csa_compress,
                                              csa_indexer_topk_e4m3, csa_quantize_e4m3,
                                              csa_indexer_topk, csa_indexer_topk_workspace_size,
                                              csa_sparse_attn, csa_workspace_status, hca_compress,
                                              hca_dense_attn)
from long_context_compressed_csa_b200.synth import randint_values, randn, to_f64
from tests.helpers import check_topk_sets, decode_e2m1, decode_e4m3, max_rel_rowwise, score_error_bound

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-5}
GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_compressed_csa_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def gv(name):
    return torch.tensor(GOLD[name]["value"], dtype=torch.float32)


def dev(x):
    return x.to(DEV).contiguous()


# ==================================================================================
# compression
# ==================================================================================
def run_csa_compress(Ca, Cb, Za, Zb, m, Ba=None, Bb=None, i0=0, i1=None, tok0=0, N_cap=None):
    B, rows, c = Ca.shape
    n = tok0 + rows
    if i1 is None:
        i1 = n // m
    N_cap = N_cap or max(i1, 1)
    out = torch.full((B, N_cap, c), float("nan"), dtype=Ca.dtype, device=DEV)
    csa_compress(Ca, Cb, Za, Zb, out, m, i0, i1, Ba=Ba, Bb=Bb, tok0=tok0)
    torch.cuda.synchronize()
    return out


def test_worked_example_compressors_fp32():
    H = gv("H")
    Ca = dev(H @ gv("W_aKV"))[None]
    Cb = dev(H @ gv("W_bKV"))[None]
    Za = dev(H @ gv("W_aZ"))[None]
    Zb = dev(H @ gv("W_bZ"))[None]
    out = run_csa_compress(Ca, Cb, Za, Zb, m=2)[0].cpu().double().numpy()
    e = math.e
    want = [[e / (e + 1), 1.0], [(4 * e**2 + e) / (2 * e**2 + e + 1), 0.75], [3 * e / (1 + 3 * e), 1.0]]
    np.testing.assert_allclose(out, want, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(out[:2], GOLD["csa_entries"]["value"], atol=3e-3)
    hout = torch.full((1, 2, 2), float("nan"), device=DEV)
    hca_compress(Ca, Za, hout, 3)
    h = hout[0].cpu().double().numpy()
    np.testing.assert_allclose(h, [[(e + 2 * e**2) / (1 + e + e**2), 1.0], [2 * e / (2 * e + 1), 2 / 3]],
                               rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("dtype,c,m", [(torch.bfloat16, 512, 4), (torch.float32, 512, 4),
                                       (torch.bfloat16, 136, 3), (torch.float32, 6, 2),
                                       (torch.bfloat16, 3, 4), (torch.bfloat16, 128, 1)])
def test_csa_compress_random(dtype, c, m):
    B, n = 2, 37 * m + m - 1          # ragged: a trailing partial block is not compressed
    S = [randn((B, n, c), 100 + i, dtype) for i in range(4)]
    Ba = randn((m, c), 110, torch.float32)
    Bb = randn((m, c), 111, torch.float32)
    out = run_csa_compress(*(dev(x) for x in S), m, Ba=dev(Ba), Bb=dev(Bb))
    N = n // m
    for b in range(B):
        ref = oracle.csa_compress(*(to_f64(x[b]) for x in S), m, Ba=to_f64(Ba), Bb=to_f64(Bb))
        err = max_rel_rowwise(out[b, :N].cpu().double().numpy(), ref)
        assert err.max() <= TOL[dtype], err.max()


def test_csa_compress_interleaved_layout_and_incremental_ranges():
    """One [n, 4c] projection buffer (ld_row = 4c), then decode-style single entries
    computed from a window of rows that starts at tok0 > 0."""
    B, n, c, m = 2, 64, 128, 4
    P = randn((B, n, 4 * c), 120, torch.bfloat16)
    Pd = dev(P)
    Ca, Cb, Za, Zb = (Pd[:, :, i * c:(i + 1) * c] for i in range(4))
    full = run_csa_compress(Ca, Cb, Za, Zb, m, N_cap=n // m)
    for b in range(B):
        ref = oracle.csa_compress(*(to_f64(P[b, :, i * c:(i + 1) * c]) for i in range(4)), m)
        assert max_rel_rowwise(full[b].cpu().double().numpy(), ref).max() <= 2e-2
    # entry i from rows m(i-1) .. m(i+1)-1 only (a ring of the last 2m token rows)
    for i in (1, 7, 15):
        lo = m * (i - 1)
        win = Pd[:, lo:m * (i + 1)]
        part = run_csa_compress(*(win[:, :, j * c:(j + 1) * c] for j in range(4)), m, i0=i,
                                i1=i + 1, tok0=lo, N_cap=n // m)
        torch.testing.assert_close(part[:, i], full[:, i], rtol=0, atol=0)


def _ref_project_compress(H, Wc, Wz, mp, Bias, i0, i1):
    """Oracle of the fused call: the plain projections, then the HCA compressor."""
    C = oracle.project(H, Wc.T)
    Z = oracle.project(H, Wz.T)
    return oracle.hca_compress(C, Z, mp, Bias, i0, i1)


@pytest.mark.parametrize("B,rows,d,c,bias,e0,e1,tok0", [
    (2, 4 * 70 + 3, 256, 256, True, 0, None, 0),      # 2 tiles of 63 entries (the last partial)
    (1, 4 * 60, 64, 128, False, 5, 40, 16),           # a sub-range, tok0 at block e0 - 1
    (3, 4 * 100, 1024, 512, True, 0, None, 0),        # several K panels and column blocks
    (2, 4 * 320 + 1, 128, 128, True, 0, None, 0),     # 6 tiles: 5 full, one ragged
    (2, 4 * 260, 192, 256, True, 70, 250, 4 * 69),    # a sub-range across 3 tiles, tok0 > 0
])
def test_csa_project_compress_matches_oracle(B, rows, d, c, bias, e0, e1, tok0):
    """Fused CSA projections + overlapped compression: the four streams H W^T in fp32 on
    the tensor cores, never stored, then the 2m-logit softmax of entry i over block i
    (a-part) and block i - 1 (b-part; none for entry 0), against the oracle's plain
    projections followed by its CSA compressor."""
    from long_context_compressed_csa_b200 import csa_project_compress
    m = 4
    H = randn((B, rows, d), 490, torch.bfloat16, scale=d ** -0.25)
    Ws = [randn((c, d), 491 + w, torch.bfloat16, scale=d ** -0.25) for w in range(4)]
    Ba = randn((m, c), 495, torch.float32) if bias else None
    Bb = randn((m, c), 496, torch.float32) if bias else None
    n = tok0 + rows
    e1 = n // m if e1 is None else e1
    out = torch.full((B, n // m + 1, c), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    csa_project_compress(dev(H), *[dev(W) for W in Ws], out, m, ws, entry_begin=e0, entry_end=e1,
                         Ba=dev(Ba) if bias else None, Bb=dev(Bb) if bias else None, tok0=tok0)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    got = out.float().cpu().numpy()
    W64 = [to_f64(W).T for W in Ws]
    for b in range(B):
        Hb = np.zeros((n, d))
        Hb[tok0:] = to_f64(H[b])
        streams = [oracle.project(Hb, W) for W in W64]
        ref = oracle.csa_compress(*streams, m, to_f64(Ba) if bias else None, to_f64(Bb) if bias else None, e0, e1)
        assert max_rel_rowwise(got[b, e0:e1], ref).max() <= TOL[torch.bfloat16]
        assert np.all(np.isnan(got[b, :e0])) and np.all(np.isnan(got[b, e1:]))


@pytest.mark.parametrize("B,rows,d,c,bias,e0,e1,tok0", [
    (2, 128 * 5 + 40, 256, 256, True, 0, None, 0),   # odd entry count, a partial block at the end
    (1, 128 * 6, 64, 128, False, 1, 4, 128),         # one K panel, one column block, a sub-range
    (3, 128 * 7, 1024, 512, True, 0, None, 0),       # several K panels and column blocks
])
def test_hca_project_compress_matches_oracle(B, rows, d, c, bias, e0, e1, tok0):
    """Fused projection + HCA compression: C = H Wc^T and Z = H Wz^T in fp32 on the tensor
    cores, never stored, then the per-column softmax pooling over each entry's 128
    tokens, against the oracle's plain projections followed by its HCA compressor."""
    from long_context_compressed_csa_b200 import hca_project_compress
    mp = 128
    H = randn((B, rows, d), 480, torch.bfloat16, scale=d ** -0.25)
    Wc = randn((c, d), 481, torch.bfloat16, scale=d ** -0.25)
    Wz = randn((c, d), 482, torch.bfloat16, scale=d ** -0.25)
    Bias = randn((mp, c), 483, torch.float32) if bias else None
    n = tok0 + rows
    e1 = n // mp if e1 is None else e1
    out = torch.full((B, n // mp + 1, c), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    hca_project_compress(dev(H), dev(Wc), dev(Wz), out, mp, ws, entry_begin=e0, entry_end=e1,
                         Bias=dev(Bias) if bias else None, tok0=tok0)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    got = out.float().cpu().numpy()
    for b in range(B):
        # the oracle sees the tokens from 0: rows before tok0 are not read, so pad them
        Hb = np.zeros((n, d))
        Hb[tok0:] = to_f64(H[b])
        ref = _ref_project_compress(Hb, to_f64(Wc), to_f64(Wz), mp, to_f64(Bias) if bias else None, e0, e1)
        assert max_rel_rowwise(got[b, e0:e1], ref).max() <= TOL[torch.bfloat16]
        assert np.all(np.isnan(got[b, :e0])) and np.all(np.isnan(got[b, e1:]))


@pytest.mark.parametrize("dtype,c,mp", [(torch.bfloat16, 512, 128), (torch.float32, 64, 128),
                                        (torch.bfloat16, 24, 5)])
def test_hca_compress_random(dtype, c, mp):
    B, n = 3, 5 * mp + 17
    C, Z = randn((B, n, c), 130, dtype), randn((B, n, c), 131, dtype)
    Bias = randn((mp, c), 132, torch.float32)
    N = n // mp
    out = torch.full((B, N, c), float("nan"), dtype=dtype, device=DEV)
    hca_compress(dev(C), dev(Z), out, mp, Bias=dev(Bias))
    for b in range(B):
        ref = oracle.hca_compress(to_f64(C[b]), to_f64(Z[b]), mp, Bias=to_f64(Bias))
        assert max_rel_rowwise(out[b].cpu().double().numpy(), ref).max() <= TOL[dtype]
    # one incremental entry from a window starting at tok0 = m' * i
    i = 3
    part = torch.zeros((B, N, c), dtype=dtype, device=DEV)
    hca_compress(dev(C[:, mp * i:mp * (i + 1)]), dev(Z[:, mp * i:mp * (i + 1)]), part, mp, i, i + 1,
                 Bias=dev(Bias), tok0=mp * i)
    torch.testing.assert_close(part[:, i], out[:, i], rtol=0, atol=0)


@pytest.mark.parametrize("B,nent,c,e0,e1,bias", [
    (2, 5000, 256, 0, None, True),      # 79 groups of 64 entries per batch, the last ragged
    (2, 5000, 256, 70, 4990, False),    # a sub-range, rows from block e0 - 1 (tok0 > 0)
    (1, 9500, 512, 0, None, True),      # two 256-column slices
])
def test_csa_compress_streaming_path(B, nent, c, e0, e1, bias):
    """Prefill-sized bf16 CSA compression, large enough (>= 148 work items of 64 entries
    x 256 columns) to run the TMA-staged streaming kernel, against the oracle on every
    entry: the b-rows loaded one block early, entry 0 without a b-part, ragged groups."""
    m = 4
    n = m * nent + 3
    e1 = nent if e1 is None else e1
    tok0 = 0 if e0 == 0 else m * (e0 - 1)
    S = [randn((B, n, c), 150 + i, torch.bfloat16) for i in range(4)]
    Ba = randn((m, c), 160, torch.float32) if bias else None
    Bb = randn((m, c), 161, torch.float32) if bias else None
    out = run_csa_compress(*(dev(x[:, tok0:]) for x in S), m, Ba=dev(Ba) if bias else None,
                           Bb=dev(Bb) if bias else None, i0=e0, i1=e1, tok0=tok0, N_cap=nent + 1)
    got = out.float().cpu().numpy()
    for b in range(B):
        ref = oracle.csa_compress(*(to_f64(x[b]) for x in S), m, Ba=to_f64(Ba) if bias else None,
                                  Bb=to_f64(Bb) if bias else None, i0=e0, i1=e1)
        assert max_rel_rowwise(got[b, e0:e1], ref).max() <= TOL[torch.bfloat16]
        assert np.all(np.isnan(got[b, :e0])) and np.all(np.isnan(got[b, e1:]))


@pytest.mark.parametrize("B,mp,nent,c,e0,bias", [
    (2, 128, 100, 512, 0, True),
    (3, 64, 120, 256, 7, False),        # a sub-range from tok0 = m' e0
    # one, three and five 32-row stages per entry: the entries of the two warp groups
    # fall on every slot alignment of the 6-stage ring, and with one stage per entry a
    # group can run several entries ahead of the other
    (1, 32, 1500, 256, 0, True),
    (1, 96, 400, 512, 3, False),
    (2, 160, 100, 256, 0, True),
])
def test_hca_compress_prefill_size(B, mp, nent, c, e0, bias):
    """Prefill-sized bf16 HCA compression, large enough (>= 148 work items of one entry x
    256 columns) to run the TMA-staged streaming kernel: m' from 32 to 160 (1 to 5
    stages of 32 rows per entry, the two warp groups on alternate entries), a sub-range
    from tok0 = m' e0, against the oracle on every entry."""
    n = mp * nent + 17
    tok0 = mp * e0
    C, Z = randn((B, n, c), 170, torch.bfloat16), randn((B, n, c), 171, torch.bfloat16)
    Bias = randn((mp, c), 172, torch.float32) if bias else None
    out = torch.full((B, nent, c), float("nan"), dtype=torch.bfloat16, device=DEV)
    hca_compress(dev(C[:, tok0:]), dev(Z[:, tok0:]), out, mp, e0, nent, Bias=dev(Bias) if bias else None,
                 tok0=tok0)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    for b in range(B):
        ref = oracle.hca_compress(to_f64(C[b]), to_f64(Z[b]), mp, Bias=to_f64(Bias) if bias else None,
                                  i0=e0, i1=nent)
        assert max_rel_rowwise(got[b, e0:], ref).max() <= TOL[torch.bfloat16]
        assert np.all(np.isnan(got[b, :e0]))


@pytest.mark.parametrize("dtype,mp", [(torch.bfloat16, 16), (torch.float32, 128)])
def test_compress_block_end_entries_match_wide_calls_bit_exactly(dtype, mp):
    """Single block-end entries, as a decode appends them (one CTA per entry, the candidate
    rows of a chunk loaded at once), against the same entries of calls over 100 entries x 2
    batch rows (one thread per column group and entry), bit for bit: CSA with biases, entry
    0 without a b-part; HCA with m' = 16 and m' = 128 (four chunks of 32 candidates).  The
    wide calls are checked against the oracle on sampled entries."""
    B, c, m, nent = 2, 512, 4, 100
    S = [randn((B, m * nent, c), 490 + i, dtype) for i in range(4)]
    Ba, Bb = randn((m, c), 495, torch.float32), randn((m, c), 496, torch.float32)
    Sd = [dev(x) for x in S]
    full = run_csa_compress(*Sd, m, Ba=dev(Ba), Bb=dev(Bb))
    for i in (0, 1, 57, 99):
        lo = max(0, m * (i - 1))
        part = run_csa_compress(*(x[:, lo:m * (i + 1)] for x in Sd), m, Ba=dev(Ba), Bb=dev(Bb), i0=i, i1=i + 1,
                                tok0=lo, N_cap=nent)
        torch.testing.assert_close(part[:, i], full[:, i], rtol=0, atol=0)
    for b in range(B):
        ref = oracle.csa_compress(*(to_f64(x[b]) for x in S), m, Ba=to_f64(Ba), Bb=to_f64(Bb), i0=0, i1=8)
        assert max_rel_rowwise(full[b, :8].double().cpu().numpy(), ref).max() <= TOL[dtype]
    n_h = mp * nent
    C, Z = randn((B, n_h, c), 497, dtype), randn((B, n_h, c), 498, dtype)
    Bias = randn((mp, c), 499, torch.float32)
    Cd, Zd = dev(C), dev(Z)
    hfull = torch.full((B, nent, c), float("nan"), dtype=dtype, device=DEV)
    hca_compress(Cd, Zd, hfull, mp, Bias=dev(Bias))
    for i in (0, 63, 99):
        part = torch.full((B, nent, c), float("nan"), dtype=dtype, device=DEV)
        hca_compress(Cd[:, mp * i:mp * (i + 1)], Zd[:, mp * i:mp * (i + 1)], part, mp, i, i + 1, Bias=dev(Bias),
                     tok0=mp * i)
        torch.cuda.synchronize()
        torch.testing.assert_close(part[:, i], hfull[:, i], rtol=0, atol=0)
    for b in range(B):
        ref = oracle.hca_compress(to_f64(C[b]), to_f64(Z[b]), mp, Bias=to_f64(Bias), i0=90, i1=100)
        assert max_rel_rowwise(hfull[b, 90:].double().cpu().numpy(), ref).max() <= TOL[dtype]


def test_compress_extreme_logits_one_hot():
    B, n, c, m = 1, 32, 64, 4
    Ca, Cb = randn((B, n, c), 140, torch.float32), randn((B, n, c), 141, torch.float32)
    Za, Zb = torch.zeros(B, n, c), torch.zeros(B, n, c)
    Za[0, 9, 5] = 80.0
    Zb[0, 6, 7] = 80.0
    out = run_csa_compress(dev(Ca), dev(Cb), dev(Za), dev(Zb), m)[0].cpu()
    assert abs(out[2, 5] - Ca[0, 9, 5]) < 1e-5 and abs(out[2, 7] - Cb[0, 6, 7]) < 1e-5


# ==================================================================================
# indexer + top-k
# ==================================================================================
def run_indexer(qI, wI, KI, t, m, k, ws=None, scores=True):
    B, nq = qI.shape[:2]
    N_cap = KI.shape[1]
    if ws is None:
        ws = torch.zeros(csa_indexer_topk_workspace_size(B, nq, N_cap, k), dtype=torch.uint8, device=DEV)
    idx = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, nq, k), float("nan"), dtype=torch.float32, device=DEV) if scores else None
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    csa_indexer_topk(qI, wI, KI, tt, m, k, idx, ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    return idx.cpu().numpy(), (sc.cpu().numpy() if scores else None), ws


def test_worked_example_indexer_fp32():
    qI = dev(gv("qI_5").reshape(1, 1, 1, 2))
    wI = dev(torch.ones(1, 1, 1))
    KI = dev(gv("KI").reshape(1, 2, 2))
    idx, sc, _ = run_indexer(qI, wI, KI, [5], m=2, k=1)
    assert idx.tolist() == [[[1]]] and sc.tolist() == [[[1.0]]]
    idx, sc, _ = run_indexer(qI, wI, KI, [5], m=2, k=2)
    assert idx.tolist() == [[[0, 1]]] and sc.tolist() == [[[0.5, 1.0]]]
    idx, _, _ = run_indexer(qI, wI, KI, [3], m=2, k=1)   # floor(3/2) = 1 visible
    assert idx.tolist() == [[[0]]]


@pytest.mark.parametrize("dtype,n_hI,cI", [(torch.bfloat16, 64, 128), (torch.bfloat16, 8, 24),
                                           (torch.float32, 16, 32)])
def test_indexer_topk_exact_on_integer_inputs(dtype, n_hI, cI):
    """Small-integer q, K, w: every score is an exact integer in fp32, so the selected set
    (with many exact ties resolved to the smaller index) must equal the oracle's."""
    B, nq, N_cap, m, k = 2, 2, 3000, 4, 257
    qI = randint_values((B, nq, n_hI, cI), 200, -2, 3, dtype)
    KI = randint_values((B, N_cap, cI), 201, -2, 3, dtype)
    wI = randint_values((B, nq, n_hI), 202, -2, 3, torch.float32)
    t = [4 * N_cap, 4 * 700 + 3, 4 * 257 + 1, 4 * 100]     # vis: 3000, 700, 257 (= k), 100
    idx, sc, ws = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for b in range(B):
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            s = oracle.index_scores(to_f64(qI[b, q]), to_f64(wI[b, q]), to_f64(KI[b]), vis)
            want = oracle.topk(s, k)
            got = idx[b, q]
            if vis <= k:   # all visible, in index order, -1 padded
                assert got.tolist() == list(range(vis)) + [-1] * (k - vis)
                assert sorted(want[:vis].tolist()) == list(range(vis))
            else:
                assert sorted(got.tolist()) == sorted(want.tolist())
            ok = got >= 0
            np.testing.assert_array_equal(sc[b, q][ok], s[got[ok]])
            assert np.all(np.isneginf(sc[b, q][~ok]))
    # the workspace is left clean: a second call gives the same sets
    idx2, _, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    for g in range(B * nq):
        assert sorted(idx2.reshape(-1, k)[g].tolist()) == sorted(idx.reshape(-1, k)[g].tolist())


def test_indexer_topk_mixed_select_paths_in_one_launch():
    """Two queries of one launch whose threshold bins differ in width: the first (0/1
    query, unit weights) crowds ~4800 keys into its threshold bin and is resolved digit
    by digit by one CTA, the second (random bf16) ranks its ~1100 candidates in every
    CTA.  Both sets must equal the oracle's except for fp32 near-ties, and a second call
    on the same workspace must repeat them."""
    B, nq, n_hI, cI, N_cap, m, k = 1, 2, 64, 128, 30000, 4, 4000
    qI = randint_values((B, nq, n_hI, cI), 270, 0, 2, torch.bfloat16)
    qI[0, 1] = randn((n_hI, cI), 275, torch.bfloat16)
    KI = randint_values((B, N_cap, cI), 271, 0, 2, torch.bfloat16)
    KI[0, :, :64] += randn((N_cap, 64), 276, torch.bfloat16, scale=1.0)   # spread for query 1
    KI = KI.to(torch.bfloat16)
    wI = torch.ones((B, nq, n_hI), dtype=torch.float32)
    wI[0, 1] = randn((n_hI,), 277, torch.float32)
    t = [4 * N_cap, 4 * N_cap]
    idx, sc, ws = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    widths = []
    for q in range(nq):
        q64, w64, K64 = to_f64(qI[0, q]), to_f64(wI[0, q]), to_f64(KI[0])
        s = oracle.index_scores(q64, w64, K64, N_cap)
        want = oracle.topk(s, k)
        u = s.astype(np.float32).view(np.uint32)
        d0 = np.where(u >> 31, ~u, u | np.uint32(0x80000000)) >> 20
        widths.append(int(np.sum(d0 == d0[want[k - 1]])))
        check_topk_sets(idx[0, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
    assert widths[0] > 4096 >= widths[1]  # one query on each select path
    idx2, _, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    for q in range(nq):
        assert sorted(idx2[0, q].tolist()) == sorted(idx[0, q].tolist())


@pytest.mark.parametrize("k,N_cap,run", [(200, 40000, 300), (1024, 262144, 2048)])
def test_indexer_topk_clustered_top_keys(k, N_cap, run):
    """The top keys crowd into a few consecutive key tiles (a run of keys scaled by 3, so
    every one of the k best lies inside it): the CTAs holding those tiles have far more
    top keys than the others, which the in-place select must place exactly as well as
    evenly spread ones.  Sets identical to the oracle's except for fp32 near-ties."""
    B, nq, n_hI, cI, m, r0 = 1, 1, 64, 128, 4, 12345
    qI = randn((B, nq, n_hI, cI), 280, torch.bfloat16)
    KI = randn((B, N_cap, cI), 281, torch.bfloat16)
    KI[0, r0:r0 + run] *= 3
    wI = randn((B, nq, n_hI), 282, torch.float32).abs()
    t = [4 * N_cap]
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    q64, w64, K64 = to_f64(qI[0, 0]), to_f64(wI[0, 0]), to_f64(KI[0])
    s = oracle.index_scores(q64, w64, K64, N_cap)
    top = oracle.topk(s, k)
    assert np.all((top >= r0) & (top < r0 + run))  # the run holds the top k
    check_topk_sets(idx[0, 0], s, k, lambda d: score_error_bound(q64, w64, K64, d))


@pytest.mark.parametrize("k,lo,hi", [(1000, 2048, 4096), (4000, 4097, 30000)])
def test_indexer_topk_wide_threshold_bin(k, lo, hi):
    """Scores that crowd into a few digit-0 bins (0/1 inputs; unit weights for the first
    query, -2..2 for the second), so the bin holding the k-th score is wide.  With
    k = 1000 it holds 2000-4000 keys: every CTA of the in-place select ranks a share of
    that candidate list.  With k = 4000 it holds over 4096: one CTA resolves it digit by
    digit instead.  Scores are exact in fp32, so the sets (ties to the smaller index)
    must equal the oracle's, and a second call on the same workspace must repeat them."""
    B, nq, n_hI, cI, N_cap, m = 1, 2, 64, 128, 30000, 4
    qI = randint_values((B, nq, n_hI, cI), 270, 0, 2, torch.bfloat16)
    KI = randint_values((B, N_cap, cI), 271, 0, 2, torch.bfloat16)
    wI = torch.ones((B, nq, n_hI), dtype=torch.float32)
    wI[0, 1] = randint_values((n_hI,), 272, -2, 3, torch.float32)
    t = [4 * N_cap, 4 * N_cap - 1]
    idx, sc, ws = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for q in range(nq):
        vis = oracle.visible(t[q], m, N_cap)
        s = oracle.index_scores(to_f64(qI[0, q]), to_f64(wI[0, q]), to_f64(KI[0]), vis)
        want = oracle.topk(s, k)
        # the threshold bin (top 12 bits of the fp32 order key) really has that width
        u = s.astype(np.float32).view(np.uint32)
        d0 = np.where(u >> 31, ~u, u | np.uint32(0x80000000)) >> 20
        assert lo <= np.sum(d0 == d0[want[k - 1]]) <= hi
        assert sorted(idx[0, q].tolist()) == sorted(want.tolist())
        np.testing.assert_array_equal(sc[0, q], s[idx[0, q]])
    idx2, _, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    for q in range(nq):
        assert sorted(idx2[0, q].tolist()) == sorted(idx[0, q].tolist())


@pytest.mark.parametrize("dtype,n_hI,cI,N_cap,k", [(torch.bfloat16, 64, 128, 20000, 512),
                                                   (torch.float32, 16, 32, 5000, 100),
                                                   (torch.bfloat16, 32, 64, 1500, 1024)])
def test_indexer_topk_random(dtype, n_hI, cI, N_cap, k):
    B, nq, m = 1, 2, 4
    qI = randn((B, nq, n_hI, cI), 210, dtype)
    KI = randn((B, N_cap, cI), 211, dtype)
    wI = randn((B, nq, n_hI), 212, torch.float32)
    t = [4 * N_cap + 2, 4 * (N_cap // 2) + 1]
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for q in range(nq):
        vis = oracle.visible(t[q], m, N_cap)
        q64, w64, K64 = to_f64(qI[0, q]), to_f64(wI[0, q]), to_f64(KI[0])
        s = oracle.index_scores(q64, w64, K64, vis)
        check_topk_sets(idx[0, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
        got = idx[0, q][idx[0, q] >= 0]
        band = score_error_bound(q64, w64, K64, got) + 1e-6 * np.abs(s[got])
        assert np.all(np.abs(sc[0, q][:len(got)] - s[got]) <= band)


@pytest.mark.parametrize("B,nq,N_cap,k,seed", [(2, 8, 40000, 512, 230), (150, 1, 1000, 100, 240),
                                              (3, 50, 1000, 100, 250)])
def test_indexer_topk_many_queries(B, nq, N_cap, k, seed):
    """16 queries: each query's scan CTAs own more key tiles than they keep on chip, so
    the in-place select also reads scores back from the workspace.  150 queries of one
    each: more queries than resident CTAs, so the scan is followed by the stand-alone
    select.  50 queries per row at random positions: the many-query scan (query blocks
    whose visible ranges differ), then one select CTA per query."""
    dtype, n_hI, cI, m = torch.bfloat16, 64, 128, 4
    qI = randn((B, nq, n_hI, cI), seed, dtype)
    KI = randn((B, N_cap, cI), seed + 1, dtype)
    wI = randn((B, nq, n_hI), seed + 2, torch.float32)
    rng = np.random.default_rng(seed + 3)
    t = [int(x) for x in rng.integers(0, 4 * N_cap + 8, size=B * nq)]
    t[0], t[1] = 4 * N_cap, 4 * (k // 2) + 3          # everything visible; fewer than k
    idx, sc, ws = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for b in range(B):
        K64 = to_f64(KI[b])
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            q64, w64 = to_f64(qI[b, q]), to_f64(wI[b, q])
            s = oracle.index_scores(q64, w64, K64, vis)
            got = idx[b, q]
            if vis <= k:
                assert got.tolist() == list(range(vis)) + [-1] * (k - vis)
            else:
                check_topk_sets(got, s, k, lambda d: score_error_bound(q64, w64, K64, d))
            sel = got[got >= 0]
            band = score_error_bound(q64, w64, K64, sel) + 1e-6 * np.abs(s[sel])
            assert np.all(np.abs(sc[b, q][:len(sel)] - s[sel]) <= band)
            assert np.all(np.isneginf(sc[b, q][len(sel):]))
    # the workspace is left clean for the next call
    idx2, _, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    assert np.array_equal(np.sort(idx2, axis=-1), np.sort(idx, axis=-1))


@pytest.mark.parametrize("dtype,cols", [(torch.bfloat16, 128), (torch.float32, 256), (torch.bfloat16, 44)])
def test_quantize_e4m3_matches_oracle_bit_exactly(dtype, cols):
    """E4M3 codes and fp32 row scales equal the oracle's (both form x * (448 / max|x|) in
    fp32 and round to nearest even), including an all-zero row and a row of large values."""
    X = randn((301, cols), 350, dtype, scale=3.0)
    X[5] = 0
    X[9] = X[9] * 1e4
    codes = torch.empty((301, cols), dtype=torch.uint8, device=DEV)
    scales = torch.empty((301,), dtype=torch.float32, device=DEV)
    csa_quantize_e4m3(dev(X), codes, scales)
    torch.cuda.synchronize()
    want_v, want_s = oracle.quantize_rows_e4m3(X.float().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), want_s)
    np.testing.assert_array_equal(decode_e4m3(codes.cpu().numpy()), want_v)


def _oracle_scores(qI, wI, KI, b, q, vis):
    return oracle.index_scores(to_f64(qI[b, q]), to_f64(wI[b, q]), to_f64(KI[b]), vis)


@pytest.mark.parametrize("n_hI,cI,B,nq,N_cap,k,seed", [
    (64, 128, 1, 40, 5000, 256, 400),    # 5 blocks of 8 queries
    (64, 128, 2, 19, 3000, 1024, 410),   # 2 rows, ragged last block, visible counts crossing k
    (32, 64, 1, 33, 2000, 100, 420),     # 16 queries per block, ragged
    (128, 128, 1, 17, 1500, 64, 430),    # 4 queries per block
])
def test_indexer_topk_prefill_chunk(n_hI, cI, B, nq, N_cap, k, seed):
    """A prefill chunk: nq consecutive query positions per batch row, scored together
    (blocks of 512 / n_hI queries resident while the key tiles stream past), then one
    select CTA per query.  Row 0 ends at the last key; row 1 starts just below k visible
    entries, and its first queries see no entry at all."""
    dtype, m = torch.bfloat16, 4
    qI = randn((B, nq, n_hI, cI), seed, dtype)
    KI = randn((B, N_cap, cI), seed + 1, dtype)
    wI = randn((B, nq, n_hI), seed + 2, torch.float32)
    starts = [4 * N_cap - 4 * nq + 3, 0][:B]
    if B > 1:
        starts[1] = 4 * (k - 3)
    t = [t0 + j for t0 in starts for j in range(nq)]
    if B > 1:
        t[nq:nq + 3] = [0, 1, 3]             # t < m: nothing visible
    idx, sc, ws = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for b in range(B):
        K64 = to_f64(KI[b])
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            q64, w64 = to_f64(qI[b, q]), to_f64(wI[b, q])
            s = oracle.index_scores(q64, w64, K64, vis)
            got = idx[b, q]
            if vis <= k:
                assert got.tolist() == list(range(vis)) + [-1] * (k - vis)
            else:
                check_topk_sets(got, s, k, lambda d: score_error_bound(q64, w64, K64, d))
            sel = got[got >= 0]
            band = score_error_bound(q64, w64, K64, sel) + 1e-6 * np.abs(s[sel])
            assert np.all(np.abs(sc[b, q][:len(sel)] - s[sel]) <= band)
            assert np.all(np.isneginf(sc[b, q][len(sel):]))
    idx2, _, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    assert np.array_equal(np.sort(idx2, axis=-1), np.sort(idx, axis=-1))


def test_indexer_topk_prefill_negative_weights():
    """Many-query path with every head weight negative: the scores are <= 0, the largest
    ones cluster near zero, and the group maxima straddle the sign (the order keys of
    +0 and of negative scores are far apart), so the select's maxima window widens."""
    B, nq, N_cap, m, k, n_hI, cI = 1, 24, 6000, 4, 300, 64, 128
    qI = randn((B, nq, n_hI, cI), 460, torch.bfloat16)
    KI = randn((B, N_cap, cI), 461, torch.bfloat16)
    wI = -randn((B, nq, n_hI), 462, torch.float32).abs()
    wI[0, 1:4] = wI[0, 1:4] * 1e-3          # three queries with scores near zero
    t = [4 * N_cap - 3 * j for j in range(nq)]
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    K64 = to_f64(KI[0])
    for q in range(nq):
        vis = oracle.visible(t[q], m, N_cap)
        q64, w64 = to_f64(qI[0, q]), to_f64(wI[0, q])
        s = oracle.index_scores(q64, w64, K64, vis)
        check_topk_sets(idx[0, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
        sel = idx[0, q]
        band = score_error_bound(q64, w64, K64, sel) + 1e-6 * np.abs(s[sel])
        assert np.all(np.abs(sc[0, q] - s[sel]) <= band)


def test_indexer_topk_prefill_exact_on_integer_inputs():
    """Many-query path on small-integer q, K, w: every score is an exact integer, so the
    selected sets, with ties resolved to the smaller index, and the scores must equal
    the oracle's exactly."""
    B, nq, N_cap, m, k, n_hI, cI = 2, 20, 3000, 4, 257, 64, 128
    qI = randint_values((B, nq, n_hI, cI), 440, -2, 3, torch.bfloat16)
    KI = randint_values((B, N_cap, cI), 441, -2, 3, torch.bfloat16)
    wI = randint_values((B, nq, n_hI), 442, -2, 3, torch.float32)
    t = [4 * N_cap - 40 + 2 * j for j in range(nq)] + [4 * 250 + 3 * j for j in range(nq)]
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k)
    for b in range(B):
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            s = _oracle_scores(qI, wI, KI, b, q, vis)
            want = oracle.topk(s, k)
            got = idx[b, q]
            if vis <= k:
                assert got.tolist() == list(range(vis)) + [-1] * (k - vis)
            else:
                assert sorted(got.tolist()) == sorted(want.tolist())
            ok = got >= 0
            np.testing.assert_array_equal(sc[b, q][ok], s[got[ok]])


def test_indexer_topk_prefill_full_size_sampled():
    """The 1M-token context's last 1024 query positions as one prefill chunk (262144
    keys, k = 1024): the launch the prefill micro-benchmark times.  Four sampled
    queries, one from each quarter of the chunk, are checked against the oracle."""
    B, nq, N_cap, m, k, n_hI, cI = 1, 1024, 262144, 4, 1024, 64, 128
    n = 1 << 20
    qI = randn((B, nq, n_hI, cI), 450, torch.bfloat16, DEV)
    KI = randn((B, N_cap, cI), 451, torch.bfloat16, DEV)
    wI = randn((B, nq, n_hI), 452, torch.float32, DEV)
    t = [n - nq + j for j in range(nq)]
    idx, sc, _ = run_indexer(qI, wI, KI, t, m, k)
    K64 = to_f64(KI[0].cpu())
    for q in (0, 300, 700, 1023):
        vis = oracle.visible(t[q], m, N_cap)
        q64, w64 = to_f64(qI[0, q].cpu()), to_f64(wI[0, q].cpu())
        s = oracle.index_scores(q64, w64, K64, vis)
        check_topk_sets(idx[0, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
        sel = idx[0, q]
        band = score_error_bound(q64, w64, K64, sel) + 1e-6 * np.abs(s[sel])
        assert np.all(np.abs(sc[0, q] - s[sel]) <= band)


@pytest.mark.parametrize("n_hI,cI,N_cap,k", [(64, 128, 20000, 512), (32, 256, 3000, 1024), (16, 128, 700, 64)])
def test_indexer_topk_e4m3(n_hI, cI, N_cap, k):
    """Top-k over E4M3 keys and in-kernel E4M3 queries against the oracle's scores of the
    same quantised operands (sets identical except for fp32 near-ties)."""
    B, nq, m = 2, 2, 4
    qI = randn((B, nq, n_hI, cI), 360, torch.bfloat16)
    KI = randn((B, N_cap, cI), 361, torch.bfloat16)
    wI = randn((B, nq, n_hI), 362, torch.float32)
    codes = torch.empty((B, N_cap, cI), dtype=torch.uint8, device=DEV)
    ksc = torch.empty((B, N_cap), dtype=torch.float32, device=DEV)
    csa_quantize_e4m3(dev(KI), codes, ksc)
    t = [m * N_cap + 3, m * (N_cap // 3) + 1, m * (k // 2), 5]      # all, a third, fewer than k, t < m
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    ws = torch.zeros(csa_indexer_topk_workspace_size(B, nq, N_cap, k), dtype=torch.uint8, device=DEV)
    idx = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, nq, k), float("nan"), dtype=torch.float32, device=DEV)
    csa_indexer_topk_e4m3(dev(qI), dev(wI), codes, ksc, tt, m, k, idx, ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        kc, ks = oracle.quantize_rows_e4m3(KI[b].float().numpy())
        K64 = kc * ks[:, None]
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            qc, qs = oracle.quantize_rows_e4m3(qI[b, q].float().numpy())
            q64, w64 = qc * qs[:, None], to_f64(wI[b, q])
            s = oracle.index_scores(q64, w64, K64, vis)
            np.testing.assert_array_equal(s, oracle.index_scores_e4m3(qI[b, q].float().numpy(), w64,
                                                                      KI[b].float().numpy(), vis))
            check_topk_sets(idx[b, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
            got = idx[b, q][idx[b, q] >= 0]
            band = score_error_bound(q64, w64, K64, got) + 1e-6 * np.abs(s[got])
            assert np.all(np.abs(sc[b, q][:len(got)] - s[got]) <= band)
    # the workspace is left clean for the next call
    idx2 = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    csa_indexer_topk_e4m3(dev(qI), dev(wI), codes, ksc, tt, m, k, idx2, ws)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx2.cpu().numpy(), axis=-1), np.sort(idx, axis=-1))


@pytest.mark.parametrize("dtype,cols", [(torch.bfloat16, 128), (torch.float32, 256), (torch.bfloat16, 8)])
def test_quantize_e2m1_matches_oracle_bit_exactly(dtype, cols):
    """E2M1 codes (two per byte, even column in the low nibble) and fp32 row scales equal
    the oracle's (both form x * (6 / max|x|) in fp32 and round to nearest even, saturating
    at 6), including an all-zero row and a row of large values."""
    from long_context_compressed_csa_b200 import csa_quantize_e2m1
    X = randn((301, cols), 370, dtype, scale=3.0)
    X[5] = 0
    X[9] = X[9] * 1e4
    codes = torch.empty((301, cols // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((301,), dtype=torch.float32, device=DEV)
    csa_quantize_e2m1(dev(X), codes, scales)
    torch.cuda.synchronize()
    want_v, want_s = oracle.quantize_rows_e2m1(X.float().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), want_s)
    np.testing.assert_array_equal(decode_e2m1(codes.cpu().numpy()), want_v)


@pytest.mark.parametrize("n_hI,cI,N_cap,k", [(64, 128, 20000, 512), (32, 256, 3000, 1024), (16, 128, 700, 64)])
def test_indexer_topk_e2m1(n_hI, cI, N_cap, k):
    """Top-k over E2M1 keys and in-kernel E4M3 queries against the oracle's scores of the
    GPU's decoded keys and the oracle-quantised queries (sets identical except for fp32
    near-ties); the scores returned match within the fp32 rounding bound."""
    from long_context_compressed_csa_b200 import csa_indexer_topk_e2m1, csa_quantize_e2m1
    B, nq, m = 2, 2, 4
    qI = randn((B, nq, n_hI, cI), 365, torch.bfloat16)
    KI = randn((B, N_cap, cI), 366, torch.bfloat16)
    wI = randn((B, nq, n_hI), 367, torch.float32)
    codes = torch.empty((B, N_cap, cI // 2), dtype=torch.uint8, device=DEV)
    ksc = torch.empty((B, N_cap), dtype=torch.float32, device=DEV)
    csa_quantize_e2m1(dev(KI), codes, ksc)
    t = [m * N_cap + 3, m * (N_cap // 3) + 1, m * (k // 2), 5]      # all, a third, fewer than k, t < m
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    ws = torch.zeros(csa_indexer_topk_workspace_size(B, nq, N_cap, k), dtype=torch.uint8, device=DEV)
    idx = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, nq, k), float("nan"), dtype=torch.float32, device=DEV)
    csa_indexer_topk_e2m1(dev(qI), dev(wI), codes, ksc, tt, m, k, idx, ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    codes_h, ksc_h = codes.cpu().numpy(), ksc.cpu().numpy().astype(np.float64)
    for b in range(B):
        K64 = decode_e2m1(codes_h[b]) * ksc_h[b][:, None]
        kc, ks = oracle.quantize_rows_e2m1(KI[b].float().numpy())
        np.testing.assert_array_equal(K64, kc * ks[:, None])  # the GPU's keys are the oracle's
        for q in range(nq):
            g = b * nq + q
            vis = oracle.visible(t[g], m, N_cap)
            qc, qs = oracle.quantize_rows_e4m3(qI[b, q].float().numpy())
            q64, w64 = qc * qs[:, None], to_f64(wI[b, q])
            s = oracle.index_scores(q64, w64, K64, vis)
            check_topk_sets(idx[b, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
            got = idx[b, q][idx[b, q] >= 0]
            band = score_error_bound(q64, w64, K64, got) + 1e-6 * np.abs(s[got])
            assert np.all(np.abs(sc[b, q][:len(got)] - s[got]) <= band)
    # the workspace is left clean for the next call
    idx2 = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    csa_indexer_topk_e2m1(dev(qI), dev(wI), codes, ksc, tt, m, k, idx2, ws)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx2.cpu().numpy(), axis=-1), np.sort(idx, axis=-1))


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_low_precision_indexer_many_queries(fmt):
    """More queries than resident CTAs (200 > 148): the low-precision scan writes the
    scores to the workspace and the stand-alone select follows.  Sets and scores against
    the oracle on the GPU's decoded keys and the oracle-quantised queries."""
    import long_context_compressed_csa_b200 as lib
    quant = lib.csa_quantize_e4m3 if fmt == "e4m3" else lib.csa_quantize_e2m1
    topk = lib.csa_indexer_topk_e4m3 if fmt == "e4m3" else lib.csa_indexer_topk_e2m1
    decode = decode_e4m3 if fmt == "e4m3" else decode_e2m1
    B, nq, n_hI, cI, N_cap, m, k = 1, 200, 64, 128, 2000, 4, 100
    qI = randn((B, nq, n_hI, cI), 385, torch.bfloat16)
    KI = randn((B, N_cap, cI), 386, torch.bfloat16)
    wI = randn((B, nq, n_hI), 387, torch.float32)
    codes = torch.empty((B, N_cap, cI if fmt == "e4m3" else cI // 2), dtype=torch.uint8, device=DEV)
    ksc = torch.empty((B, N_cap), dtype=torch.float32, device=DEV)
    quant(dev(KI), codes, ksc)
    t = [m * (N_cap // 2) + 4 * q for q in range(nq)]  # visible counts 1000 .. 1199
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    ws = torch.zeros(csa_indexer_topk_workspace_size(B, nq, N_cap, k), dtype=torch.uint8, device=DEV)
    idx = torch.full((B, nq, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((B, nq, k), float("nan"), dtype=torch.float32, device=DEV)
    topk(dev(qI), dev(wI), codes, ksc, tt, m, k, idx, ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    K64 = decode(codes[0].cpu().numpy()) * ksc[0].cpu().numpy().astype(np.float64)[:, None]
    for q in (0, 57, 123, 199):
        vis = oracle.visible(t[q], m, N_cap)
        qc, qs = oracle.quantize_rows_e4m3(qI[0, q].float().numpy())
        q64, w64 = qc * qs[:, None], to_f64(wI[0, q])
        s = oracle.index_scores(q64, w64, K64, vis)
        check_topk_sets(idx[0, q], s, k, lambda d: score_error_bound(q64, w64, K64, d))
        got = idx[0, q]
        band = score_error_bound(q64, w64, K64, got) + 1e-6 * np.abs(s[got])
        assert np.all(np.abs(sc[0, q] - s[got]) <= band)


def test_indexer_wait_timeout_is_reported_then_cleared():
    """Failure detection without a GPU fault: a wait budget of a few cycles for the grid
    meeting of the in-place top-k (the workspace's test hook) makes that bounded wait run
    out; the call then reports CSA_ERR_TIMEOUT through the workspace status, every CTA
    still exits, and after the status word and the budget are cleared the next call on
    the same workspace matches the oracle."""
    from long_context_compressed_csa_b200 import csa_workspace_set_wait_budget, csa_workspace_zero
    n_hI, cI, m, k, N = 64, 128, 4, 512, 65536
    qI = randn((1, 1, n_hI, cI), 560, torch.bfloat16)
    wI = randn((1, 1, n_hI), 561, torch.float32)
    KI = randn((1, N, cI), 562, torch.bfloat16)
    t = [m * N]
    ws = torch.zeros(csa_indexer_topk_workspace_size(1, 1, N, k), dtype=torch.uint8, device=DEV)
    csa_workspace_set_wait_budget(ws, 8)
    idx0 = torch.empty((1, 1, k), dtype=torch.int32, device=DEV)
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(1, 1)
    csa_indexer_topk(dev(qI), dev(wI), dev(KI), tt, m, k, idx0, ws)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == -7
    csa_workspace_zero(ws[:16])  # the status word and the budget
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), t, m, k, ws=ws)
    assert csa_workspace_status(ws) == 0
    q64, w64, K64 = to_f64(qI[0, 0]), to_f64(wI[0, 0]), to_f64(KI[0])
    s = oracle.index_scores(q64, w64, K64, N)
    check_topk_sets(idx[0, 0], s, k, lambda d: score_error_bound(q64, w64, K64, d))


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_low_precision_key_cache_decode_loop(fmt):
    """A CSA decode loop whose indexer keys live as E4M3 (one byte) or E2M1 (half a byte)
    codes with one fp32 scale per key: the prefill keys are quantised once, and each key
    appended at a block end is formed by csa_compress (bf16) and quantised as it is
    formed.  Stage-wise checks at every step: each new key's codes and scale are
    bit-exact against the oracle's quantisation of the GPU's bf16 key, and the step's
    top-k set matches the oracle's scores of the GPU's decoded keys and the
    oracle-quantised query (near-ties within the fp32 rounding bound plus 1e-6
    relative)."""
    import long_context_compressed_csa_b200 as lib
    quant = lib.csa_quantize_e4m3 if fmt == "e4m3" else lib.csa_quantize_e2m1
    topk = lib.csa_indexer_topk_e4m3 if fmt == "e4m3" else lib.csa_indexer_topk_e2m1
    decode = decode_e4m3 if fmt == "e4m3" else decode_e2m1
    oquant = oracle.quantize_rows_e4m3 if fmt == "e4m3" else oracle.quantize_rows_e2m1
    B, m, cI, n_hI, k, N0, steps = 1, 4, 128, 64, 256, 3000, 13
    n0 = m * N0
    N_cap = N0 + steps // m + 2
    SI = [randn((B, n0 + steps, cI), 380 + i, torch.bfloat16) for i in range(4)]
    SId = [dev(x) for x in SI]
    kI = torch.empty((B, N_cap, cI), dtype=torch.bfloat16, device=DEV)
    K8 = torch.zeros((B, N_cap, cI if fmt == "e4m3" else cI // 2), dtype=torch.uint8, device=DEV)
    KS = torch.zeros((B, N_cap), dtype=torch.float32, device=DEV)
    csa_compress(*(x[:, :n0] for x in SId), kI, m, 0, N0)
    quant(kI[:, :N0], K8[:, :N0], KS[:, :N0])
    ws = torch.zeros(csa_indexer_topk_workspace_size(B, 1, N_cap, k), dtype=torch.uint8, device=DEV)
    for j in range(steps):
        t = n0 + j
        qI = randn((B, 1, n_hI, cI), 390 + j, torch.bfloat16)
        wI = randn((B, 1, n_hI), 400 + j, torch.float32)
        idx = torch.full((B, 1, k), -7, dtype=torch.int32, device=DEV)
        tt = torch.tensor([[t]], dtype=torch.int64, device=DEV)
        topk(dev(qI), dev(wI), K8, KS, tt, m, k, idx, ws)
        torch.cuda.synchronize()
        assert csa_workspace_status(ws) == 0
        vis = oracle.visible(t, m, N_cap)
        K64 = decode(K8[0, :vis].cpu().numpy()) * KS[0, :vis].cpu().numpy().astype(np.float64)[:, None]
        qc, qs = oracle.quantize_rows_e4m3(qI[0, 0].float().numpy())
        q64, w64 = qc * qs[:, None], to_f64(wI[0, 0])
        s = oracle.index_scores(q64, w64, K64, vis)
        check_topk_sets(idx.cpu().numpy()[0, 0], s, k, lambda d: score_error_bound(q64, w64, K64, d))
        if (t + 1) % m == 0:  # the token completes entry i: form it, then quantise it
            i = (t + 1) // m - 1
            lo = m * (i - 1)
            csa_compress(*(x[:, lo:lo + 2 * m] for x in SId), kI, m, i, i + 1, tok0=lo)
            quant(kI[:, i:i + 1], K8[:, i:i + 1], KS[:, i:i + 1])
            torch.cuda.synchronize()
            rc, rs = oquant(kI[0, i].float().cpu().numpy())
            np.testing.assert_array_equal(decode(K8[0, i].cpu().numpy()), rc)
            assert KS[0, i].item() == np.float32(rs)


def test_indexer_degenerate_cases():
    dtype, n_hI, cI, N_cap, m = torch.bfloat16, 64, 128, 700, 4
    qI = randn((1, 3, n_hI, cI), 220, dtype)
    KI = torch.zeros((1, N_cap, cI), dtype=dtype)      # all scores exactly 0: ties everywhere
    wI = randn((1, 3, n_hI), 221, torch.float32)
    idx, sc, _ = run_indexer(dev(qI), dev(wI), dev(KI), [0, 4 * 5, 4 * N_cap], m, 64)
    assert idx[0, 0].tolist() == [-1] * 64                     # nothing visible
    assert idx[0, 1].tolist() == list(range(5)) + [-1] * 59    # fewer visible than k
    assert sorted(idx[0, 2].tolist()) == list(range(64))       # all tied: smallest indices
    assert np.all(sc[0, 2] == 0)


# ==================================================================================
# attention
# ==================================================================================
def run_sparse(q, cache, idx, out_dtype=torch.float32, scale=0.0):
    B, nq, n_h, c = q.shape
    k = idx.shape[2]
    ws = torch.zeros(csa_attn_workspace_size(B, nq, n_h, c, k), dtype=torch.uint8, device=DEV)
    out = torch.full((B, nq, n_h, c), float("nan"), dtype=out_dtype, device=DEV)
    lse = torch.full((B, nq, n_h), float("nan"), device=DEV)
    csa_sparse_attn(q, cache, idx, out, ws, lse=lse, scale=scale)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def run_dense(q, cache, t, mp, out_dtype=torch.float32):
    B, nq, n_h, c = q.shape
    N_cap = cache.shape[1]
    ws = torch.zeros(csa_attn_workspace_size(B, nq, n_h, c, N_cap), dtype=torch.uint8, device=DEV)
    out = torch.full((B, nq, n_h, c), float("nan"), dtype=out_dtype, device=DEV)
    lse = torch.full((B, nq, n_h), float("nan"), device=DEV)
    tt = torch.tensor(t, dtype=torch.int64, device=DEV).reshape(B, nq)
    hca_dense_attn(q, cache, tt, mp, out, ws, lse=lse)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def test_worked_example_attention_fp32():
    e = math.e
    C = torch.tensor([[e / (e + 1), 1.0], [(4 * e**2 + e) / (2 * e**2 + e + 1), 0.75],
                      [3 * e / (1 + 3 * e), 1.0]], dtype=torch.float32)
    q = dev(gv("cQ_5").reshape(1, 1, 1, 2))
    o, lse = run_sparse(q, dev(C[None]), dev(torch.tensor([[[1]]], dtype=torch.int32)))
    np.testing.assert_allclose(o[0, 0, 0], C[1].numpy(), rtol=1e-6)
    np.testing.assert_allclose(o[0, 0, 0], GOLD["csa_output_k1"]["value"], atol=3e-3)
    o, _ = run_sparse(q, dev(C[None]), dev(torch.tensor([[[0, 1]]], dtype=torch.int32)))
    np.testing.assert_allclose(o[0, 0, 0], [1.412288, 0.832019], atol=2e-6)
    Hc = torch.tensor([[(e + 2 * e**2) / (1 + e + e**2), 1.0], [2 * e / (2 * e + 1), 2 / 3]])
    o, _ = run_dense(q, dev(Hc[None]), [5], 3)
    np.testing.assert_allclose(o[0, 0, 0], Hc[0].numpy(), rtol=1e-6)


def _ref_attn(q, cache, sel, scale=None):
    out, lse = oracle.mqa(q, cache, sel, scale)
    return out, lse


@pytest.mark.parametrize("dtype,n_h,c,k", [(torch.bfloat16, 128, 512, 1024),
                                           (torch.bfloat16, 128, 512, 200),
                                           (torch.float32, 8, 64, 300),
                                           (torch.bfloat16, 20, 40, 77)])
def test_sparse_attn_random(dtype, n_h, c, k):
    B, nq, N_cap = 2, 1, 3000
    q = randn((B, nq, n_h, c), 300, dtype)
    cache = randn((B, N_cap, c), 301, dtype)
    g = torch.Generator().manual_seed(302)
    idx = torch.stack([torch.randperm(N_cap, generator=g)[:k] for _ in range(B * nq)]).reshape(B, nq, k)
    idx = idx.to(torch.int32)
    idx[0, 0, ::7] = -1                                  # padding slots are skipped
    o, lse = run_sparse(dev(q), dev(cache), dev(idx))
    for b in range(B):
        ref, ref_lse = _ref_attn(to_f64(q[b, 0]), to_f64(cache[b]), idx[b, 0].numpy())
        assert max_rel_rowwise(o[b, 0], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(lse[b, 0], ref_lse, atol=2e-3 if dtype == torch.bfloat16 else 1e-5,
                                   rtol=0)


def test_sparse_attn_bf16_output_scale_and_empty():
    B, nq, n_h, c, N_cap, k = 1, 2, 128, 512, 500, 64
    q = randn((B, nq, n_h, c), 310, torch.bfloat16)
    cache = randn((B, N_cap, c), 311, torch.bfloat16)
    idx = torch.randint(0, N_cap, (B, nq, k), generator=torch.Generator().manual_seed(312)).to(torch.int32)
    idx[0, 1] = -1                                       # query 1: nothing selected
    o, lse = run_sparse(dev(q), dev(cache), dev(idx), out_dtype=torch.bfloat16, scale=0.03)
    ref, ref_lse = _ref_attn(to_f64(q[0, 0]), to_f64(cache[0]), idx[0, 0].numpy(), 0.03)
    assert max_rel_rowwise(o[0, 0], ref).max() <= 2e-2
    np.testing.assert_allclose(lse[0, 0], ref_lse, atol=2e-3)
    assert np.all(o[0, 1] == 0) and np.all(np.isneginf(lse[0, 1]))


@pytest.mark.parametrize("dtype,n_h,c", [(torch.bfloat16, 128, 512), (torch.float32, 16, 64)])
def test_dense_attn_random(dtype, n_h, c):
    B, nq, N_cap, mp = 3, 1, 1024, 128
    q = randn((B, nq, n_h, c), 320, dtype)
    cache = randn((B, N_cap, c), 321, dtype)
    t = [mp * N_cap + 5, mp * 333 + 127, 100]            # vis 1024, 333, 0
    o, lse = run_dense(dev(q), dev(cache), t, mp)
    for b in range(B):
        vis = oracle.visible(t[b], mp, N_cap)
        if vis == 0:
            assert np.all(o[b, 0] == 0) and np.all(np.isneginf(lse[b, 0]))
            continue
        ref, ref_lse = _ref_attn(to_f64(q[b, 0]), to_f64(cache[b]), np.arange(vis, dtype=np.int32))
        assert max_rel_rowwise(o[b, 0], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(lse[b, 0], ref_lse, atol=2e-3 if dtype == torch.bfloat16 else 1e-5,
                                   rtol=0)


@pytest.mark.parametrize("B,N_cap,vis", [
    (1, 200, [75]),                                          # one 32-entry chunk per split
    (8, 2048, [2048, 1000, 700, 64, 63, 0, 130, 1]),         # CTA pairs, four 64-entry chunks per split
])
def test_dense_attn_ignores_rows_past_visible(B, N_cap, vis):
    """Cache rows at or past the visible count hold NaN: a split whose range the count cuts
    (a partial chunk), or that lies past it, must neither read them into the output nor
    leave them in shared memory for the products."""
    n_h, c, mp = 128, 512, 128
    q = randn((B, 1, n_h, c), 480, torch.bfloat16)
    cache = randn((B, N_cap, c), 481, torch.bfloat16)
    for b, v in enumerate(vis):
        cache[b, v:] = float("nan")
    t = [mp * v + (b * 37) % mp for b, v in enumerate(vis)]
    o, lse = run_dense(dev(q), dev(cache), t, mp)
    for b, v in enumerate(vis):
        assert oracle.visible(t[b], mp, N_cap) == v
        if v == 0:
            assert np.all(o[b, 0] == 0) and np.all(np.isneginf(lse[b, 0]))
            continue
        ref, ref_lse = _ref_attn(to_f64(q[b, 0]), to_f64(cache[b]), np.arange(v, dtype=np.int32))
        assert np.all(np.isfinite(o[b, 0]))
        assert max_rel_rowwise(o[b, 0], ref).max() <= TOL[torch.bfloat16]
        np.testing.assert_allclose(lse[b, 0], ref_lse, atol=2e-3, rtol=0)


def test_attn_many_queries_and_workspace_reuse():
    """80 queries of 128 heads in one call (one CTA pair per query, padding inside one
    list); then one dense workspace reused across calls whose visible counts, hence split
    plans, differ."""
    dtype, n_h, c = torch.bfloat16, 128, 512
    B, nq, N_cap, k = 1, 80, 512, 96
    q = randn((B, nq, n_h, c), 330, dtype)
    cache = randn((B, N_cap, c), 331, dtype)
    g = torch.Generator().manual_seed(332)
    idx = torch.stack([torch.randperm(N_cap, generator=g)[:k] for _ in range(nq)]).to(torch.int32)
    idx[3, 5:20] = -1                                    # padding inside one list
    o, lse = run_sparse(dev(q), dev(cache), dev(idx.reshape(B, nq, k)))
    for j in (0, 3, 41, 79):
        sel = idx[j].numpy()
        ref, ref_lse = _ref_attn(to_f64(q[0, j]), to_f64(cache[0]), sel[sel >= 0])
        assert max_rel_rowwise(o[0, j], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(lse[0, j], ref_lse, atol=2e-3, rtol=0)
    # dense, one workspace, growing then shrinking visible counts
    mp, Nh = 128, 4096
    qd = randn((1, 1, n_h, c), 333, dtype)
    cd = randn((1, Nh, c), 334, dtype)
    ws = torch.zeros(csa_attn_workspace_size(1, 1, n_h, c, Nh), dtype=torch.uint8, device=DEV)
    for tpos in (mp * 64 + 3, mp * Nh, mp * 700 + 1, mp * 65):
        out = torch.full((1, 1, n_h, c), float("nan"), dtype=torch.float32, device=DEV)
        lsed = torch.full((1, 1, n_h), float("nan"), device=DEV)
        tt = torch.tensor([tpos], dtype=torch.int64, device=DEV).reshape(1, 1)
        hca_dense_attn(dev(qd), dev(cd), tt, mp, out, ws, lse=lsed)
        torch.cuda.synchronize()
        assert csa_workspace_status(ws) == 0
        vis = oracle.visible(tpos, mp, Nh)
        ref, ref_lse = _ref_attn(to_f64(qd[0, 0]), to_f64(cd[0]), np.arange(vis, dtype=np.int32))
        assert max_rel_rowwise(out.cpu().numpy()[0, 0], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(lsed.cpu().numpy()[0, 0], ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_attn_prefill_chunk_direct_output(out_dtype):
    """A prefill chunk of 100 (sparse) and 90 (dense) queries: one CTA pair per query, so
    the split kernel writes the final output and lse itself (no combine pass), over
    several 64-entry chunks per pair.  Every query is checked, including dense queries
    that see no entry (output 0, lse -inf) and a sparse list with padding."""
    dtype, n_h, c = torch.bfloat16, 128, 512
    B, nq, N_cap, k = 1, 100, 4096, 300
    q = randn((B, nq, n_h, c), 470, dtype)
    cache = randn((B, N_cap, c), 471, dtype)
    g = torch.Generator().manual_seed(472)
    idx = torch.stack([torch.randperm(N_cap, generator=g)[:k] for _ in range(nq)]).to(torch.int32)
    idx[7, 100:250] = -1                                 # padding inside one list
    o, lse = run_sparse(dev(q), dev(cache), dev(idx.reshape(B, nq, k)), out_dtype=out_dtype)
    tol = TOL[dtype]  # the bf16 output is held to the same bound as the fp32 one
    for j in range(nq):
        sel = idx[j].numpy()
        ref, ref_lse = _ref_attn(to_f64(q[0, j]), to_f64(cache[0]), sel[sel >= 0])
        assert max_rel_rowwise(o[0, j], ref).max() <= tol
        np.testing.assert_allclose(lse[0, j], ref_lse, atol=2e-3, rtol=0)
    mp, Nh, nqd = 16, 1500, 90
    qd = randn((1, nqd, n_h, c), 473, dtype)
    cd = randn((1, Nh, c), 474, dtype)
    t = [mp * 1500 - 40 * j for j in range(nqd)]
    t[5], t[6] = 3, mp - 1                               # nothing visible
    od, lsed = run_dense(dev(qd), dev(cd), t, mp, out_dtype=out_dtype)
    for j in range(nqd):
        vis = oracle.visible(t[j], mp, Nh)
        if vis == 0:
            assert np.all(od[0, j] == 0) and np.all(np.isneginf(lsed[0, j]))
            continue
        ref, ref_lse = _ref_attn(to_f64(qd[0, j]), to_f64(cd[0]), np.arange(vis, dtype=np.int32))
        assert max_rel_rowwise(od[0, j], ref).max() <= tol
        np.testing.assert_allclose(lsed[0, j], ref_lse, atol=2e-3, rtol=0)


@pytest.mark.parametrize("dtype,n_h,c", [(torch.bfloat16, 128, 512), (torch.float32, 16, 64)])
def test_sparse_and_dense_attn_with_window(dtype, n_h, c):
    """Sliding-window branch: the window entries of tokens max(0, t-n_win+1) .. t, read
    from a ring buffer (token p at row p % win_cap), join the softmax of the selected
    (sparse) or visible (dense) compressed entries."""
    B, nq, N_cap, k, mp, n_win, win_cap = 2, 2, 3000, 256, 16, 128, 160
    q = randn((B, nq, n_h, c), 340, dtype)
    cache = randn((B, N_cap, c), 341, dtype)
    win = randn((B, win_cap, c), 342, dtype)
    g = torch.Generator().manual_seed(343)
    idx = torch.stack([torch.randperm(N_cap, generator=g)[:k] for _ in range(B * nq)]).to(torch.int32)
    idx[1, :k] = -1                                       # only window entries for this query
    idx[2, 100:] = -1
    tpos = [1000, 40, 0, mp * N_cap + 7]                  # wrapped ring, partial window, t = 0, all visible
    tt = torch.tensor(tpos, dtype=torch.int64, device=DEV).reshape(B, nq)
    qd, cd, wd = dev(q), dev(cache), dev(win)
    # sparse
    ws = torch.zeros(csa_attn_workspace_size(B, nq, n_h, c, k + n_win), dtype=torch.uint8, device=DEV)
    out = torch.full((B, nq, n_h, c), float("nan"), dtype=torch.float32, device=DEV)
    lse = torch.full((B, nq, n_h), float("nan"), device=DEV)
    csa_sparse_attn(qd, cd, dev(idx.reshape(B, nq, k)), out, ws, lse=lse, win=wd, t=tt, n_win=n_win)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws) == 0
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    for gq in range(B * nq):
        b, j = divmod(gq, nq)
        rows = to_f64(win[b])[oracle.window_positions(tpos[gq], n_win) % win_cap]
        ref, ref_lse = oracle.mqa_window(to_f64(q[b, j]), to_f64(cache[b]), idx[gq].numpy(), rows)
        assert max_rel_rowwise(o[b, j], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(l[b, j], ref_lse, atol=2e-3 if dtype == torch.bfloat16 else 1e-5, rtol=0)
    # dense
    ws2 = torch.zeros(csa_attn_workspace_size(B, nq, n_h, c, N_cap + n_win), dtype=torch.uint8, device=DEV)
    out2 = torch.full((B, nq, n_h, c), float("nan"), dtype=torch.float32, device=DEV)
    lse2 = torch.full((B, nq, n_h), float("nan"), device=DEV)
    hca_dense_attn(qd, cd, tt, mp, out2, ws2, lse=lse2, win=wd, n_win=n_win)
    torch.cuda.synchronize()
    assert csa_workspace_status(ws2) == 0
    o2, l2 = out2.cpu().numpy(), lse2.cpu().numpy()
    for gq in range(B * nq):
        b, j = divmod(gq, nq)
        vis = oracle.visible(tpos[gq], mp, N_cap)
        rows = to_f64(win[b])[oracle.window_positions(tpos[gq], n_win) % win_cap]
        ref, ref_lse = oracle.mqa_window(to_f64(q[b, j]), to_f64(cache[b]), np.arange(vis, dtype=np.int32), rows)
        assert max_rel_rowwise(o2[b, j], ref).max() <= TOL[dtype]
        np.testing.assert_allclose(l2[b, j], ref_lse, atol=2e-3 if dtype == torch.bfloat16 else 1e-5, rtol=0)


# ==================================================================================
# end to end: streams -> caches -> indexer/top-k -> sparse attention; HCA likewise
# ==================================================================================
def test_end_to_end_csa_and_hca_decode():
    """Streams -> caches -> indexer/top-k -> sparse attention, and streams -> HCA cache ->
    dense attention, checked stage by stage: each oracle stage consumes the GPU's output
    of the stage before it (the bf16 caches, the GPU's indexer keys, the GPU's selected
    indices), so every stage is held to its own tolerance.  The top-k band is the fp32
    rounding bound of the two scores plus 1e-6 relative (the near-tie rule); the sparse
    attention is checked whatever the set comparison found."""
    dtype = torch.bfloat16
    B, n, m, mp, c, cI, n_h, n_hI, k = 1, 4096, 4, 128, 512, 128, 128, 64, 128
    S = [randn((B, n, c), 400 + i, dtype) for i in range(4)]
    SI = [randn((B, n, cI), 410 + i, dtype) for i in range(4)]
    H = [randn((B, n, c), 420 + i, dtype) for i in range(2)]
    q = randn((B, 1, n_h, c), 430, dtype)
    qh = randn((B, 1, n_h, c), 433, dtype)
    qI = randn((B, 1, n_hI, cI), 431, dtype)
    wI = randn((B, 1, n_hI), 432, torch.float32)
    N, Nh, t = n // m, n // mp, n
    cache = torch.empty((B, N, c), dtype=dtype, device=DEV)
    kI = torch.empty((B, N, cI), dtype=dtype, device=DEV)
    hcache = torch.empty((B, Nh, c), dtype=dtype, device=DEV)
    csa_compress(*(dev(x) for x in S), cache, m)
    csa_compress(*(dev(x) for x in SI), kI, m)
    hca_compress(dev(H[0]), dev(H[1]), hcache, mp)
    idx, _, _ = run_indexer(dev(qI), dev(wI), kI, [t], m, k)
    o, _ = run_sparse(dev(q), cache, dev(torch.from_numpy(idx)))
    oh, _ = run_dense(dev(qh), hcache, [t], mp)

    # stage 1: the three caches against the oracle's compressors on the same streams
    gpu_cache = cache[0].float().cpu().numpy().astype(np.float64)
    gpu_kI = kI[0].float().cpu().numpy().astype(np.float64)
    gpu_h = hcache[0].float().cpu().numpy().astype(np.float64)
    ref_cache = oracle.csa_compress(*(to_f64(x[0]) for x in S), m)
    ref_kI = oracle.csa_compress(*(to_f64(x[0]) for x in SI), m)
    ref_h = oracle.hca_compress(to_f64(H[0][0]), to_f64(H[1][0]), mp)
    assert max_rel_rowwise(gpu_cache, ref_cache).max() <= 2e-2
    assert max_rel_rowwise(gpu_kI, ref_kI).max() <= 2e-2
    assert max_rel_rowwise(gpu_h, ref_h).max() <= 2e-2
    # stage 2: top-k on the GPU's keys; the sets agree except for near-ties within the
    # fp32 rounding bound of both scores plus 1e-6 relative
    q64, w64 = to_f64(qI[0, 0]), to_f64(wI[0, 0])
    s = oracle.index_scores(q64, w64, gpu_kI, oracle.visible(t, m, N))
    check_topk_sets(idx[0, 0], s, k, lambda d: score_error_bound(q64, w64, gpu_kI, d))
    # stage 3: sparse attention over the GPU's own selection on the GPU's cache
    sel = idx[0, 0][idx[0, 0] >= 0]
    ref_o, _ = oracle.mqa(to_f64(q[0, 0]), gpu_cache, sel)
    assert max_rel_rowwise(o[0, 0], ref_o).max() <= 2e-2
    # dense attention over every visible entry of the GPU's HCA cache
    ref_oh, _ = oracle.mqa(to_f64(qh[0, 0]), gpu_h, np.arange(oracle.visible(t, mp, Nh), dtype=np.int32))
    assert max_rel_rowwise(oh[0, 0], ref_oh).max() <= 2e-2
