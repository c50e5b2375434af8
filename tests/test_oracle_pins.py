"""Pins for the fp64 CPU oracle: what the pages and mathematics fix, not the oracle itself.

Source: "DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch" ([P1]) - the six-token
worked example (sections 3-10), its printed softmax vectors and entries, the indexer
and top-k numerical checks (sections 6.4, 7), the single-element attention check
(section 8) and the ledger (sections 1, 12.1).  Printed decimals are rounded on the
page, so they are checked to 3e-3 while the closed forms derived from the same
numbers are checked to 1e-12.  Each pin is chosen so that a plausible slip in the
oracle (dropped b-stream, wrong block offset, softmax over the wrong axis, missing
ReLU, wrong scale, off-by-one visibility, wrong tie order) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))
E = math.e
TOL_PRINTED = GOLD["printed_tolerance"]


def g(name):
    return np.array(GOLD[name]["value"], dtype=np.float64)


def streams():
    H = g("H")
    return (oracle.project(H, g("W_aKV")), oracle.project(H, g("W_bKV")),
            oracle.project(H, g("W_aZ")), oracle.project(H, g("W_bZ")))


# ----------------------------------------------------------------------------------
# worked example: projections, compressors, indexer, top-k, attention
# ----------------------------------------------------------------------------------
def test_projection_reproduces_printed_streams():
    Ca, Cb, Za, Zb = streams()
    for name, got in (("Ca", Ca), ("Cb", Cb), ("Za", Za), ("Zb", Zb)):
        np.testing.assert_array_equal(got, g(name), err_msg=name)


def test_csa_entries_closed_form():
    Ca, Cb, Za, Zb = streams()
    C = oracle.csa_compress(Ca, Cb, Za, Zb, m=2)
    assert C.shape == (3, 2)
    want = np.array([
        [E / (E + 1), 1.0],                                   # section 5, C_0
        [(4 * E**2 + E) / (2 * E**2 + E + 1), 0.75],          # section 5, C_1
        [3 * E / (1 + 3 * E), 1.0],                           # C_2 ("analogous", derived)
    ])
    np.testing.assert_allclose(C, want, rtol=0, atol=1e-12)


def test_csa_entries_printed():
    Ca, Cb, Za, Zb = streams()
    C = oracle.csa_compress(Ca, Cb, Za, Zb, m=2)
    np.testing.assert_allclose(C[:2], g("csa_entries"), rtol=0, atol=TOL_PRINTED)


def _indicator_weights(compress, n, c, row_count, entry, col, **kw):
    """Softmax weight of every candidate row, read off the compressor by feeding a value
    stream that is 1 on one token row and 0 elsewhere (output = that row's weight)."""
    out = []
    for row in range(row_count):
        ind = np.zeros((n, c))
        ind[row, col] = 1.0
        out.append(compress(ind, entry, **kw)[col])
    return np.array(out)


def test_csa_softmax_weights_printed():
    Ca, Cb, Za, Zb = streams()
    sm = GOLD["csa_softmax"]

    def w_a(block, col):
        # weight of a-stream rows 2*block, 2*block+1 (b-stream values zero)
        ws = []
        for r in range(2):
            ind = np.zeros((6, 2)); ind[2 * block + r, col] = 1.0
            ws.append(oracle.csa_compress(ind, np.zeros((6, 2)), Za, Zb, m=2)[block, col])
        return ws

    def w_b(block, col):
        ws = []
        for r in range(2):
            row = 2 * (block - 1) + r
            if row < 0:
                ws.append(0.0)
                continue
            ind = np.zeros((6, 2)); ind[row, col] = 1.0
            ws.append(oracle.csa_compress(np.zeros((6, 2)), ind, Za, Zb, m=2)[block, col])
        return ws

    for block in (0, 1):
        for col in (0, 1):
            got = np.array(w_a(block, col) + w_b(block, col))
            want = np.array(sm["block%d_col%d" % (block, col)])
            np.testing.assert_allclose(got, want, atol=TOL_PRINTED)
            assert abs(got.sum() - 1.0) < 1e-12          # section 4 numerical check
    # block 1 column 0 closed form: [e^2, e, 1, e^2] / (2e^2 + e + 1)
    d = 2 * E**2 + E + 1
    got = np.array(w_a(1, 0) + w_b(1, 0))
    np.testing.assert_allclose(got, [E**2 / d, E / d, 1 / d, E**2 / d], atol=1e-12)


def test_hca_entries_closed_form_and_printed():
    H = g("H")
    C = oracle.project(H, g("W_aKV"))
    Z = oracle.project(H, g("W_aZ"))
    out = oracle.hca_compress(C, Z, m_prime=3)
    want = np.array([[(E + 2 * E**2) / (1 + E + E**2), 1.0], [2 * E / (2 * E + 1), 2.0 / 3.0]])
    np.testing.assert_allclose(out, want, atol=1e-12)
    np.testing.assert_allclose(out, g("hca_entries"), atol=TOL_PRINTED)


def test_hca_softmax_weights_printed():
    H = g("H")
    Z = oracle.project(H, g("W_aZ"))
    sm = GOLD["hca_softmax"]
    for block in (0, 1):
        for col in (0, 1):
            ws = []
            for r in range(3):
                ind = np.zeros((6, 2)); ind[3 * block + r, col] = 1.0
                ws.append(oracle.hca_compress(ind, Z, m_prime=3)[block, col])
            np.testing.assert_allclose(ws, sm["block%d_col%d" % (block, col)], atol=TOL_PRINTED)
            assert abs(sum(ws) - 1.0) < 1e-12


def test_indexer_queries_scores_printed():
    H = g("H")
    t = GOLD["params"]["t"]
    cQ = oracle.project(H[t:t + 1], g("W_DQ"))[0]
    np.testing.assert_array_equal(cQ, g("cQ_5"))
    qI = oracle.project(cQ[None], g("W_IUQ"))            # [1, n_hI * cI] = [1, 2]
    np.testing.assert_array_equal(qI[0], g("qI_5"))
    wI = oracle.project(H[t:t + 1], g("W_w"))[0]
    assert wI[0] == GOLD["wI_5"]["value"]
    s = oracle.index_scores(qI.reshape(1, 2), wI, g("KI"))
    np.testing.assert_array_equal(s, g("index_scores"))


def test_visibility_and_topk_printed():
    p = GOLD["params"]
    assert oracle.visible(p["t"], p["m"], 3) == GOLD["visible_csa"]["value"]
    assert oracle.visible(p["t"], p["m_prime"], 2) == GOLD["visible_hca"]["value"]
    s = oracle.index_scores(g("qI_5")[None], np.array([1.0]), g("KI"))
    np.testing.assert_array_equal(oracle.topk(s, 1), g("topk_k1").astype(np.int32))


def test_csa_attention_printed_and_k2_closed_form():
    Ca, Cb, Za, Zb = streams()
    C = oracle.csa_compress(Ca, Cb, Za, Zb, m=2)
    q = oracle.project(g("cQ_5")[None], g("W_UQ"))       # [1, 2]
    o, lse = oracle.mqa(q, C, np.array([1], np.int32))
    np.testing.assert_allclose(o[0], C[1], atol=1e-15)   # single value: output = value
    np.testing.assert_allclose(o[0], g("csa_output_k1"), atol=TOL_PRINTED)
    # k = 2 at t = 5: logits q.C_s / sqrt(2), weights and output in closed form
    c0 = E / (E + 1)
    c1 = (4 * E**2 + E) / (2 * E**2 + E + 1)
    l0, l1 = c0 / math.sqrt(2), c1 / math.sqrt(2)
    w1 = 1.0 / (1.0 + math.exp(l0 - l1))
    want = (1 - w1) * np.array([c0, 1.0]) + w1 * np.array([c1, 0.75])
    o2, lse2 = oracle.mqa(q, C, np.array([0, 1], np.int32))
    np.testing.assert_allclose(o2[0], want, atol=1e-12)
    np.testing.assert_allclose(o2[0], [1.412288, 0.832019], atol=1e-6)
    assert abs(lse2[0] - math.log(math.exp(l0) + math.exp(l1))) < 1e-12


def test_hca_attention_printed():
    H = g("H")
    C = oracle.hca_compress(oracle.project(H, g("W_aKV")), oracle.project(H, g("W_aZ")), 3)
    vis = oracle.visible(5, 3, C.shape[0])
    o, _ = oracle.mqa(g("cQ_5")[None], C, np.arange(vis, dtype=np.int32))
    np.testing.assert_allclose(o[0], C[0], atol=1e-15)
    np.testing.assert_allclose(o[0], g("hca_output"), atol=TOL_PRINTED)


# ----------------------------------------------------------------------------------
# compressor invariants and reductions
# ----------------------------------------------------------------------------------
def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("m", [1, 2, 4])
def test_csa_convex_and_constant(m):
    n, c = 6 * m, 5
    Ca, Cb, Za, Zb = (rnd(s, n, c) for s in range(4))
    out = oracle.csa_compress(Ca, Cb, Za, Zb, m)
    for i in range(n // m):
        cand_a = Ca[m * i:m * i + m]
        cand = cand_a if i == 0 else np.vstack([cand_a, Cb[m * (i - 1):m * i]])
        assert np.all(out[i] <= cand.max(0) + 1e-12) and np.all(out[i] >= cand.min(0) - 1e-12)
    const = np.tile(np.arange(c, dtype=np.float64), (n, 1))
    out = oracle.csa_compress(const, const, Za, Zb, m)
    np.testing.assert_allclose(out, np.tile(np.arange(c), (n // m, 1)), atol=1e-12)


def test_csa_equal_logits_give_mean():
    m, n, c = 4, 16, 3
    Ca, Cb = rnd(1, n, c), rnd(2, n, c)
    Z = np.full((n, c), 0.37)
    out = oracle.csa_compress(Ca, Cb, Z, Z, m)
    np.testing.assert_allclose(out[0], Ca[0:4].mean(0), atol=1e-12)      # padding excluded
    for i in range(1, n // m):
        want = np.vstack([Ca[4 * i:4 * i + 4], Cb[4 * i - 4:4 * i]]).mean(0)
        np.testing.assert_allclose(out[i], want, atol=1e-12)


def test_csa_one_hot_limits_through_logits_and_biases():
    m, n, c = 4, 12, 3
    Ca, Cb = rnd(3, n, c), rnd(4, n, c)
    Za, Zb = np.zeros((n, c)), np.zeros((n, c))
    Za[9, 1] = 60.0                  # entry 2, a-row r=1, column 1
    Zb[6, 2] = 60.0                  # b-row of entry 2 (previous block rows 4..7), r=2
    out = oracle.csa_compress(Ca, Cb, Za, Zb, m)
    assert abs(out[2, 1] - Ca[9, 1]) < 1e-12
    assert abs(out[2, 2] - Cb[6, 2]) < 1e-12
    # the bias is indexed by position within the block and shared by every block
    Ba, Bb = np.zeros((m, c)), np.zeros((m, c))
    Ba[3, 0] = 60.0
    out = oracle.csa_compress(Ca, Cb, np.zeros((n, c)), np.zeros((n, c)), m, Ba=Ba, Bb=Bb)
    for i in range(n // m):
        assert abs(out[i, 0] - Ca[m * i + 3, 0]) < 1e-12
    Bb[0, 1] = 60.0
    out = oracle.csa_compress(Ca, Cb, np.zeros((n, c)), np.zeros((n, c)), m, Ba=None, Bb=Bb)
    for i in range(1, n // m):
        assert abs(out[i, 1] - Cb[m * (i - 1), 1]) < 1e-12
    # a per-column constant added to every logit leaves the softmax unchanged
    Za, Zb = rnd(5, n, c), rnd(6, n, c)
    shift = np.tile(rnd(7, 1, c), (m, 1))
    np.testing.assert_allclose(oracle.csa_compress(Ca, Cb, Za, Zb, m, Ba=shift, Bb=shift),
                               oracle.csa_compress(Ca, Cb, Za, Zb, m), atol=1e-12)


def test_csa_reduces_to_hca_pooling_of_each_stream():
    m, n, c = 4, 20, 6
    Ca, Cb, Za, Zb = (rnd(10 + s, n, c) for s in range(4))
    ninf = np.full((n, c), -np.inf)
    # b-stream switched off: entry i = m-pooling of a-stream block i
    np.testing.assert_allclose(oracle.csa_compress(Ca, Cb, Za, ninf, m),
                               oracle.hca_compress(Ca, Za, m), atol=1e-12)
    # a-stream switched off: entry i >= 1 = m-pooling of b-stream block i-1
    out = oracle.csa_compress(Ca, Cb, ninf, Zb, m)
    np.testing.assert_allclose(out[1:], oracle.hca_compress(Cb, Zb, m)[:-1], atol=1e-12)


def test_csa_brute_force_against_scipy_softmax():
    m, n, c = 3, 12, 4
    Ca, Cb, Za, Zb = (rnd(20 + s, n, c) for s in range(4))
    Ba, Bb = rnd(30, m, c), rnd(31, m, c)
    out = oracle.csa_compress(Ca, Cb, Za, Zb, m, Ba=Ba, Bb=Bb)
    for i in range(n // m):
        la, va = Za[m * i:m * i + m] + Ba, Ca[m * i:m * i + m]
        if i == 0:
            L, V = la, va
        else:
            L = np.vstack([la, Zb[m * i - m:m * i] + Bb])
            V = np.vstack([va, Cb[m * i - m:m * i]])
        np.testing.assert_allclose(out[i], (softmax(L, axis=0) * V).sum(0), atol=1e-12)


def test_compress_entry_ranges_are_consistent():
    m, n, c = 4, 32, 5
    Ca, Cb, Za, Zb = (rnd(40 + s, n, c) for s in range(4))
    full = oracle.csa_compress(Ca, Cb, Za, Zb, m)
    np.testing.assert_array_equal(oracle.csa_compress(Ca, Cb, Za, Zb, m, i0=3, i1=5), full[3:5])
    fullh = oracle.hca_compress(Ca, Za, 8)
    np.testing.assert_array_equal(oracle.hca_compress(Ca, Za, 8, i0=2, i1=4), fullh[2:4])


def test_hca_brute_force_and_bias():
    mp, n, c = 8, 32, 3
    C, Z, Bias = rnd(50, n, c), rnd(51, n, c), rnd(52, mp, c)
    out = oracle.hca_compress(C, Z, mp, Bias=Bias)
    for i in range(n // mp):
        L = Z[mp * i:mp * i + mp] + Bias
        np.testing.assert_allclose(out[i], (softmax(L, axis=0) * C[mp * i:mp * i + mp]).sum(0),
                                   atol=1e-12)


# ----------------------------------------------------------------------------------
# indexer, top-k, attention
# ----------------------------------------------------------------------------------
def test_index_scores_brute_force_relu_and_linearity():
    n_hI, cI, N = 5, 7, 40
    qI, KI, wI = rnd(60, n_hI, cI), rnd(61, N, cI), rnd(62, n_hI)
    s = oracle.index_scores(qI, wI, KI)
    np.testing.assert_allclose(s, np.maximum(KI @ qI.T, 0.0) @ wI, atol=1e-12)
    # ReLU: a head whose dot products are all negative contributes nothing
    KIpos = np.abs(KI)
    qneg = qI.copy(); qneg[0] = -np.abs(qneg[0])
    s1 = oracle.index_scores(qneg, wI, KIpos)
    s2 = oracle.index_scores(qneg[1:], wI[1:], KIpos)
    np.testing.assert_allclose(s1, s2, atol=1e-12)
    # linear in w, and truncated at nvis
    np.testing.assert_allclose(oracle.index_scores(qI, 2 * wI, KI), 2 * s, atol=1e-12)
    np.testing.assert_array_equal(oracle.index_scores(qI, wI, KI, nvis=11), s[:11])


def test_topk_against_stable_sort_ties_and_padding():
    rng = np.random.default_rng(70)
    s = rng.integers(0, 6, size=50).astype(np.float64)        # many exact ties
    for k in (1, 7, 13, 50):
        want = np.argsort(-s, kind="stable")[:k]
        np.testing.assert_array_equal(oracle.topk(s, k), want.astype(np.int32))
    got = oracle.topk(s[:5], 8)
    assert sorted(got[:5].tolist()) == list(range(5)) and list(got[5:]) == [-1, -1, -1]
    assert list(oracle.topk(np.zeros(0), 3)) == [-1, -1, -1]
    # largest scores win regardless of position; ties resolved to the smaller index
    s = np.array([0.5, 2.0, 2.0, -1.0, 3.0])
    assert list(oracle.topk(s, 2)) == [4, 1]


def test_visibility_floor_and_cap():
    assert oracle.visible(0, 4, 10) == 0
    assert oracle.visible(3, 4, 10) == 0
    assert oracle.visible(4, 4, 10) == 1
    assert oracle.visible(8192, 4, 4096) == 2048
    assert oracle.visible(10**6, 4, 100) == 100
    assert oracle.visible(131072, 128, 1024) == 1024


def test_mqa_brute_force_lse_permutation_and_padding():
    n_h, c, N = 4, 8, 30
    q, cache = rnd(80, n_h, c), rnd(81, N, c)
    sel = np.array([3, 17, 0, 29, 8], np.int32)
    o, lse = oracle.mqa(q, cache, sel)
    logits = q @ cache[sel].T / math.sqrt(c)
    np.testing.assert_allclose(o, softmax(logits, axis=1) @ cache[sel], atol=1e-12)
    np.testing.assert_allclose(lse, logsumexp(logits, axis=1), atol=1e-12)
    o2, lse2 = oracle.mqa(q, cache, sel[::-1].copy())
    np.testing.assert_allclose(o2, o, atol=1e-12)
    o3, lse3 = oracle.mqa(q, cache, np.array([-1, 3, 17, -1, 0, 29, 8, -1], np.int32))
    np.testing.assert_allclose(o3, o, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, atol=1e-12)
    # zero query: uniform weights -> mean of the selected values
    o4, _ = oracle.mqa(np.zeros((1, c)), cache, sel)
    np.testing.assert_allclose(o4[0], cache[sel].mean(0), atol=1e-12)
    # explicit scale
    o5, lse5 = oracle.mqa(q, cache, sel, scale=0.25)
    np.testing.assert_allclose(lse5, logsumexp(q @ cache[sel].T * 0.25, axis=1), atol=1e-12)
    # nothing visible
    o6, lse6 = oracle.mqa(q, cache, np.array([-1, -1], np.int32))
    assert np.all(o6 == 0) and np.all(np.isneginf(lse6))


def test_hca_dense_equals_sparse_over_all_visible():
    n, c, mp = 64, 6, 8
    C, Z, q = rnd(90, n, c), rnd(91, n, c), rnd(92, 3, c)
    cache = oracle.hca_compress(C, Z, mp)
    t = 45
    vis = oracle.visible(t, mp, cache.shape[0])
    assert vis == 5
    o, _ = oracle.mqa(q, cache, np.arange(vis, dtype=np.int32))
    o_perm, _ = oracle.mqa(q, cache, np.random.default_rng(0).permutation(vis).astype(np.int32))
    np.testing.assert_allclose(o, o_perm, atol=1e-12)


def test_round_bf16_ties_to_even():
    vals = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.5, 0.0, 65504.0])
    got = oracle.round_bf16(vals)
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 4 * 2**-8, 1.0, -2.5, 0.0, 65536.0])


# ----------------------------------------------------------------------------------
# ledger ([P1] sections 1 and 12.1)
# ----------------------------------------------------------------------------------
def test_ledger_ratios():
    L = GOLD["ledger"]
    led = oracle.kv_ledger(n=1)
    assert led["csa_bytes"] == L["csa_bytes_per_token_layer"]
    assert led["hca_bytes"] == L["hca_bytes_per_token_layer"]
    assert led["csa_over_gqa"] == L["csa_over_gqa"]
    assert led["hca_over_gqa"] == 8 / 2048
    assert abs(led["hca_over_gqa"] - L["hca_over_gqa_printed"]) < 1e-4
    assert abs(led["mix_over_gqa"] - L["mix_numerator"] / L["mix_denominator"]) < 1e-15
    assert abs(led["mix_over_gqa"] - L["mix_over_gqa_printed"]) < 1e-3
    led2 = oracle.kv_ledger(n=1, kv_factor=2)
    assert led2["gqa_bytes"] == L["gqa_bytes_per_token_layer_section1"]
    assert led2["csa_over_gqa"] == 0.0625
    assert led["indexer_key_bytes"] == 64
    from oracle.ledger import raw_request_bytes
    assert raw_request_bytes() == 10**6 * 61 * 4096
    assert abs(raw_request_bytes() - L["raw_request_bytes_1M_61_layers"]) / 2.5e11 < 0.01


# ==================================================================================
# sliding-window branch (bhhxx.wiki "MHA -> ... -> CSA/HCA" section 6: W_t and the
# concatenation of window and compressed key/value entries under one softmax)
# ==================================================================================
def test_window_positions_pins():
    # W_t = {max(1, t-n+1), ..., t} on 1-based positions, i.e. max(0, t-n+1) .. t here
    assert oracle.window_positions(0, 128).tolist() == [0]
    assert oracle.window_positions(5, 128).tolist() == [0, 1, 2, 3, 4, 5]
    w = oracle.window_positions(1000, 128)
    assert len(w) == 128 and w[0] == 873 and w[-1] == 1000 and np.all(np.diff(w) == 1)
    assert oracle.window_positions(127, 128).tolist() == list(range(128))
    assert oracle.window_positions(128, 128).tolist() == list(range(1, 129))
    assert oracle.window_positions(7, 1).tolist() == [7]
    assert oracle.window_positions(-1, 4).size == 0 and oracle.window_positions(9, 0).size == 0


def test_window_mqa_closed_form_two_entries():
    """One compressed entry and one window entry, c = 2, one head: the output is the
    softmax(logit) mix of the two in closed form."""
    a, b = 1.3, -0.4
    q = np.array([[1.0, 2.0]])
    cache = np.array([[a, 0.0]])           # logit = a / sqrt(2)
    win = np.array([[0.0, b]])             # logit = 2b / sqrt(2)
    out, lse = oracle.mqa_window(q, cache, np.array([0]), win)
    la, lb = a / np.sqrt(2.0), 2 * b / np.sqrt(2.0)
    pa = np.exp(la) / (np.exp(la) + np.exp(lb))
    np.testing.assert_allclose(out[0], [pa * a, (1 - pa) * b], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], np.log(np.exp(la) + np.exp(lb)), rtol=0, atol=1e-14)


def test_window_mqa_invariants():
    rng = np.random.default_rng(7)
    n_h, c, N = 3, 8, 20
    q, cache = rng.standard_normal((n_h, c)), rng.standard_normal((N, c))
    win = rng.standard_normal((5, c))
    sel = np.array([4, -1, 11, 2], dtype=np.int32)
    out, lse = oracle.mqa_window(q, cache, sel, win)
    # the order of the window rows (and of the selection) does not matter
    out2, lse2 = oracle.mqa_window(q, cache, sel[::-1], win[::-1])
    np.testing.assert_allclose(out2, out, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    # window only (every compressed slot padded) equals plain MQA over the window rows
    ow, lw = oracle.mqa_window(q, cache, np.full(3, -1, np.int32), win)
    ow2, lw2 = oracle.mqa(q, win, np.arange(5, dtype=np.int32))
    np.testing.assert_allclose(ow, ow2, atol=1e-13)
    np.testing.assert_allclose(lw, lw2, atol=1e-13)
    # no window rows: plain sparse MQA
    o0, l0 = oracle.mqa_window(q, cache, sel, np.zeros((0, c)))
    o1, l1 = oracle.mqa(q, cache, sel)
    np.testing.assert_allclose(o0, o1, atol=1e-14)
    np.testing.assert_allclose(l0, l1, atol=1e-14)
    # a window row equal to a selected compressed row counts as that entry twice
    od, ld = oracle.mqa_window(q, cache, np.array([4, 11], np.int32), cache[[4]])
    oe, le = oracle.mqa(q, cache, np.array([4, 4, 11], np.int32))
    np.testing.assert_allclose(od, oe, atol=1e-13)
    np.testing.assert_allclose(ld, le, atol=1e-13)
    # lse combines like a union: exp(lse) = exp(lse_comp) + exp(lse_win)
    lc = oracle.mqa(q, cache, sel)[1]
    np.testing.assert_allclose(np.exp(lse), np.exp(lc) + np.exp(lw2), rtol=1e-12)


# ==================================================================================
# FP8 (E4M3) indexer operands (reading of [P1] section 6.4 "FP4 indexer"; format chosen:
# E4M3 codes with one fp32 scale per row)
# ==================================================================================
def _e4m3_table():
    """Every finite E4M3 value, decoded from the 8-bit codes by the format definition
    (sign, 4-bit exponent with bias 7, 3-bit mantissa, subnormals at exponent 0;
    exponent 15 with mantissa 7 is NaN)."""
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(-v if s else v)
    return np.unique(np.array(vals))


def test_e4m3_rounding_pins():
    tab = _e4m3_table()
    assert tab.max() == 448.0 and tab.min() == -448.0 and len(tab) == 253  # +-0 merge
    # every representable value is a fixed point
    np.testing.assert_array_equal(oracle.round_e4m3(tab.astype(np.float32)), tab)
    # midpoints between neighbours round to the one with an even mantissa
    pos = tab[tab >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = oracle.round_e4m3(mids.astype(np.float32))
    for mid, g, a, b in zip(mids, got, pos[:-1], pos[1:]):
        assert g in (a, b)
        # the even neighbour: code mantissa bit 0 clear; on the grid, a/step even
        e = max(np.floor(np.log2(a)) if a > 0 else -6, -6)
        step = 2.0 ** (e - 3)
        assert (g / step) % 2 == 0 or g == b == 2 ** (e + 1)
    # saturation, sign symmetry, nearest rounding away from midpoints
    np.testing.assert_array_equal(oracle.round_e4m3(np.float32([500.0, -1e6, 449.0])), [448, -448, 448])
    rng = np.random.default_rng(3)
    x = rng.uniform(-400, 400, 2000).astype(np.float32)
    r = oracle.round_e4m3(x)
    idx = np.abs(tab[None, :] - x[:, None].astype(np.float64)).argmin(axis=1)
    dist_best = np.abs(tab[idx] - x)
    np.testing.assert_array_equal(np.abs(r - x), dist_best)   # nearest (ties aside)
    np.testing.assert_array_equal(oracle.round_e4m3(-x), -r)


def test_e4m3_row_quantisation_and_scores():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((50, 128)).astype(np.float32)
    X[7] = 0.0
    codes, scale = oracle.quantize_rows_e4m3(X)
    assert scale[7] == 0 and np.all(codes[7] == 0)
    amax = np.abs(X).max(axis=1)
    np.testing.assert_array_equal(scale[:7], (amax[:7] / np.float32(448)).astype(np.float32))
    # the largest entry of each row maps to +-448; every code is an E4M3 value
    rows = np.arange(50) != 7
    assert np.all(np.abs(codes[rows]).max(axis=1) == 448.0)
    assert np.all(np.isin(codes, _e4m3_table()))
    # relative error of E4M3 is at most 2^-4 of the value above the subnormal range
    deq = codes * scale[:, None]
    big = np.abs(X) >= 2.0 ** -6 * scale[:, None]
    assert np.all(np.abs(deq - X)[big] <= 2.0 ** -4 * np.abs(X)[big] + 1e-30)
    # scores on E4M3 operands stay within the operand error of the exact scores
    qI, wI, KI = rng.standard_normal((16, 128)), rng.standard_normal(16), rng.standard_normal((300, 128))
    s8 = oracle.index_scores_e4m3(qI, wI, KI)
    s = oracle.index_scores(qI, wI, KI)
    bound = np.abs(wI) @ (np.abs(qI) @ np.abs(KI).T) * (2 * 2.0 ** -4 + 2.0 ** -8) + 1e-9
    assert np.all(np.abs(s8 - s) <= bound)
    assert np.corrcoef(s8, s)[0, 1] > 0.99


# ==================================================================================
# FP4 (E2M1) indexer keys (reading of [P1] section 6.4 "FP4 indexer"; format chosen:
# E2M1 codes with one fp32 scale per key, the query E4M3 per head)
# ==================================================================================
def _e2m1_table():
    """Every E2M1 value, decoded from the 4-bit codes by the format definition (sign,
    2-bit exponent with bias 1, 1-bit mantissa, subnormal at exponent 0)."""
    vals = []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        v = (m / 2.0) if e == 0 else (1 + m / 2.0) * 2.0 ** (e - 1)
        vals.append(-v if s else v)
    return np.unique(np.array(vals))


def test_e2m1_rounding_pins():
    tab = _e2m1_table()
    np.testing.assert_array_equal(tab[tab >= 0], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(oracle.round_e2m1(tab.astype(np.float32)), tab)
    # midpoints go to the neighbour whose code has mantissa bit 0
    mids = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    np.testing.assert_array_equal(oracle.round_e2m1(mids), [0, 1, 1, 2, 2, 4, 4])
    np.testing.assert_array_equal(oracle.round_e2m1(-mids), -np.array([0, 1, 1, 2, 2, 4, 4.0]))
    # saturation and nearest rounding away from midpoints
    np.testing.assert_array_equal(oracle.round_e2m1(np.float32([6.5, 100.0, -7.0, 5.01, 0.26, 0.24])),
                                  [6, 6, -6, 6, 0.5, 0])
    rng = np.random.default_rng(5)
    x = rng.uniform(-6, 6, 4000).astype(np.float32)
    r = oracle.round_e2m1(x)
    idx = np.abs(tab[None, :] - x[:, None].astype(np.float64)).argmin(axis=1)
    np.testing.assert_array_equal(np.abs(r - x), np.abs(tab[idx] - x))


def test_e2m1_row_quantisation_and_scores():
    # a hand-worked row: max|x| = 6, so the factor is 1 and the codes are E2M1(x)
    codes, scale = oracle.quantize_rows_e2m1(np.float32([[6.0, 3.0, 1.4, -0.2, 0.0, 5.2, -2.6, 0.8]]))
    assert scale[0] == 1.0
    np.testing.assert_array_equal(codes[0], [6, 3, 1.5, -0, 0, 6, -3, 1])
    rng = np.random.default_rng(6)
    X = rng.standard_normal((60, 128)).astype(np.float32)
    X[9] = 0.0
    codes, scale = oracle.quantize_rows_e2m1(X)
    assert scale[9] == 0 and np.all(codes[9] == 0)
    amax = np.abs(X).max(axis=1)
    rows = np.arange(60) != 9
    np.testing.assert_array_equal(scale[rows], (amax[rows] / np.float32(6)).astype(np.float32))
    assert np.all(np.abs(codes[rows]).max(axis=1) == 6.0)   # the largest entry maps to +-6
    assert np.all(np.isin(codes, _e2m1_table()))
    # E2M1 error: at most a quarter of max(|x|, scale) (half a grid step)
    deq = codes * scale[:, None]
    tol = 0.25 * np.maximum(np.abs(X), scale[:, None]) * (1 + 1e-6)
    assert np.all(np.abs(deq - X) <= tol)
    # scores with E2M1 keys and E4M3 queries stay within the operands' error
    qI, wI, KI = rng.standard_normal((16, 128)), rng.standard_normal(16), rng.standard_normal((300, 128))
    s4 = oracle.index_scores_e2m1(qI, wI, KI)
    s = oracle.index_scores(qI, wI, KI)
    kc, ks = oracle.quantize_rows_e2m1(KI)
    dk = 0.25 * (np.abs(KI) + ks[:, None])                 # key error bound per element
    dq = 2.0 ** -4 * np.abs(qI) + 2.0 ** -9 * np.abs(qI).max(axis=1, keepdims=True) / 448
    bound = np.abs(wI) @ ((np.abs(qI) + dq) @ dk.T + dq @ np.abs(KI).T) + 1e-9
    assert np.all(np.abs(s4 - s) <= bound)
    assert np.corrcoef(s4, s)[0, 1] > 0.9
