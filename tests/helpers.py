"""Comparison helpers shared by the GPU parity tests (no method arithmetic here beyond
the error metrics and the fp32 rounding bound of a score)."""
import numpy as np

U32 = 2.0 ** -24  # unit roundoff of fp32


def max_rel_rowwise(got, ref):
    """max |got - ref| / max |ref| over the last axis, for every leading index."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return num / den


def score_error_bound(qI, wI, KI, idx):
    """Worst-case |fp32 score - exact score| for entries idx (fp32 sums of exact products,
    ReLU 1-Lipschitz): (cI + n_hI + 2) * 2u * sum_h |w_h| sum_j |q_hj K_sj|."""
    n_hI, cI = qI.shape
    mag = (np.abs(KI[idx]) @ np.abs(qI).T) @ np.abs(wI)
    return (cI + n_hI + 2) * 2 * U32 * mag


def check_topk_sets(got_idx, oracle_scores, k, band_fn, rel=1e-6):
    """The GPU top-k set equals the oracle's except for near-ties: every index in the
    symmetric difference must score within its rounding band (plus 1e-6 relative) of
    the oracle's k-th largest score."""
    got = np.asarray(got_idx)
    vis = oracle_scores.shape[0]
    if vis <= k:
        assert list(got[:vis]) == list(range(vis))
        assert np.all(got[vis:] == -1)
        return 0
    assert np.all((got >= 0) & (got < vis)), "index out of the visible range"
    assert len(set(got.tolist())) == k, "duplicate indices"
    order = np.argsort(-oracle_scores, kind="stable")
    want = set(order[:k].tolist())
    sk = oracle_scores[order[k - 1]]
    diff = sorted(want.symmetric_difference(set(got.tolist())))
    if diff:
        d = np.array(diff)
        band = band_fn(d) + band_fn(np.array([order[k - 1]]))[0] + rel * abs(sk)
        gap = np.abs(oracle_scores[d] - sk)
        assert np.all(gap <= band), "top-k differs beyond near-ties: %s" % list(
            zip(diff, gap.tolist(), band.tolist()))
    return len(diff)


def decode_e4m3(codes):
    """Values of E4M3 byte codes (numpy uint8 array), decoded from the format definition:
    sign, 4-bit exponent with bias 7, 3-bit mantissa, subnormals at exponent 0."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    v = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7.0))
    assert not np.any((e == 15) & (m == 7)), "NaN code"
    return np.where(s == 1, -v, v)


def decode_e2m1(packed):
    """Values of E2M1 codes packed two per byte (numpy uint8 array [..., n]), the even
    element in the low nibble, decoded from the format definition: sign, 2-bit exponent
    with bias 1, 1-bit mantissa, subnormal at exponent 0.  Returns [..., 2 n]."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    c = np.stack([b & 15, b >> 4], axis=-1).reshape(b.shape[:-1] + (2 * b.shape[-1],))
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    v = np.where(e == 0, m / 2.0, (1 + m / 2.0) * 2.0 ** (e - 1.0))
    return np.where(s == 1, -v, v)
