"""Plain fp64 CPU oracle for the CSA / HCA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
``--impl reference`` leg may import this package.  The product library never imports,
links or calls it; the two share no code.  The arithmetic lives in ``csa_oracle.c``
(compiled here with gcc into ``liboracle.so``); this module only marshals numpy arrays.

Sources:
  "DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch" (cited as [P1]) sections 3-12;
  bhhxx.wiki "MHA -> ... -> CSA/HCA", section 6.2.2 (cited as [P4]).

Parity pins: tests/test_oracle_pins.py (worked example in closed form, printed values,
invariants, brute force against library routines, ledger).  No function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile csa_oracle.c with gcc (plain -O2, no fast-math) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.oracle_project.argtypes = [dp, dp, i64, i64, i64, dp]
            lib.oracle_csa_compress.argtypes = [dp, dp, dp, dp, dp, dp, i64, i64, i64, i64, i64, dp]
            lib.oracle_hca_compress.argtypes = [dp, dp, dp, i64, i64, i64, i64, i64, dp]
            lib.oracle_visible.argtypes = [i64, i64, i64]
            lib.oracle_visible.restype = i64
            lib.oracle_window.argtypes = [i64, i64, ctypes.POINTER(ctypes.c_int64)]
            lib.oracle_window.restype = i64
            lib.oracle_index_scores.argtypes = [dp, dp, dp, i64, i64, i64, dp]
            lib.oracle_topk.argtypes = [dp, i64, i64, ctypes.POINTER(ctypes.c_int32)]
            lib.oracle_mqa.argtypes = [dp, dp, ctypes.POINTER(ctypes.c_int32), i64, i64, i64,
                                       ctypes.c_double, dp, dp]
            _lib = lib
    return _lib


def _d(a):
    """Contiguous float64 copy (or view) of ``a``."""
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def project(H, W):
    """out = H @ W by the plain triple loop ([P1] section 3)."""
    H, W = _d(H), _d(W)
    n, d = H.shape
    d2, c = W.shape
    assert d == d2
    out = np.empty((n, c), np.float64)
    _load().oracle_project(_ptr(H), _ptr(W), n, d, c, _ptr(out))
    return out


def csa_compress(Ca, Cb, Za, Zb, m, Ba=None, Bb=None, i0=0, i1=None):
    """CSA overlapped compressor ([P1] sections 4-5): entries i0 <= i < i1, [i1-i0, c]."""
    Ca, Cb, Za, Zb = _d(Ca), _d(Cb), _d(Za), _d(Zb)
    n, c = Ca.shape
    for a in (Cb, Za, Zb):
        assert a.shape == (n, c)
    if i1 is None:
        i1 = n // m
    assert 0 <= i0 <= i1 and m * i1 <= n
    Ba = None if Ba is None else _d(Ba)
    Bb = None if Bb is None else _d(Bb)
    if Ba is not None:
        assert Ba.shape == (m, c)
    if Bb is not None:
        assert Bb.shape == (m, c)
    out = np.empty((i1 - i0, c), np.float64)
    _load().oracle_csa_compress(_ptr(Ca), _ptr(Cb), _ptr(Za), _ptr(Zb), _ptr(Ba), _ptr(Bb),
                                n, c, m, i0, i1, _ptr(out))
    return out


def hca_compress(C, Z, m_prime, Bias=None, i0=0, i1=None):
    """HCA compressor ([P1] section 10): entries i0 <= i < i1, [i1-i0, c]."""
    C, Z = _d(C), _d(Z)
    n, c = C.shape
    assert Z.shape == (n, c)
    if i1 is None:
        i1 = n // m_prime
    assert 0 <= i0 <= i1 and m_prime * i1 <= n
    Bias = None if Bias is None else _d(Bias)
    if Bias is not None:
        assert Bias.shape == (m_prime, c)
    out = np.empty((i1 - i0, c), np.float64)
    _load().oracle_hca_compress(_ptr(C), _ptr(Z), _ptr(Bias), n, c, m_prime, i0, i1, _ptr(out))
    return out


def visible(t, m, N_cap):
    """Number of compressed entries query t may see: min(floor(t/m), N_cap) ([P1] s.7)."""
    return int(_load().oracle_visible(int(t), int(m), int(N_cap)))


def index_scores(qI, wI, KI, nvis=None):
    """I[s] = sum_h w[h] ReLU(q[h].K[s]) for s < nvis ([P1] section 6.4)."""
    qI, wI, KI = _d(qI), _d(wI), _d(KI)
    n_hI, cI = qI.shape
    assert wI.shape == (n_hI,)
    if nvis is None:
        nvis = KI.shape[0]
    assert KI.shape[1] == cI and nvis <= KI.shape[0]
    out = np.empty((nvis,), np.float64)
    _load().oracle_index_scores(_ptr(qI), _ptr(wI), _ptr(KI), nvis, n_hI, cI, _ptr(out))
    return out


def topk(scores, k):
    """Indices of the k largest scores, ties to the smaller index, -1 padded ([P1] s.7)."""
    scores = _d(scores)
    idx = np.empty((k,), np.int32)
    _load().oracle_topk(_ptr(scores), scores.shape[0], k, _ptr(idx, ctypes.c_int32))
    return idx


def mqa(q, cache, sel, scale=None):
    """Shared-KV MQA over the entries ``sel`` (-1 skipped) ([P1] section 8).

    Returns (out [n_h, c], lse [n_h]); scale defaults to 1/sqrt(c).
    """
    q, cache = _d(q), _d(cache)
    n_h, c = q.shape
    assert cache.shape[1] == c
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    assert sel.ndim == 1
    if sel.size:
        assert sel.max() < cache.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(c)
    out = np.empty((n_h, c), np.float64)
    lse = np.empty((n_h,), np.float64)
    _load().oracle_mqa(_ptr(q), _ptr(cache) if cache.size else _ptr(np.zeros(1)),
                       _ptr(sel, ctypes.c_int32) if sel.size else None, sel.size, n_h, c,
                       float(scale), _ptr(out), _ptr(lse))
    return out, lse


def window_positions(t, n_win):
    """Token positions of the sliding-window branch for the query at position t:
    max(0, t - n_win + 1) .. t (bhhxx.wiki "MHA -> ... -> CSA/HCA" section 6, W_t)."""
    pos = np.empty((max(int(n_win), 1),), np.int64)
    n = _load().oracle_window(int(t), int(n_win), _ptr(pos, ctypes.c_int64))
    return pos[:n].copy()


def mqa_window(q, cache, sel, win_rows, scale=None):
    """MQA whose shared key/value set is the selected compressed entries ``sel`` (-1
    skipped) concatenated with the sliding-window entries ``win_rows`` [n, c] (bhhxx.wiki
    section 6: "concat sliding window key/value entries and compressed entries"), under
    one softmax.  Returns (out [n_h, c], lse [n_h])."""
    cache, win_rows = _d(cache), _d(win_rows).reshape(-1, _d(cache).shape[1])
    sel = np.ascontiguousarray(sel, dtype=np.int32).reshape(-1)
    keys = np.concatenate([cache, win_rows], axis=0)
    sel2 = np.concatenate([sel, cache.shape[0] + np.arange(win_rows.shape[0], dtype=np.int32)])
    return mqa(q, keys, sel2, scale)


# ----------------------------------------------------------------------------------
# FP8 (E4M3) indexer keys and queries.  The pages run the indexer in FP4 ([P1] section 6.4:
# scoring "performed in FP4 precision", viable because the scores are never
# exponentiated) and note FP4 has the peak of FP8 on current hardware ([P1] section 12);
# the block-scale format is not given.  The reading used: OCP E4M3 codes (1 sign, 4
# exponent bits with bias 7, 3 mantissa bits, subnormals, largest finite 448, no
# infinities) with one fp32 scale per row (per key, per query head) = max|x| / 448; the
# codes are E4M3(x * (448 / max|x|)).
# ----------------------------------------------------------------------------------
E4M3_MAX = 448.0


def round_e4m3(x):
    """Round fp32 values to the nearest E4M3 value, ties to even, saturating at +-448
    (the format's definition; as float64)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    # grid spacing at |x|: 2^(e - 3) for the binade [2^e, 2^(e+1)), e >= -6; 2^-9 below 2^-6
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    r = np.round(a / step) * step          # np.round: half to even
    r = np.minimum(r, E4M3_MAX)
    return np.where(a > 0, np.copysign(r, x), 0.0 * x)


def quantize_rows_e4m3(X):
    """Per-row E4M3 quantisation: dequantisation scale = max|x| / 448 and quantisation
    factor r = 448 / max|x|, both one fp32 division per row; code = E4M3(x * r) with the
    product in fp32 (rows of zeros: scale 0, codes 0).  Returns (values of the codes
    [rows, cols] float64, scales [rows] float64)."""
    X = np.asarray(X, dtype=np.float32)
    X2 = X.reshape(-1, X.shape[-1])
    amax = np.max(np.abs(X2), axis=1).astype(np.float32)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    r = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    q = (X2 * r[:, None]).astype(np.float32)
    codes = np.where(amax[:, None] > 0, round_e4m3(q), 0.0)
    return codes.reshape(X.shape), scale.astype(np.float64).reshape(X.shape[:-1])


def index_scores_e4m3(qI, wI, KI, nvis=None):
    """[P1] section 6.4 scores on E4M3 operands: q^I (per head) and K^I (per key) are
    quantised by quantize_rows_e4m3 and the boxed formula is evaluated in fp64 on the
    dequantised values (code x scale)."""
    qc, qs = quantize_rows_e4m3(qI)
    kc, ks = quantize_rows_e4m3(KI)
    return index_scores(qc * qs[:, None], wI, kc * ks[:, None], nvis)


# ----------------------------------------------------------------------------------
# FP4 (E2M1) indexer keys.  [P1] section 6.4 runs the indexer's products in FP4; the
# element and scale formats are not given.  The reading used: OCP E2M1 codes (1 sign, 2
# exponent bits with bias 1, 1 mantissa bit, one subnormal 0.5; values 0, 0.5, 1, 1.5,
# 2, 3, 4, 6) with one fp32 scale per key = max|x| / 6; the codes are E2M1(x * (6 /
# max|x|)), the product in fp32, rounded to nearest even and saturated at +-6.  The
# query stays E4M3 per head (quantize_rows_e4m3): the key cache is what the scan streams,
# the query is 16 KB.
# ----------------------------------------------------------------------------------
E2M1_MAX = 6.0
E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # magnitudes of codes 0..7


def round_e2m1(x):
    """Round fp32 values to the nearest E2M1 value, ties to the even code (mantissa bit
    0), saturating at +-6 (the format's definition; as float64)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E2M1_MAX)
    # grid spacing at |x|: 0.5 below 2, 1 in [2, 4), 2 in [4, 6]
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    r = np.round(a / step) * step  # np.round: half to even, which is the even code here
    r = np.minimum(r, E2M1_MAX)
    return np.where(a > 0, np.copysign(r, x), 0.0 * x)


def quantize_rows_e2m1(X):
    """Per-row E2M1 quantisation: dequantisation scale = max|x| / 6 and quantisation
    factor r = 6 / max|x|, both one fp32 division per row; code = E2M1(x * r) with the
    product in fp32 (rows of zeros: scale 0, codes 0).  Returns (values of the codes
    [rows, cols] float64, scales [rows] float64)."""
    X = np.asarray(X, dtype=np.float32)
    X2 = X.reshape(-1, X.shape[-1])
    amax = np.max(np.abs(X2), axis=1).astype(np.float32)
    scale = (amax / np.float32(E2M1_MAX)).astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    r = (np.float32(E2M1_MAX) / safe).astype(np.float32)
    q = (X2 * r[:, None]).astype(np.float32)
    codes = np.where(amax[:, None] > 0, round_e2m1(q), 0.0)
    return codes.reshape(X.shape), scale.astype(np.float64).reshape(X.shape[:-1])


def index_scores_e2m1(qI, wI, KI, nvis=None):
    """[P1] section 6.4 scores with E2M1 keys (quantize_rows_e2m1, one scale per key) and
    E4M3 query heads (quantize_rows_e4m3, one scale per head); the boxed formula is
    evaluated in fp64 on the dequantised values (code x scale)."""
    qc, qs = quantize_rows_e4m3(qI)
    kc, ks = quantize_rows_e2m1(KI)
    return index_scores(qc * qs[:, None], wI, kc * ks[:, None], nvis)


def round_bf16(x):
    """Round float64/float32 values to the nearest bfloat16 (ties to even), as float64.

    This is the storage rounding of a bf16 compressed cache (the pages do not fix the
    cache precision; the reading used is bf16 round-to-nearest-even).  Written here
    independently of the CUDA library's conversion.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(f)
    out = r.astype(np.uint32).view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out


from .ledger import kv_ledger  # noqa: E402  (pure arithmetic of [P1] section 12)

__all__ = ["build", "project", "csa_compress", "hca_compress", "visible", "index_scores",
           "topk", "mqa", "round_bf16", "kv_ledger"]
