"""ctypes marshalling for libcsa_b200.so: pointers, sizes and the current stream only."""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libcsa_b200.so")

CSA_BF16 = 0
CSA_F32 = 1

_lock = threading.Lock()
_lib = None

i32, i64, f32, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

_SIGS = {
    "csa_status_string": ([i32], ctypes.c_char_p),
    "csa_version": ([], i32),
    "csa_workspace_zero": ([vp, sz, vp], i32),
    "csa_compress": ([vp, vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, i64, i32, i32, i32, i64, i64,
                      i32, vp], i32),
    "hca_compress": ([vp, vp, i64, i64, i64, i64, vp, vp, i64, i32, i32, i32, i64, i64, i32, vp], i32),
    "hca_project_compress": ([vp, i64, i64, i64, i64, vp, vp, i32, vp, vp, i64, i32, i32, i32, i64, i64, vp, sz,
                              vp], i32),
    "csa_project_compress": ([vp, i64, i64, i64, i64, vp, vp, vp, vp, i32, vp, vp, vp, i64, i32, i32, i32, i64, i64,
                              vp, sz, vp], i32),
    "csa_indexer_topk_workspace_size": ([i32, i32, i64, i32], sz),
    "csa_workspace_status": ([vp, vp], i32),
    "csa_workspace_set_wait_budget": ([vp, i64, vp], i32),
    "csa_indexer_topk": ([vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, i32, vp, vp, vp, sz, i32, vp],
                         i32),
    "csa_indexer_topk_noalloc": ([vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, i32, vp, vp, i32, vp], i32),
    "csa_indexer_topk_noalloc_status": ([vp], i32),
    "csa_attn_workspace_size": ([i32, i32, i32, i32, i64], sz),
    "csa_sparse_attn": ([vp, vp, vp, i32, i32, i32, i32, i64, i32, f32, vp, vp, vp, sz, i32, i32, vp],
                        i32),
    "hca_dense_attn": ([vp, vp, vp, i32, i32, i32, i32, i64, i32, f32, vp, vp, vp, sz, i32, i32, vp],
                       i32),
    "csa_quantize_e4m3": ([vp, i64, i32, i64, vp, vp, i32, vp], i32),
    "csa_indexer_topk_e4m3": ([vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, i32, vp, vp, vp, sz, vp], i32),
    "csa_quantize_e2m1": ([vp, i64, i32, i64, vp, vp, i32, vp], i32),
    "csa_indexer_topk_e2m1": ([vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, i32, vp, vp, vp, sz, vp], i32),
    "csa_sparse_attn_window": ([vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i32, i32, i64, f32, vp, vp,
                                vp, sz, i32, i32, vp], i32),
    "hca_dense_attn_window": ([vp, vp, vp, vp, i32, i32, i32, i32, i64, i32, i32, i64, f32, vp, vp, vp,
                               sz, i32, i32, vp], i32),
}


class CSAError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, csa_status_string(status), status))


def library():
    """Load libcsa_b200.so (raises if it has not been built: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise ImportError("libcsa_b200.so not found at %s; build it with "
                                  "`python -m long_context_compressed_csa_b200.build`" % library_path)
            lib = ctypes.CDLL(library_path)
            for name, (args, res) in _SIGS.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def csa_status_string(status: int) -> str:
    return library().csa_status_string(int(status)).decode()


def csa_version() -> int:
    return int(library().csa_version())


def _check(fn, status):
    if status != 0:
        raise CSAError(fn, status)


def _dtype(t):
    import torch
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.float32:
        return CSA_F32
    raise TypeError("unsupported dtype %s (bf16 or fp32)" % t.dtype)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def csa_workspace_zero(ws, stream=None):
    _cuda(ws)
    _check("csa_workspace_zero", library().csa_workspace_zero(_ptr(ws), ws.numel() * ws.element_size(),
                                                              _stream(stream)))


def csa_compress(Ca, Cb, Za, Zb, out, m, entry_begin=0, entry_end=None, Ba=None, Bb=None,
                 tok0=0, stream=None):
    """CSA overlapped compression into ``out[:, entry_begin:entry_end]``.

    Ca, Cb, Za, Zb: [B, rows, c] views (same strides, last dim contiguous) holding token
    rows tok0 .. tok0+rows-1.  out: [B, N_cap, c] of the same dtype.  Ba, Bb: fp32 [m, c].
    """
    _cuda(Ca, Cb, Za, Zb, out, Ba, Bb)
    B, rows, c = Ca.shape
    for x in (Cb, Za, Zb):
        assert x.shape == Ca.shape and x.stride() == Ca.stride() and x.dtype == Ca.dtype
    assert Ca.stride(2) == 1 and out.stride(2) == 1 and out.dtype == Ca.dtype
    n = tok0 + rows
    if entry_end is None:
        entry_end = n // m
    assert out.shape[0] == B and out.shape[2] == c and out.shape[1] >= entry_end
    _check("csa_compress", library().csa_compress(
        _ptr(Ca), _ptr(Cb), _ptr(Za), _ptr(Zb), Ca.stride(1), Ca.stride(0), tok0, n,
        _ptr(Ba), _ptr(Bb), _ptr(out), out.stride(0), B, c, m, entry_begin, entry_end,
        _dtype(Ca), _stream(stream)))


def hca_compress(C, Z, out, m_prime, entry_begin=0, entry_end=None, Bias=None, tok0=0,
                 stream=None):
    """HCA compression into ``out[:, entry_begin:entry_end]`` (see csa_compress)."""
    _cuda(C, Z, out, Bias)
    B, rows, c = C.shape
    assert Z.shape == C.shape and Z.stride() == C.stride() and Z.dtype == C.dtype
    assert C.stride(2) == 1 and out.stride(2) == 1 and out.dtype == C.dtype
    n = tok0 + rows
    if entry_end is None:
        entry_end = n // m_prime
    assert out.shape[0] == B and out.shape[2] == c and out.shape[1] >= entry_end
    _check("hca_compress", library().hca_compress(
        _ptr(C), _ptr(Z), C.stride(1), C.stride(0), tok0, n, _ptr(Bias), _ptr(out), out.stride(0),
        B, c, m_prime, entry_begin, entry_end, _dtype(C), _stream(stream)))


def hca_project_compress(H, Wc, Wz, out, m_prime, workspace, entry_begin=0, entry_end=None, Bias=None, tok0=0,
                         stream=None):
    """Fused HCA projection + compression into ``out[:, entry_begin:entry_end]``: H [B, rows, d]
    bf16 token rows (token tok0 + r at row r), Wc and Wz [c, d] bf16 (output column j's weights
    in row j), out [B, N', c] bf16, workspace >= 256 bytes (zeroed once)."""
    _cuda(H, Wc, Wz, out, Bias, workspace)
    B, rows, d = H.shape
    c = Wc.shape[0]
    assert Wc.shape == (c, d) and Wz.shape == (c, d) and Wc.is_contiguous() and Wz.is_contiguous()
    assert H.stride(2) == 1 and out.stride(2) == 1 and H.dtype == Wc.dtype == Wz.dtype == out.dtype
    n = tok0 + rows
    if entry_end is None:
        entry_end = n // m_prime
    assert out.shape[0] == B and out.shape[2] == c and out.shape[1] >= entry_end
    _check("hca_project_compress", library().hca_project_compress(
        _ptr(H), H.stride(1), H.stride(0), tok0, n, _ptr(Wc), _ptr(Wz), d, _ptr(Bias), _ptr(out), out.stride(0),
        B, c, m_prime, entry_begin, entry_end, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def csa_project_compress(H, Wa_kv, Wb_kv, Wa_z, Wb_z, out, m, workspace, entry_begin=0, entry_end=None, Ba=None,
                         Bb=None, tok0=0, stream=None):
    """Fused CSA projections + overlapped compression into ``out[:, entry_begin:entry_end]``:
    H [B, rows, d] bf16 (token tok0 + r at row r), the four weights [c, d] bf16 (output column
    j's weights in row j), out [B, N, c] bf16, workspace >= 256 bytes (zeroed once)."""
    _cuda(H, Wa_kv, Wb_kv, Wa_z, Wb_z, out, Ba, Bb, workspace)
    B, rows, d = H.shape
    c = Wa_kv.shape[0]
    for W in (Wa_kv, Wb_kv, Wa_z, Wb_z):
        assert W.shape == (c, d) and W.is_contiguous() and W.dtype == H.dtype
    assert H.stride(2) == 1 and out.stride(2) == 1 and out.dtype == H.dtype
    n = tok0 + rows
    if entry_end is None:
        entry_end = n // m
    assert out.shape[0] == B and out.shape[2] == c and out.shape[1] >= entry_end
    _check("csa_project_compress", library().csa_project_compress(
        _ptr(H), H.stride(1), H.stride(0), tok0, n, _ptr(Wa_kv), _ptr(Wb_kv), _ptr(Wa_z), _ptr(Wb_z), d,
        _ptr(Ba), _ptr(Bb), _ptr(out), out.stride(0), B, c, m, entry_begin, entry_end, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_indexer_topk_workspace_size(B, nq, N_cap, k) -> int:
    return int(library().csa_indexer_topk_workspace_size(B, nq, N_cap, k))


def csa_indexer_topk(qI, wI, KI, t, m, k, idx_out, workspace, scores_out=None, stream=None):
    """Indexer scores + top-k.  qI [B,nq,n_hI,cI], wI fp32 [B,nq,n_hI], KI [B,N_cap,cI],
    t int64 [B,nq] (device), idx_out int32 [B,nq,k], workspace uint8 (zeroed once)."""
    _cuda(qI, wI, KI, t, idx_out, workspace, scores_out)
    B, nq, n_hI, cI = qI.shape
    N_cap = KI.shape[1]
    assert KI.shape == (B, N_cap, cI) and KI.is_contiguous() and qI.is_contiguous()
    assert wI.shape == (B, nq, n_hI) and wI.is_contiguous()
    assert t.numel() == B * nq and idx_out.shape == (B, nq, k) and idx_out.is_contiguous()
    _check("csa_indexer_topk", library().csa_indexer_topk(
        _ptr(qI), _ptr(wI), _ptr(KI), _ptr(t), B, nq, N_cap, n_hI, cI, m, k, _ptr(idx_out),
        _ptr(scores_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _dtype(qI), _stream(stream)))


def csa_indexer_topk_noalloc(qI, wI, KI, t, m, k, idx_out, scores_out=None, stream=None):
    """csa_indexer_topk without a workspace argument, for callers that cannot allocate:
    scratch comes from a fixed 8 MiB device array inside the library (one per GPU), so
    calls must not overlap on the GPU and the problem must fit in it."""
    _cuda(qI, wI, KI, t, idx_out, scores_out)
    B, nq, n_hI, cI = qI.shape
    N_cap = KI.shape[1]
    assert KI.shape == (B, N_cap, cI) and KI.is_contiguous() and qI.is_contiguous()
    assert wI.shape == (B, nq, n_hI) and wI.is_contiguous()
    assert t.numel() == B * nq and idx_out.shape == (B, nq, k) and idx_out.is_contiguous()
    _check("csa_indexer_topk_noalloc", library().csa_indexer_topk_noalloc(
        _ptr(qI), _ptr(wI), _ptr(KI), _ptr(t), B, nq, N_cap, n_hI, cI, m, k, _ptr(idx_out),
        _ptr(scores_out), _dtype(qI), _stream(stream)))


def csa_indexer_topk_noalloc_status(stream=None) -> int:
    """Status word of the no-allocation variant's fixed scratch after the work enqueued on
    the stream: 0, or -7 (CSA_ERR_TIMEOUT) if a device-side wait of the last
    csa_indexer_topk_noalloc call gave up.  The next such call clears it."""
    return int(library().csa_indexer_topk_noalloc_status(_stream(stream)))


def csa_workspace_status(workspace, stream=None) -> int:
    """0, or -7 (CSA_ERR_TIMEOUT) if a device-side wait of an earlier call gave up."""
    return int(library().csa_workspace_status(_ptr(workspace), _stream(stream)))


def csa_workspace_set_wait_budget(workspace, cycles, stream=None):
    """Test hook: the wait budget (SM cycles) of the indexer's grid-wide meeting, kept in
    the workspace; 0 restores the default."""
    _cuda(workspace)
    _check("csa_workspace_set_wait_budget",
           library().csa_workspace_set_wait_budget(_ptr(workspace), int(cycles), _stream(stream)))


def csa_attn_workspace_size(B, nq, n_h, c, max_entries) -> int:
    return int(library().csa_attn_workspace_size(B, nq, n_h, c, max_entries))


def csa_quantize_e4m3(x, codes, scales, stream=None):
    """Per-row E4M3 codes (uint8 tensor, same shape as x) and fp32 scales (x.shape[:-1]) of
    x [..., cols] (bf16 or fp32, rows contiguous)."""
    _cuda(x, codes, scales)
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    assert x.is_contiguous() and codes.is_contiguous() and scales.is_contiguous()
    assert codes.shape == x.shape and codes.element_size() == 1 and scales.numel() == rows
    _check("csa_quantize_e4m3", library().csa_quantize_e4m3(
        _ptr(x), rows, cols, cols, _ptr(codes), _ptr(scales), _dtype(x), _stream(stream)))


def csa_indexer_topk_e4m3(qI, wI, KI8, KI_scale, t, m, k, idx_out, workspace, scores_out=None, stream=None):
    """csa_indexer_topk on E4M3 keys KI8 [B,N_cap,cI] (uint8) with scales [B,N_cap]; qI bf16."""
    _cuda(qI, wI, KI8, KI_scale, t, idx_out, workspace, scores_out)
    B, nq, n_hI, cI = qI.shape
    N_cap = KI8.shape[1]
    assert qI.is_contiguous() and KI8.is_contiguous() and KI_scale.is_contiguous()
    assert KI8.shape == (B, N_cap, cI) and KI_scale.shape == (B, N_cap) and idx_out.shape == (B, nq, k)
    _check("csa_indexer_topk_e4m3", library().csa_indexer_topk_e4m3(
        _ptr(qI), _ptr(wI), _ptr(KI8), _ptr(KI_scale), _ptr(t), B, nq, N_cap, n_hI, cI, m, k, _ptr(idx_out),
        _ptr(scores_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_quantize_e2m1(x, codes, scales, stream=None):
    """Per-row E2M1 codes (uint8 tensor [..., cols / 2], two codes per byte) and fp32
    scales (x.shape[:-1]) of x [..., cols] (bf16 or fp32, rows contiguous)."""
    _cuda(x, codes, scales)
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    assert x.is_contiguous() and codes.is_contiguous() and scales.is_contiguous()
    assert codes.shape == x.shape[:-1] + (cols // 2,) and codes.element_size() == 1 and scales.numel() == rows
    _check("csa_quantize_e2m1", library().csa_quantize_e2m1(
        _ptr(x), rows, cols, cols, _ptr(codes), _ptr(scales), _dtype(x), _stream(stream)))


def csa_indexer_topk_e2m1(qI, wI, KI4, KI_scale, t, m, k, idx_out, workspace, scores_out=None, stream=None):
    """csa_indexer_topk on E2M1 keys KI4 [B,N_cap,cI/2] (uint8, two codes per byte) with
    scales [B,N_cap]; qI bf16."""
    _cuda(qI, wI, KI4, KI_scale, t, idx_out, workspace, scores_out)
    B, nq, n_hI, cI = qI.shape
    N_cap = KI4.shape[1]
    assert qI.is_contiguous() and KI4.is_contiguous() and KI_scale.is_contiguous()
    assert KI4.shape == (B, N_cap, cI // 2) and KI_scale.shape == (B, N_cap) and idx_out.shape == (B, nq, k)
    _check("csa_indexer_topk_e2m1", library().csa_indexer_topk_e2m1(
        _ptr(qI), _ptr(wI), _ptr(KI4), _ptr(KI_scale), _ptr(t), B, nq, N_cap, n_hI, cI, m, k, _ptr(idx_out),
        _ptr(scores_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_sparse_attn(q, cache, idx, out, workspace, lse=None, scale=0.0, stream=None,
                    win=None, t=None, n_win=0):
    """MQA of q [B,nq,n_h,c] over cache [B,N_cap,c] rows idx int32 [B,nq,k] (-1 = pad).

    With ``win`` [B,win_cap,c] (ring buffer, token p at row p % win_cap), device int64
    positions ``t`` [B,nq] and ``n_win`` >= 1, the window entries of tokens
    max(0, t-n_win+1) .. t join the same softmax (csa_sparse_attn_window)."""
    _cuda(q, cache, idx, out, workspace, lse, win, t)
    B, nq, n_h, c = q.shape
    N_cap = cache.shape[1]
    k = idx.shape[2]
    assert q.is_contiguous() and cache.is_contiguous() and idx.is_contiguous() and out.is_contiguous()
    assert cache.shape[0] == B and cache.shape[2] == c and idx.shape[:2] == (B, nq) and out.shape == q.shape
    out_bf16 = 1 if out.dtype.itemsize == 2 else 0
    ws_bytes = workspace.numel() * workspace.element_size()
    if win is None:
        _check("csa_sparse_attn", library().csa_sparse_attn(
            _ptr(q), _ptr(cache), _ptr(idx), B, nq, n_h, c, N_cap, k, float(scale), _ptr(out), _ptr(lse),
            _ptr(workspace), ws_bytes, _dtype(q), out_bf16, _stream(stream)))
        return
    assert win.is_contiguous() and win.shape[0] == B and win.shape[2] == c and t.numel() == B * nq
    _check("csa_sparse_attn_window", library().csa_sparse_attn_window(
        _ptr(q), _ptr(cache), _ptr(idx), _ptr(win), _ptr(t), B, nq, n_h, c, N_cap, k, int(n_win),
        win.shape[1], float(scale), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _dtype(q), out_bf16,
        _stream(stream)))


def hca_dense_attn(q, cache, t, m_prime, out, workspace, lse=None, scale=0.0, stream=None,
                   win=None, n_win=0):
    """Dense MQA of q [B,nq,n_h,c] over cache [B,N_cap,c] rows s < floor(t/m').

    With ``win`` [B,win_cap,c] and ``n_win`` >= 1, the window entries of tokens
    max(0, t-n_win+1) .. t join the same softmax (hca_dense_attn_window)."""
    _cuda(q, cache, t, out, workspace, lse, win)
    B, nq, n_h, c = q.shape
    N_cap = cache.shape[1]
    assert q.is_contiguous() and cache.is_contiguous() and out.is_contiguous()
    assert t.numel() == B * nq and cache.shape[0] == B and cache.shape[2] == c and out.shape == q.shape
    out_bf16 = 1 if out.dtype.itemsize == 2 else 0
    ws_bytes = workspace.numel() * workspace.element_size()
    if win is None:
        _check("hca_dense_attn", library().hca_dense_attn(
            _ptr(q), _ptr(cache), _ptr(t), B, nq, n_h, c, N_cap, m_prime, float(scale), _ptr(out),
            _ptr(lse), _ptr(workspace), ws_bytes, _dtype(q), out_bf16, _stream(stream)))
        return
    assert win.is_contiguous() and win.shape[0] == B and win.shape[2] == c
    _check("hca_dense_attn_window", library().hca_dense_attn_window(
        _ptr(q), _ptr(cache), _ptr(t), _ptr(win), B, nq, n_h, c, N_cap, m_prime, int(n_win), win.shape[1],
        float(scale), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _dtype(q), out_bf16,
        _stream(stream)))
