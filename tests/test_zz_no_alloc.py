"""csa_indexer_topk_noalloc: the indexer + top-k for callers that cannot allocate device
memory (scratch comes from a fixed array inside the library instead of a workspace).

Its output must match csa_indexer_topk's on the same inputs, on two calls in a row (the
second call runs on whatever the first left in the shared scratch).  This file is
collected last so that a failure here does not stop a -x run before the other tests.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _run(fn_kind, qI, wI, KI, t, m, k):
    from long_context_compressed_csa_b200 import (csa_indexer_topk, csa_indexer_topk_noalloc,
                                                  csa_indexer_topk_workspace_size)
    B, nq = qI.shape[:2]
    idx = torch.full((B, nq, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, nq, k), float("nan"), dtype=torch.float32, device="cuda")
    if fn_kind == "workspace":
        ws = torch.zeros(csa_indexer_topk_workspace_size(B, nq, KI.shape[1], k), dtype=torch.uint8,
                         device="cuda")
        csa_indexer_topk(qI, wI, KI, t, m, k, idx, ws, scores_out=sc)
    else:
        from long_context_compressed_csa_b200 import csa_indexer_topk_noalloc_status
        csa_indexer_topk_noalloc(qI, wI, KI, t, m, k, idx, scores_out=sc)
        # a device-side timeout would show here (the next call clears it)
        assert csa_indexer_topk_noalloc_status() == 0
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


def _same_selection(a, b):
    (ia, sa), (ib, sb) = a, b
    for g in range(ia.shape[0] * ia.shape[1]):
        x, y = ia.reshape(-1, ia.shape[-1])[g], ib.reshape(-1, ib.shape[-1])[g]
        px, py = np.argsort(x, kind="stable"), np.argsort(y, kind="stable")
        np.testing.assert_array_equal(x[px], y[py])
        np.testing.assert_array_equal(sa.reshape(-1, sa.shape[-1])[g][px], sb.reshape(-1, sb.shape[-1])[g][py])


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    from long_context_compressed_csa_b200 import build
    from long_context_compressed_csa_b200.synth import randn
    build.build()
    m, k = 4, 512
    cases = [
        # tensor-core path (bf16, 64 heads x 128), two queries, one with fewer than k visible
        (randn((1, 2, 64, 128), 700, torch.bfloat16), randn((1, 2, 64), 701, torch.float32),
         randn((1, 40000, 128), 702, torch.bfloat16), [[4 * 40000, 4 * 300 + 1]]),
        # a second, different problem right after: CUDA-core path (fp32, 16 heads x 32)
        (randn((2, 1, 16, 32), 710, torch.float32), randn((2, 1, 16), 711, torch.float32),
         randn((2, 9000, 32), 712, torch.float32), [[4 * 9000 + 3], [4 * 5000]]),
        # then a chunk of 16 queries (the many-query scan, which leaves the digit-0
        # histograms untouched, then one select CTA per query), starting from the scratch
        # the two calls above left behind; visible counts from below k to all keys
        (randn((1, 16, 64, 128), 720, torch.bfloat16), randn((1, 16, 64), 721, torch.float32),
         randn((1, 3000, 128), 722, torch.bfloat16), [[4 * 100 + 800 * j for j in range(16)]]),
    ]
    for qI, wI, KI, t in cases:
        qI, wI, KI = qI.cuda(), wI.cuda(), KI.cuda()
        tt = torch.tensor(t, dtype=torch.int64, device="cuda")
        ref = _run("workspace", qI, wI, KI, tt, m, k)
        got = _run("noalloc", qI, wI, KI, tt, m, k)
        _same_selection(got, ref)
        assert np.all(got[0] >= -1)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from long_context_compressed_csa_b200 import CSAError, csa_indexer_topk_noalloc
    qI = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    wI = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    KI = torch.zeros((1, 1 << 20, 128), dtype=torch.bfloat16, device="cuda")  # ~21 MB of scratch needed
    t = torch.full((1, 1), 4 << 20, dtype=torch.int64, device="cuda")
    idx = torch.empty((1, 1, 64), dtype=torch.int32, device="cuda")
    with pytest.raises(CSAError) as e:
        csa_indexer_topk_noalloc(qI, wI, KI, t, 4, 64, idx)
    assert e.value.status == -4
