"""Benchmark: hybrid CSA + HCA decode at a 1M-token context on B200.

Workload ("hybrid_1m_decode"): batch 1, n = 2^20 prefilled tokens; a CSA layer with
m = 4 (262144 compressed entries of c = 512, indexer keys c^I = 128, n_h^I = 64,
k = 1024) and an HCA layer with m' = 128 (8192 entries), n_h = 128 query heads, bf16
caches, fp32 accumulation.  A step is one generated token through one CSA + HCA layer
pair: csa_indexer_topk -> csa_sparse_attn -> hca_dense_attn, plus the incremental
csa_compress (KV cache and indexer keys) when the token completes an m-block and
hca_compress when it completes an m'-block.  Eight independent layer pairs are
visited in turn (token j passes through pairs 0..7, like consecutive layers), so the
73 MiB a step reads is evicted from the 126 MB L2 before the same pair is read again.

Prints one JSON line.  `value` = layer-pair decode steps per second with every input
resident in HBM (device-timed CUDA events around CUDA-graph replays); `e2e` = the same
steps driven eagerly through the C ABI with each step's inputs copied from pinned host
memory and both outputs copied back.  `--impl reference` times the fp64 CPU oracle on
the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode tokens/s at 128K–1M ctx; achieved HBM GB/s vs ~8 TB/s peak"
WORKLOAD = "hybrid_1m_decode"
N_PAIRS = 8
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one scan_tc_kernel launch
# over 262144 keys, per key format, from one ncu capture of the current kernel each: bf16
# 67.21 MB read + 0.59 MB written (algorithmic 67.11 MB), E4M3 34.71 MB read (34.60 MB),
# E2M1 17.93 MB read (17.83 MB).  Must be retaken (or set to None) when the kernel changes.
SCAN_TRAFFIC_BYTES = {"bf16": 67_799_296, "e4m3": 34_714_880, "e2m1": 17_927_680}
IDX_SAMPLE = 8  # steps per CUDA graph; the indexer call of each graph's first step is timed


def max_over_ranks(x, device="cpu"):
    """Max of a per-rank float over all ranks of the default process group (the value
    itself on one rank).  The device is the group's: "cuda" under NCCL, "cpu" under gloo."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(steps_per_rank, world, ms_max):
    """Steps per second of the whole job: every rank's steps over the slowest rank's time."""
    return steps_per_rank * world / (ms_max / 1000.0)


def workload_config(world, kI_format="bf16"):
    """The `config` object of both arms' JSON line (the 1M-token hybrid decode)."""
    return {"workload": WORKLOAD, "kI_format": kI_format, "n": 1 << 20, "B": 1, "c": 512, "m": 4, "m_prime": 128, "k": 1024,
            "n_h": 128, "n_hI": 64, "cI": 128, "pairs_rotated": N_PAIRS,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2: 8 layer pairs rotated (73 MiB read per step, "
                  "584 MiB between revisits of a pair)",
            "step": "one token through one CSA+HCA layer pair (indexer+top-k, sparse MQA, "
                    "dense MQA, incremental compress at block ends)"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = np.array([float(r[1]) for r in rows])
        mx = float(rows[0][2])
        load = sm[sm >= 0.5 * sm.max()] if sm.max() > 0 else sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, nm in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


# ----------------------------------------------------------------------------------
# workload state on one GPU
# ----------------------------------------------------------------------------------
class HybridDecode:
    """Eight CSA + HCA layer pairs prefilled at n = 2^20, ready for decode steps."""

    def __init__(self, torch, steps_total, seed=5000, n=1 << 20, device="cuda", kI_format="bf16"):
        import long_context_compressed_csa_b200 as lib
        from long_context_compressed_csa_b200.synth import randn, randint_values
        self.torch, self.lib = torch, lib
        self.n, self.m, self.mp, self.c, self.cI = n, 4, 128, 512, 128
        self.n_h, self.n_hI, self.k = 128, 64, 1024
        self.dev = device
        # indexer keys as E4M3 (one byte) or E2M1 (half a byte) codes + one fp32 scale per key
        self.kfmt = kI_format
        self.e4m3, self.e2m1 = kI_format == "e4m3", kI_format == "e2m1"
        self.quant = self.e4m3 or self.e2m1
        bf16 = torch.bfloat16
        self.tokens = (steps_total + N_PAIRS - 1) // N_PAIRS + 1
        T = self.tokens
        self.N = n // self.m
        self.Nh = n // self.mp
        self.N_cap = self.N + T // self.m + 1
        self.Nh_cap = self.Nh + T // self.mp + 1
        self.hist = 2 * self.m  # stream rows kept from before the decode (for block i-1)
        c, cI = self.c, self.cI
        self.row_width = 4 * (c + cI) + 2 * c  # elements of one token's decode stream rows
        self.pairs = []
        t0 = time.time()
        for p in range(N_PAIRS):
            s = seed + 100 * p
            P = {}
            P["cache"] = torch.empty((1, self.N_cap, c), dtype=bf16, device=device)
            P["kI"] = torch.empty((1, self.N_cap, cI), dtype=bf16, device=device)
            P["hcache"] = torch.empty((1, self.Nh_cap, c), dtype=bf16, device=device)
            # prefill compress through the library (streams generated in slices)
            self._prefill(P, s)
            if self.quant:  # quantise the prefill keys once; the bf16 cache stays the staging of new keys
                P["kI8"] = torch.zeros((1, self.N_cap, cI if self.e4m3 else cI // 2), dtype=torch.uint8,
                                       device=device)
                P["kIs"] = torch.zeros((1, self.N_cap), dtype=torch.float32, device=device)
                self._quantize(P, 0, self.N)
            # decode-time stream rows, one interleaved row per token (the 4 CSA streams, the
            # 4 indexer-key streams, the 2 HCA streams), so that a token's new rows are one
            # contiguous copy: tokens n - hist .. n + T - 1 (CSA), n .. n + T - 1 (HCA)
            P["rows"] = randn((1, self.hist + T, self.row_width), s + 10, bf16, device)
            R = P["rows"]
            P["dec"] = [R[:, :, i * c:(i + 1) * c] for i in range(4)]
            P["decI"] = [R[:, :, 4 * c + i * cI:4 * c + (i + 1) * cI] for i in range(4)]
            P["decH"] = [R[:, self.hist:, 4 * (c + cI) + i * c:4 * (c + cI) + (i + 1) * c] for i in range(2)]
            self.pairs.append(P)
        torch.cuda.synchronize()
        log("prefill of %d layer pairs: %.1f s" % (N_PAIRS, time.time() - t0))
        # per-step queries: a pool of 64 distinct sets reused cyclically
        self.nQ = 64
        self.q = randn((self.nQ, 1, 1, self.n_h, c), seed + 1, bf16, device)
        self.qh = randn((self.nQ, 1, 1, self.n_h, c), seed + 2, bf16, device)
        self.qI = randn((self.nQ, 1, 1, self.n_hI, cI), seed + 3, bf16, device)
        self.wI = randn((self.nQ, 1, 1, self.n_hI), seed + 4, torch.float32, device)
        self.tpos = torch.arange(n, n + T, dtype=torch.int64, device=device).reshape(T, 1, 1)
        # outputs and workspaces (one set per pair so steps never share scratch in flight)
        self.idx = torch.empty((1, 1, self.k), dtype=torch.int32, device=device)
        self.obuf = torch.empty((2, 1, 1, self.n_h, c), dtype=torch.float32, device=device)
        self.o, self.oh = self.obuf[0], self.obuf[1]  # CSA and HCA outputs, adjacent
        self.ws_topk = torch.zeros(lib.csa_indexer_topk_workspace_size(1, 1, self.N_cap, self.k),
                                   dtype=torch.uint8, device=device)
        self.ws_attn = torch.zeros(lib.csa_attn_workspace_size(1, 1, self.n_h, c, self.k),
                                   dtype=torch.uint8, device=device)
        self.ws_hattn = torch.zeros(lib.csa_attn_workspace_size(1, 1, self.n_h, c, self.Nh_cap),
                                    dtype=torch.uint8, device=device)

    def _prefill(self, P, s):
        torch, lib = self.torch, self.lib
        from long_context_compressed_csa_b200.synth import randn
        bf16 = torch.bfloat16
        c, cI, m, mp = self.c, self.cI, self.m, self.mp
        chunk = 1 << 17  # tokens per slice (multiple of m')
        for lo in range(0, self.n, chunk):
            hi = min(self.n, lo + chunk)
            base = max(0, lo - m)  # block i-1 of the first entry of the slice
            rows = hi - base
            S = [randn((1, rows, c), s * 1000 + lo // chunk * 8 + i, bf16, self.dev) for i in range(4)]
            lib.csa_compress(*S, P["cache"], m, lo // m, hi // m, tok0=base)
            del S
            SI = [randn((1, rows, cI), s * 1000 + 500 + lo // chunk * 8 + i, bf16, self.dev) for i in range(4)]
            lib.csa_compress(*SI, P["kI"], m, lo // m, hi // m, tok0=base)
            del SI
            H = [randn((1, hi - lo, c), s * 1000 + 900 + lo // chunk * 8 + i, bf16, self.dev) for i in range(2)]
            lib.hca_compress(H[0], H[1], P["hcache"], mp, lo // mp, hi // mp, tok0=lo)
            del H

    # one step: token j through layer pair p (part 0: indexer + top-k, part 1: the rest)
    def step(self, p, j, q=None, qh=None, qI=None, wI=None, part=None, o=None, oh=None):
        lib = self.lib
        P = self.pairs[p]
        o = self.o if o is None else o
        oh = self.oh if oh is None else oh
        qs = j % self.nQ
        q = self.q[qs] if q is None else q
        qh = self.qh[qs] if qh is None else qh
        qI = self.qI[qs] if qI is None else qI
        wI = self.wI[qs] if wI is None else wI
        t = self.tpos[j]
        if part in (None, 0):
            if self.e4m3:
                lib.csa_indexer_topk_e4m3(qI, wI, P["kI8"], P["kIs"], t, self.m, self.k, self.idx, self.ws_topk)
            elif self.e2m1:
                lib.csa_indexer_topk_e2m1(qI, wI, P["kI8"], P["kIs"], t, self.m, self.k, self.idx, self.ws_topk)
            else:
                lib.csa_indexer_topk(qI, wI, P["kI"], t, self.m, self.k, self.idx, self.ws_topk)
        if part == 0:
            return
        lib.csa_sparse_attn(q, P["cache"], self.idx, o, self.ws_attn)
        lib.hca_dense_attn(qh, P["hcache"], t, self.mp, oh, self.ws_hattn)
        tok = self.n + j
        if (tok + 1) % self.m == 0:  # token completes CSA block i = (tok+1)/m - 1
            i = (tok + 1) // self.m - 1
            lo = self.m * (i - 1)            # first row needed (block i-1 through stream b)
            r0 = lo - (self.n - self.hist)   # row in the decode buffers
            win = [x[:, r0:r0 + 2 * self.m] for x in P["dec"]]
            lib.csa_compress(*win, P["cache"], self.m, i, i + 1, tok0=lo)
            winI = [x[:, r0:r0 + 2 * self.m] for x in P["decI"]]
            lib.csa_compress(*winI, P["kI"], self.m, i, i + 1, tok0=lo)
            if self.quant:  # the new key, quantised as it is formed
                self._quantize(P, i, i + 1)
        if (tok + 1) % self.mp == 0:
            i = (tok + 1) // self.mp - 1
            lo = self.mp * i
            r0 = lo - self.n
            lib.hca_compress(P["decH"][0][:, r0:r0 + self.mp], P["decH"][1][:, r0:r0 + self.mp],
                             P["hcache"], self.mp, i, i + 1, tok0=lo)

    def _quantize(self, P, lo, hi):
        f = self.lib.csa_quantize_e4m3 if self.e4m3 else self.lib.csa_quantize_e2m1
        f(P["kI"][:, lo:hi], P["kI8"][:, lo:hi], P["kIs"][:, lo:hi])

    def key_bytes(self):
        """HBM bytes of one indexer key as the scan reads it (codes + scale)."""
        return self.cI + 4 if self.e4m3 else self.cI // 2 + 4 if self.e2m1 else self.cI * 2

    def step_bytes(self, j):
        """Algorithmic HBM bytes of step j: indexer keys scanned + selected entries +
        HCA entries read (+ the stream rows and entries of any compression)."""
        tok = self.n + j
        vis = tok // self.m
        visH = tok // self.mp
        b = vis * self.key_bytes() + self.k * self.c * 2 + visH * self.c * 2
        if (tok + 1) % self.m == 0:
            b += 4 * 2 * self.m * (self.c + self.cI) * 2 + (self.c + self.cI) * 2
        if (tok + 1) % self.mp == 0:
            b += 2 * self.mp * self.c * 2 + self.c * 2
        return b


def kernel_launches_per_step(dec, j):
    tok = dec.n + j
    n = 1 + 2 + 2  # indexer (scan with the select in place), sparse attn (+combine), dense attn (+combine)
    if (tok + 1) % dec.m == 0:
        n += 3 if dec.quant else 2
    if (tok + 1) % dec.mp == 0:
        n += 1
    return n


# ----------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload, on the host's cores)
# ----------------------------------------------------------------------------------
def _oracle_inputs(workload, seed):
    """Seeded inputs of one decode step of `workload` for the oracle (float64 numpy)."""
    import torch
    from long_context_compressed_csa_b200.synth import randn, to_f64
    bf = torch.bfloat16
    if workload == "hybrid_1m_decode":
        n, m, mp, c, cI, n_h, n_hI = 1 << 20, 4, 128, 512, 128, 128, 64
        return {"KI": to_f64(randn((n // m, cI), seed, bf)), "hc": to_f64(randn((n // mp, c), seed + 1, bf)),
                "rows": to_f64(randn((4096, c), seed + 2, bf)),  # CSA entries, indexed mod 4096
                "q": to_f64(randn((n_h, c), seed + 3, bf)), "qI": to_f64(randn((n_hI, cI), seed + 4, bf)),
                "wI": to_f64(randn((n_hI,), seed + 5, torch.float32))}
    if workload in ("csa_decode_8k", "csa_prefill_decode_b4_256k"):
        n = 8192 if workload == "csa_decode_8k" else 262144
        m, c, cI, n_h, n_hI = 4, 512, 128, 128, 64
        return {"KI": to_f64(randn((n // m, cI), seed, bf)), "cache": to_f64(randn((n // m, c), seed + 1, bf)),
                "q": to_f64(randn((n_h, c), seed + 3, bf)), "qI": to_f64(randn((n_hI, cI), seed + 4, bf)),
                "wI": to_f64(randn((n_hI,), seed + 5, torch.float32))}
    if workload == "hca_decode_b16_128k":
        return {"hc": to_f64(randn((1024, 512), seed + 1, bf)), "q": to_f64(randn((128, 512), seed + 3, bf))}
    raise ValueError(workload)


def _oracle_step(workload, x, j, kI_format="bf16"):
    """One decode step of one sequence through the oracle (the unit of the workload's
    metric divided by its batch)."""
    import oracle
    if workload == "hybrid_1m_decode":
        t = (1 << 20) + j
        score = {"e4m3": oracle.index_scores_e4m3, "e2m1": oracle.index_scores_e2m1}.get(kI_format,
                                                                                         oracle.index_scores)
        s = score(x["qI"], x["wI"], x["KI"], oracle.visible(t, 4, x["KI"].shape[0]))
        sel = oracle.topk(s, 1024)
        oracle.mqa(x["q"], x["rows"][sel % x["rows"].shape[0]], np.arange(1024, dtype=np.int32))
        oracle.mqa(x["q"], x["hc"], np.arange(oracle.visible(t, 128, x["hc"].shape[0]), dtype=np.int32))
    elif workload in ("csa_decode_8k", "csa_prefill_decode_b4_256k"):
        k = 512 if workload == "csa_decode_8k" else 1024
        N = x["KI"].shape[0]
        s = oracle.index_scores(x["qI"], x["wI"], x["KI"], oracle.visible(4 * N + j, 4, N))
        oracle.mqa(x["q"], x["cache"], oracle.topk(s, k))
    else:
        oracle.mqa(x["q"], x["hc"], np.arange(1024, dtype=np.int32))


def _oracle_worker(workload, seed, steps, barrier, queue, kI_format="bf16", warmup=1, budget_s=None):
    x = _oracle_inputs(workload, seed)
    t_w = time.monotonic()
    for j in range(max(1, warmup)):  # warm: loads the oracle library (untimed)
        _oracle_step(workload, x, -1 - j, kI_format)
    per_step = (time.monotonic() - t_w) / max(1, warmup)
    if budget_s is not None:  # a bounded sample: as many of the steps as fit the budget
        steps = max(1, min(steps, int(budget_s / max(per_step, 1e-9))))
    barrier.wait()
    t0 = time.monotonic()
    for j in range(steps):
        _oracle_step(workload, x, j + 1, kI_format)
    queue.put((t0, time.monotonic(), steps))


# per-sequence oracle steps of each workload in one worker, about 10-30 s of CPU work in all
ORACLE_STEPS = {"hybrid_1m_decode": 1, "csa_decode_8k": 20, "hca_decode_b16_128k": 8,
                "csa_prefill_decode_b4_256k": 3}
ORACLE_MAX_WORKERS = 16


def cpu_baseline(workload="hybrid_1m_decode", seed=77, steps=None, kI_format="bf16", warmup=1, total=None,
                 budget_s=None):
    """The oracle timed on the host's cores: one spawned process per core (at most
    ORACLE_MAX_WORKERS), each running whole decode steps of its own sequence after a
    common barrier; value = all steps / the wall time of the concurrent region, in the
    workload's unit (a layer-pair step of the hybrid workload is one token).  With
    `total`, the processes share that many steps; with `budget_s`, each runs at most the
    steps that fit that many seconds (measured on its warm-up steps)."""
    import multiprocessing as mp_
    host = len(os.sched_getaffinity(0))
    P = max(1, min(host, ORACLE_MAX_WORKERS))
    steps = steps or ORACLE_STEPS[workload]
    if total is not None:
        steps = max(1, -(-total // P))
    ctx = mp_.get_context("spawn")  # never fork a process that has touched the GPU
    barrier, queue = ctx.Barrier(P), ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(workload, seed + 1000 * w, steps, barrier, queue, kI_format,
                                                      warmup, budget_s))
             for w in range(P)]
    for pr in procs:
        pr.start()
    res = [queue.get(timeout=600) for _ in range(P)]
    for pr in procs:
        pr.join()
    wall = max(r[1] for r in res) - min(r[0] for r in res)
    unit = "layer-pair decode steps/s" if workload == "hybrid_1m_decode" else "decode tokens/s"
    what = {"hybrid_1m_decode": "one CSA+HCA layer pair at t=2^20 (indexer over 262144 %skeys, full-sort "
                                "top-1024, 128-head MQA over 1024 + 8192 entries)"
                                % ({"e4m3": "E4M3-quantised ", "e2m1": "E2M1-quantised "}.get(kI_format, "")),
            "csa_decode_8k": "one CSA layer at t=8192 (indexer over 2048 keys, top-512, 128-head MQA "
                             "over 512 entries)",
            "hca_decode_b16_128k": "one sequence's HCA dense MQA at t=131072 (128 heads over 1024 entries)",
            "csa_prefill_decode_b4_256k": "one sequence's CSA step at t=262144 (indexer over 65536 keys, "
                                          "top-1024, 128-head MQA over 1024 entries)"}[workload]
    done = sum(r[2] for r in res)
    return {"value": done / wall, "unit": unit, "cores": P, "host_cores": host, "kind": "oracle",
            "sample": "%d processes x %d decode steps of %s, fp64 oracle, one process per core"
                      % (P, -(-done // P), what) + ("" if budget_s is None else
                                                     " (at most %.0f s of steps per process)" % budget_s),
            "seconds": wall, "steps_done": done}


# ----------------------------------------------------------------------------------
# single-kernel micro runs (profiling and per-kernel rooflines)
# ----------------------------------------------------------------------------------
def micro(kind, iters, rotate=4, nq_prefill=1024, batch=16):
    """Time one entry point alone on the 1M workload's shapes (compress kernels on the
    B=16 x 128K HCA and B=4 x 256K CSA prefill shapes), rotating over `rotate` input
    sets so repeated launches do not hit L2.  Prints one JSON line (not the bench line)."""
    import torch
    import long_context_compressed_csa_b200 as lib
    from long_context_compressed_csa_b200 import build
    from long_context_compressed_csa_b200.synth import randn
    build.build()
    bf16 = torch.bfloat16
    dev = "cuda"
    n, m, mp, c, cI, n_h, n_hI, k = 1 << 20, 4, 128, 512, 128, 128, 64, 1024
    N, Nh = n // m, n // mp
    t = torch.full((1, 1), n, dtype=torch.int64, device=dev)
    calls, nbytes, flops = [], 0, 0
    if kind == "indexer_prefill":
        # a prefill chunk: the context's last nq_prefill query positions scored and
        # selected in one call (the many-query tensor-core scan, then one select CTA per
        # query); the contraction's flops are 2 * n_hI * cI per visible (query, key) pair
        nq = nq_prefill
        KIs = [randn((1, N, cI), 900 + r, bf16, dev) for r in range(rotate)]
        qI, wI = randn((1, nq, n_hI, cI), 892, bf16, dev), randn((1, nq, n_hI), 893, torch.float32, dev)
        tq = torch.arange(n - nq, n, dtype=torch.int64, device=dev).reshape(1, nq)
        idx = torch.empty((1, nq, k), dtype=torch.int32, device=dev)
        ws = torch.zeros(lib.csa_indexer_topk_workspace_size(1, nq, N, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_indexer_topk(qI, wI, KIs[r], tq, m, k, idx, ws) for r in range(rotate)]
        vis = [min((n - nq + j) // m, N) for j in range(nq)]
        nbytes = N * cI * 2 + nq * (n_hI * cI * 2 + n_hI * 4 + k * 4)
        flops = 2 * n_hI * cI * sum(vis)
    elif kind == "sparse_prefill":
        # sparse MQA for a prefill chunk: nq_prefill queries, each over its own k selected
        # entries of the 1M-token CSA cache (indices drawn per query, as the prefill
        # indexer returns them); flops 2 * 2 * n_h * c per (query, selected entry)
        nq = nq_prefill
        caches = [randn((1, N, c), 910 + r, bf16, dev) for r in range(2)]
        q = randn((1, nq, n_h, c), 925, bf16, dev)
        g = torch.Generator(device="cpu").manual_seed(926)
        idx = torch.stack([torch.randperm(N, generator=g)[:k] for _ in range(nq)]).to(torch.int32)
        idx = idx.reshape(1, nq, k).to(dev)
        o = torch.empty((1, nq, n_h, c), dtype=torch.float32, device=dev)
        ws = torch.zeros(lib.csa_attn_workspace_size(1, nq, n_h, c, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_sparse_attn(q, caches[r], idx, o, ws) for r in range(2)]
        nbytes = nq * k * c * 2
        flops = 4 * n_h * c * k * nq
    elif kind == "indexer":
        KIs = [randn((1, N, cI), 900 + r, bf16, dev) for r in range(rotate)]
        qI, wI = randn((1, 1, n_hI, cI), 890, bf16, dev), randn((1, 1, n_hI), 891, torch.float32, dev)
        idx = torch.empty((1, 1, k), dtype=torch.int32, device=dev)
        ws = torch.zeros(lib.csa_indexer_topk_workspace_size(1, 1, N, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_indexer_topk(qI, wI, KIs[r], t, m, k, idx, ws) for r in range(rotate)]
        nbytes = N * cI * 2
    elif kind == "sparse":
        caches = [randn((1, N, c), 910 + r, bf16, dev) for r in range(rotate)]
        q = randn((1, 1, n_h, c), 920, bf16, dev)
        g = torch.Generator(device="cpu").manual_seed(921)
        idx = torch.randperm(N, generator=g)[:k].to(torch.int32).reshape(1, 1, k).to(dev)
        o = torch.empty((1, 1, n_h, c), dtype=torch.float32, device=dev)
        ws = torch.zeros(lib.csa_attn_workspace_size(1, 1, n_h, c, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_sparse_attn(q, caches[r], idx, o, ws) for r in range(rotate)]
        nbytes = k * c * 2
    elif kind == "indexer_e4m3":
        # the same scan and top-k over E4M3 keys (1 byte per element + one fp32 scale per key)
        KIs = [randn((1, N, cI), 900 + r, bf16, dev) for r in range(rotate)]
        K8s = [torch.empty((1, N, cI), dtype=torch.uint8, device=dev) for _ in range(rotate)]
        KSs = [torch.empty((1, N), dtype=torch.float32, device=dev) for _ in range(rotate)]
        for r in range(rotate):
            lib.csa_quantize_e4m3(KIs[r], K8s[r], KSs[r])
        del KIs
        qI, wI = randn((1, 1, n_hI, cI), 890, bf16, dev), randn((1, 1, n_hI), 891, torch.float32, dev)
        idx = torch.empty((1, 1, k), dtype=torch.int32, device=dev)
        ws = torch.zeros(lib.csa_indexer_topk_workspace_size(1, 1, N, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_indexer_topk_e4m3(qI, wI, K8s[r], KSs[r], t, m, k, idx, ws)
                 for r in range(rotate)]
        nbytes = N * (cI + 4)
    elif kind == "indexer_e2m1":
        # the same scan and top-k over E2M1 keys (half a byte per element + one fp32 scale per key)
        KIs = [randn((1, N, cI), 900 + r, bf16, dev) for r in range(rotate)]
        K4s = [torch.empty((1, N, cI // 2), dtype=torch.uint8, device=dev) for _ in range(rotate)]
        KSs = [torch.empty((1, N), dtype=torch.float32, device=dev) for _ in range(rotate)]
        for r in range(rotate):
            lib.csa_quantize_e2m1(KIs[r], K4s[r], KSs[r])
        del KIs
        qI, wI = randn((1, 1, n_hI, cI), 890, bf16, dev), randn((1, 1, n_hI), 891, torch.float32, dev)
        idx = torch.empty((1, 1, k), dtype=torch.int32, device=dev)
        ws = torch.zeros(lib.csa_indexer_topk_workspace_size(1, 1, N, k), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.csa_indexer_topk_e2m1(qI, wI, K4s[r], KSs[r], t, m, k, idx, ws)
                 for r in range(rotate)]
        nbytes = N * (cI // 2 + 4)
    elif kind in ("sparse_window", "dense_window"):
        # the same calls with the sliding-window branch: 128 raw-token entries from a ring
        # buffer join the softmax (V4-Pro window size)
        n_win, win_cap = 128, 256
        wins = [randn((1, win_cap, c), 915 + r, bf16, dev) for r in range(rotate)]
        q = randn((1, 1, n_h, c), 920, bf16, dev)
        o = torch.empty((1, 1, n_h, c), dtype=torch.float32, device=dev)
        if kind == "sparse_window":
            caches = [randn((1, N, c), 910 + r, bf16, dev) for r in range(rotate)]
            g = torch.Generator(device="cpu").manual_seed(921)
            idx = torch.randperm(N, generator=g)[:k].to(torch.int32).reshape(1, 1, k).to(dev)
            ws = torch.zeros(lib.csa_attn_workspace_size(1, 1, n_h, c, k + n_win), dtype=torch.uint8, device=dev)
            calls = [lambda r=r: lib.csa_sparse_attn(q, caches[r], idx, o, ws, win=wins[r], t=t, n_win=n_win)
                     for r in range(rotate)]
            nbytes = (k + n_win) * c * 2
        else:
            caches = [randn((1, Nh, c), 930 + r, bf16, dev) for r in range(rotate * 4)]
            ws = torch.zeros(lib.csa_attn_workspace_size(1, 1, n_h, c, Nh + n_win), dtype=torch.uint8, device=dev)
            calls = [lambda r=r: lib.hca_dense_attn(q, caches[r], t, mp, o, ws, win=wins[r % rotate], n_win=n_win)
                     for r in range(rotate * 4)]
            nbytes = (Nh + n_win) * c * 2
    elif kind == "dense":
        caches = [randn((1, Nh, c), 930 + r, bf16, dev) for r in range(rotate * 4)]
        q = randn((1, 1, n_h, c), 940, bf16, dev)
        o = torch.empty((1, 1, n_h, c), dtype=torch.float32, device=dev)
        ws = torch.zeros(lib.csa_attn_workspace_size(1, 1, n_h, c, Nh), dtype=torch.uint8, device=dev)
        calls = [lambda r=r: lib.hca_dense_attn(q, caches[r], t, mp, o, ws) for r in range(rotate * 4)]
        nbytes = Nh * c * 2
    elif kind == "hca_compress":
        B, nn = 16, 131072
        C, Z = randn((B, nn, c), 950, bf16, dev), randn((B, nn, c), 951, bf16, dev)
        out = torch.empty((B, nn // mp, c), dtype=bf16, device=dev)
        calls = [lambda: lib.hca_compress(C, Z, out, mp)]
        nbytes = 2 * B * nn * c * 2 + B * (nn // mp) * c * 2
    elif kind == "hca_project_compress":
        # fused projection + HCA compression over the HCA prefill shape (B = 16 x 128K
        # tokens) with model width d = 4096 (not given by the pages); flops 2 * d * 2c per token
        B, nn, d = batch, 131072, 4096
        H = randn((B, nn, d), 970, bf16, dev, scale=d ** -0.25)
        Wc, Wz = randn((c, d), 971, bf16, dev, scale=d ** -0.25), randn((c, d), 972, bf16, dev, scale=d ** -0.25)
        out = torch.empty((B, nn // mp, c), dtype=bf16, device=dev)
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)
        calls = [lambda: lib.hca_project_compress(H, Wc, Wz, out, mp, ws)]
        nbytes = B * nn * d * 2 + 2 * c * d * 2 + B * (nn // mp) * c * 2
        flops = 2 * B * nn * d * 2 * c
    elif kind == "csa_project_compress":
        # fused CSA projections + compression over the CSA prefill shape (B = 4 x 256K
        # tokens), d = 4096; flops 2 * d * 4c per token
        B, nn, d = batch, 262144, 4096
        H = randn((B, nn, d), 980, bf16, dev, scale=d ** -0.25)
        Ws = [randn((c, d), 981 + w, bf16, dev, scale=d ** -0.25) for w in range(4)]
        out = torch.empty((B, nn // m, c), dtype=bf16, device=dev)
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)
        calls = [lambda: lib.csa_project_compress(H, *Ws, out, m, ws)]
        nbytes = B * nn * d * 2 + 4 * c * d * 2 + B * (nn // m) * c * 2
        flops = 2 * B * nn * d * 4 * c
    elif kind == "csa_compress":
        B, nn = 4, 262144
        S = [randn((B, nn, c), 960 + i, bf16, dev) for i in range(4)]
        out = torch.empty((B, nn // m, c), dtype=bf16, device=dev)
        calls = [lambda: lib.csa_compress(*S, out, m)]
        nbytes = 4 * B * nn * c * 2 + B * (nn // m) * c * 2
    else:
        raise SystemExit("unknown --micro kind %r" % kind)
    for f in calls:
        f()
    torch.cuda.synchronize()
    # all timed calls captured in one CUDA graph with an event record node before and
    # after each call, so neither host launch latency nor host pacing is timed
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(iters)]
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for i in range(iters):
            evs[i][0].record()
            calls[i % len(calls)]()
            evs[i][1].record()
    gr.replay()  # warm-up
    torch.cuda.synchronize()
    gr.replay()
    torch.cuda.synchronize()
    us = np.array([a.elapsed_time(b) * 1e3 for a, b in evs])
    hbm, tf, src = peaks()
    gbs = nbytes / (np.median(us) * 1e-6) / 1e9
    line = {"micro": kind, "iters": iters, "us_median": float(np.median(us)),
            "us_mean": float(us.mean()), "us_min": float(us.min()),
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "peak_gbs": hbm,
            "frac": gbs / hbm, "peak_source": src}
    if flops:
        tfs = flops / (np.median(us) * 1e-6) / 1e12
        line.update({"algorithmic_flops": flops, "achieved_tflops": tfs, "peak_tflops": tf,
                     "tensor_frac": tfs / tf})
        if kind.endswith("_prefill"):
            line["queries"] = nq_prefill
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------
# timing helpers
# ----------------------------------------------------------------------------------
def graph_replay_ms(torch, fns, reps):
    """Capture the calls `fns` once in one CUDA graph and replay it `reps` times, each
    replay bracketed by CUDA events on the stream it is launched on; returns the
    per-replay milliseconds (after one untimed replay)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        out.append(a.elapsed_time(b))
    del g
    return np.array(out)


def back_to_back_launch_us(torch, fns, reps=8):
    """Per-launch device time of a call issued back to back: `fns` (>= 64 calls, inputs
    rotated so they stream from HBM) captured in one graph and replayed `reps` times;
    each replay gives one sample = its duration / len(fns).  No event node sits between
    the calls, so each launch keeps its overlap with its neighbours as in a step."""
    ms = graph_replay_ms(torch, fns, reps)
    per = ms * 1e3 / len(fns)
    return {"median_us": float(np.median(per)), "mean_us": float(per.mean()), "min_us": float(per.min()),
            "max_us": float(per.max()), "samples": int(reps), "timed_launches": int(reps * len(fns))}


def time_step_graphs(torch, step, s_lo, s_hi, group=IDX_SAMPLE):
    """Steps s_lo..s_hi-1 captured in CUDA graphs of `group` consecutive steps and replayed
    in order between two CUDA events; returns the elapsed milliseconds."""
    graphs = []
    for a0 in range(s_lo, s_hi, group):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for s in range(a0, min(a0 + group, s_hi)):
                step(s)
        graphs.append(g)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for g in graphs:
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del graphs
    return a.elapsed_time(b)


def roofline_obj(kernel, nbytes, t, hbm, src, traffic, how):
    ach = nbytes / (t["mean_us"] * 1e-6) / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
            "frac": ach / hbm, "peak_source": src + " (burst copy)", "traffic": traffic,
            "algorithmic_bytes_per_launch": nbytes, "avg_launch_us": t["mean_us"],
            "median_launch_us": t["median_us"],
            "frac_at_median": nbytes / (t["median_us"] * 1e-6) / 1e9 / hbm,
            "timed_launches": t["timed_launches"], "samples": t["samples"], "how": how}


HOW_B2B = ("%d back-to-back launches per CUDA graph (inputs rotated over independent layer caches, "
           "no event node between calls), %d graph replays each timed by CUDA events on the launching "
           "stream: avg = mean of the replays' per-launch times, median = their median")


# ----------------------------------------------------------------------------------
# presets: the other workload configurations, each with its own timed units
# ----------------------------------------------------------------------------------
def preset_config(name, extra=None):
    from long_context_compressed_csa_b200.synth import WORKLOADS
    cfg = {"workload": name}
    cfg.update(WORKLOADS[name])
    cfg.update(extra or {})
    return cfg


def run_preset(torch, name, args, world, rank):
    """Configs other than the 1M hybrid decode (one layer, B sequences):
      csa_decode_8k              prefill compress of both caches; step = indexer + top-k +
                                 sparse MQA for the query at t = 8192
      hca_decode_b16_128k        hca_compress over all 16 x 131072 tokens; step = dense MQA
                                 of 16 queries (one per sequence) at t = 131072
      csa_prefill_decode_b4_256k prefill compress of both caches; steps = 64 decode tokens per
                                 sequence (indexer + top-k + sparse MQA of 4 queries, with the
                                 incremental compression of both caches every m = 4 tokens)
    Independent layer caches are rotated so that a step's inputs stream from HBM.
    `value` = decode tokens per second (B tokens per step)."""
    import long_context_compressed_csa_b200 as lib
    from long_context_compressed_csa_b200.synth import randn
    bf16, dev = torch.bfloat16, "cuda"
    hbm, tf, src = peaks()
    W = max(3, args.warmup)
    seed = 7000 + 17 * rank
    c, cI, n_h, n_hI, m, mp = 512, 128, 128, 64, 4, 128
    if name == "hca_decode_b16_128k":
        B, n = 16, 131072
        Nh = n // mp
        L = 8  # 8 x 16.8 MB of entries between revisits of a layer
        caches = [torch.empty((B, Nh, c), dtype=bf16, device=dev) for _ in range(L)]
        pre_ms = []
        for l in range(L):  # prefill: 4.3 GB of C and Z per layer, compressed as one call
            C = randn((B, n, c), seed + 10 * l, bf16, dev)
            Z = randn((B, n, c), seed + 10 * l + 1, bf16, dev)
            lib.hca_compress(C, Z, caches[l], mp)  # warm
            pre_ms.append(float(np.median(graph_replay_ms(torch, [lambda: lib.hca_compress(C, Z, caches[l], mp)], 3))))
            del C, Z
        q = randn((L, B, 1, n_h, c), seed + 5, bf16, dev)
        t = torch.full((B, 1), n, dtype=torch.int64, device=dev)
        o = torch.empty((B, 1, n_h, c), dtype=torch.float32, device=dev)
        ws = torch.zeros(lib.csa_attn_workspace_size(B, 1, n_h, c, Nh), dtype=torch.uint8, device=dev)
        step = lambda s: lib.hca_dense_attn(q[s % L], caches[s % L], t, mp, o, ws)
        step_bytes = B * Nh * c * 2
        launches_per_step = 2
        pre_bytes = 2 * B * n * c * 2 + B * Nh * c * 2
        dom = ("hca_dense_attn (attn_pair_kernel + attn_combine), 16 queries x 1024 entries",
               step_bytes, [lambda s=s: step(s) for s in range(64)])
    else:
        B, n, k = (1, 8192, 512) if name == "csa_decode_8k" else (4, 262144, 1024)
        N = n // m
        L = 64 if B == 1 else 4  # 64 x 2.5 MB, or 4 x 336 MB, between revisits of a layer
        steps_dec = 64 if B == 4 else 0  # decode tokens appended per sequence
        N_cap = N + steps_dec // m + 1
        caches = [torch.empty((B, N_cap, c), dtype=bf16, device=dev) for _ in range(L)]
        kIs = [torch.empty((B, N_cap, cI), dtype=bf16, device=dev) for _ in range(L)]
        rw = 4 * (c + cI)  # one token's rows of the 4 cache streams and the 4 key streams
        hist = 2 * m
        rows = [randn((B, hist + steps_dec, rw), seed + 10 * l + 9, bf16, dev) for l in range(L)]
        pre_ms = []
        if B == 1:  # all layers' streams first, so none is still in L2 when compressed
            S = [randn((B, n, rw), seed + 10 * l, bf16, dev) for l in range(L)]
            fns = []
            for l in range(L):
                v = [S[l][:, :, i * c:(i + 1) * c] for i in range(4)]
                vI = [S[l][:, :, 4 * c + i * cI:4 * c + (i + 1) * cI] for i in range(4)]
                fns.append(lambda v=v, l=l: lib.csa_compress(*v, caches[l], m, 0, N))
                fns.append(lambda vI=vI, l=l: lib.csa_compress(*vI, kIs[l], m, 0, N))
            for f in fns:
                f()
            pre_ms = list(graph_replay_ms(torch, fns, 3) / L)
            del S, fns
        else:
            for l in range(L):  # 5.4 GB of streams per layer, one layer at a time
                S = randn((B, n, rw), seed + 10 * l, bf16, dev)
                v = [S[:, :, i * c:(i + 1) * c] for i in range(4)]
                vI = [S[:, :, 4 * c + i * cI:4 * c + (i + 1) * cI] for i in range(4)]
                fns = [lambda: lib.csa_compress(*v, caches[l], m, 0, N),
                       lambda: lib.csa_compress(*vI, kIs[l], m, 0, N)]
                for f in fns:
                    f()
                pre_ms.append(float(np.median(graph_replay_ms(torch, fns, 3))))
                del S, v, vI, fns
        nQ = 16
        q = randn((nQ, B, 1, n_h, c), seed + 5, bf16, dev)
        qI = randn((nQ, B, 1, n_hI, cI), seed + 6, bf16, dev)
        wI = randn((nQ, B, 1, n_hI), seed + 7, torch.float32, dev)
        T = max(1, steps_dec)
        tpos = torch.arange(n, n + T, dtype=torch.int64, device=dev).reshape(T, 1, 1).expand(T, B, 1).contiguous()
        idx = torch.empty((B, 1, k), dtype=torch.int32, device=dev)
        o = torch.empty((B, 1, n_h, c), dtype=torch.float32, device=dev)
        ws_t = torch.zeros(lib.csa_indexer_topk_workspace_size(B, 1, N_cap, k), dtype=torch.uint8, device=dev)
        ws_a = torch.zeros(lib.csa_attn_workspace_size(B, 1, n_h, c, k), dtype=torch.uint8, device=dev)

        def step(s):
            l, j = s % L, (s // L) % T  # token j of every sequence through layer l
            lib.csa_indexer_topk(qI[s % nQ], wI[s % nQ], kIs[l], tpos[j], m, k, idx, ws_t)
            lib.csa_sparse_attn(q[s % nQ], caches[l], idx, o, ws_a)
            tok = n + j
            if steps_dec and (tok + 1) % m == 0:  # the token completes entry i
                i = (tok + 1) // m - 1
                lo = m * (i - 1)
                r0 = lo - (n - hist)
                R = rows[l][:, r0:r0 + 2 * m]
                lib.csa_compress(*[R[:, :, a * c:(a + 1) * c] for a in range(4)], caches[l], m, i, i + 1, tok0=lo)
                lib.csa_compress(*[R[:, :, 4 * c + a * cI:4 * c + (a + 1) * cI] for a in range(4)], kIs[l], m,
                                 i, i + 1, tok0=lo)

        def bytes_of(s):
            j = (s // L) % T
            tok = n + j
            b = B * ((tok // m) * cI * 2 + k * c * 2)
            if steps_dec and (tok + 1) % m == 0:
                b += B * (4 * 2 * m * (c + cI) * 2 + (c + cI) * 2)
            return b
        launches_per_step = 3
        pre_bytes = B * (4 * n * (c + cI) * 2 + N * (c + cI) * 2)
        dom = ("csa_indexer_topk (scan_tc_kernel with the top-k select in place), %d x %d keys" % (B, N),
               B * N * cI * 2,
               [lambda l=l: lib.csa_indexer_topk(qI[l % nQ], wI[l % nQ], kIs[l % L], tpos[0], m, k, idx, ws_t)
                for l in range(64)])
    # steps: a whole number of layer rotations, at least the requested count
    K = max(args.steps, L)
    if name == "csa_prefill_decode_b4_256k":
        K = max(K, L * 64)  # 64 decode tokens per sequence through every layer
    K = (K + L - 1) // L * L
    for s in range(min(W, 8)):
        step(s)
    torch.cuda.synchronize()
    time_step_graphs(torch, step, 0, W)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ms = time_step_graphs(torch, step, W, W + K)
    clocks = sampler.stop()
    ms_all = max_over_ranks(ms, "cuda")
    if name == "hca_decode_b16_128k":
        total_bytes = K * step_bytes
        gpu_launches = K * launches_per_step
    else:
        total_bytes = sum(bytes_of(s) for s in range(W, W + K))
        gpu_launches = sum(3 + (2 if steps_dec and (n + (s // L) % T + 1) % m == 0 else 0)
                           for s in range(W, W + K))
    t_dom = back_to_back_launch_us(torch, dom[2], reps=8)
    step_gbs = total_bytes / (ms / 1e3) / 1e9
    pre_us = float(np.median(pre_ms)) * 1e3
    line = {
        "metric": METRIC, "value": whole_job_rate(K * B, world, ms_all), "unit": "decode tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms_all / K,
        "us_per_step": ms_all / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": preset_config(name, {"layers_rotated": L, "parallelism": "replicas" if world > 1 else "single",
                                       "l2": "inputs larger than L2: %d independent layer caches rotated" % L}),
        "roofline": roofline_obj(dom[0], dom[1], t_dom, hbm, src, None, HOW_B2B % (len(dom[2]), 8)),
        "step_roofline": {"achieved": step_gbs, "peak": hbm, "unit": "GB/s", "frac": step_gbs / hbm,
                          "bytes_per_step": total_bytes / K},
        "prefill_compress": {"us": pre_us, "bytes": pre_bytes, "achieved": pre_bytes / (pre_us * 1e-6) / 1e9,
                             "peak": hbm, "unit": "GB/s", "frac": pre_bytes / (pre_us * 1e-6) / 1e9 / hbm},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        base = cpu_baseline(name)
        line["cpu_baseline"] = {k2: base[k2] for k2 in ("value", "unit", "cores", "host_cores", "kind", "sample")}
    return line


# ----------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["hybrid_1m_decode", "csa_decode_8k", "hca_decode_b16_128k",
                             "csa_prefill_decode_b4_256k"],
                    help="the configuration timed (default: the 1M-token hybrid decode)")
    ap.add_argument("--kI-format", default="bf16", choices=["bf16", "e4m3", "e2m1"],
                    help="indexer keys of the hybrid decode: bf16 (default), E4M3 or E2M1 codes with one "
                         "fp32 scale per key, every appended key quantised as it is formed")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--micro", default=None,
                    help="time one entry point alone: indexer, indexer_e4m3, indexer_e2m1, indexer_prefill, "
                         "sparse, sparse_prefill, dense, sparse_window, dense_window, csa_compress, "
                         "hca_compress, hca_project_compress, csa_project_compress")
    ap.add_argument("--nq", type=int, default=1024,
                    help="query positions of the indexer_prefill / sparse_prefill chunk")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences of the *_project_compress micro-benchmarks (16 HCA, 4 CSA)")
    ap.add_argument("--iters", type=int, default=20)
    args = ap.parse_args()
    if args.micro:
        bdef = 4 if args.micro == "csa_project_compress" else 16
        return micro(args.micro, args.iters, nq_prefill=args.nq, batch=args.batch or bdef)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle
        oracle.build()
        # the K timed steps are shared by the host processes (each on its own sequence),
        # after at most 2 untimed steps each; every process stops at ~90 s of steps, so a
        # run with the default K still ends within a few minutes
        base = cpu_baseline(args.workload, kI_format=args.kI_format, warmup=min(2, max(1, args.warmup)),
                            total=max(1, args.steps), budget_s=90.0)
        cfg = workload_config(args.gpus, args.kI_format) if args.workload == WORKLOAD else preset_config(args.workload)
        line = {"impl": "reference", "metric": METRIC, "value": base["value"], "unit": base["unit"],
                "n_gpus": args.gpus, "steps": base["steps_done"], "warmup": min(2, max(1, args.warmup)),
                "ms_per_step": 1000.0 / base["value"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": cfg,
                "cpu_baseline": {k: base[k] for k in ("value", "unit", "cores", "host_cores", "kind", "sample")},
                "e2e": {"value": base["value"], "unit": base["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    from long_context_compressed_csa_b200 import build
    if rank == 0:
        build.build()
        if not args.no_cpu:
            import oracle
            oracle.build()
    if world > 1:
        dist.barrier()

    if args.workload != WORKLOAD:
        line = run_preset(torch, args.workload, args, world, rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    W, K = max(3, args.warmup), args.steps
    dec = HybridDecode(torch, W + K, seed=5000 + 17 * rank, kI_format=args.kI_format)
    stream = torch.cuda.current_stream()

    # ---- capture the steps in CUDA graphs of N_PAIRS consecutive steps (one token through
    # the 8 layer pairs; every pointer and position is baked in), so the kernels of
    # consecutive steps keep their programmatic overlap.  In the first step of each graph,
    # event record nodes bracket the indexer call to time it on the device; the other
    # steps carry no event nodes, which would cut that overlap. ----
    def make_graph(s0, s1):
        g = torch.cuda.CUDAGraph()
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        with torch.cuda.graph(g):
            for s in range(s0, s1):
                p, j = s % N_PAIRS, s // N_PAIRS
                if s == s0:
                    ev[0].record()
                dec.step(p, j, part=0)
                if s == s0:
                    ev[1].record()
                dec.step(p, j, part=1)
        return g, ev

    def graph_ranges(lo, hi):
        return [(s, min(s + IDX_SAMPLE, hi)) for s in range(lo, hi, IDX_SAMPLE)]

    # eager warm-up of every code path once (outside any graph), then build graphs
    for s in range(min(W, 8)):
        dec.step(s % N_PAIRS, s // N_PAIRS)
    torch.cuda.synchronize()
    # re-run the prefill positions: eager steps above advanced nothing persistent except
    # the incremental entries they recomputed, which the graphs recompute identically.
    t0 = time.time()
    warm_graphs = [make_graph(a0, a1) for a0, a1 in graph_ranges(0, W)]
    graphs = [make_graph(a0, a1) for a0, a1 in graph_ranges(W, W + K)]
    torch.cuda.synchronize()
    log("captured %d graphs of up to %d steps in %.1f s" % (len(warm_graphs) + len(graphs), IDX_SAMPLE,
                                                            time.time() - t0))

    for g, _ in warm_graphs:
        g.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for g, _ in graphs:
        g.replay()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = start.elapsed_time(end)
    idx_ms = np.array([ev[0].elapsed_time(ev[1]) for _, ev in graphs])
    ms_all = max_over_ranks(ms, "cuda")
    del graphs, warm_graphs

    bytes_total = sum(dec.step_bytes(s // N_PAIRS) for s in range(W, W + K))
    launches = sum(kernel_launches_per_step(dec, s // N_PAIRS) for s in range(W, W + K))
    hbm, tf, src = peaks()
    value = whole_job_rate(K, world, ms_all)

    # ---- dominant kernel: the indexer (scan over every visible key, then top-k), timed
    # back to back over the 8 layer pairs' keys at the first timed token position ----
    j0 = W // N_PAIRS
    vis = (dec.n + j0) // dec.m
    idx_bytes = vis * dec.key_bytes()
    t_idx = back_to_back_launch_us(
        torch, [lambda p=p: dec.step(p, j0, part=0) for _ in range(8) for p in range(N_PAIRS)], reps=8)
    log("indexer+topk per launch: back to back mean %.2f us, median %.2f us; in the step (event nodes) "
        "mean %.2f us over %d; step %.2f us" % (t_idx["mean_us"], t_idx["median_us"], idx_ms.mean() * 1e3,
                                                len(idx_ms), ms * 1e3 / K))
    step_gbs = bytes_total / (ms / 1000.0) / 1e9

    # ---- end to end through the C ABI with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, dec, W, min(K, 512), world)

    roof = roofline_obj("csa_indexer_topk%s (scan_tc_kernel: indexer scan with the top-k select in place)"
                        % ("" if not dec.quant else "_" + dec.kfmt), idx_bytes, t_idx, hbm, src,
                        SCAN_TRAFFIC_BYTES.get(dec.kfmt), HOW_B2B % (64, 8))
    roof["in_step_event_nodes_us_mean"] = float(idx_ms.mean() * 1e3)
    roof["in_step_event_nodes_samples"] = int(len(idx_ms))
    line = {
        "metric": METRIC, "value": value, "unit": "layer-pair decode steps/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms_all / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(world, args.kI_format),
        "roofline": roof,
        "step_roofline": {"achieved": step_gbs, "peak": hbm, "unit": "GB/s", "frac": step_gbs / hbm,
                          "bytes_per_step": bytes_total / K},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu:
        base = cpu_baseline(kI_format=args.kI_format)
        line["cpu_baseline"] = {k: base[k] for k in ("value", "unit", "cores", "host_cores", "kind", "sample")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(torch, dec, W, K, world):
    """Steps through the C ABI with each step's inputs from pinned host memory (the new
    token's stream rows, q, q^I, w^I, the HCA query) and both outputs back to pinned host:
    three copies per step (the four queries share one staging buffer, the new token's rows
    of all ten streams are one interleaved row, the two outputs are adjacent)."""
    c, cI = dec.c, dec.cI
    nQ = 8
    parts = [dec.q[:nQ], dec.qh[:nQ], dec.qI[:nQ], dec.wI[:nQ]]
    sizes = [x[0].numel() * x.element_size() for x in parts]
    offs = [0]
    for z in sizes:
        offs.append(offs[-1] + (z + 255) // 256 * 256)
    hstage = torch.empty((nQ, offs[-1]), dtype=torch.uint8).pin_memory()
    for x, o0, z in zip(parts, offs, sizes):
        hstage[:, o0:o0 + z].copy_(x.reshape(nQ, -1).view(torch.uint8).cpu())
    # two staging and two output sets, alternating by step parity, so that a step's
    # copies overlap its neighbours' kernels
    dstage = [torch.empty((offs[-1],), dtype=torch.uint8, device="cuda") for _ in range(2)]
    dqs = [[d[o0:o0 + z].view(x.dtype).view(x[0].shape) for x, o0, z in zip(parts, offs, sizes)] for d in dstage]
    hrows = torch.randn((nQ, dec.row_width), dtype=torch.float32).to(torch.bfloat16).pin_memory()
    obufs = [dec.obuf, torch.empty_like(dec.obuf)]
    houts = [torch.empty(dec.obuf.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(sizes) + hrows[0].numel() * 2
    d2h = houts[0].numel() * 4

    def one(s):  # eager form: every copy and call on the current stream
        p, j = s % N_PAIRS, s // N_PAIRS
        qs, par = s % nQ, s & 1
        dstage[par].copy_(hstage[qs], non_blocking=True)
        dec.pairs[p]["rows"][0, dec.hist + j].copy_(hrows[qs], non_blocking=True)  # the new token's rows
        dq, dqh, dqI, dwI = dqs[par]
        dec.step(p, j, q=dq, qh=dqh, qI=dqI, wI=dwI, o=obufs[par][0], oh=obufs[par][1])
        houts[par].copy_(obufs[par], non_blocking=True)

    def capture_group(s0, s1):
        """Steps s0..s1-1 with the input copies on one side stream and the output copies on
        another, ordered by events: step s waits for its inputs; the inputs of step s+2
        wait for step s's kernels (same staging set); step s+2's kernels wait for step s's
        output copy (same output set).  Both side streams rejoin at the end."""
        main = torch.cuda.current_stream()
        up, down = side_streams
        fork = torch.cuda.Event()
        fork.record(main)
        up.wait_event(fork)
        down.wait_event(fork)
        done_k = {}   # step -> event after its kernels
        done_d = {}   # step -> event after its output copy
        for s in range(s0, s1):
            p, j = s % N_PAIRS, s // N_PAIRS
            qs, par = s % nQ, s & 1
            if s - 2 in done_k:
                up.wait_event(done_k[s - 2])
            with torch.cuda.stream(up):
                dstage[par].copy_(hstage[qs], non_blocking=True)
                dec.pairs[p]["rows"][0, dec.hist + j].copy_(hrows[qs], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(up)
            main.wait_event(ready)
            if s - 2 in done_d:
                main.wait_event(done_d[s - 2])
            dq, dqh, dqI, dwI = dqs[par]
            dec.step(p, j, q=dq, qh=dqh, qI=dqI, wI=dwI, o=obufs[par][0], oh=obufs[par][1])
            done_k[s] = torch.cuda.Event()
            done_k[s].record(main)
            down.wait_event(done_k[s])
            with torch.cuda.stream(down):
                houts[par].copy_(obufs[par], non_blocking=True)
            done_d[s] = torch.cuda.Event()
            done_d[s].record(down)
        for st in (up, down):
            join = torch.cuda.Event()
            join.record(st)
            main.wait_event(join)

    side_streams = (torch.cuda.Stream(), torch.cuda.Stream())
    for s in range(W):
        one(s)
    torch.cuda.synchronize()
    # The same calls as a serving loop issues them: each group of IDX_SAMPLE steps (one
    # token through the layer pairs) captured once, with its copies, in a CUDA graph and
    # replayed; every replay still moves each step's inputs and outputs over PCIe.
    how = ("C-ABI calls of each step with its pinned host->device input copies and "
           "device->host output copies, captured in CUDA graphs of %d steps and replayed; "
           "the copies run on side streams, overlapping the neighbouring steps' kernels" % IDX_SAMPLE)
    graphs = []
    try:
        for s0 in range(W, W + K, IDX_SAMPLE):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                capture_group(s0, min(s0 + IDX_SAMPLE, W + K))
            graphs.append(g)
        torch.cuda.synchronize()
    except Exception as exc:  # capture refused: time the eager calls instead
        log("e2e graph capture failed (%s); timing eager calls" % exc)
        graphs = []
        how = "eager C-ABI calls per step; pinned host->device inputs and device->host outputs inside the timed region"
        torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graphs:
        graphs[0].replay()  # warm-up replay
        torch.cuda.synchronize()
    a.record()
    if graphs:
        for g in graphs:
            g.replay()
    else:
        for s in range(W, W + K):
            one(s)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    del graphs
    # the same steps issued eagerly from the host, one C-ABI call at a time (no graphs):
    # what a host-driven serving loop pays for launch latency
    Ke = min(K, 256)
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a2.record()
    for s in range(W, W + Ke):
        one(s)
    b2.record()
    torch.cuda.synchronize()
    ms_e = a2.elapsed_time(b2)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms, ms_e], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, ms_e = float(t[0].item()), float(t[1].item())
    return {"value": K * world / (ms / 1000.0), "unit": "layer-pair decode steps/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": K,
            "how": how,
            "eager": {"value": Ke * world / (ms_e / 1000.0), "steps": Ke,
                      "how": "the same calls and copies issued eagerly from the host, one C-ABI call at a "
                             "time on one stream (no CUDA graphs)"}}


if __name__ == "__main__":
    sys.exit(main())
