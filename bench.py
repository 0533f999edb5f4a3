"""Benchmark of the sparse-attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference] [--index bf16|fp8]

One step = the whole hot path over one batch: lightning-indexer scores -> top-K (+sink/window) ->
sparse MLA gather-attention, for the 16-query decode batch over L = 131072 cached tokens
(K = 2048, H_I = 64, d_I = 128, 128 heads, 576/512 bf16 latent).  Inputs are seeded synthetic
tensors (lsa_synth) resident in HBM before timing; L2 is flushed (256 MB write) before every step,
outside the per-step CUDA events.  Rank 0 prints one JSON line.

N > 1 (torchrun): every rank runs an independent replica of the same decode batch (the path has no
exchange step on one node here: replicas only), timed per rank, max over ranks.

"e2e" is the same step through the C-ABI with host buffers: every step copies its inputs from pinned host
memory, runs the three calls and copies the output back.  The sequence is captured once as a CUDA graph and
replayed per step (the form a serving loop uses); "eager_ms_per_step" is the same sequence issued call by call.

At N = 1 the line also carries "long_context": per-stage times of the 1M-token decode (FP8 token path,
hierarchical selection, micro-block selection), of the hybrid attention and the group-wise block selection at
128K, and of the 10M-token Flat bucket workload (--no-configs skips them), and "prefill_chunk": the latency of one
causal prefill chunk (8192 queries, FP8 scan + bf16 re-rank, K = 2048 + sink 4 + window 128) with its per-stage
times (--no-prefill skips it).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

import lsa_synth as S

ROOT = os.path.dirname(os.path.abspath(__file__))
CONFIG = "decode128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s), used only when no FP8 measurement is committed
FP8_PEAK_FILE = os.path.join(ROOT, "profiles", "fp8_peak.json")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def fp8_peak():
    """(e4m3 dense TFLOP/s burst, sustained, source): the committed measurement of this machine's B200s
    (`python bench.py --measure-tensor-peaks`), else the bf16 peak x the nominal ratio."""
    if os.path.exists(FP8_PEAK_FILE):
        d = json.load(open(FP8_PEAK_FILE))
        return float(d["fp8_e4m3_tflops"]), float(d["fp8_e4m3_tflops_sustained"]), "measured (profiles/fp8_peak.json)"
    pk, src = peaks()
    return pk["bf16_tflops"] * FP8_OVER_BF16, pk["bf16_tflops_sustained"] * FP8_OVER_BF16, src + " bf16 x2 (nominal)"


def measure_tensor_peaks(device, seconds: float = 4.0):
    """Dense GEMM throughput of this GPU with the library GEMMs: torch._scaled_mm e4m3 x e4m3 -> bf16 and
    torch.matmul bf16, 8192^3 (2 N^3 flops each).  Burst = best of 10 single launches (CUDA events); sustained =
    back-to-back launches for `seconds`, with the SM clock sampled meanwhile.  No clock or power setting is
    touched."""
    n = 8192
    torch.manual_seed(0)
    a16 = torch.randn(n, n, device=device, dtype=torch.bfloat16)
    b16 = torch.randn(n, n, device=device, dtype=torch.bfloat16)
    a8 = a16.to(torch.float8_e4m3fn)
    b8 = b16.to(torch.float8_e4m3fn).t().contiguous().t()  # column-major, as _scaled_mm wants
    one = torch.ones((), device=device, dtype=torch.float32)
    ops = {"fp8_e4m3": lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
           "bf16": lambda: torch.matmul(a16, b16)}
    flops = 2.0 * n ** 3
    res = {}
    for name, f in ops.items():
        for _ in range(5):
            f()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        with ClockSampler(device.index or 0) as clk:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps, t0 = 0, time.perf_counter()
            e0.record()
            while time.perf_counter() - t0 < seconds:
                for _ in range(20):
                    f()
                reps += 20
                torch.cuda.synchronize()
            e1.record()
            e1.synchronize()
            ms = e0.elapsed_time(e1)
        res[name] = {"burst_tflops": round(flops / (best * 1e-3) / 1e12, 1),
                     "sustained_tflops": round(flops * reps / (ms * 1e-3) / 1e12, 1), "clocks": clk.summary()}
    return {"fp8_e4m3_tflops": res["fp8_e4m3"]["burst_tflops"],
            "fp8_e4m3_tflops_sustained": res["fp8_e4m3"]["sustained_tflops"],
            "bf16_tflops_same_run": res["bf16"]["burst_tflops"],
            "bf16_tflops_sustained_same_run": res["bf16"]["sustained_tflops"],
            "clocks": {k: v["clocks"] for k, v in res.items()},
            "gpu": torch.cuda.get_device_name(device),
            "how": "torch._scaled_mm(e4m3 [8192,8192] x e4m3 [8192,8192] col-major, unit scales, bf16 out) and "
                   "torch.matmul bf16 8192^3, 2*N^3 flops: best of 10 CUDA-event launches (burst) and back-to-back "
                   f"launches for {seconds:.0f} s (sustained)"}


# ------------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                if out.returncode == 0 and out.stdout.strip():
                    self.samples.append([x.strip() for x in out.stdout.strip().split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if len(s) > 5 + i and s[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------------------


class DecodeStep:
    """Resident tensors and the three C-ABI calls of one decode step."""

    def __init__(self, wl: S.Workload, index_dtype: str, device):
        import sparse_long_context_lightning_b200 as lsa

        self.lsa = lsa
        self.wl = wl
        self.fp8 = index_dtype == "fp8"
        q_I, w = S.index_queries(wl, "cpu")
        k_I = S.index_keys(wl, q_I, device)
        self.q_I, self.w = q_I.to(device), w.to(device)
        k_I_bf16 = k_I
        if self.fp8:
            self.q_in, self.q_scale = S.quantize_e4m3_rows(self.q_I)
            self.k_in, self.k_scale = S.quantize_e4m3_rows(k_I)
        else:
            self.q_in, self.q_scale, self.k_in, self.k_scale = self.q_I, None, k_I, None
        self.q_pos = wl.q_pos().to(device)
        self.q = S.attn_queries(wl, device)
        self.kv = S.latent_cache(wl, device)
        B, L = wl.B, wl.L
        self.kmax = wl.K + wl.sink + wl.window
        self.scores = torch.empty(B, L, device=device)
        self.idx = torch.empty(B, self.kmax, dtype=torch.int32, device=device)
        self.cnt = torch.empty(B, dtype=torch.int32, device=device)
        self.out = torch.empty(B, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(B, wl.H, device=device)
        self.ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, L, self.kmax, wl.H), device)
        if self.fp8:
            # FP8 scan keeps the top 2K, then the exact bf16 re-rank keeps K of them
            self.k2 = 2 * wl.K
            self.cand = torch.empty(B, self.k2 + wl.sink + wl.window, dtype=torch.int32, device=device)
            self.ccnt = torch.empty(B, dtype=torch.int32, device=device)
            self.k_bf16 = k_I_bf16
            self.ws_rf = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_REFINE, B, self.cand.shape[1], wl.K), device)

    def index(self):
        self.lsa.lsa_index_score(self.q_in, self.w, self.k_in, self.q_pos, self.scores,
                                 q_scale=self.q_scale, k_scale=self.k_scale)

    def topk(self):
        wl = self.wl
        if self.fp8:
            self.lsa.lsa_topk_select(self.scores, wl.L, self.k2, wl.sink, wl.window, self.q_pos, self.cand, self.ccnt)
            self.lsa.lsa_topk_refine(self.q_I, self.w, self.k_bf16, self.cand, self.ccnt, wl.K, wl.sink, wl.window,
                                     self.q_pos, self.idx, self.cnt, self.ws_rf)
        else:
            self.lsa.lsa_topk_select(self.scores, wl.L, wl.K, wl.sink, wl.window, self.q_pos, self.idx, self.cnt)

    def attn(self):
        self.lsa.lsa_sparse_attn(self.q, self.kv, self.idx, self.cnt, self.wl.scale, self.out, self.lse, self.ws)


def algorithmic_work(wl: S.Workload, counts: np.ndarray, fp8: bool):
    """Bytes / flops each stage must touch (what the method reads and writes, nothing re-read)."""
    B, L = wl.B, wl.L
    vis = L  # decode: every cached key is visible
    idx_elem = 1 if fp8 else 2
    index_flops = 2.0 * B * wl.H_I * wl.d_I * vis
    index_bytes = vis * wl.d_I * idx_elem + (vis * 4 if fp8 else 0) + B * vis * 4 + B * wl.H_I * (wl.d_I * idx_elem + 4)
    topk_bytes = B * vis * 4 + B * (wl.K + wl.sink + wl.window) * 4
    if fp8:  # top-2K of the FP8 scores, then the bf16 re-rank reads 2K key rows per query
        topk_bytes += B * 2 * wl.K * (4 + wl.d_I * 2 + 4)
    n_rows = float(counts.sum())
    attn_bytes = n_rows * wl.d_qk * 2 + B * wl.H * wl.d_qk * 2 + B * wl.H * wl.d_v * 2 + B * wl.H * 4 + n_rows * 4
    attn_flops = 2.0 * n_rows * wl.H * (wl.d_qk + wl.d_v)
    return {"index": (index_flops, index_bytes), "topk": (0.0, topk_bytes), "attn": (attn_flops, attn_bytes)}


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        p = os.path.join(ROOT, "sparse_long_context_lightning_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d:
        return None
    if d.get("source_hash") != kernel_source_hash(d.get("sources", [])):
        return None
    return d.get("dram_bytes_per_launch")


STAGE_KERNEL = {"index": ("k_index_score_tc", ["k_index_tc.cu"]),
                "topk": ("k_topk_cluster", ["k_topk.cu"]),
                "attn": ("k_sparse_attn_2p", ["k_attn_2p.cu"])}
# kernels each stage launches per step (the e2e leg adds none of ours)
LAUNCHES = {"index": 1, "topk": 1, "attn": 1}


def dynamic_recall(idx_a, cnt_a, idx_b, cnt_b, q_pos, sink: int, window: int):
    """Mean and min over rows of |A_dyn & B_dyn| / |B_dyn|, the sink and window positions left out (B is the
    reference selection)."""
    ia, ca, ib, cb, qp = (t.cpu().numpy() for t in (idx_a, cnt_a, idx_b, cnt_b, q_pos))
    rec = []
    for r in range(ia.shape[0]):
        lo = max(int(qp[r]) - window + 1, 0) if window > 0 else int(qp[r]) + 1
        a, b = ia[r, : ca[r]], ib[r, : cb[r]]
        a = a[(a >= sink) & (a < lo)]
        b = b[(b >= sink) & (b < lo)]
        rec.append(np.intersect1d(a, b).size / max(b.size, 1))
    return {"mean": round(float(np.mean(rec)), 5), "min": round(float(np.min(rec)), 5), "rows": len(rec)}


def fp8_decode(device, l2_flush, bf16_step, iters: int = 10):
    """The decode step with the FP8 indexer (e4m3 scan -> top-2K -> exact bf16 re-rank -> K): per-stage times, the
    scan's fraction of the measured e4m3 peak, and the recall of its selection against the bf16 path's (which the
    parity tests pin to the exact top-K up to ties), on the dynamic part."""
    wl = bf16_step.wl
    step = DecodeStep(wl, "fp8", device)
    st = _time_stages([step.index, step.topk, step.attn], l2_flush, iters)
    step.index()
    step.topk()
    bf16_step.index()
    bf16_step.topk()
    torch.cuda.synchronize()
    counts = step.cnt.cpu().numpy()
    work = algorithmic_work(wl, counts, True)
    p8, _, p8_src = fp8_peak()
    res = {"workload": f"{CONFIG} with the e4m3 indexer (per-row scales), top-2K + exact bf16 re-rank to K",
           "stages": {"index": _stage(st[0], work["index"][1], work["index"][0], p8),
                      "topk_rerank": _stage(st[1], work["topk"][1]),
                      "attn": _stage(st[2], work["attn"][1], work["attn"][0], peaks()[0]["bf16_tflops"])},
           "ms_per_step": round(float(st.sum()), 5), "queries_per_s": round(wl.B / (float(st.sum()) * 1e-3), 1),
           "fp8_peak_tflops": p8, "fp8_peak_source": p8_src,
           "recall_vs_bf16_selection": dynamic_recall(step.idx, step.cnt, bf16_step.idx, bf16_step.cnt, step.q_pos,
                                                      wl.sink, wl.window)}
    del step
    torch.cuda.empty_cache()
    return res


def prefill_chunk(device, l2_flush, iters: int = 3):
    """Latency of one causal prefill chunk: 8192 queries at positions 122880..131071 over L = 131072, FP8
    scan + exact bf16 re-rank to K = 2048, sink 4 + window 128, attention over the selected rows.
    Inputs resident in HBM; L2 flushed before each iteration, outside the events."""
    wl = S.WORKLOADS["prefill"]
    step = DecodeStep(wl, "fp8", device)
    stream = torch.cuda.current_stream()

    def once(ev):
        ev[0].record(stream)
        step.index()
        ev[1].record(stream)
        step.topk()
        ev[2].record(stream)
        step.attn()
        ev[3].record(stream)

    l2_flush()
    once([torch.cuda.Event(enable_timing=True) for _ in range(4)])  # warm-up
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(iters)]
    for i in range(iters):
        l2_flush()
        once(evs[i])
    torch.cuda.synchronize()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(iters)])
    ms = float(per.sum(axis=1).mean())
    st = per.mean(axis=0)
    # the FP8 scan's rate against the measured e4m3 peak: 2 H_I d_I flops per visible (query, key) pair
    pairs = float(sum(int(p) + 1 for p in wl.q_pos().tolist()))
    scan_flops = 2.0 * wl.H_I * wl.d_I * pairs
    p8, _, p8_src = fp8_peak()
    # recall of the FP8 selection against the bf16 path's on every row (bf16 scores into the same buffer)
    idx8, cnt8 = step.idx.clone(), step.cnt.clone()
    step.lsa.lsa_index_score(step.q_I, step.w, step.k_bf16, step.q_pos, step.scores)
    step.lsa.lsa_topk_select(step.scores, wl.L, wl.K, wl.sink, wl.window, step.q_pos, step.idx, step.cnt)
    torch.cuda.synchronize()
    rec = dynamic_recall(idx8, cnt8, step.idx, step.cnt, step.q_pos, wl.sink, wl.window)
    del step, idx8, cnt8
    torch.cuda.empty_cache()
    return {"workload": "prefill: 8192 causal queries (q_pos 122880..131071), L=131072, FP8 scan + bf16 re-rank, "
                        "K=2048 + sink 4 + window 128, H=128", "ms": round(ms, 3),
            "stages_ms": {"index": round(float(st[0]), 3), "topk": round(float(st[1]), 3), "attn": round(float(st[2]), 3)},
            "index_scan": {"algorithmic_flops": scan_flops, "achieved_tflops": round(scan_flops / (st[0] * 1e-3) / 1e12, 1),
                           "tensor_frac": round(scan_flops / (st[0] * 1e-3) / 1e12 / p8, 4), "peak_tflops": p8,
                           "peak_source": p8_src},
            "recall_vs_bf16_selection": rec,
            "queries_per_s": round(wl.B / (ms * 1e-3), 1), "iterations": iters}


class BucketStep:
    """Representative (bucket / micro-block) selection then attention: the C-ABI calls of one step of the
    micro-block (4-token blocks, top-512 + tail) or Flat (64-member buckets, top-32) variant.  The
    representatives and their bf16 split are built once before timing (the untimed precompute)."""

    def __init__(self, wl: S.Workload, device):
        import sparse_long_context_lightning_b200 as lsa

        self.lsa, self.wl = lsa, wl
        q_I, w = S.index_queries(wl, "cpu")
        k_I = S.index_keys(wl, q_I, device)
        self.q_I, self.w = q_I.to(device), w.to(device)
        self.members = S.bucket_members(wl, device) if wl.mode == "flat" else None
        nb = self.members.shape[0] if self.members is not None else wl.L // wl.bsz
        self.cen = torch.empty(nb, wl.d_I, device=device)
        lsa.lsa_pool_keys(k_I, self.cen, wl.bsz, members=self.members)
        del k_I
        # cached beside the representatives: their exact bf16 split for the tensor-core scoring
        self.split = torch.empty(3, nb, wl.d_I, dtype=torch.bfloat16, device=device)
        lsa.lsa_split_representatives(self.cen, self.split)
        self.q_pos = wl.q_pos().to(device)
        self.idx = torch.empty(wl.B, wl.kmax, dtype=torch.int32, device=device)
        self.cnt = torch.empty(wl.B, dtype=torch.int32, device=device)
        self.ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET_MIN, wl.B, nb, wl.M), device)
        self.q = S.attn_queries(wl, device)
        self.kv = S.latent_cache(wl, device)
        self.out = torch.empty(wl.B, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(wl.B, wl.H, device=device)
        self.ws_a = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, wl.B, wl.L, wl.kmax, wl.H), device)
        self.nb = nb

    def select(self):
        wl = self.wl
        self.lsa.lsa_bucket_select_split(self.q_I, self.w, self.split, self.members, wl.bsz, wl.M, wl.sink, wl.window,
                                         wl.L, self.q_pos, self.idx, self.cnt, self.ws)

    def attn(self):
        self.lsa.lsa_sparse_attn(self.q, self.kv, self.idx, self.cnt, self.wl.scale, self.out, self.lse, self.ws_a)


class HiStep:
    """Hierarchical selection (pages of 128 tokens, 8-token sub-blocks, top-1024 pages, token top-K on the
    recalled tokens) beside the flat bf16 indexer + top-K over the same keys, then attention.  The sub-block
    means and their bf16 split are built once before timing (the untimed precompute)."""

    P, BSUB, M = 128, 8, 1024

    def __init__(self, wl: S.Workload, device):
        import sparse_long_context_lightning_b200 as lsa

        self.lsa, self.wl = lsa, wl
        q_I, w = S.index_queries(wl, "cpu")
        self.k = S.index_keys(wl, q_I, device)
        self.q_I, self.w = q_I.to(device), w.to(device)
        nsub = wl.L // self.BSUB
        means = torch.empty(nsub, wl.d_I, device=device)
        lsa.lsa_pool_keys(self.k, means, self.BSUB)
        self.split = torch.empty(3, nsub, wl.d_I, dtype=torch.bfloat16, device=device)
        lsa.lsa_split_representatives(means, self.split)
        del means
        self.q_pos = wl.q_pos().to(device)
        kmax = wl.K + wl.sink + wl.window
        self.idx = torch.empty(wl.B, kmax, dtype=torch.int32, device=device)
        self.cnt = torch.empty(wl.B, dtype=torch.int32, device=device)
        self.ws = lsa.workspace(lsa.lsa_hi_workspace_size(wl.B, wl.L, self.P, self.BSUB, self.M, wl.K, wl.sink,
                                                          wl.window), device)
        self.scores = torch.empty(wl.B, wl.L, device=device)
        self.fidx = torch.empty_like(self.idx)
        self.fcnt = torch.empty_like(self.cnt)
        self.q = S.attn_queries(wl, device)
        self.kv = S.latent_cache(wl, device)
        self.out = torch.empty(wl.B, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(wl.B, wl.H, device=device)
        self.ws_a = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, wl.B, wl.L, kmax, wl.H), device)

    def hi(self):
        wl = self.wl
        self.lsa.lsa_hi_select(self.q_I, self.w, self.k, self.split, self.P, self.BSUB, self.M, wl.K, wl.sink,
                               wl.window, self.q_pos, self.idx, self.cnt, self.ws)

    def flat(self):
        wl = self.wl
        self.lsa.lsa_index_score(self.q_I, self.w, self.k, self.q_pos, self.scores)
        self.lsa.lsa_topk_select(self.scores, wl.L, wl.K, wl.sink, wl.window, self.q_pos, self.fidx, self.fcnt)

    def attn(self):
        self.lsa.lsa_sparse_attn(self.q, self.kv, self.idx, self.cnt, self.wl.scale, self.out, self.lse, self.ws_a)


class MsaStep:
    """Group-wise block selection (G groups of the 64 index heads, each keeping its top-KB 128-token blocks by
    max-pooled token score plus the local block) and each query-head group's attention over its own blocks."""

    def __init__(self, wl: S.Workload, device, G: int, KB: int):
        import sparse_long_context_lightning_b200 as lsa

        self.lsa, self.wl, self.G, self.KB = lsa, wl, G, KB
        q_I, w = S.index_queries(wl, "cpu")
        self.k = S.index_keys(wl, q_I, device)
        self.q_I, self.w = q_I.to(device), w.to(device)
        self.q_pos = wl.q_pos().to(device)
        ld = (G * KB + 1) * 128
        self.idx = torch.empty(wl.B, ld, dtype=torch.int32, device=device)
        self.gmask = torch.empty(wl.B, ld, dtype=torch.uint8, device=device)
        self.cnt = torch.empty(wl.B, dtype=torch.int32, device=device)
        self.ws = lsa.workspace(lsa.lsa_msa_workspace_size(wl.B, wl.L, G, KB), device)
        self.q = S.attn_queries(wl, device)
        self.kv = S.latent_cache(wl, device)
        self.out = torch.empty(wl.B, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(wl.B, wl.H, device=device)
        self.ws_a = lsa.workspace(lsa.lsa_msa_attn_workspace_size(wl.B, ld, G), device)

    def select(self):
        self.lsa.lsa_msa_select(self.q_I, self.w, self.k, self.G, self.KB, self.q_pos, self.idx, self.gmask,
                                self.cnt, self.ws)

    def attn(self):
        self.lsa.lsa_msa_attn(self.q, self.kv, self.idx, self.gmask, self.cnt, self.G, self.wl.scale, self.out,
                              self.lse, self.ws_a)


def _time_stages(stages, l2_flush, iters):
    """Mean CUDA-event time (ms) of each callable in `stages`, run in order, L2 flushed before each pass."""
    stream = torch.cuda.current_stream()
    n = len(stages)

    def once(ev):
        ev[0].record(stream)
        for j, f in enumerate(stages):
            f()
            ev[j + 1].record(stream)

    for _ in range(3):
        l2_flush()
        once([torch.cuda.Event(enable_timing=True) for _ in range(n + 1)])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(iters)]
    for i in range(iters):
        l2_flush()
        once(evs[i])
    torch.cuda.synchronize()
    return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n)] for i in range(iters)]).mean(axis=0)


def _stage(ms, nbytes, flops=None, peak_tflops=None, pipe="tensor"):
    hbm = peaks()[0]["hbm_gbs"]
    d = {"ms": round(float(ms), 5), "algorithmic_bytes": int(nbytes),
         "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)}
    if flops:
        d["algorithmic_flops"] = float(flops)
        d["achieved_tflops"] = round(flops / (ms * 1e-3) / 1e12, 2)
        d[f"{pipe}_frac"] = round(flops / (ms * 1e-3) / 1e12 / peak_tflops, 4)
    return d


def long_context_configs(device, l2_flush, iters: int = 10, only=None):
    """Per-stage times of the long-context workloads (one GPU, inputs resident, L2 flushed before each pass):
    1M-token decode with the FP8 token path, 1M-token decode with micro-block selection, and the 10M-token
    Flat bucket workload.  Each stage's fraction is against the measured HBM copy peak (and, for the indexer,
    the FP8 tensor peak = measured bf16 x 2)."""
    res = {}
    bf16 = peaks()[0]["bf16_tflops"]

    def want(name):  # --only: a comma-separated subset of the workloads (a short run, e.g. to profile one kernel)
        return only is None or name in only

    if want("decode1m_fp8"):
        # 1M tokens, FP8 scan -> top-2K -> exact bf16 re-rank -> attention
        wl = S.WORKLOADS["decode1m"]
        step = DecodeStep(wl, "fp8", device)
        st = _time_stages([step.index, step.topk, step.attn], l2_flush, iters)
        rows = float(step.cnt.sum().item())
        B, L = wl.B, wl.L
        ix_bytes = L * wl.d_I + L * 4 + B * L * 4 + B * wl.H_I * wl.d_I + B * wl.H_I * 8
        ix_flops = 2.0 * B * wl.H_I * wl.d_I * L
        tk_bytes = B * L * 4 + B * 2 * wl.K * (wl.d_I * 2 + 4) + B * step.kmax * 4
        at_bytes = rows * (wl.d_qk * 2 + 4) + B * wl.H * (wl.d_qk * 2 + wl.d_v * 2 + 4)
        res["decode1m_fp8"] = {
            "workload": "B=4 decode queries, L=1048576, e4m3 indexer (H_I=64, d_I=128), top-4096 + exact bf16 re-rank "
                        "to K=2048, sink 4 + window 128, H=128",
            "stages": {"index": _stage(st[0], ix_bytes, ix_flops, fp8_peak()[0]), "topk_rerank": _stage(st[1], tk_bytes),
                       "attn": _stage(st[2], at_bytes)},
            "ms": round(float(st.sum()), 5), "queries_per_s": round(B / (float(st.sum()) * 1e-3), 1)}
        del step
        torch.cuda.empty_cache()
    if want("decode1m_hi"):
        # 1M tokens, hierarchical selection (bf16) against the flat bf16 indexer + top-K on the same keys
        wl = S.WORKLOADS["decode1m"]
        hstep = HiStep(wl, device)
        st = _time_stages([hstep.hi, hstep.attn, hstep.flat], l2_flush, iters)
        B, L = wl.B, wl.L
        recalled = HiStep.M * HiStep.P
        sub_flops = 3 * 2.0 * B * wl.H_I * wl.d_I * (L // HiStep.BSUB)
        tok_flops = 2.0 * B * wl.H_I * wl.d_I * recalled
        hi_bytes = (L // HiStep.BSUB) * wl.d_I * 6 + B * recalled * (wl.d_I * 2 + 8)
        hrows = float(hstep.cnt.sum().item())
        h_at_bytes = hrows * (wl.d_qk * 2 + 4) + B * wl.H * (wl.d_qk * 2 + wl.d_v * 2 + 4)
        res["decode1m_hi"] = {
            "workload": "B=4 decode queries, L=1048576, bf16 indexer keys; pages of 128 tokens, 8-token sub-block means "
                        "(cached bf16 split), top-1024 pages (131072 recalled tokens), exact token top-2048 on them, "
                        "sink 4 + window 128, H=128",
            "stages": {"hi_select": _stage(st[0], hi_bytes, sub_flops + tok_flops, bf16), "attn": _stage(st[1], h_at_bytes)},
            "flat_select_ms": round(float(st[2]), 5),
            "ms": round(float(st[0] + st[1]), 5), "queries_per_s": round(B / (float(st[0] + st[1]) * 1e-3), 1)}
        del hstep
        torch.cuda.empty_cache()
    if want("decode128k_hfa"):
        # the pages' fixed / dynamic split (sink 16 + window 1024 + 1024 sparse) at 128K: the attention as one
        # gather pass over the row and as the hybrid operator (contiguous part on a second stream, LSE merge)
        wl = S.Workload("decode128k_si", L=131072, B=16, H_I=64, d_I=128, K=1024, H=128, sink=16, window=1024,
                        needles="cos06", n_needles=1310)
        step = DecodeStep(wl, "bf16", device)
        step.index()
        step.topk()
        ws_h = step.lsa.workspace(step.lsa.lsa_workspace_size(step.lsa.LSA_OP_HYBRID_ATTN, wl.B, wl.L, step.kmax, wl.H,
                                                              wl.sink, wl.window), device)

        def hybrid():
            step.lsa.lsa_hybrid_attn(step.q, step.kv, step.idx, step.cnt, wl.sink, wl.window, step.q_pos, wl.scale,
                                     step.out, step.lse, ws_h)

        st = _time_stages([step.attn, hybrid], l2_flush, iters)
        rows = float(step.cnt.sum().item())
        at_bytes = rows * (wl.d_qk * 2 + 4) + wl.B * wl.H * (wl.d_qk * 2 + wl.d_v * 2 + 4)
        res["decode128k_hfa"] = {
            "workload": "B=16 decode queries, L=131072, sink 16 + window 1024 + top-1024 sparse (the pages' 1:1 fixed / "
                        "dynamic budget), H=128",
            "stages": {"attn_single_pass": _stage(st[0], at_bytes), "attn_hybrid": _stage(st[1], at_bytes)}}
        del step, ws_h
        torch.cuda.empty_cache()
    if want("decode128k_msa"):
        # group-wise block selection at 128K: 8 groups, each its top-16 blocks of 128 (2048 tokens per group) + the
        # local block; the attention stage reads each group's rows for its 16 query heads
        wl = S.WORKLOADS["decode128k"]
        mstep = MsaStep(wl, device, G=8, KB=16)
        st = _time_stages([mstep.select, mstep.attn], l2_flush, iters)
        B, L = wl.B, wl.L
        nblk = L // 128
        sel_bytes = L * wl.d_I * 2 + B * 8 * nblk * 4 + B * mstep.idx.shape[1] * 5
        sel_flops = 2.0 * B * wl.H_I * wl.d_I * L
        rows = float(mstep.cnt.sum().item())
        gm = mstep.gmask.cpu().numpy()
        grp_rows = float(sum(int(((gm[b, : int(c)] >> g) & 1).sum()) for b, c in enumerate(mstep.cnt.cpu().tolist())
                             for g in range(8)))
        at_bytes = rows * (wl.d_qk * 2 + 4) + B * wl.H * (wl.d_qk * 2 + wl.d_v * 2 + 4)
        res["decode128k_msa"] = {
            "workload": "B=16 decode queries, L=131072, bf16 indexer (H_I=64 as 8 groups of 8 heads), top-16 blocks of "
                        "128 per group + the local block, H=128 (8 groups of 16 query heads)",
            "stages": {"msa_select": _stage(st[0], sel_bytes, sel_flops, bf16), "attn": _stage(st[1], at_bytes)},
            "union_rows_per_query": round(rows / B, 1), "group_rows_per_query": round(grp_rows / B, 1),
            "ms": round(float(st.sum()), 5), "queries_per_s": round(B / (float(st.sum()) * 1e-3), 1)}
        del mstep
        torch.cuda.empty_cache()
    if want("decode1m_mb") or want("flat10m") or want("flat10m_tree"):
        for name in ("decode1m_mb", "flat10m"):
            if not (want(name) or (name == "flat10m" and want("flat10m_tree"))):
                continue
            wl = S.WORKLOADS[name]
            bstep = BucketStep(wl, device)
            st = _time_stages([bstep.select, bstep.attn], l2_flush, iters)
            B = wl.B
            rows = float(bstep.cnt.sum().item())
            sel_bytes = bstep.nb * wl.d_I * 6 + B * bstep.nb * 4 + B * wl.kmax * 4 + \
                (B * wl.M * wl.bsz * 4 if wl.mode == "flat" else 0)
            sel_flops = 2.0 * B * wl.H_I * wl.d_I * bstep.nb
            at_bytes = rows * (wl.d_qk * 2 + 4) + B * wl.H * (wl.d_qk * 2 + wl.d_v * 2 + 4)
            desc = ("B=4 decode queries, L=1048576, 4-token mean-pooled blocks (fp32, scored from their cached exact "
                    "3 x bf16 split on tensor cores), top-512 blocks + tail + sink 4 + window 128, H=128"
                    if name == "decode1m_mb" else
                    "B=8 decode queries, L=10000000, 156250 Flat buckets of 64 (fp32 representatives scored from their "
                    "cached exact 3 x bf16 split on tensor cores), top-32 buckets + sink 4 + window 512, H=128, "
                    "11.5 GB latent cache")
            res[name] = {"workload": desc,
                         "stages": {"bucket_select": _stage(st[0], sel_bytes, 3 * sel_flops, bf16),
                                    "attn": _stage(st[1], at_bytes)},
                         "ms": round(float(st.sum()), 5), "queries_per_s": round(B / (float(st.sum()) * 1e-3), 1)}
            if name == "flat10m":
                # the Tree form over the same buckets: parents of 64 consecutive buckets, top-64 parents, then the
                # top-32 of their 4096 children; timed beside Flat, with the share of Flat's positions it keeps
                F, M2 = 64, 64
                lsa_ = bstep.lsa
                NP = -(-bstep.nb // F)
                par = torch.empty(NP, wl.d_I, device=device)
                lsa_.lsa_tree_parents(bstep.cen, F, par)
                t_idx, t_cnt = torch.empty_like(bstep.idx), torch.empty_like(bstep.cnt)
                ws_t = lsa_.workspace(lsa_.lsa_tree_workspace_size(B, NP, F, M2, wl.M), device)

                def tree():  # children from the cached split of the centres, on the tensor cores
                    lsa_.lsa_tree_select_split(bstep.q_I, bstep.w, bstep.split, par, F, bstep.members, M2, wl.M, wl.sink,
                                               wl.window, wl.L, bstep.q_pos, t_idx, t_cnt, ws_t)

                st_t = _time_stages([tree], l2_flush, iters)
                bstep.select()
                tree()
                torch.cuda.synchronize()
                fi, fc, ti, tc = bstep.idx.cpu(), bstep.cnt.cpu(), t_idx.cpu(), t_cnt.cpu()
                kept = [len(np.intersect1d(fi[b, : fc[b]].numpy(), ti[b, : tc[b]].numpy())) / max(int(fc[b]), 1)
                        for b in range(B)]
                t_bytes = NP * wl.d_I * 4 + B * M2 * F * (wl.d_I * 4 + 8) + B * wl.kmax * 4
                t_flops = 2.0 * B * wl.H_I * wl.d_I * (NP + M2 * F)
                res["flat10m_tree"] = {
                    "workload": "flat10m's buckets as a two-level tree: 2442 parents of 64 consecutive buckets (mean "
                                "centres), top-64 parents, top-32 of their 4096 children (scored on the tensor cores "
                                "from the centres' cached bf16 split), + sink 4 + window 512",
                    "stages": {"tree_select": _stage(st_t[0], t_bytes)}, "tree_select_flops": t_flops,
                    "flat_select_ms": round(float(st[0]), 5),
                    "share_of_flat_positions_kept": round(float(np.mean(kept)), 4)}
                del par, t_idx, t_cnt, ws_t
            del bstep
            torch.cuda.empty_cache()
    return res


def max_over_ranks(vals: torch.Tensor, world: int) -> torch.Tensor:
    """Element-wise max over the ranks (the slowest rank's times); identity for one process."""
    if world > 1:
        torch.distributed.all_reduce(vals, op=torch.distributed.ReduceOp.MAX)
    return vals


def job_rate(per_rank_units: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units every rank processed, over the slowest rank's time."""
    return per_rank_units * world / (ms * 1e-3)


def run_gpu(args, rank, world, local_rank):
    import sparse_long_context_lightning_b200 as lsa

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    wl = S.WORKLOADS[CONFIG]
    step = DecodeStep(wl, args.index, device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=device)
    flush_rd = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.int32, device=device)

    def l2_flush():
        # write a buffer larger than L2, then read another one: L2 ends up cold and clean, so the step
        # neither hits cached inputs nor pays for writing back the flush's dirty lines
        flush.zero_()
        torch.sum(flush_rd)

    stream = torch.cuda.current_stream()
    launches = dict(LAUNCHES)
    if step.fp8:
        launches["topk"] = 4  # top-2K, re-score, top-K of the candidates, assemble
    launches["attn"] = 2 if lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, wl.B, wl.L, step.kmax, wl.H) > 0 else 1  # + combine

    def one_step(ev, stage_events: bool):
        # the timed steps record events only around the whole step, so consecutive kernels overlap their
        # launches (programmatic dependent launch) as in a serving loop; the stage breakdown comes from a
        # second pass of the same steps with an event between the stages
        ev[0].record(stream)
        step.index()
        if stage_events:
            ev[1].record(stream)
        step.topk()
        if stage_events:
            ev[2].record(stream)
        step.attn()
        ev[3].record(stream)

    for _ in range(args.warmup):
        l2_flush()
        one_step([torch.cuda.Event(enable_timing=True) for _ in range(4)], True)
    torch.cuda.synchronize()
    counts = step.cnt.cpu().numpy()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        t0 = time.perf_counter()
        for i in range(args.steps):
            l2_flush()  # outside the step's events
            one_step(evs[i], False)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    if world > 1:
        torch.distributed.barrier()
    step_ms = float(np.mean([evs[i][0].elapsed_time(evs[i][3]) for i in range(args.steps)]))
    # stage breakdown (not the headline): the same steps with events between the stages
    evs_st = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        l2_flush()
        one_step(evs_st[i], True)
    torch.cuda.synchronize()
    per = np.array([[evs_st[i][j].elapsed_time(evs_st[i][j + 1]) for j in range(3)] for i in range(args.steps)])
    stage_ms = per.mean(axis=0)
    stage_sum_ms = float(per.sum(axis=1).mean())

    # e2e: host (pinned) inputs -> H2D -> the three calls -> D2H of the result, every step
    h_q_in = step.q_in.cpu().pin_memory()
    h_w = step.w.cpu().pin_memory()
    h_qs = step.q_scale.cpu().pin_memory() if step.q_scale is not None else None
    h_qI = step.q_I.cpu().pin_memory() if step.fp8 else None  # the FP8 mode's re-rank reads the bf16 queries
    h_q = step.q.cpu().pin_memory()
    h_qpos = step.q_pos.cpu().pin_memory()
    h_out = torch.empty_like(step.out, device="cpu").pin_memory()
    h_lse = torch.empty_like(step.lse, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_q_in, h_w, h_q, h_qpos, h_qs, h_qI) if t is not None)
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
    side = torch.cuda.Stream(device=device)

    def e2e_body():
        # the attention queries (the largest input) cross PCIe on a second stream while the indexer and the
        # top-K run; the attention waits for them
        cur = torch.cuda.current_stream()
        side.wait_stream(cur)
        with torch.cuda.stream(side):
            step.q.copy_(h_q, non_blocking=True)
        step.q_in.copy_(h_q_in, non_blocking=True)
        step.w.copy_(h_w, non_blocking=True)
        if h_qs is not None:
            step.q_scale.copy_(h_qs, non_blocking=True)
            step.q_I.copy_(h_qI, non_blocking=True)
        step.q_pos.copy_(h_qpos, non_blocking=True)
        step.index()
        step.topk()
        cur.wait_stream(side)
        step.attn()
        h_out.copy_(step.out, non_blocking=True)
        h_lse.copy_(step.lse, non_blocking=True)

    def e2e_time(run):
        ms = []
        for i in range(args.warmup + args.steps):
            l2_flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run()
            e1.record(stream)
            e1.synchronize()
            if i >= args.warmup:
                ms.append(e0.elapsed_time(e1))
        return float(np.mean(ms))

    # eagerly (one host call per copy and per C-ABI call), then the same sequence captured once as a CUDA graph
    # and replayed: the serving form, where the host launches a step with one call
    e2e_eager = e2e_time(e2e_body)
    e2e_mode = "cuda-graph"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            e2e_body()
        torch.cuda.synchronize()
        e2e_step = e2e_time(graph.replay)
    except Exception as exc:  # capture unsupported here: report the eager figure
        print(f"[bench] CUDA-graph capture of the e2e step failed ({exc}); reporting the eager e2e", file=sys.stderr)
        graph, e2e_mode, e2e_step = None, "eager", e2e_eager
    del graph

    # max over ranks
    vals = max_over_ranks(torch.tensor([step_ms, e2e_step, stage_sum_ms, *stage_ms.tolist()], dtype=torch.float64,
                                       device=device), world)
    step_ms, e2e_step, stage_sum_ms = float(vals[0]), float(vals[1]), float(vals[2])
    stage_ms = vals[3:].cpu().numpy()
    if rank != 0:
        return None
    prefill = None if (args.no_prefill or world > 1) else prefill_chunk(device, l2_flush)
    fp8_line = None if (args.no_configs or world > 1 or step.fp8) else fp8_decode(device, l2_flush, step)
    only = set(args.only.split(",")) if args.only else None
    long_ctx = None if (args.no_configs or world > 1) else long_context_configs(device, l2_flush, only=only)

    pk, pk_src = peaks()
    work = algorithmic_work(wl, counts, step.fp8)
    tensor_peak = fp8_peak()[0] if step.fp8 else pk["bf16_tflops"]
    stages = {}
    for j, name in enumerate(("index", "topk", "attn")):
        flops, nbytes = work[name]
        t = stage_ms[j] * 1e-3
        gbs = nbytes / t / 1e9
        st = {"ms": round(float(stage_ms[j]), 5), "algorithmic_bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
              "hbm_frac": round(gbs / pk["hbm_gbs"], 4)}
        if flops:
            tf = flops / t / 1e12
            st.update({"algorithmic_flops": flops, "achieved_tflops": round(tf, 2),
                       "tensor_frac": round(tf / tensor_peak, 4)})
        stages[name] = st
    dom = max(stages, key=lambda k: stages[k]["ms"])
    kname, _ = STAGE_KERNEL[dom]
    tkey = kname  # the committed DRAM traffic of this kernel in this mode, if any
    if step.fp8 and dom == "index":
        tkey = "k_index_score_tc<fp8>"
    elif step.fp8 and dom == "topk":  # the FP8 mode's selection stage is four launches
        kname, tkey = "k_topk_cluster (top-2K) + k_rescore_tc + k_refine_assemble + k_topk_cluster", None
    if dom == "index":
        roof = {"bound": "tensor", "achieved": stages[dom]["achieved_tflops"], "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": stages[dom]["tensor_frac"]}
    else:
        roof = {"bound": "hbm", "achieved": stages[dom]["achieved_gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": stages[dom]["hbm_frac"]}
    roof.update({"kernel": kname, "peak_source": fp8_peak()[2] if (dom == "index" and step.fp8) else pk_src,
                 "traffic": committed_traffic(tkey) if tkey else None})
    qps = job_rate(wl.B, world, step_ms)
    n_launch = sum(launches.values()) * args.steps
    return {
        "metric": "sparse decode queries/s @L=128K,K=2048",
        "value": round(qps, 1),
        "unit": "queries/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if not step.fp8 else "e4m3-index/bf16-attn",
        "data": "synthetic (lsa_synth, seed 0)",
        "config": {"workload": f"{CONFIG}: B=16 decode queries, L=131072, H_I=64, d_I=128, K=2048, H=128, "
                               f"latent 576/512 bf16", "index_dtype": args.index, "global_batch": wl.B * world,
                   "seq_len": wl.L, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (256 MB write + 256 MB read), outside the step's CUDA events"},
        "gather_hbm_gbs": stages["attn"]["achieved_gbs"],
        "stages": stages,
        "stages_sum_ms": round(stage_sum_ms, 5),
        "stages_note": "per-stage times from a second pass of the same steps with CUDA events between the stages "
                       "(those events also stop the stages' launches from overlapping); ms_per_step is timed with "
                       "events around each whole step only",
        "roofline": roof,
        "e2e": {"value": round(job_rate(wl.B, world, e2e_step), 1), "unit": "queries/s",
                "ms_per_step": round(e2e_step, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "mode": e2e_mode, "eager_ms_per_step": round(e2e_eager, 5)},
        "gpu_launches": n_launch,
        "clocks": clk.summary(),
        "wall_s_timed_region": round(wall, 4),
        "fp8_decode": fp8_line,
        "prefill_chunk": prefill,
        "long_context": long_ctx,
    }


# ------------------------------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline, and the --impl reference arm)
# ------------------------------------------------------------------------------------------------


def oracle_queries(budget_s: float, max_queries: int = 1000, stages: dict | None = None):
    """Run the fp64 oracle on decode queries of the same workload until budget_s elapses.

    Per query: indexer scores over all 131072 keys, top-K + union, attention over the selected
    latent rows (gathered from the same synthetic cache).  Returns (queries, seconds, threads); when
    ``stages`` is given it receives each stage's seconds summed over the queries.
    """
    from oracle import lsa_oracle as O

    wl = S.WORKLOADS[CONFIG]
    q_I, w = S.index_queries(wl)
    k_I = S.index_keys(wl, q_I)
    kf = O.bf16_to_f64(k_I.view(torch.int16).numpy())
    qf = O.bf16_to_f64(q_I.view(torch.int16).numpy())
    wf = w.numpy().astype(np.float64)
    q = S.attn_queries(wl)
    done, t0 = 0, time.perf_counter()
    acc = {"index": 0.0, "topk": 0.0, "attn": 0.0}
    while done < max_queries:
        b = done % wl.B
        ta = time.perf_counter()
        sc = O.index_score(qf[b: b + 1], wf[b: b + 1], kf, np.array([wl.L - 1]))
        tb = time.perf_counter()
        sel, _, _ = O.topk_row(sc[0], wl.L - 1, wl.K, wl.sink, wl.window)
        tc = time.perf_counter()
        rows = S.latent_rows(wl, torch.as_tensor(sel))
        O.sparse_mla_attn(O.bf16_to_f64(q[b].view(torch.int16).numpy()), O.bf16_to_f64(rows.view(torch.int16).numpy()),
                          wl.scale)
        td = time.perf_counter()
        acc["index"] += tb - ta
        acc["topk"] += tc - tb
        acc["attn"] += td - tc
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    if stages is not None:
        stages.update(acc)
    return done, dt, torch.get_num_threads()


def _oracle_pipeline(wl, O, q_I, w, kf, rows, q_pos_of):
    """Oracle time per stage over query rows `rows`: indexer scores over the visible keys, top-K with the sink /
    window union, attention over the selected latent rows.  Returns (rows done, {stage: seconds})."""
    qf = O.bf16_to_f64(q_I.view(torch.int16).numpy())
    wf = w.numpy().astype(np.float64)
    acc = {"index": 0.0, "topk": 0.0, "attn": 0.0}
    for b in rows:
        qp = int(q_pos_of(b))
        ta = time.perf_counter()
        sc = O.index_score(qf[b: b + 1], wf[b: b + 1], kf[: qp + 1], np.array([qp]))
        tb = time.perf_counter()
        sel, _, _ = O.topk_row(sc[0], qp, wl.K, wl.sink, wl.window)
        tc = time.perf_counter()
        qa = S.normal_bf16_rows(S.ST_Q, torch.arange(b * wl.H, (b + 1) * wl.H), wl.d_qk)
        kv = S.latent_rows(wl, torch.as_tensor(sel))
        O.sparse_mla_attn(O.bf16_to_f64(qa.view(torch.int16).numpy()), O.bf16_to_f64(kv.view(torch.int16).numpy()),
                          wl.scale)
        td = time.perf_counter()
        acc["index"] += tb - ta
        acc["topk"] += tc - tb
        acc["attn"] += td - tc
    return len(rows), acc


def oracle_configs():
    """The oracle on the other workloads, each on a bounded sample, as rows (queries) per second per stage.
    Input generation and the untimed precompute (representatives) are outside the timed stages."""
    from oracle import lsa_oracle as O

    def rates(n, acc):
        tot = sum(acc.values())
        return {"queries_per_s": round(n / tot, 4), "queries": n,
                "stage_queries_per_s": {k: round(n / v, 3) for k, v in acc.items() if v > 0}}

    res = {}
    wl = S.WORKLOADS["tiny"]
    q_I, w = S.index_queries(wl)
    kf = O.bf16_to_f64(S.index_keys(wl, q_I).view(torch.int16).numpy())
    n, acc = _oracle_pipeline(wl, O, q_I, w, kf, [0] * 20, lambda b: wl.L - 1)
    res["tiny"] = dict(rates(n, acc), sample="the one decode query, 20 times")
    wl = S.WORKLOADS["decode1m"]
    q_I, w = S.index_queries(wl)
    kf = O.bf16_to_f64(S.index_keys(wl, q_I).view(torch.int16).numpy())
    n, acc = _oracle_pipeline(wl, O, q_I, w, kf, [0], lambda b: wl.L - 1)
    res["decode1m"] = dict(rates(n, acc), sample="1 of the 4 decode queries (bf16 indexer over all 1048576 keys)")
    del kf
    wl = S.WORKLOADS["prefill"]
    q_I, w = S.index_queries(wl)
    kf = O.bf16_to_f64(S.index_keys(wl, q_I).view(torch.int16).numpy())
    qpos = wl.q_pos()
    n, acc = _oracle_pipeline(wl, O, q_I, w, kf, [0, wl.B // 2, wl.B - 1], lambda b: int(qpos[b]))
    res["prefill"] = dict(rates(n, acc), sample="3 of the 8192 causal query rows (first, middle, last), bf16 indexer")
    del kf
    # flat10m: the oracle's Flat selection and attention for one query over a table of the first 1/16 of the
    # buckets (their representatives built from their member keys beforehand, like the cached GPU table)
    wl = S.WORKLOADS["flat10m"]
    q_I, w = S.index_queries(wl)
    mem = S.bucket_members(wl)
    nb = mem.shape[0] // 16
    msub = mem[:nb]
    keys = S.index_key_rows(wl, q_I, msub.reshape(-1).long())
    reps = O.pool_keys(O.bf16_to_f64(keys.view(torch.int16).numpy()).reshape(-1, wl.d_I),
                       np.arange(nb * wl.bsz).reshape(nb, wl.bsz))
    qf = O.bf16_to_f64(q_I.view(torch.int16).numpy())
    wf = w.numpy().astype(np.float64)
    ta = time.perf_counter()
    bs = O.bucket_scores(qf[:1], wf[:1], reps)
    sel, _, _ = O.bucket_select_row(bs[0], wl.L - 1, wl.M, wl.sink, wl.window, members=msub.numpy())
    tb = time.perf_counter()
    qa = S.normal_bf16_rows(S.ST_Q, torch.arange(0, wl.H), wl.d_qk)
    kv = S.latent_rows(wl, torch.as_tensor(sel))
    O.sparse_mla_attn(O.bf16_to_f64(qa.view(torch.int16).numpy()), O.bf16_to_f64(kv.view(torch.int16).numpy()),
                      wl.scale)
    tc = time.perf_counter()
    res["flat10m"] = {"sample": f"1 decode query; bucket table = the first {nb} of {mem.shape[0]} buckets",
                      "buckets_scored_and_selected_per_s": round(nb / (tb - ta), 1),
                      "attention_queries_per_s": round(1.0 / (tc - tb), 3), "attention_rows": int(len(sel))}
    return res


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world=1):
    """The oracle on the host cores; under torchrun only rank 0 runs it (the others return None at once)."""
    if rank != 0:
        return None
    # warm-up steps are untimed oracle queries; each timed step is one bounded sample (<= 2 queries)
    for _ in range(min(args.warmup, 1)):
        oracle_queries(0.0, 1)
    qs, secs = 0, 0.0
    for _ in range(args.steps):
        n, dt, _ = oracle_queries(5.0, 2)
        qs += n
        secs += dt
    v = qs / secs
    cores = blas_threads()
    return {"metric": "sparse decode queries/s @L=128K,K=2048", "value": round(v, 4), "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (lsa_synth, seed 0)", "impl": "reference",
            "config": {"workload": f"{CONFIG}: B=16 decode queries, L=131072, H_I=64, d_I=128, K=2048, H=128, "
                                   f"latent 576/512 bf16", "sample": "<= 2 decode queries per step"},
            "cpu_baseline": {"value": round(v, 4), "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": f"{qs} decode queries of the workload (full indexer over L, top-K, attention)"},
            "e2e": {"value": round(v, 4), "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lsa", choices=["lsa", "reference"])
    ap.add_argument("--index", default="bf16", choices=["bf16", "fp8"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill-chunk latency measurement")
    ap.add_argument("--only", default=None,
                    help="long-context workloads to run, comma-separated (decode1m_fp8, decode1m_hi, decode128k_hfa, "
                         "decode128k_msa, decode1m_mb, flat10m, flat10m_tree); default all")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the long-context workloads (1M-token FP8 / micro-block decode, 10M-token Flat)")
    ap.add_argument("--measure-tensor-peaks", action="store_true",
                    help="measure the dense e4m3 and bf16 GEMM peaks of this GPU, print them as JSON and exit")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.measure_tensor_peaks:
        print(json.dumps(measure_tensor_peaks(torch.device("cuda", 0))), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    res = run_gpu(args, rank, world, local_rank)
    if res is not None:
        if not args.no_cpu_baseline and world == 1:
            st = {}
            n, dt, _ = oracle_queries(12.0, stages=st)
            res["cpu_baseline"] = {"value": round(n / dt, 4), "unit": "queries/s", "cores": blas_threads(),
                                   "kind": "oracle", "sample": f"{n} decode queries of the workload "
                                                                f"(fp64 indexer over L=131072, top-K, attention)",
                                   "stage_queries_per_s": {k: round(n / v, 3) for k, v in st.items() if v > 0},
                                   "other_workloads": oracle_configs() if not args.no_configs else None}
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
