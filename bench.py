"""Benchmark of the DSA hot path on B200: prefill tokens/s at 128K and decode
queries/s at B=64 x 32K, with roofline fractions and the CPU oracle beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path (indexer -> top-k -> sparse MLA)
over the prefill workload: one causal prefill of L = 131072 tokens, queries
scored in 4096-row chunks against the full causal prefix (inputs resident in
HBM, far larger than L2, so no flush is needed). Under torchrun each rank
runs its own independent prefill (weak scaling, no data-path collective);
the reported time is the max over ranks. The decode workload (64 sequences
x 32768 tokens, paged cache) is timed in the same run, with an L2 flush
before every iteration, and reported under "decode".

--impl reference times the CPU oracle (the plain C implementation the tests
compare against) on the host cores, on a stratified sample of query rows of
the same workload, and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "DSA tokens/s: prefill@128K & decode queries/s B=64@32K; % of FP8/HBM roofline"
PREFILL_CFG = 4
DECODE_CFG = 3


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--L", type=int, default=0, help="override the prefill length (testing)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--path", default="fused", choices=["fused", "scores"],
                    help="fused: dsa_forward_fused (top-k fused into the indexer, no score rows "
                         "in HBM); scores: dsa_forward (each chunk's scores in HBM, read back by "
                         "the top-k)")
    ap.add_argument("--profile", default="", choices=["", "chunk", "decode"],
                    help="small cases for ncu captures: chunk = the last 4096 query rows of the "
                         "128K prefill against its whole 131072-key caches (about 1.5 GB on the "
                         "device), one whole-path call per step; decode = the B=64 x 32768 decode "
                         "alone. Prints one JSON line with the per-call time")
    ap.add_argument("--next", action="store_true",
                    help="also time dense causal and sliding-window attention beside DSA at 16K")
    ap.add_argument("--shard", default="problems", choices=["problems", "rows"],
                    help="problems: one prefill per GPU (weak scaling, the default); rows: one "
                         "prefill's query rows split over the GPUs by causal cost (strong "
                         "scaling)")
    return ap.parse_args()


# ------------------------------------------------------------------ ranks

class Ranks:
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE). The only
    collectives are the timing barrier and the max of the per-rank times; the
    problems themselves are independent. `backend` "gloo" keeps everything on
    the CPU (tests without GPUs)."""

    def __init__(self, gpus, backend="nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.dev = "cuda" if backend == "nccl" else "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
            self.pg = dist
        elif backend == "nccl" and torch.cuda.is_available():
            torch.cuda.set_device(0)
        self.gpus = gpus

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, maxm, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                maxm = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": maxm,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------ work counts

def prefill_work(L, Hi, H, k):
    """Algorithmic work of one causal prefill (no masked pairs, no re-reads)."""
    pairs = L * (L + 1) // 2                               # causal (t, s) pairs
    sel = sum(min(t + 1, k) for t in range(L))             # selected (t, key) pairs
    idx_flops = 2 * 128 * Hi * pairs
    mla_flops = 2 * (576 + 512) * H * sel
    # bytes each stage must move at least once
    idx_bytes = L * Hi * 128 + L * 128 + L * 4 * 2 + L * Hi * 4 + L * k * 4
    mla_bytes = L * H * 576 * 2 + L * 576 * 2 + L * k * 4 + L * H * 512 * 2 + L * H * 4
    return dict(pairs=pairs, sel=sel, idx_flops=idx_flops, mla_flops=mla_flops,
                idx_bytes=idx_bytes, mla_bytes=mla_bytes)


def decode_work(lens, nq, Hi, H, k):
    ctx = [int(n) for n in lens]
    idx_bytes = sum(n * (128 + 4) for n in ctx) + len(ctx) * nq * (Hi * 128 + Hi * 4 + 4)
    sel = sum(min(n - nq + j + 1, k) for n in ctx for j in range(nq))
    mla_bytes = sel * 1152 + len(ctx) * nq * H * (576 * 2 + 512 * 2 + 4)
    idx_flops = sum(2 * 128 * Hi * (n - nq + j + 1) for n in ctx for j in range(nq))
    mla_flops = 2 * (576 + 512) * H * sel
    return dict(idx_bytes=idx_bytes, mla_bytes=mla_bytes, idx_flops=idx_flops,
                mla_flops=mla_flops, sel=sel)


# The committed ncu summary of each kernel's DRAM traffic: a line
#   "traffic: <bytes> bytes per launch (...); source sha256 <16 hex digits>"
# taken on a small case and scaled to one launch of the bench's workload. The
# figure is used only while the kernel's source still has that hash.
TRAFFIC_SUMMARY = {"sparse_mla": ("profiles/ncu_sparse_mla_chunk_L131072.md",
                                  "sparse_attention_long_02_b200/csrc/sparse_mla.cu"),
                   "indexer": ("profiles/ncu_indexer_filter_chunk_L131072.md",
                               "sparse_attention_long_02_b200/csrc/indexer.cu")}


def traffic_from_profile(kernel):
    """(bytes per launch, summary file) from the committed ncu summary, or
    (None, reason) when there is none or the kernel has changed since."""
    import hashlib
    import re
    summary, source = TRAFFIC_SUMMARY[kernel]
    try:
        text = open(os.path.join(ROOT, summary)).read()
        src = open(os.path.join(ROOT, source), "rb").read()
    except OSError:
        return None, f"no summary {summary}"
    m = re.search(r"^traffic: ([0-9.eE+]+) bytes per launch.*source sha256 ([0-9a-f]{16})", text,
                  re.M)
    if not m:
        return None, f"no traffic line in {summary}"
    if hashlib.sha256(src).hexdigest()[:16] != m.group(2):
        return None, f"{source} has changed since {summary} was captured"
    return float(m.group(1)), summary


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# --------------------------------------------------------- GPU measurement

def _ev():
    return torch.cuda.Event(enable_timing=True)


def prefill_inputs(L, rank):
    import dataclasses
    cfg = dataclasses.replace(W.CONFIGS[PREFILL_CFG], seed=W.CONFIGS[PREFILL_CFG].seed + 1000 * rank)
    return cfg, W.make_prefill(cfg, device="cuda", L=L)


class Prefill:
    """Preallocated buffers and one call of the whole path per step."""

    def __init__(self, dsa, cfg, inp, path="scores"):
        self.dsa, self.cfg, self.inp, self.path = dsa, cfg, inp, path
        T, H, k = inp["T"], inp["H"], inp["k"]
        self.chunk = cfg.chunk or T
        size = dsa.forward_fused_workspace_size if path == "fused" else dsa.forward_workspace_size
        self.run = dsa.forward_fused if path == "fused" else dsa.forward
        self.ws = torch.empty(size(T, inp["S"], inp["Hi"], H, k, self.chunk),
                              dtype=torch.uint8, device="cuda")
        self.out = torch.empty(T, H, 512, dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
        self.idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
        # per chunk: indexer + top-k (scores), or sample indexer, threshold, filter
        # indexer, select and recompute (fused); then one sparse MLA launch
        self.launches = (5 if path == "fused" else 2) * math.ceil(T / self.chunk) + 1

    def step(self):
        i = self.inp
        self.run(i["q8"], i["q_scale"], i["k8"], i["k_scale"], i["w"], i["q"], i["kv"],
                         i["k"], i["scale"], i["sm_scale"], chunk=self.chunk, idx=self.idx,
                         out=self.out, lse=self.lse, workspace=self.ws)

    def stages(self, reps=2):
        """Per-stage device time of one step (ms), events around each stage call."""
        d, i = self.dsa, self.inp
        T, S, Hi, k = i["T"], i["S"], i["Hi"], i["k"]
        ld = (S + 3) // 4 * 4
        if self.ws.numel() >= self.chunk * ld * 4:
            scores = self.ws[: self.chunk * ld * 4].view(torch.float32).view(self.chunk, ld)
        else:                                 # the fused path's workspace holds no score rows
            scores = torch.empty(self.chunk, ld, dtype=torch.float32, device="cuda")
        tot = {"indexer": 0.0, "topk": 0.0, "sparse_mla": 0.0}
        for _ in range(reps):
            for c0 in range(0, T, self.chunk):
                n = min(self.chunk, T - c0)
                e0, e1, e2 = _ev(), _ev(), _ev()
                e0.record()
                d.indexer_scores(i["q8"][c0:c0 + n], i["q_scale"][c0:c0 + n], i["k8"], i["k_scale"],
                                 i["w"][c0:c0 + n], i["scale"], q_pos0=c0, scores=scores[:n])
                e1.record()
                d.topk(scores[:n], S, k, q_pos0=c0, idx=self.idx[c0:c0 + n])
                e2.record()
                e2.synchronize()
                tot["indexer"] += e0.elapsed_time(e1)
                tot["topk"] += e1.elapsed_time(e2)
            e0, e1 = _ev(), _ev()
            e0.record()
            d.sparse_mla(i["q"], i["kv"], self.idx, i["sm_scale"], out=self.out, lse=self.lse)
            e1.record()
            e1.synchronize()
            tot["sparse_mla"] += e0.elapsed_time(e1)
        return {s: v / reps for s, v in tot.items()}


class RowShard:
    """This rank's share of one prefill: whole chunks of rows, balanced over the
    ranks by causal cost (dsa_plan_prefill_chunks; every rank computes the same
    plan), each run as its own dsa_forward over the key prefix its rows see.
    The caches are whole on every GPU; no data crosses between GPUs."""

    def __init__(self, dsa, cfg, inp, world, rank, path="fused"):
        self.dsa, self.inp = dsa, inp
        T, H, k = inp["T"], inp["H"], inp["k"]
        self.chunk = cfg.chunk or T
        self.starts = dsa.plan_prefill_chunks(T, inp["S"], inp["Hi"], H, k, self.chunk, world,
                                              rank)
        size = dsa.forward_fused_workspace_size if path == "fused" else dsa.forward_workspace_size
        self.run = dsa.forward_fused if path == "fused" else dsa.forward
        self.ws = torch.empty(size(self.chunk, inp["S"], inp["Hi"], H, k, self.chunk),
                              dtype=torch.uint8, device="cuda")
        self.out = torch.empty(T, H, 512, dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
        self.idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
        # per chunk: sample indexer, threshold, filter indexer, select, recompute and sparse
        # MLA (fused), or indexer, top-k and sparse MLA (scores)
        self.launches = (6 if path == "fused" else 3) * len(self.starts)
        self.rows = sum(min(self.chunk, T - c0) for c0 in self.starts)

    def step(self):
        i = self.inp
        cut = lambda x, a, b: None if x is None else x[a:b]
        for c0 in self.starts:
            e = min(c0 + self.chunk, i["T"])
            self.run(i["q8"][c0:e], cut(i["q_scale"], c0, e), i["k8"][:e],
                     cut(i["k_scale"], 0, e), i["w"][c0:e], i["q"][c0:e], i["kv"][:e],
                     i["k"], i["scale"], i["sm_scale"], q_pos0=c0, chunk=self.chunk,
                     idx=self.idx[c0:e], out=self.out[c0:e], lse=self.lse[c0:e],
                     workspace=self.ws)


def time_steps(fn, steps, warmup, ranks, dsa, clock_gpu):
    for _ in range(warmup):
        fn()
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {dsa.STATUS.get(st, st)}")
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(clock_gpu) as clk:
        e0, e1 = _ev(), _ev()
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        e1.synchronize()
    torch.cuda.synchronize()
    ranks.barrier()
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {dsa.STATUS.get(st, st)}")
    return ranks.max(e0.elapsed_time(e1) / steps), clk.summary()


def e2e_prefill(pf, steps):
    """The whole prefill through the public API from pinned host buffers, every
    copy inside the timed region. The two caches go up first; then, per chunk
    of rows, the chunk's queries go up on one copy stream, the chunk runs on the
    compute stream (the path's entry point with the chunk's q_pos0, against the
    key prefix its rows see) and its output comes down on another copy stream,
    so the upload of chunk c+1 and the download of chunk c-1 run under chunk
    c's compute."""
    i, dsa, chunk = pf.inp, pf.dsa, pf.chunk
    T, S, k = i["T"], i["S"], i["k"]
    row_names = [n for n in ("q8", "q_scale", "w", "q") if i[n] is not None]
    cache_names = [n for n in ("k8", "k_scale", "kv") if i[n] is not None]
    host = {}
    for n in row_names + cache_names:
        h = torch.empty(i[n].shape, dtype=i[n].dtype, pin_memory=True)
        h.copy_(i[n])
        host[n] = h
    out_h = torch.empty(pf.out.shape, dtype=pf.out.dtype, pin_memory=True)
    lse_h = torch.empty(pf.lse.shape, dtype=pf.lse.dtype, pin_memory=True)
    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    size = (dsa.forward_fused_workspace_size if pf.path == "fused"
            else dsa.forward_workspace_size)
    ws = torch.empty(size(chunk, S, i["Hi"], i["H"], k, chunk), dtype=torch.uint8, device="cuda")
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    starts = list(range(0, T, chunk))
    cut = lambda x, a, b: None if x is None else x[a:b]

    def step():
        up.wait_stream(comp)
        with torch.cuda.stream(up):
            for n in cache_names:
                i[n].copy_(host[n], non_blocking=True)
        for c0 in starts:
            c1 = min(c0 + chunk, T)
            with torch.cuda.stream(up):
                for n in row_names:
                    i[n][c0:c1].copy_(host[n][c0:c1], non_blocking=True)
            comp.wait_stream(up)
            pf.run(i["q8"][c0:c1], cut(i["q_scale"], c0, c1), i["k8"][:c1], cut(i["k_scale"], 0, c1),
                   i["w"][c0:c1], i["q"][c0:c1], i["kv"][:c1], k, i["scale"], i["sm_scale"],
                   q_pos0=c0, chunk=chunk, idx=pf.idx[c0:c1], out=pf.out[c0:c1],
                   lse=pf.lse[c0:c1], workspace=ws)
            down.wait_stream(comp)
            with torch.cuda.stream(down):
                out_h[c0:c1].copy_(pf.out[c0:c1], non_blocking=True)
                lse_h[c0:c1].copy_(pf.lse[c0:c1], non_blocking=True)
        comp.wait_stream(down)

    step()
    torch.cuda.synchronize()
    e0, e1 = _ev(), _ev()
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del host, ws
    return ms, h2d, d2h


def time_decode(dsa, steps, warmup, cfg_id=DECODE_CFG):
    cfg = W.CONFIGS[cfg_id]
    inp = W.make_decode(cfg, device="cuda")
    g = inp
    B, nq, k = inp["B"], inp["nq"], inp["k"]
    ws = torch.empty(dsa.decode_workspace_size(B, nq, inp["max_blocks"], inp["Hi"], inp["H"], k),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(B, nq, inp["H"], 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, nq, inp["H"], dtype=torch.float32, device="cuda")
    idx = torch.empty(B, nq, k, dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def full():
        dsa.decode_paged(g["q8"], g["q_scale"], g["w"], g["q"], g["k8_pool"], g["k_scale_pool"],
                         g["kv_pool"], g["block_table"], g["seq_len"], k, inp["scale"],
                         inp["sm_scale"], idx=idx, out=out, lse=lse, workspace=ws)

    def mla():
        dsa.sparse_mla_decode_paged(g["q"], g["kv_pool"], g["block_table"], g["seq_len"], idx,
                                    inp["sm_scale"], out=out, lse=lse)

    res = {}
    for name, fn in (("total", full), ("sparse_mla", mla)):
        for _ in range(warmup):
            fn()
        times = []
        for _ in range(steps):
            flush.zero_()                                   # L2 flush, outside the events
            e0, e1 = _ev(), _ev()
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        res[name] = statistics.median(times)
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in decode: {dsa.STATUS.get(st, st)}")
    work = decode_work(inp["seq_len"].cpu().tolist(), nq, inp["Hi"], inp["H"], k)
    return res, work, B * nq, inp


def _time(fn, steps, warmup, flush=None):
    """Median device time of fn (ms) over `steps` calls after `warmup`, an
    optional L2 flush before each (outside the events)."""
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        e0, e1 = _ev(), _ev()
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def time_next(dsa, pf, path="scores"):
    """DSA beside dense causal attention (the same MLA kernel with every causal
    key, slots generated in the kernel) over the context length, for prefill
    (prefixes of the 128K prefill's inputs: the first L rows against the first
    L keys are an L-token causal prefill) and for decode (B = 64 sequences of
    one context length, paged). Also sliding-window attention at 16K, the
    projection and the warm-up objective."""
    i = pf.inp
    H, k, sm = i["H"], i["k"], i["sm_scale"]
    res = {"workload": "prefill: the first L rows of the L=131072 prefill (4096-row chunks, k=2048, "
                       "indexer 64x128 FP8, MLA 128 heads); dsa = " +
                       ("dsa_forward_fused" if path == "fused" else "dsa_forward") +
                       ", dense = dsa_dense_causal_mla (every causal key); decode: B=64 sequences "
                       "of the given context, nq=1, paged, L2 flushed before each call"}
    prefill = []
    for L in (4096, 16384, 65536, 131072):
        chunk = min(4096, L)
        size = dsa.forward_fused_workspace_size if path == "fused" else dsa.forward_workspace_size
        run = dsa.forward_fused if path == "fused" else dsa.forward
        ws = torch.empty(size(L, L, i["Hi"], H, k, chunk), dtype=torch.uint8, device="cuda")
        out = torch.empty(L, H, 512, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(L, H, dtype=torch.float32, device="cuda")
        cut = lambda x: None if x is None else x[:L]

        def dsa_call():
            run(i["q8"][:L], cut(i["q_scale"]), i["k8"][:L], cut(i["k_scale"]), i["w"][:L],
                i["q"][:L], i["kv"][:L], k, i["scale"], sm, chunk=chunk, out=out, lse=lse,
                workspace=ws, return_idx=False)

        def dense_call():
            dsa.dense_causal_mla(i["q"][:L], i["kv"][:L], sm, out=out, lse=lse)

        reps = 1 if L > 65536 else 2
        t_dsa = _time(dsa_call, reps, 1)
        t_dense = _time(dense_call, reps, 1)
        prefill.append({"L": L, "dsa_ms": t_dsa, "dense_ms": t_dense,
                        "dsa_tokens_per_s": L / (t_dsa * 1e-3),
                        "dense_tokens_per_s": L / (t_dense * 1e-3), "speedup": t_dense / t_dsa})
        del ws, out, lse
        torch.cuda.empty_cache()
    res["prefill"] = prefill
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    decode = []
    for ctx in (4096, 16384, 32768, 65536, 131072):
        cfg = W.Config(94, "decode_curve", "decode", k=2048, Hi=64, H=128, seed=7, B=64, ctx=ctx)
        d = W.make_decode(cfg, device="cuda")
        B, nq = d["B"], d["nq"]
        ws = torch.empty(dsa.decode_workspace_size(B, nq, d["max_blocks"], d["Hi"], d["H"], 2048),
                         dtype=torch.uint8, device="cuda")
        out = torch.empty(B, nq, d["H"], 512, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, nq, d["H"], dtype=torch.float32, device="cuda")

        def dsa_dec():
            dsa.decode_paged(d["q8"], d["q_scale"], d["w"], d["q"], d["k8_pool"], d["k_scale_pool"],
                             d["kv_pool"], d["block_table"], d["seq_len"], 2048, d["scale"],
                             d["sm_scale"], out=out, lse=lse, workspace=ws)

        def dense_dec():
            dsa.dense_causal_mla_decode_paged(d["q"], d["kv_pool"], d["block_table"], d["seq_len"],
                                              d["sm_scale"], out=out, lse=lse)

        t_dsa = _time(dsa_dec, 5, 2, flush)
        t_dense = _time(dense_dec, 5, 2, flush)
        decode.append({"ctx": ctx, "dsa_ms": t_dsa, "dense_ms": t_dense,
                       "dsa_queries_per_s": B * nq / (t_dsa * 1e-3),
                       "dense_queries_per_s": B * nq / (t_dense * 1e-3),
                       "speedup": t_dense / t_dsa})
        del d, ws, out, lse
        torch.cuda.empty_cache()
    res["decode"] = decode
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the DSA-vs-dense runs: {dsa.STATUS.get(st, st)}")
    # sliding-window attention (window k) at 16K, on the same MLA kernel
    L = 16384
    swa_idx = dsa.window_indices(L, L, k, k)
    out = torch.empty(L, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, H, dtype=torch.float32, device="cuda")
    t_swa = _time(lambda: dsa.sparse_mla(i["q"][:L], i["kv"][:L], swa_idx, sm, out=out, lse=lse),
                  3, 2)
    res["swa_16k"] = {"window": k, "ms": t_swa, "tokens_per_s": L / (t_swa * 1e-3)}
    del swa_idx, out, lse
    torch.cuda.empty_cache()
    res["projection"] = time_projection(dsa, 3, 2)
    res["warmup_objective"] = time_warmup(dsa, 3, 2)
    return res


def time_warmup(dsa, steps, warmup, L=2048):
    """The indexer's warm-up objective on one L-token prefill: the
    head-mean dense attention target (lse from the sparse MLA over dense index sets),
    the KL with its gradient on the indexer scores, and the backward to q, k, w."""
    cfg = W.Config(93, "warmup", "prefill", k=L, Hi=64, H=128, seed=6, L=L)
    inp = W.make_prefill(cfg, device="cuda")
    idx = dsa.window_indices(L, L, L, L)
    out = torch.empty(L, inp["H"], 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, inp["H"], dtype=torch.float32, device="cuda")
    ws = torch.empty(dsa.lib().dsa_attention_probs_workspace_size(L, L, inp["H"]),
                     dtype=torch.uint8, device="cuda")
    state = {}

    def target():
        dsa.sparse_mla(inp["q"], inp["kv"], idx, inp["sm_scale"], out=out, lse=lse)
        state["p"] = dsa.attention_probs_mean(inp["q"], inp["kv"], lse, inp["sm_scale"],
                                              workspace=ws)

    def kl():
        I = dsa.indexer_scores(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"],
                               inp["scale"])
        state["loss"], state["grad"] = dsa.indexer_kl(I, state["p"], L)

    bws = torch.empty(dsa.lib().dsa_indexer_backward_workspace_size(L, L, inp["Hi"]),
                      dtype=torch.uint8, device="cuda")

    def backward():
        dsa.indexer_backward(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"],
                             inp["scale"], state["grad"], workspace=bws)

    res = {"workload": f"prefill L={L}, 128 MLA heads, 64 indexer heads: target (dense MLA "
                       "for lse + head-mean weights), KL + gradient, backward to q, k, w"}
    for name, fn in (("target", target), ("kl", kl), ("backward", backward)):
        for _ in range(warmup):
            fn()
        e0, e1 = _ev(), _ev()
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        e1.synchronize()
        res[name] = {"ms": e0.elapsed_time(e1) / steps}
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the warm-up objective: {dsa.STATUS.get(st, st)}")
    res["loss_mean"] = float(state["loss"].mean())
    return res


def time_projection(dsa, steps, warmup, T=4096, d=4096, Hi=64):
    """Step 1 of the workflow (hidden states -> FP8 indexer inputs) for one 4096-token
    chunk; the width d is not given by the pages."""
    inp = W.make_projection(T, d, Hi, seed=5, device="cuda")
    ws = torch.empty(dsa.lib().dsa_project_workspace_size(T, Hi), dtype=torch.uint8,
                     device="cuda")

    def run():
        dsa.project_indexer_inputs(inp["h"], inp["wt"], inp["rope"], Hi, workspace=ws)

    for _ in range(warmup):
        run()
    e0, e1 = _ev(), _ev()
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the projection: {dsa.STATUS.get(st, st)}")
    flops = 2.0 * T * d * (Hi * 128 + 128 + Hi)
    tf = flops / (ms * 1e-3) / 1e12
    pk = peaks()
    return {"workload": f"T={T} tokens, d={d}, Hi={Hi}: GEMM to {Hi * 128 + 128 + Hi} outputs, "
                        "rotary on q and k, per-token FP8", "ms": ms,
            "tokens_per_s": T / (ms * 1e-3), "achieved": tf, "unit": "TFLOP/s",
            "peak": pk["bf16_sus"], "frac": tf / pk["bf16_sus"]}


# ------------------------------------------------------------ CPU oracle

def oracle_sample(inp, n_rows=32, threads=None):
    """Time the CPU oracle on query rows spread evenly over t (incl. the last).

    Each row runs the whole path (indexer over its causal prefix, top-k, sparse
    MLA). Rows are independent; they are shared out over host threads (the C
    oracle releases the GIL). Since the sample is stratified in t, rows/s
    estimates the oracle's tokens/s on the full workload.
    """
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or os.cpu_count() or 1
    T, k = inp["T"], inp["k"]
    rows = sorted(set(min(T - 1, int((i + 0.5) * T / n_rows)) for i in range(n_rows)) | {T - 1})
    r = torch.tensor(rows)
    host = dict(k8=inp["k8"].cpu(), k_scale=None if inp["k_scale"] is None else inp["k_scale"].cpu(),
                kv=inp["kv"].cpu(), q8=inp["q8"][r.to(inp["q8"].device)].cpu(),
                w=inp["w"][r.to(inp["w"].device)].cpu(), q=inp["q"][r.to(inp["q"].device)].cpu(),
                q_scale=None if inp["q_scale"] is None else inp["q_scale"][r.to(inp["q8"].device)].cpu())

    def one(i):
        t = rows[i]
        qs = None if host["q_scale"] is None else host["q_scale"][i:i + 1]
        I = oracle.indexer(host["q8"][i:i + 1], qs, host["k8"], host["k_scale"], host["w"][i:i + 1],
                           inp["scale"], q_pos0=t)
        sel = oracle.topk(I, [min(t + 1, inp["S"])], k)
        oracle.sparse_mla(host["q"][i:i + 1], host["kv"], sel, inp["sm_scale"])

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, range(len(rows))))
    wall = time.perf_counter() - t0
    return dict(value=len(rows) / wall, unit="tokens/s", cores=threads, kind="oracle",
                sample=f"{len(rows)} query rows of the L={T} prefill, evenly spaced in t "
                       f"(incl. the last), whole path per row, {threads} threads; "
                       f"{wall:.1f} s wall", wall_s=wall, cpu_model=cpu_model(),
                host_cpus=os.cpu_count())


def oracle_decode_sample(inp, n_seqs=8, threads=None):
    """Time the CPU oracle's paged decode on a sample of the batch's sequences,
    stratified by context length (every n-th by length, so queries/s on the
    sample estimates the whole batch's); rows run in parallel on host threads."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or os.cpu_count() or 1
    lens = inp["seq_len"].cpu().numpy()
    order = np.argsort(lens, kind="stable")
    B, nq = len(lens), inp["nq"]
    seqs = sorted({int(order[min(B - 1, int((i + 0.5) * B / n_seqs))]) for i in range(n_seqs)})
    as_np = {"q8": np.uint8, "q_scale": np.float32, "w": np.float32, "q": np.uint16,
             "k8_pool": np.uint8, "k_scale_pool": np.float32, "kv_pool": np.uint16,
             "block_table": np.int32, "seq_len": np.int32}
    host = dict(inp)
    for name, dt in as_np.items():                  # one host copy, shared by the threads
        host[name] = oracle._np(inp[name], dt)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda b: oracle.decode(host, seqs=[b]), seqs))
    wall = time.perf_counter() - t0
    ctx = [int(lens[b]) for b in seqs]
    return dict(value=len(seqs) * nq / wall, unit="queries/s", cores=threads, kind="oracle",
                sample=f"{len(seqs)} of the {B} sequences (every {B // len(seqs)}-th by context "
                       f"length: {min(ctx)}..{max(ctx)} tokens), {nq} queries each, whole path per "
                       f"query, {threads} threads; {wall:.1f} s wall", wall_s=wall)


def cpu_model():
    """The host CPU's model name, from /proc/cpuinfo (None where it is absent)."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ------------------------------------------------------------------- main

def config_obj(L, chunk):
    return {"workload": f"prefill L={L} causal, 4096-row chunks, k=2048, indexer 64x128 FP8, "
                        "MLA 128 heads x (512+64) bf16; decode B=64 x 32768 paged",
            "L": L, "chunk": chunk, "k": 2048, "Hi": 64, "H": 128,
            "l2": "prefill inputs exceed L2 (no flush); decode: 256 MB L2 flush per iteration"}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    L = args.L or W.CONFIGS[PREFILL_CFG].L
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    cfg = W.CONFIGS[PREFILL_CFG]
    inp = W.make_prefill(cfg, device=dev, L=L)
    for _ in range(args.warmup):
        oracle_sample(inp, n_rows=8)
    vals, walls, last = [], [], None
    for _ in range(args.steps):
        last = oracle_sample(inp)
        vals.append(last["value"])
        walls.append(last["wall_s"])
    v = statistics.mean(vals)
    last["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(walls), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_obj(L, cfg.chunk), "cpu_baseline": last,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args, dsa):
    """One small case per step, for ncu captures of single kernels (see --profile)."""
    if args.profile == "decode":
        dres, dwork, nq, _ = time_decode(dsa, max(args.steps, 1), args.warmup)
        print(json.dumps({"profile": "decode", "ms": dres, "queries": nq,
                          "mla_bytes": dwork["mla_bytes"], "idx_bytes": dwork["idx_bytes"]}))
        return
    cfg = W.CONFIGS[PREFILL_CFG]
    L = args.L or cfg.L
    chunk = cfg.chunk or 4096
    inp = W.make_prefill(cfg, device="cuda", L=L, rows=(L - chunk, L))
    torch.cuda.empty_cache()
    T, S, H, k = inp["T"], inp["S"], inp["H"], inp["k"]
    fused = args.path == "fused"
    size = dsa.forward_fused_workspace_size if fused else dsa.forward_workspace_size
    run = dsa.forward_fused if fused else dsa.forward
    ws = torch.empty(size(T, S, inp["Hi"], H, k, chunk), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")

    def step():
        run(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"], inp["q"], inp["kv"], k,
            inp["scale"], inp["sm_scale"], q_pos0=inp["q_pos0"], chunk=chunk, idx=idx, out=out,
            lse=lse, workspace=ws)

    for _ in range(args.warmup):
        step()
    e0, e1 = _ev(), _ev()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    e1.synchronize()
    st = dsa.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the profile case: {dsa.STATUS.get(st, st)}")
    line = {"profile": "chunk", "path": args.path, "rows": [L - chunk, L], "keys": S,
            "ms_per_call": e0.elapsed_time(e1) / max(args.steps, 1),
            "device_bytes": torch.cuda.memory_allocated()}
    if fused:
        line["fallback_rows"] = dsa.forward_fused_fallback_rows(ws, T, S, k, chunk)
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.profile:
        import sparse_attention_long_02_b200 as dsa
        torch.cuda.set_device(0)
        run_profile_case(args, dsa)
        return
    ranks = Ranks(args.gpus)
    import sparse_attention_long_02_b200 as dsa
    pk = peaks()
    fp8_sus = 2 * pk["bf16_sus"]
    fp8_burst = 2 * pk["bf16"]
    rows_mode = args.shard == "rows"
    # rows: every rank holds the same prefill and runs its share of the rows
    cfg, inp = prefill_inputs(args.L or W.CONFIGS[PREFILL_CFG].L, 0 if rows_mode else ranks.rank)
    L = inp["T"]
    shard = None
    if rows_mode:
        shard = RowShard(dsa, cfg, inp, ranks.world, ranks.rank, args.path)
        ms, clocks = time_steps(shard.step, args.steps, args.warmup, ranks, dsa, ranks.local)
        tokens = L
        del shard.ws, shard.out, shard.lse, shard.idx
        torch.cuda.empty_cache()
        pf = Prefill(dsa, cfg, inp, args.path)
    else:
        pf = Prefill(dsa, cfg, inp, args.path)
        ms, clocks = time_steps(pf.step, args.steps, args.warmup, ranks, dsa, ranks.local)
        tokens = L * ranks.world
    value = tokens / (ms / 1e3)
    # rows of the last timed step whose threshold missed and that were
    # recomputed on CUDA cores (the fused path keeps the count in its workspace)
    fallback_rows = (dsa.forward_fused_fallback_rows(pf.ws, inp["T"], inp["S"], inp["k"], pf.chunk)
                     if args.path == "fused" and not rows_mode else None)

    work = prefill_work(L, inp["Hi"], inp["H"], inp["k"])
    st = pf.stages()
    # each stage is timed on its own (events around one call), so its fraction
    # is of the burst peak; the sustained peak's fraction is given beside it
    stages = {
        "indexer": {"ms": st["indexer"], "bound": "tensor", "unit": "TFLOP/s",
                    "achieved": work["idx_flops"] / (st["indexer"] * 1e-3) / 1e12,
                    "peak": fp8_burst, "peak_sustained": fp8_sus,
                    "note": "scores-mode launches (dsa_indexer_scores), 32 chunks"},
        "topk": {"ms": st["topk"]},
        "sparse_mla": {"ms": st["sparse_mla"], "bound": "tensor", "unit": "TFLOP/s",
                       "achieved": work["mla_flops"] / (st["sparse_mla"] * 1e-3) / 1e12,
                       "peak": pk["bf16"], "peak_sustained": pk["bf16_sus"]},
    }
    for s in stages.values():
        if "peak" in s:
            s["frac"] = s["achieved"] / s["peak"]
            s["frac_sustained"] = s["achieved"] / s["peak_sustained"]
    dom = max(("indexer", "sparse_mla"), key=lambda s: st[s])
    launches_per_step = {"indexer": math.ceil(L / pf.chunk), "sparse_mla": 1}[dom]
    traffic, traffic_src = traffic_from_profile(dom)
    roof = {"kernel": dom, "bound": "tensor", "achieved": stages[dom]["achieved"],
            "peak": stages[dom]["peak"], "unit": "TFLOP/s", "frac": stages[dom]["frac"],
            "frac_sustained": stages[dom]["frac_sustained"],
            "traffic": traffic, "traffic_unit": "bytes per launch", "traffic_src": traffic_src,
            "launches_per_step": launches_per_step,
            "peak_src": f"{pk['src']} burst bf16 (the stage is timed alone)" +
                        (" x2 (FP8/BF16 nominal ratio)" if dom == "indexer" else "")}
    t_roof = max(work["idx_flops"] / (fp8_sus * 1e12), work["idx_bytes"] / (pk["hbm"] * 1e9)) + \
        max(work["mla_flops"] / (pk["bf16_sus"] * 1e12), work["mla_bytes"] / (pk["hbm"] * 1e9))

    config = config_obj(L, pf.chunk)
    config["path"] = ("dsa_forward_fused: top-k fused into the indexer, no score rows in HBM"
                      if args.path == "fused" else
                      "dsa_forward: each chunk's scores in HBM, top-k beside the next indexer")
    if fallback_rows is not None:
        config["fallback_rows"] = fallback_rows
    if rows_mode:
        config["shard"] = (f"rows: the {math.ceil(L / pf.chunk)} chunks of one prefill over "
                           f"{ranks.world} GPU(s) by causal cost; rank 0 runs "
                           f"{len(shard.starts)} chunks ({shard.rows} rows)")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ranks.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong" if rows_mode else "weak",
            "vs_baseline": None,
            "dtype": "fp8 indexer / bf16 MLA, fp32 accumulate", "data": "synthetic",
            "config": config, "clocks": clocks,
            "gpu_launches": (shard.launches if rows_mode else pf.launches) * args.steps,
            "roofline": roof, "stages": stages,
            "end_to_end_roofline": {"ms": 1e3 * t_roof, "frac": 1e3 * t_roof / ms}}
    if not args.no_decode:
        dres, dwork, nqueries, dinp = time_decode(dsa, max(args.steps, 10), args.warmup)
        mla_gbs = dwork["mla_bytes"] / (dres["sparse_mla"] * 1e-3) / 1e9
        line["decode"] = {
            "workload": "B=64 x 32768, nq=1, paged (block 64), k=2048, 64x128 FP8 indexer, "
                        "MLA 128 heads", "value": nqueries * ranks.world / (dres["total"] * 1e-3),
            "unit": "queries/s", "ms": dres["total"],
            "sparse_mla": {"ms": dres["sparse_mla"], "bound": "hbm", "achieved": mla_gbs,
                           "peak": pk["hbm"], "unit": "GB/s", "frac": mla_gbs / pk["hbm"]},
            "indexer_topk_ms": dres["total"] - dres["sparse_mla"]}
        # decode is HBM-bound in both stages: the indexer's algorithmic bytes (the
        # visible k8 rows, scales, q8, w, idx out) and the MLA's (selected rows, q, out,
        # lse), each at the measured copy bandwidth, or its flops at the tensor peak
        it_ms = dres["total"] - dres["sparse_mla"]
        t_idx = max(dwork["idx_bytes"] / (pk["hbm"] * 1e9), dwork["idx_flops"] / (fp8_sus * 1e12))
        t_mla = max(dwork["mla_bytes"] / (pk["hbm"] * 1e9),
                    dwork["mla_flops"] / (pk["bf16_sus"] * 1e12))
        line["decode"]["indexer_topk"] = {
            "ms": it_ms, "bound": "hbm", "unit": "GB/s",
            "achieved": dwork["idx_bytes"] / (it_ms * 1e-3) / 1e9, "peak": pk["hbm"],
            "frac": 1e3 * t_idx / it_ms,
            "note": "indexer + top-k timed together, against the indexer's algorithmic bytes"}
        line["decode"]["end_to_end_roofline"] = {"ms": 1e3 * (t_idx + t_mla),
                                                 "frac": 1e3 * (t_idx + t_mla) / dres["total"]}
        vres, vwork, vq, vinp = time_decode(dsa, max(args.steps, 10), args.warmup, cfg_id=5)
        vgbs = vwork["mla_bytes"] / (vres["sparse_mla"] * 1e-3) / 1e9
        line["decode_varlen"] = {
            "workload": "B=128, contexts log-uniform in [512, 131072], nq=2 causal, paged, "
                        "k=2048", "value": vq * ranks.world / (vres["total"] * 1e-3),
            "unit": "queries/s", "ms": vres["total"],
            "sparse_mla": {"ms": vres["sparse_mla"], "bound": "hbm", "achieved": vgbs,
                           "peak": pk["hbm"], "unit": "GB/s", "frac": vgbs / pk["hbm"]}}
    if args.next:
        line["next"] = time_next(dsa, pf, args.path)
    if not args.no_e2e and not rows_mode:       # e2e: the default mode's whole prefill per GPU
        e_ms, h2d, d2h = e2e_prefill(pf, max(1, min(args.steps, 3)))
        line["e2e"] = {"value": tokens / (ranks.max(e_ms) / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if ranks.rank == 0 and ranks.world == 1 and not args.no_cpu:
        cb = oracle_sample(inp)
        one = oracle_sample(inp, n_rows=8, threads=1)
        cb["single_thread"] = {k: one[k] for k in ("value", "unit", "cores", "sample", "wall_s")}
        if not args.no_decode:
            cb["decode"] = oracle_decode_sample(dinp)
            cb["decode"]["workload"] = "decode B=64 x 32768, nq=1 (the GPU decode line's)"
            vcb = oracle_decode_sample(vinp)
            vcb["workload"] = "decode B=128, contexts log-uniform in [512, 131072], nq=2"
            cb["decode_varlen"] = vcb
        line["cpu_baseline"] = cb
    ranks.close()
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
