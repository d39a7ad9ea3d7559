"""Benchmark of the shared-index top-k sparse KV attention hot path on B200.

One bench step = one denoising block of the workload, for L independent layer
copies (distinct K/V caches, queries and outputs, so every step streams from
HBM rather than L2):
  * selection of the NEXT block (dsa_select, all L layers) on a second stream,
  * overlapped with the T-1 sparse steps of the CURRENT block
    (dsa_sparse_attn x (T-1) x L) on the main stream, which reuse the indices
    selected one step earlier (ping-pong index buffers).
The step is captured once into CUDA graphs and replayed.  `value` is algorithmic
HBM bytes (selected K/V + block Q/O per sparse step; prefix K/V + Q/O per
selection) over device time, summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs are independent replicas (the path has no exchange step);
torch.distributed/NCCL is used only for the barrier and the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_27_b200 import workloads as W  # noqa: E402

METRIC = "sparse block-step µs & HBM GB/s (% roofline) at 128K, k=1024; select-pass ms"
WORKLOAD_TEXT = {
    "128k": "128k: 1 seq, prefix N=131072, block B=32, Hq=32, Hkv=8 (GQA 4), d=128, page=16, "
            "top-k 1024 tokens (64 pages), 32 steps/block, bf16 N(0,1) with 0.5% needle pages; "
            "selection of block n+1 on a second stream overlapped with block n's sparse steps",
    "8k": "8k: 1 seq, N=8192, B=32, Hq=32, Hkv=8, d=128, page=16, top-k 512 tokens, 32 steps",
    "32k": "32k: 1 seq, N=32768, B=32, Hq=28, Hkv=4, d=128, page=64, top-k 1024 tokens, 32 steps",
    "tiny": "tiny: 1 seq, N=1024, B=4, Hq=4, Hkv=1, d=64, page=16, top-k 128 tokens, 4 steps, "
            "8 planted needle pages",
    "batched": "batched: 8 seqs, N~U[16K,64K], B=32, Hq=32, Hkv=8, d=128, page=16, "
               "top-k in {512,1024,2048}, 32 steps, random page table",
}


# ------------------------------------------------------------------ bytes/flops
def sparse_bytes(w) -> int:
    """Selected K/V + block Q/O bytes of one sparse step (per layer)."""
    sel = sum(min(int(w.topk[s]), w.n_pages(s) * w.P) for s in range(w.S)) * w.Hkv * w.d * 2 * 2
    qo = 2 * w.S * w.B * w.Hq * w.d * 2
    return sel + qo


def select_bytes(w) -> int:
    """Prefix K/V + block Q/O bytes of one selection pass (per layer)."""
    kv = sum(int(w.n_ctx[s]) for s in range(w.S)) * w.Hkv * w.d * 2 * 2
    return kv + 2 * w.S * w.B * w.Hq * w.d * 2


def sparse_flops(w) -> int:
    keys = sum(min(int(w.topk[s]), w.n_pages(s) * w.P) + w.B for s in range(w.S)) / w.S
    return int(4 * w.S * w.B * w.Hq * keys * w.d)


def select_flops(w) -> int:
    return int(4 * w.B * w.Hq * w.d * sum(int(w.n_ctx[s]) for s in range(w.S)))


# ---------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_sha() -> str:
    """Hash of the kernel sources with comments and blank lines removed: editing a
    comment keeps the recorded traffic, any change to the code drops it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_27_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())
        h.update(name.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches this source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(f"{kernel}@{workload}")
    if not rec or rec.get("source_sha") != kernel_source_sha():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms in the background."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in self.rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torch.distributed.run sets RANK/LOCAL_RANK/WORLD_SIZE).
    The process group carries only the barrier and the max-over-ranks time; the
    "gloo" backend serves the CPU tests of this plumbing."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    elif n_gpus > 1:
        raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run")
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- CPU baseline
def oracle_block(w, steps, seqs=None):
    """The fp64 oracle on one block of one layer: selection + `steps` sparse steps, for
    the first `seqs` sequences of the batch (all by default).  Returns the seconds."""
    import oracle
    S = w.S if seqs is None else min(seqs, w.S)
    pt = None if w.page_table is None else w.page_table.numpy()[:S]
    n_ctx, topk = w.n_ctx.numpy()[:S], w.topk.numpy()[:S]
    inputs = [tuple(x[:S] for x in w.step_inputs(t)) for t in range(2, 2 + steps)]
    t0 = time.perf_counter()
    r = oracle.select(W.bits(w.q1[:S]), W.bits(w.k_cache), W.bits(w.v_cache), n_ctx, topk,
                      page_table=pt, max_pages=w.max_pages)
    for q, bk, bv in inputs:
        oracle.sparse(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache), n_ctx, r.idx, r.cnt,
                      W.bits(bk), W.bits(bv), page_table=pt, max_pages=w.max_pages)
    return time.perf_counter() - t0


def sample_bytes(w, steps, seqs=None):
    """Algorithmic bytes of oracle_block's sample."""
    S = w.S if seqs is None else min(seqs, w.S)
    kv = sum(int(w.n_ctx[s]) for s in range(S)) * w.Hkv * w.d * 2 * 2
    sel = sum(min(int(w.topk[s]), w.n_pages(s) * w.P) for s in range(S)) * w.Hkv * w.d * 2 * 2
    qo = 2 * S * w.B * w.Hq * w.d * 2
    return kv + qo + steps * (sel + qo)


def block_time_shape(dsa, names=("8k", "32k", "128k"), reps=20):
    """One layer of a denoising block at several context lengths, with a GEMM stand-in
    for the FFN (two bf16 matmuls, d_model = Hq*d, d_ff = 4*d_model, S*B tokens, random
    weights; cuBLAS through torch).  Per context: the selection pass (exact attention of
    the block's queries over the prefix, the dense stand-in), the sparse step and the FFN
    in microseconds (eager launches, CUDA events), attention's share of a block's time
    and the block speed-up of shared-index sparse attention over exact attention at every
    step: 32 x (exact + ffn) / (select + 31 x sparse + 32 x ffn)."""
    out = {}
    cur = torch.cuda.current_stream()
    for name in names:
        w = W.make(name, 0)
        dw = dsa.DeviceWorkload(w)
        dm = w.Hq * w.d
        g = torch.Generator(device="cuda")
        g.manual_seed(1)
        x = torch.randn((w.S * w.B, dm), device="cuda", generator=g, dtype=torch.float32).to(torch.bfloat16)
        w1 = (torch.randn((dm, 4 * dm), device="cuda", generator=g, dtype=torch.float32) / dm ** 0.5).to(torch.bfloat16)
        w2 = (torch.randn((4 * dm, dm), device="cuda", generator=g, dtype=torch.float32) / (4 * dm) ** 0.5).to(torch.bfloat16)
        ffn = lambda i: torch.matmul(torch.matmul(x, w1), w2)  # noqa: E731
        for i in range(3):
            dw.select()
            dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1)
            ffn(i)
        sel_us = 1e3 * timed(lambda i: dw.select(), reps, cur)
        sp_us = 1e3 * timed(lambda i: dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1), reps, cur)
        ffn_us = 1e3 * timed(ffn, reps, cur)
        T = w.T
        sparse_block = sel_us + (T - 1) * sp_us + T * ffn_us
        dense_block = T * (sel_us + ffn_us)
        out[name] = {"select_us": round(sel_us, 1), "sparse_step_us": round(sp_us, 2),
                     "ffn_us": round(ffn_us, 2),
                     "attention_share_sparse": round((sel_us + (T - 1) * sp_us) / sparse_block, 3),
                     "attention_share_exact": round(T * sel_us / dense_block, 3),
                     "block_speedup": round(dense_block / sparse_block, 2)}
        del dw, x, w1, w2
    return out


def cpu_baseline(w):
    """The oracle as it stands on the host cores: one block of one layer (the selection
    pass plus T-1 sparse steps); of a batch, its first sequence only (a bounded sample)."""
    import oracle
    steps = w.T - 1
    seqs = 1 if w.S > 1 else None
    secs = oracle_block(w, steps, seqs)
    nbytes = sample_bytes(w, steps, seqs)
    what = "its first sequence" if seqs else "the whole workload"
    return {"value": round(nbytes / secs / 1e9, 6), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(secs, 3),
            "sample": f"one block of one layer of the {w.name} workload ({what}): the selection "
                      f"pass plus {steps} sparse steps ({nbytes} algorithmic bytes) in {secs:.2f} s"}


def run_reference(args, world, rank):
    """--impl reference: the fp64 oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    w = W.make(args.workload, 0)
    steps = w.T - 1
    nbytes = select_bytes(w) + steps * sparse_bytes(w)
    for _ in range(args.warmup):
        oracle_block(w, steps)
    secs = [oracle_block(w, steps) for _ in range(args.steps)]
    total = sum(secs)
    value = nbytes * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload),
                   "unit_of_work": "one block of one layer (selection + T-1 sparse steps)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"one block of one layer of the {args.workload} workload per "
                                   f"step ({nbytes} algorithmic bytes)"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU bench
class Bench:
    def __init__(self, w, layers: int, dsa, select_sms: int = 0):
        self.w, self.L, self.dsa = w, layers, dsa
        dev = torch.device("cuda")
        T, S = w.T, w.S
        self.main = torch.cuda.current_stream()   # a non-default stream set by run_ours
        self.side = torch.cuda.Stream()           # the selection of the next block
        self.h2d = torch.cuda.Stream()            # end-to-end runs: inputs in, ahead of use
        self.d2h = torch.cuda.Stream()            # end-to-end runs: outputs out, behind
        # L independent layer copies of the KV cache
        self.k = torch.empty((layers, *w.k_cache.shape), dtype=torch.bfloat16, device=dev)
        self.v = torch.empty_like(self.k)
        kb, vb = w.k_cache.to(dev), w.v_cache.to(dev)
        self.k.copy_(kb.unsqueeze(0).expand_as(self.k))
        self.v.copy_(vb.unsqueeze(0).expand_as(self.v))
        del kb, vb
        # per-step inputs (step 1 = selection queries), one copy per layer
        steps = [w.step_inputs(t) for t in range(1, T + 1)]
        self.host_q = torch.stack([s[0] for s in steps]).pin_memory()     # [T, S, B, Hq, d]
        self.host_bk = torch.stack([s[1] for s in steps]).pin_memory()    # [T, S, B, Hkv, d]
        self.host_bv = torch.stack([s[2] for s in steps]).pin_memory()
        self.q = self.host_q.to(dev).unsqueeze(0).repeat(layers, 1, 1, 1, 1, 1).contiguous()
        self.bk = self.host_bk.to(dev).unsqueeze(0).repeat(layers, 1, 1, 1, 1, 1).contiguous()
        self.bv = self.host_bv.to(dev).unsqueeze(0).repeat(layers, 1, 1, 1, 1, 1).contiguous()
        self.n_ctx = w.n_ctx.to(dev)
        self.topk = w.topk.to(dev)
        self.page_table = None if w.page_table is None else w.page_table.to(dev)
        # the sparse steps reuse indices the selection wrote one block earlier (on the side
        # stream, joined by an event): each gathers its pages before the kernel ahead of it ends
        self.dims = dsa.dims_for(self.q[0, 0], self.k[0], w.max_pages, w.kmax, self.page_table,
                                 sm_limit=select_sms, early_gather=1)
        self.idx = torch.full((2, layers, S, w.Hkv, w.kmax), -1, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros((2, layers, S, w.Hkv), dtype=torch.int32, device=dev)
        self.o_sel = torch.empty((layers, *w.q1.shape), dtype=torch.bfloat16, device=dev)
        # one output per (layer, later step): an output copied to the host end to end
        # is never overwritten by a later kernel
        self.o_sp = torch.empty((layers, T - 1, *w.q1.shape), dtype=torch.bfloat16, device=dev)
        self.ws_sel = dsa.Workspace(dsa.select_workspace_size(self.dims), dev)
        self.ws_sp = dsa.Workspace(dsa.sparse_workspace_size(self.dims), dev)
        self.host_o = torch.empty((T, *w.q1.shape), dtype=torch.bfloat16).pin_memory()
        self.host_o_sel = torch.empty(w.q1.shape, dtype=torch.bfloat16).pin_memory()
        self.host_idx = torch.empty((w.S, w.Hkv, w.kmax), dtype=torch.int32).pin_memory()

    # one call each -------------------------------------------------------------
    def select(self, l, buf, stream):
        self.dsa.dsa_select(self.q[l, 0], self.k[l], self.v[l], self.n_ctx, self.w.P, self.topk,
                            self.idx[buf, l], self.o_sel[l], stream, dims=self.dims,
                            cnt_out=self.cnt[buf, l], workspace=self.ws_sel)

    def sparse(self, l, t, buf, stream):
        self.dsa.dsa_sparse_attn(self.q[l, t], self.k[l], self.v[l], self.idx[buf, l],
                                 self.bk[l, t], self.bv[l, t], self.o_sp[l, t - 1], stream,
                                 dims=self.dims, n_ctx=self.n_ctx, idx_cnt=self.cnt[buf, l],
                                 workspace=self.ws_sp)

    # the block step: select(next) on the side stream || sparse(current) on main
    def block_step(self, cur, e2e=False):
        nxt = 1 - cur
        L, T = self.L, self.w.T
        main, side = self.main, self.side
        if not e2e:
            side.wait_stream(main)
            with torch.cuda.stream(side):
                for l in range(L):
                    self.select(l, nxt, side)
            for t in range(1, T):
                for l in range(L):
                    self.sparse(l, t, cur, main)
            main.wait_stream(side)
            return
        # End to end: every call's inputs are copied in from pinned host memory on a
        # copy stream, ahead of their use (an event per call gates it), and every
        # output is copied back on another stream once its kernel is done, so that
        # the copies overlap the kernels.
        side.wait_stream(main)
        self.h2d.wait_stream(main)
        self.d2h.wait_stream(main)
        ready = {}
        with torch.cuda.stream(self.h2d):
            for t in range(T):
                for l in range(L):
                    self.q[l, t].copy_(self.host_q[t], non_blocking=True)
                    if t > 0:
                        self.bk[l, t].copy_(self.host_bk[t], non_blocking=True)
                        self.bv[l, t].copy_(self.host_bv[t], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(self.h2d)
                    ready[(l, t)] = ev
        for l in range(L):
            side.wait_event(ready[(l, 0)])
            self.select(l, nxt, side)
            done = torch.cuda.Event()
            done.record(side)
            self.d2h.wait_event(done)
            with torch.cuda.stream(self.d2h):
                self.host_o_sel.copy_(self.o_sel[l], non_blocking=True)
                self.host_idx.copy_(self.idx[nxt, l], non_blocking=True)
        for t in range(1, T):
            for l in range(L):
                main.wait_event(ready[(l, t)])
                self.sparse(l, t, cur, main)
                done = torch.cuda.Event()
                done.record(main)
                self.d2h.wait_event(done)
                with torch.cuda.stream(self.d2h):
                    self.host_o[t].copy_(self.o_sp[l, t - 1], non_blocking=True)
        main.wait_stream(side)
        main.wait_stream(self.h2d)
        main.wait_stream(self.d2h)

    def h2d_d2h_bytes(self):
        w, L = self.w, self.L
        q = self.host_q[0].numel() * 2
        blk = self.host_bk[0].numel() * 2
        h2d = L * (q + (w.T - 1) * (q + 2 * blk))
        d2h = L * (q + self.host_idx.numel() * 4 + (w.T - 1) * q)
        return h2d, d2h

    def capture(self, e2e=False):
        graphs = []
        for cur in (0, 1):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.main, capture_error_mode="relaxed"):
                self.block_step(cur, e2e)
            graphs.append(g)
        return graphs

    def capture_sparse_only(self):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.main, capture_error_mode="relaxed"):
            for t in range(1, self.w.T):
                for l in range(self.L):
                    self.sparse(l, t, 0, self.main)
        return g


def timed(fn, reps, stream):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(reps):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / reps  # ms


def run_ours(args, world, rank, local):
    from block_sparse_attention_27_b200 import build as build_mod
    from block_sparse_attention_27_b200 import dsa
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the CUDA library has no CPU path)")
    build_mod.build()
    dsa.load()
    torch.cuda.set_device(local)
    main_stream = torch.cuda.Stream()   # graphs cannot be captured on the legacy stream
    with torch.cuda.stream(main_stream):
        _run_ours(args, world, rank, local, dsa)


LAYERS = {"128k": 64, "8k": 64, "32k": 64, "tiny": 64, "batched": 4}


def measure(w, layers, dsa, steps, warmup, world, select_sms=0, clocks=None, e2e=False):
    """The block step of workload `w` over `layers` independent layer copies: the
    overlapped step (selection of the next block on the side stream, the T-1 sparse
    steps of the current block on the main stream) captured in CUDA graphs and
    replayed, then the selection alone and the sparse steps alone (their own graph),
    and end to end if asked.  Times in ms / us from CUDA events on the launching
    stream; the step time is the max over ranks."""
    b = Bench(w, layers, dsa, select_sms)
    T, L = w.T, layers
    for l in range(L):  # block 0's indices; every kernel warmed up eagerly
        b.select(l, 0, b.main)
    torch.cuda.synchronize()
    b.sparse(0, 1, 0, b.main)
    torch.cuda.synchronize()
    graphs = b.capture()
    for i in range(warmup):
        graphs[i % 2].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if clocks is not None:
        with clocks:
            ms = timed(lambda i: graphs[(warmup + i) % 2].replay(), steps, b.main)
    else:
        ms = timed(lambda i: graphs[(warmup + i) % 2].replay(), steps, b.main)
    barrier(world)
    ms = max_over_ranks(ms, world)
    del graphs
    status_sel, status_sp = b.ws_sel.status(), b.ws_sp.status()
    if status_sel != dsa.DSA_OK or status_sp != dsa.DSA_OK:
        raise SystemExit(f"{w.name}: device status: select {status_sel}, sparse {status_sp}")
    # the parts alone: the selection (eager launches over the layers) and the
    # sparse steps (their own graph)
    reps = 3
    sel_ms = timed(lambda i: [b.select(l, 0, b.main) for l in range(L)], reps, b.main) / L
    torch.cuda.synchronize()
    sel_full_ms = sel_ms
    if select_sms:  # the pass alone on the whole device, as a caller without a second stream runs it
        dims_sm = b.dims
        b.dims = dsa.dims_for(b.q[0, 0], b.k[0], w.max_pages, w.kmax, b.page_table, early_gather=1)
        b.ws_sel = dsa.Workspace(dsa.select_workspace_size(b.dims), "cuda")
        for l in range(L):
            b.select(l, 0, b.main)
        sel_full_ms = timed(lambda i: [b.select(l, 0, b.main) for l in range(L)], reps, b.main) / L
        torch.cuda.synchronize()
        b.dims = dims_sm
    g_sp = b.capture_sparse_only()
    g_sp.replay()
    sp_us = 1e3 * timed(lambda i: g_sp.replay(), reps, b.main) / ((T - 1) * L)
    del g_sp
    out = {"b": b, "ms": ms, "sel_ms": sel_ms, "sel_full_ms": sel_full_ms, "sp_us": sp_us,
           "launches_per_step": L * (dsa.select_launches(b.dims) + (T - 1) * dsa.kernels_per_call(1)),
           "sparse_kernel": dsa.sparse_kernel(b.dims), "select_sms": select_sms}
    if e2e:
        e2e_graphs = b.capture(e2e=True)
        for i in range(2):
            e2e_graphs[i % 2].replay()
        out["e2e_ms"] = max_over_ranks(timed(lambda i: e2e_graphs[i % 2].replay(), steps, b.main), world)
        del e2e_graphs
        out["h2d"], out["d2h"] = b.h2d_d2h_bytes()
    return out


def config_entry(w, m, layers, hbm_peak, world, cpu):
    """One workload's numbers for the JSON line (the headline's sub-objects use the
    same fields)."""
    T = w.T
    sel_b, sp_b = select_bytes(w), sparse_bytes(w)
    sel_gbs = sel_b / (m["sel_full_ms"] * 1e-3) / 1e9
    sp_gbs = sp_b / (m["sp_us"] * 1e-6) / 1e9
    serial = layers * (m["sel_ms"] + (T - 1) * m["sp_us"] * 1e-3)
    e = {"workload": WORKLOAD_TEXT.get(w.name, w.name), "layers_rotated": layers,
         "step_ms": round(m["ms"], 4),
         "step_gbs": round(world * layers * (sel_b + (T - 1) * sp_b) / (m["ms"] * 1e-3) / 1e9, 1),
         "sparse_step_us": round(m["sp_us"], 3), "sparse_step_gbs": round(sp_gbs, 1),
         "sparse_frac": round(sp_gbs / hbm_peak, 4), "sparse_bytes": sp_b,
         "sparse_kernel": ("resident, clusters of %d" % (m["sparse_kernel"] - 1)
                           if m["sparse_kernel"] > 1 else "streaming"),
         "select_pass_ms": round(m["sel_full_ms"], 4), "select_pass_gbs": round(sel_gbs, 1),
         "select_pass_ms_in_step": round(m["sel_ms"], 4),
         "select_frac": round(sel_gbs / hbm_peak, 4), "select_bytes": sel_b,
         "overlap": {"what": f"makespan of the block step (the selection of the next block on a "
                             f"second stream beside the {T - 1} sparse steps of the current one, "
                             f"{layers} layers) against the sum of the parts timed alone",
                     "select_sms": m["select_sms"] or "all",
                     "serial_ms": round(serial, 4), "makespan_ms": round(m["ms"], 4),
                     "gain": round(serial / m["ms"] - 1.0, 4)}}
    if cpu:
        e["oracle"] = cpu_baseline(w)
    return e


def _run_ours(args, world, rank, local, dsa):
    w = W.make(args.workload, 0)
    hbm_peak, tc_peak, peak_kind = load_peaks()
    T, L = w.T, args.layers
    clk = ClockSampler(local)
    m = measure(w, L, dsa, args.steps, args.warmup, world, args.select_sms, clocks=clk, e2e=True)
    b, ms, sel_ms, sp_us = m["b"], m["ms"], m["sel_full_ms"], m["sp_us"]
    step_bytes = L * (select_bytes(w) + (T - 1) * sparse_bytes(w))
    launches_per_step = m["launches_per_step"]
    e2e_ms, h2d, d2h = m["e2e_ms"], m["h2d"], m["d2h"]
    head = config_entry(w, m, L, hbm_peak, world, cpu=False)
    host_q = b.host_q
    del m, b
    torch.cuda.empty_cache()

    # MAGE's central quantity (outside the timed region): recall of the page set in
    # use at each step against that step's own top-k, for the reused step-1 set
    # and for a refresh every 8 steps
    from block_sparse_attention_27_b200 import recall as R
    dw = dsa.DeviceWorkload(w)
    qs = [host_q[t].cuda() for t in range(T)]
    rec_reused = R.step_recall(dw, qs)
    rec_anchor8 = R.step_recall(dw, qs, anchor=8)
    # exact step-1 output: what it costs beyond the selection pass (which writes its
    # row log-sum-exps as well): the block-only sparse pass and the LSE merge
    lse_sel = torch.empty(w.q1.shape[:3], dtype=torch.float32, device="cuda")
    lse_blk, lse_all = torch.empty_like(lse_sel), torch.empty_like(lse_sel)
    no_pages = torch.zeros_like(dw.cnt)
    o_all = torch.empty_like(dw.o_sel)
    dw.select(lse_out=lse_sel)

    def exact_extra(_):
        o_blk = dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1, cnt=no_pages, lse_out=lse_blk)
        dsa.dsa_merge_attn(dw.o_sel, lse_sel, o_blk, lse_blk, o_all, lse_all)
    for i in range(3):
        exact_extra(i)
    exact_us = 1e3 * timed(exact_extra, 20, torch.cuda.current_stream())
    # head-adaptive budget (Step-dLLM): one budget of Hkv*kp pages per sequence shared
    # by its KV heads; its selection pass and a sparse step on the ragged per-head
    # counts, beside a per-head sparse step timed the same way (eager launches)
    cur = torch.cuda.current_stream()
    dwh = dsa.DeviceWorkload(w, head_budget=1)
    for i in range(3):
        dwh.select()
    hb_sel_ms = timed(lambda i: dwh.select(), 20, cur)
    for i in range(3):
        dwh.sparse(dwh.q1, dwh.blk_k1, dwh.blk_v1)
        dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1)
    hb_sp_us = 1e3 * timed(lambda i: dwh.sparse(dwh.q1, dwh.blk_k1, dwh.blk_v1), 50, cur)
    ph_sp_us = 1e3 * timed(lambda i: dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1), 50, cur)
    hb_cnt = dwh.cnt.cpu().numpy()
    # prefix-part reuse (LoSA): a sparse step whose tokens are all stable reads its
    # prefix parts from the caches and loads no page; one with every token active
    # computes them and refreshes the caches
    c_o = torch.empty_like(dw.q1)
    c_l = torch.empty(w.q1.shape[:3], dtype=torch.float32, device="cuda")
    on = torch.ones((w.S, w.B), dtype=torch.uint8, device="cuda")
    off = torch.zeros_like(on)
    for i in range(3):
        dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1, active=on, cache=(c_o, c_l))
    losa_active_us = 1e3 * timed(lambda i: dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1, active=on,
                                                       cache=(c_o, c_l)), 50, cur)
    losa_stable_us = 1e3 * timed(lambda i: dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1, active=off,
                                                       cache=(c_o, c_l)), 50, cur)
    del dw, dwh, qs, c_o, c_l
    shape = block_time_shape(dsa)
    torch.cuda.empty_cache()

    # the other workloads, timed the same way (each its own graphs over its own
    # layer copies; the batched workload holds ~1.3 GB of cache per layer, so fewer)
    others = {}
    for name in [c for c in args.configs.split(",") if c and c != "none" and c != args.workload]:
        wc = W.make(name, 0)
        mc = measure(wc, LAYERS.get(name, 64), dsa, args.steps, args.warmup, world, args.select_sms)
        others[name] = config_entry(wc, mc, LAYERS.get(name, 64), hbm_peak, world,
                                     cpu=(world == 1 and not args.no_cpu_baseline))
        del mc, wc
        torch.cuda.empty_cache()

    if rank != 0:
        return
    sel_b, sp_b = select_bytes(w), sparse_bytes(w)
    value = world * step_bytes / (ms * 1e-3) / 1e9
    sel_gbs = sel_b / (sel_ms * 1e-3) / 1e9
    sp_gbs = sp_b / (sp_us * 1e-6) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload),
                   "step": f"one denoising block over {L} independent layer copies: selection "
                           f"of the next block ({L} x dsa_select, second stream) overlapped with "
                           f"{T - 1} x {L} dsa_sparse_attn of the current block",
                   "layers_rotated": L,
                   "select_sms": args.select_sms or "all",
                   "l2": f"inputs larger than L2: {L} distinct K/V caches, queries and outputs "
                         f"({step_bytes / 1e9:.1f} GB of algorithmic traffic per step)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "sparse_step_us": round(sp_us, 3),
        "sparse_step_gbs": round(sp_gbs, 1),
        "select_pass_ms": round(sel_ms, 4),
        "select_pass_gbs": round(sel_gbs, 1),
        "select_pass_ms_in_step": head["select_pass_ms_in_step"],
        # the kernel that takes most of the step: the sparse step
        "roofline": {"bound": "hbm", "kernel": "sparse step (dsa_sparse_attn)",
                     "achieved": round(sp_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(sp_gbs / hbm_peak, 4),
                     "traffic": recorded_traffic("sparse", args.workload),
                     "algorithmic_bytes_per_launch": sp_b, "peak_kind": peak_kind,
                     "share_of_step": round(L * (T - 1) * sp_us * 1e-3 / ms, 3)},
        "roofline_select": {"bound": "hbm", "kernel": "selection pass (dsa_select)",
                            "achieved": round(sel_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                            "frac": round(sel_gbs / hbm_peak, 4),
                            "traffic": recorded_traffic("select", args.workload),
                            "algorithmic_bytes_per_launch": sel_b, "peak_kind": peak_kind,
                            "timed": "alone on the whole device (one cooperative launch)"},
        "overlap": head["overlap"],
        "sparse_kernel": head["sparse_kernel"],
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "how": "inputs of every call copied in from pinned host memory on a copy stream "
                       "ahead of use, every output copied back on another stream, inside the "
                       "timed graphs"},
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk.summary(),
        "tensor_tflops_select": round(select_flops(w) / (sel_ms * 1e-3) / 1e12, 1),
        "tensor_peak_tflops": tc_peak,
        "recall": {"what": "mean over (seq, KV head) of |pages in use & step t's exact top-k| / "
                           "|exact top-k|, steps 2..T, selections by dsa_select",
                   "reused_step1_mean": round(float(np.mean(rec_reused[1:])), 4),
                   "reused_step1_min": round(float(np.min(rec_reused[1:])), 4),
                   "anchor_every_8_mean": round(float(np.mean(rec_anchor8[1:])), 4)},
        "exact_step1_extra_us": round(exact_us, 2),
        "head_budget": {"what": "one budget of Hkv*kp pages per sequence shared by its KV heads "
                                "(dsa_dims.head_budget = 1); eager launches",
                        "select_pass_ms": round(hb_sel_ms, 4),
                        "sparse_step_us": round(hb_sp_us, 2),
                        "per_head_sparse_step_us": round(ph_sp_us, 2),
                        "pages_per_head_min": int(hb_cnt.min()),
                        "pages_per_head_max": int(hb_cnt.max())},
        "prefix_reuse": {"what": "sparse step with the prefix part of stable tokens reused from "
                                 "caches (dsa_dims.active); eager launches",
                         "all_active_us": round(losa_active_us, 2),
                         "all_stable_us": round(losa_stable_us, 2),
                         "per_head_sparse_step_us": round(ph_sp_us, 2)},
        "block_time_shape": {"what": "one layer, GEMM stand-in for the FFN (d_ff = 4 d_model, "
                                     "random bf16 weights, cuBLAS): selection pass as exact "
                                     "attention, attention share of a block and block speed-up "
                                     "of sparse over exact attention at every step; eager launches",
                             **shape},
    }
    line["configs"] = others
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line, ensure_ascii=False), flush=True)




def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="128k", choices=list(WORKLOAD_TEXT))
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default="8k,32k,batched,tiny",
                    help="other workloads timed the same way and reported under 'configs' "
                         "(comma list, or 'none')")
    ap.add_argument("--select-sms", type=int, default=56,
                    help="SMs the selection pass may hold in the block step (dsa_dims.sm_limit; "
                         "0 = all, one cooperative launch that holds the device).  56 gives "
                         "groups of 7 CTAs launched as clusters, so that the selection of the "
                         "next block runs beside the sparse steps (at 128K: 21.5 ms per step "
                         "against 21.7 with 64 SMs and 23.8 with 48)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        # the oracle needs no GPU and no process group: rank 0 runs, the others exit
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
