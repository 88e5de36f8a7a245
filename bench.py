#!/usr/bin/env python
"""Benchmark of the absorbed MLA decode on B200.

One step = one mla_decode_absorbed call (query absorption, split-KV attention over the
latent cache, log-sum-exp merge, W_UV) for the DeepSeek-V3-shaped workload: 32 sequences
of 4096 cached tokens, 128 heads, d_c = 512, d_hR = 64, bf16 storage, fp32 accumulation.
Inputs are resident in HBM when the timed region starts; L2 is flushed between steps,
outside the per-step events: a 256 MiB buffer is written, then another 256 MiB buffer is
read, so L2 holds none of the step's inputs and no dirty line of the flush is written back
inside the next step (the write-only flush is timed too and reported beside it).

Prints ONE JSON line (rank 0).  `--impl reference` times the float64 CPU oracle instead.
Multi-GPU (torchrun): every rank decodes its own batch (weak scaling, no collective on the
data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
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

import workloads  # noqa: E402

METRIC = "MLA decode tokens/s + latent-cache GB/s, % roofline (H=128,d_c=512,ctx 4k)"
WORKLOAD = "v3_decode_b32_ctx4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FLUSH_BYTES = 256 << 20


class L2Flush:
    """Evicts the step's data from L2 between steps.  The write (256 MiB, twice the L2) leaves
    L2 full of dirty lines, which the next step would write back to HBM while it reads its
    own data; the read of a second 256 MiB buffer that follows displaces them, so the lines
    left in L2 are clean.  `clean=False` is the write alone."""

    def __init__(self, dev, clean: bool = True):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if clean else None

    def __call__(self):
        self.w.zero_()
        if self.r is not None:
            torch.sum(self.r)


# ------------------------------------------------------------------ arithmetic

def alg_step(w: workloads.Workload) -> dict:
    """Bytes the method must move and flops it must do for one decode step."""
    L = workloads.lengths(w)
    tokens = int(L.sum())
    e = 2  # bf16
    cache = tokens * w.row * e
    weights = 2 * w.H * w.qk_nope * w.d_c * e            # W_UK and W_UV (qk_nope = v_head)
    q = w.B * w.H * (w.qk_nope + w.d_hR) * e
    out = w.B * w.H * w.v_head * e
    flops_attn = tokens * w.H * (2 * w.row + 2 * w.d_c)    # scores over 576 + P.c over 512
    flops_proj = 2 * w.B * w.H * w.qk_nope * w.d_c * 2     # absorption and W_UV
    return {"bytes": cache + weights + q + out, "cache_bytes": cache, "flops": flops_attn + flops_proj,
            "attn_flops": flops_attn, "tokens": tokens}


FP8_ROW_BYTES = 656   # E4M3 codes (512) + bf16 rotary key (128) + fp32 scale (4) + padding (12)


def alg_step_fp8(w: workloads.Workload) -> dict:
    """alg_step over FP8 cache rows: 656 bytes per token instead of 1152."""
    a = alg_step(w)
    cache = a["tokens"] * FP8_ROW_BYTES
    a["bytes"] += cache - a["cache_bytes"]
    a["cache_bytes"] = cache
    return a


def alg_multi(w: workloads.Workload) -> dict:
    """Bytes and flops of one multi-token decode step: each sequence's L + q_len rows read
    once, new token t attending to the first L + t + 1 of them."""
    L = workloads.lengths(w)
    rows = int((L + w.q_len).sum())
    e = 2
    cache = rows * w.row * e
    weights = 2 * w.H * w.qk_nope * w.d_c * e
    n = w.B * w.q_len
    q = n * w.H * (w.qk_nope + w.d_hR) * e
    out = n * w.H * w.v_head * e
    attended = int(sum(int(l) + t + 1 for l in L for t in range(w.q_len)))
    flops_attn = attended * w.H * (2 * w.row + 2 * w.d_c)
    flops_proj = 2 * n * w.H * w.qk_nope * w.d_c * 2
    return {"bytes": cache + weights + q + out, "cache_bytes": cache, "flops": flops_attn + flops_proj,
            "attn_flops": flops_attn, "tokens": rows}


def paged_layout(w, inp, seed):
    """The contiguous rows of `inp` laid out in 64-token pages of a shuffled page pool:
    (pages [n_pages, 64, row], block_table int32 [B, max_blocks], seq_lens int32 [B])."""
    offs = inp["offsets"].numpy().astype(np.int64)
    L = offs[1:] - offs[:-1]
    npg = (L + 63) // 64
    max_blocks = max(int(npg.max()), 1)
    total = int(npg.sum())
    perm = np.random.default_rng(seed).permutation(total)
    pages = torch.zeros(total, 64, w.row, dtype=inp["cache"].dtype)
    table = np.zeros((w.B, max_blocks), dtype=np.int32)
    k = 0
    for b in range(w.B):
        for j in range(int(npg[b])):
            p = int(perm[k])
            k += 1
            table[b, j] = p
            n = int(min(64, L[b] - 64 * j))
            pages[p, :n] = inp["cache"][offs[b] + 64 * j: offs[b] + 64 * j + n]
    return pages, torch.from_numpy(table), torch.from_numpy(L.astype(np.int32))


def alg_layer(w: workloads.Workload) -> dict:
    """Bytes and flops of one full decode-layer step: append the new token, project the
    query, absorbed attention over L + 1 rows, W_UV, W_O.  The same figures serve the folded
    weights: they are the method's, and the folded products only add to what is moved."""
    L = workloads.lengths(w) + 1
    tokens = int(L.sum())
    e = 2 if w.dtype == "bf16" else 4
    qh = w.qk_nope + w.d_hR
    w_bytes = (w.row * w.d_model + w.H * qh * w.d_model + w.d_model * w.H * w.v_head
               + 2 * w.H * w.qk_nope * w.d_c) * e
    act = (w.B * w.d_model * 2 + w.B * w.row) * e
    flops = (2 * w.B * w.d_model * (w.row + w.H * qh) + tokens * w.H * (2 * w.row + 2 * w.d_c)
             + 4 * w.B * w.H * w.qk_nope * w.d_c + 2 * w.B * w.H * w.v_head * w.d_model)
    return {"bytes": tokens * w.row * e + w_bytes + act, "flops": flops, "tokens": w.B}


def alg_prefill(w: workloads.Workload) -> dict:
    """Bytes and flops of one causal prefill step (K/V materialised)."""
    n = w.B * w.ctx
    e = 2
    qh = w.qk_nope + w.d_hR
    w_bytes = (w.row * w.d_model + w.H * qh * w.d_model + 2 * w.H * w.qk_nope * w.d_c) * e
    io = (n * w.d_model + n * w.row + n * w.H * w.v_head) * e
    causal_pairs = w.B * w.ctx * (w.ctx + 1) // 2
    flops = (2 * n * w.d_model * (w.row + w.H * qh) + 2 * n * w.d_c * w.H * (w.qk_nope + w.v_head)
             + causal_pairs * w.H * 2 * (qh + w.v_head))
    return {"bytes": w_bytes + io, "flops": flops, "tokens": n}


def alg_kernel_bytes(name: str, w: workloads.Workload) -> int:
    """Algorithmic bytes of one launch of the kernel that dominates the step: the cache rows
    it attends over (1152 B per token, or 656 B for FP8 rows) plus the queries it reads."""
    L = workloads.lengths(w)
    cache = int(L.sum()) * (FP8_ROW_BYTES if name.endswith("_fp8") else w.row * 2)
    if name.startswith("tc_"):
        return cache + w.B * w.H * w.row * 2
    return cache + w.B * w.H * (w.d_c * 4 + w.d_hR * 2)


def alg_kernel_flops(name: str, w: workloads.Workload) -> int:
    """Algorithmic flops of one launch of the attention kernel: per attended token and head,
    2 x (d_c + d_hR) for the score and 2 x d_c for P c."""
    tokens = int(workloads.lengths(w).sum())
    return tokens * w.H * (2 * w.row + 2 * w.d_c)


def peaks() -> tuple:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0), "fallback"


def traffic_for(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source has not
    changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d["sha256"]:
        return None
    return d["bytes_per_launch"]


# ---------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        inside = [p for t, p in self.samples if t0 <= t <= t1]
        used = inside or [p for _, p in self.samples]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for p in used for n, v in zip(names, p[5:9]) if v.lower() == "active"})
        sm = [float(p[1]) for p in used if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for p in used if p[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(used), "samples_in_timed_region": len(inside)}


# ----------------------------------------------------------------- distributed

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


def rank_workload(w: workloads.Workload, rank: int) -> workloads.Workload:
    """Each rank decodes its own batch of the same shape (its own seed)."""
    return w if rank == 0 else workloads.shrink(w, seed=w.seed + 1000 * rank)


# ------------------------------------------------------------------ CPU oracle

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def time_oracle_units(w: workloads.Workload, inp: dict, budget_s: float, min_units: int = 2,
                      max_units: int = 10 ** 6, tokens: int = 0, threads: int = 1):
    """Run the float64 naive oracle on seeded (b, h) units until `budget_s` of wall time is
    spent, on `threads` host threads (the oracle's C routine runs outside the interpreter
    lock, one unit per thread at a time).  With tokens > 0 each unit attends over only its
    first `tokens` rows; the naive cost is linear in the rows attended, so a unit's time
    scales by (rows of the unit / tokens).  Throughput = units done / wall time, scaled to
    the full step of B x H units."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    offs = inp["offsets"].numpy().astype(np.int64)
    rng = np.random.default_rng(0)
    units = [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(min(max_units, 1 << 16))]
    lib = oracle.load()
    lock = threading.Lock()
    state = {"next": 0, "done": 0, "scaled": 0.0, "busy": 0.0}
    t_start = time.perf_counter()

    def worker():
        while True:
            with lock:
                i = state["next"]
                over = time.perf_counter() - t_start >= budget_s and i >= min_units
                if i >= len(units) or i >= max_units or over:
                    return
                state["next"] = i + 1
            b, h = units[i]
            T = int(offs[b + 1] - offs[b])
            n = T if tokens <= 0 else max(1, min(T, tokens))
            rows = inp["cache"][offs[b]:offs[b] + n]
            t = time.perf_counter()
            oracle.attend(inp["q_nope"][b, h], inp["q_rope"][b, h], rows, inp["W_UK"][h], inp["W_UV"][h],
                          w.scale, absorbed=False, lib=lib)
            dt = time.perf_counter() - t
            with lock:
                state["done"] += 1
                state["scaled"] += T / n
                state["busy"] += dt

    with ThreadPoolExecutor(max_workers=threads) as ex:
        for f in [ex.submit(worker) for _ in range(threads)]:
            f.result()
    wall = time.perf_counter() - t_start
    done = state["done"]
    # full-row units per second of wall time, over all threads
    rate = state["scaled"] / wall
    step_s = w.B * w.H / rate
    what = "all rows" if tokens <= 0 else f"its first {tokens} rows (time scaled to all rows)"
    return {"value": w.B / step_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} seeded (sequence, head) units of {w.name}, each over {what}, through the naive "
                      f"float64 oracle (K and V materialised) on {threads} host thread(s) for {wall:.1f} s; "
                      f"the full step ({w.B * w.H} units) extrapolated from the units per second",
            "step_s_extrapolated": step_s, "unit_s_mean": state["busy"] / max(done, 1)}


# ------------------------------------------------------------------------ arms

def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = workloads.make_inputs(w)
    import oracle
    oracle.load()
    # calibrate: rows per second of the naive oracle, then size each step's sample so the
    # whole run (warm-up + timed) takes about args.reference_seconds
    cores = host_cores()
    cal = time_oracle_units(w, inp, 0.0, min_units=2, max_units=2, tokens=256)
    rows_per_s = 256.0 / cal["unit_s_mean"]   # rows per second of one thread
    per_step = args.reference_seconds / (args.steps + args.warmup)
    # each step is one unit per host thread, over the first `tokens` rows of its sequence
    tokens = int(max(16, min(w.ctx or 10 ** 9, per_step * rows_per_s)))
    time_oracle_units(w, inp, 0.0, min_units=cores * args.warmup, max_units=cores * args.warmup, tokens=tokens,
                      threads=cores)
    r = time_oracle_units(w, inp, 0.0, min_units=cores * args.steps, max_units=cores * args.steps, tokens=tokens,
                          threads=cores)
    line = {"impl": "reference", "metric": METRIC, "value": r["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["step_s_extrapolated"] * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": r["value"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, world):
    return {"workload": w.name, "B_per_gpu": w.B, "ctx": w.ctx, "H": w.H, "d_c": w.d_c, "d_hR": w.d_hR,
            "qk_nope": w.qk_nope, "v_head": w.v_head, "global_batch": w.B * world,
            "parallelism": f"replicas{world}",
            "l2": "flushed between steps, outside the step events: 256 MiB written, then another 256 MiB read "
                  "(no dirty flush line is written back inside a step); ms_per_step_write_only_flush is the "
                  "same step after the write alone",
            **({"q_len": w.q_len} if w.kind == "decode_multi" else {})}


def build_step(w, inp, dev, mla):
    """Device inputs, the library call of one step, and what an end-to-end step copies."""
    g = {k: v.to(dev) for k, v in inp.items()}
    dims = mla.make_dims(w.H, w.d_model, w.d_c, w.d_hR, w.qk_nope, w.v_head, w.dtype)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if w.kind == "decode_attn":
        weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
        out = torch.empty(w.B, w.H, w.v_head, dtype=dt, device=dev)
        ws = mla.workspace(mla.mla_decode_workspace_size(dims, w.B), dev)

        def step():
            mla.mla_decode_absorbed(dims, weights, g["cache"], g["offsets"], out, ws, q_nope=g["q_nope"],
                                    q_rope=g["q_rope"])
        h2d = [("q_nope", inp["q_nope"]), ("q_rope", inp["q_rope"])]
        return g, dims, weights, out, step, h2d, alg_step(w), w.B
    if w.kind == "decode_fp8":
        weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
        out = torch.empty(w.B, w.H, w.v_head, dtype=dt, device=dev)
        ws = mla.workspace(mla.mla_decode_workspace_size(dims, w.B), dev)
        # the cache in FP8 rows, quantised once before the timed steps
        cache8 = torch.empty(g["cache"].shape[0], mla.mla_fp8_row_bytes(dims), dtype=torch.uint8, device=dev)
        mla.mla_quantize_cache_fp8(dims, g["cache"], cache8)
        del g["cache"]

        def step():
            mla.mla_decode_absorbed_fp8(dims, weights, cache8, g["offsets"], out, ws, g["q_nope"], g["q_rope"])
        h2d = [("q_nope", inp["q_nope"]), ("q_rope", inp["q_rope"])]
        return g, dims, weights, out, step, h2d, alg_step_fp8(w), w.B
    if w.kind == "decode_multi":
        weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
        out = torch.empty(w.B, w.q_len, w.H, w.v_head, dtype=dt, device=dev)
        pages, table, lens = paged_layout(w, inp, w.seed)
        pages, table, lens = pages.to(dev), table.to(dev), lens.to(dev)
        del g["cache"]   # the pages hold the rows
        ws = mla.workspace(mla.mla_decode_multi_workspace_size(dims, w.B, w.q_len, table.shape[1]), dev)

        def step():
            mla.mla_decode_absorbed_paged_multi(dims, weights, pages, table, lens, out, ws, q_nope=g["q_nope"],
                                                q_rope=g["q_rope"])
        h2d = [("q_nope", inp["q_nope"]), ("q_rope", inp["q_rope"])]
        return g, dims, weights, out, step, h2d, alg_multi(w), w.B * w.q_len
    if w.kind == "decode_layer":
        weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"], g["W_Q"], g["W_O"], fold=w.fold)
        out = torch.empty(w.B, w.d_model, dtype=dt, device=dev)
        ws = mla.workspace(mla.mla_decode_workspace_size(dims, w.B), dev)
        L = workloads.lengths(w)
        offs = inp["offsets"].numpy().astype(np.int64)
        q_pos = torch.from_numpy(L.astype(np.int32)).to(dev)
        slot = torch.from_numpy(offs[:-1] + L).to(dev)
        if w.history == "hidden":   # small fp32 layer: build the history by appending
            cache = torch.zeros(int(offs[-1]), w.row, dtype=dt, device=dev)
            pos = np.tile(np.arange(w.ctx), w.B).astype(np.int32)
            hs = (offs[:-1, None] + np.arange(w.ctx)[None]).reshape(-1)
            mla.mla_append_cache(dims, g["h_hist"].reshape(-1, w.d_model), g["W_DKV"], g["W_KR"],
                                 torch.from_numpy(pos).to(dev), torch.from_numpy(hs).to(dev), cache)
        else:
            cache = g["cache"]

        def step():   # append the new token at position L, then decode it over L + 1 rows
            mla.mla_append_cache(dims, g["h_new"], g["W_DKV"], g["W_KR"], q_pos, slot, cache)
            mla.mla_decode_absorbed(dims, weights, cache, g["offsets"], out, ws, h=g["h_new"], q_pos=q_pos)
        return g, dims, weights, out, step, [("h_new", inp["h_new"])], alg_layer(w), w.B
    # prefill
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"], g["W_Q"])
    cache = torch.zeros(w.B * w.ctx, w.row, dtype=dt, device=dev)
    out = torch.empty(w.B, w.ctx, w.H, w.v_head, dtype=dt, device=dev)
    ws = mla.workspace(mla.mla_prefill_workspace_size(dims, w.B, w.ctx), dev)

    def step():
        mla.mla_prefill_causal(dims, weights, g["h"], g["W_DKV"], g["W_KR"], cache, out, ws)
    return g, dims, weights, out, step, [("h", inp["h"])], alg_prefill(w), w.B * w.ctx


def run_ours(args, w0):
    world, rank, local = dist_init()
    import compressed_kv_cache_absorbed_b200 as mla
    w = rank_workload(w0, rank)
    inp = workloads.make_inputs(w)
    dev = torch.device("cuda", local)
    g, dims, weights, out, step, h2d, a, units = build_step(w, inp, dev, mla)
    flush = L2Flush(dev)
    flush_w = L2Flush(dev, clean=False)
    stream = torch.cuda.current_stream()

    # warm-up
    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    st, det = mla.mla_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} ({det}) during warm-up")

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    time.sleep(0.3 if clocks else 0)

    def timed_pass(profile: bool, fl=flush):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        if profile:
            mla.mla_profile_report(reset=True)
            mla.mla_profile_enable(True)
        barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        for i in range(args.steps):
            fl()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t1 = time.time()
        barrier()
        prof = None
        if profile:
            mla.mla_profile_enable(False)
            prof = mla.mla_profile_report(reset=True)
        return [a_.elapsed_time(b_) for a_, b_ in ev], prof, t0, t1

    # timed region: per-step CUDA events, the L2 flush between them (outside the events);
    # the library's kernels chain with programmatic dependent launch.  The step time is the
    # median of the per-step events (p10 / p90 reported beside it), max over ranks.
    step_ms, _, t0, t1 = timed_pass(False)
    ms = max_over_ranks(float(np.median(step_ms)))
    pct = {"p10": max_over_ranks(float(np.percentile(step_ms, 10))),
           "p90": max_over_ranks(float(np.percentile(step_ms, 90))),
           "mean": max_over_ranks(float(np.mean(step_ms)))}
    # second timed pass: CUDA events around every library launch on its stream give each
    # kernel's live launch duration (events between launches stop the kernels from
    # overlapping, so this pass is slower than the first)
    prof_ms, prof, _, _ = timed_pass(True)
    # the same steps after the write-only flush (its dirty lines are written back in the step)
    wo_ms, _, _, _ = timed_pass(False, flush_w)
    ms_wo = max_over_ranks(float(np.median(wo_ms)))
    ms_prof = max_over_ranks(float(np.median(prof_ms)))
    clk = clocks.summary(t0, t1) if clocks else None
    if clocks:
        clocks.stop()

    # end to end with host buffers: every step copies its inputs from pinned host memory and
    # its output back.  The decode workloads go through the C-ABI call that takes host
    # buffers (mla_decode_absorbed_host: the copies run inside the call); the others copy
    # with torch around the device call.
    pinned = [(g[k], v.pin_memory()) for k, v in h2d]
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    if w.kind == "decode_attn":
        ws_h = mla.workspace(mla.mla_decode_workspace_size(dims, w.B), dev)
        qn_h, qr_h = pinned[0][1], pinned[1][1]

        def e2e_step():
            mla.mla_decode_absorbed_host(dims, weights, g["cache"], g["offsets"], qn_h, qr_h, out_h, ws_h)
    else:
        def e2e_step():
            for dst, src in pinned:
                dst.copy_(src, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
    ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps + args.warmup):
        flush()
        j = i - args.warmup
        if j >= 0:
            ev3[j][0].record(stream)
        e2e_step()
        if j >= 0:
            ev3[j][1].record(stream)
    torch.cuda.synchronize()
    e2e_all = [a_.elapsed_time(b_) for a_, b_ in ev3]
    e2e_ms = max_over_ranks(float(np.median(e2e_all)))
    e2e_pct = {"p10": max_over_ranks(float(np.percentile(e2e_all, 10))),
               "p90": max_over_ranks(float(np.percentile(e2e_all, 90)))}
    st, det = mla.mla_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} ({det})")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and w.kind == "decode_attn":
        cores = host_cores()
        one = time_oracle_units(w, inp, args.cpu_seconds / 4)
        cpu = time_oracle_units(w, inp, args.cpu_seconds, min_units=cores, threads=cores)
        cpu["single_core"] = {"value": one["value"], "unit": "tokens/s", "sample": one["sample"]}
        cpu["nproc"] = cores
        for k in ("step_s_extrapolated", "unit_s_mean"):
            cpu.pop(k, None)

    if rank == 0:
        pk, pk_kind = peaks()
        dom = max(prof, key=lambda k: prof[k][1])
        n_launch, dom_ms = prof[dom]
        launch_s = dom_ms / n_launch * 1e-3
        launches_per_step = sum(v[0] for v in prof.values()) / args.steps
        step_s = ms * 1e-3
        roof_s = max(a["bytes"] / (pk["hbm_gbs"] * 1e9), a["flops"] / (pk["bf16_tflops"] * 1e12))
        if w.kind == "decode_fp8":
            # FP8 rows halve the bytes: the attention kernel sits on the tensor side of the ridge
            kflops = alg_kernel_flops(dom, w)
            kbytes = alg_kernel_bytes(dom, w)
            tf = kflops / launch_s / 1e12
            roofline = {"kernel": dom, "bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                        "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"], "traffic": traffic_for(dom),
                        "alg_flops_per_launch": kflops, "launch_us": launch_s * 1e6,
                        "peak_source": f"{pk_kind} bf16_tflops (fp16 operands run at the bf16 rate)",
                        "hbm_side": {"alg_bytes_per_launch": kbytes, "achieved_gbs": kbytes / launch_s / 1e9,
                                     "frac": kbytes / launch_s / 1e9 / pk["hbm_gbs"]}}
            metric, unit = "MLA decode tokens/s over an FP8 latent cache (H=128,d_c=512,ctx 4k)", "tokens/s"
        elif w.kind == "decode_attn":
            kbytes = alg_kernel_bytes(dom, w)
            achieved = kbytes / launch_s / 1e9
            roofline = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": traffic_for(dom),
                        "alg_bytes_per_launch": kbytes, "launch_us": launch_s * 1e6,
                        "peak_source": f"{pk_kind} hbm_gbs"}
            # the absorbed decode sits next to the ridge point: report the tensor side too
            kflops = alg_kernel_flops(dom, w)
            tf = kflops / launch_s / 1e12
            roofline["tensor_side"] = {
                "alg_flops_per_launch": kflops, "achieved_tflops": tf, "peak": pk["bf16_tflops"],
                "frac": tf / pk["bf16_tflops"], "peak_sustained": pk["bf16_tflops_sustained"],
                "frac_sustained": tf / pk["bf16_tflops_sustained"],
                "intensity_flop_per_byte": kflops / kbytes,
                "ridge_flop_per_byte": pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)}
            metric, unit = METRIC, "tokens/s"
        else:
            # whole-step roofline: these steps chain several kernels of different bounds
            bound = "tensor" if a["flops"] / (pk["bf16_tflops"] * 1e12) > a["bytes"] / (pk["hbm_gbs"] * 1e9) else "hbm"
            achieved = a["flops"] / step_s / 1e12 if bound == "tensor" else a["bytes"] / step_s / 1e9
            peak = pk["bf16_tflops"] if bound == "tensor" else pk["hbm_gbs"]
            roofline = {"kernel": "step", "bound": bound, "achieved": achieved, "peak": peak,
                        "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": achieved / peak,
                        "traffic": None, "dominant_kernel": dom, "dominant_launch_us": launch_s * 1e6,
                        "peak_source": f"{pk_kind} " + ("bf16_tflops" if bound == "tensor" else "hbm_gbs")}
            metric = {"decode_layer": "MLA decode-layer tokens/s (append + q proj + absorbed attention + W_UV + W_O)",
                      "decode_multi": "MLA multi-token decode tokens/s (q_len new tokens per sequence, paged cache)",
                      "prefill": "MLA causal prefill tokens/s (K/V materialised)"}[w.kind]
            unit = "tokens/s"
        line = {
            "metric": metric, "value": world * units / step_s, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_step_stats": {"stat": "median of the per-step CUDA events", **pct},
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": config_of(w, world),
            "step_roofline": {"alg_bytes": a["bytes"], "alg_flops": a["flops"], "roofline_us": roof_s * 1e6,
                              "frac": roof_s / step_s, "tflops": a["flops"] / step_s / 1e12,
                              "peaks": f"{pk_kind}: hbm {pk['hbm_gbs']} GB/s, bf16 {pk['bf16_tflops']} TFLOP/s"},
            "roofline": roofline,
            "kernels": {k: {"launches": v[0], "avg_us": v[1] / v[0] * 1e3} for k, v in prof.items()},
            "ms_per_step_with_kernel_events": ms_prof,
            "ms_per_step_write_only_flush": ms_wo,
            "e2e": {"value": world * units / (e2e_ms * 1e-3), "unit": unit,
                    "h2d_bytes_per_step": int(sum(v.numel() * v.element_size() for _, v in h2d)),
                    "d2h_bytes_per_step": int(out.numel() * out.element_size()), "ms_per_step": e2e_ms,
                    "ms_p10": e2e_pct["p10"], "ms_p90": e2e_pct["p90"],
                    "api": "mla_decode_absorbed_host" if w.kind == "decode_attn" else "device call + torch copies",
                    "note": "latent cache and weights stay resident in HBM (decode state)"},
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "clocks": clk,
            "cpu_baseline": cpu,
            "decode_path": "tcgen05" if mla.mla_decode_path(dims) == 1 else "cuda-core",
        }
        if w.kind in ("decode_attn", "decode_fp8"):
            line["latent_cache_GBps"] = a["cache_bytes"] / step_s / 1e9
        print(json.dumps(line), flush=True)
    weights.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        if w.kind != "decode_attn":
            ap.error("the reference arm times the oracle on the decode workloads")
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
