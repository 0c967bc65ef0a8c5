"""Benchmark: routed-attention decode queries/s at 64K context on B200.

One step = one fused decode (chunk routing, group routing, gather, exact
attention) for a batch of independent 64K-token sequences with Qwen3-30B-A3B
attention shapes (32 query heads, 4 KV heads, head dim 128; chunk 128, group 16,
top-32 chunks + sink + local, top-4 groups). Inputs are seeded synthetic data
resident in HBM; the L2 cache is flushed between steps and only the decode
launches are inside the device-timed events.

  python bench.py [--gpus N --steps K --warmup W --batch B] [--impl reference]

Under torchrun each rank runs its own batch (weak scaling, no collective on the
data path); the reported time is the max over ranks. Rank 0 prints one JSON line.
``--impl reference`` times the CPU oracle on a bounded sample instead.
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
import types
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "routed-attn decode queries/s at 64K ctx; achieved HBM GB/s vs B200 peak"
UNIT = "queries/s"
W64 = synth.DECODE_64K
SWEEP = (4096, 8192, 16384, 32768, 65536)


# --------------------------------------------------------------------------- bytes


def decode_bytes(L: int, w=W64) -> int:
    """Algorithmic HBM bytes of one decode query (all KV heads) at context L.

    Candidate chunk summaries (nf-2 per KV head), group summaries of the routed
    chunks, K and V of the routed tokens, q in (bf16), out (fp32) and lse (fp32).
    """
    C, g, d, hkv, hq = w.chunk, w.group, w.head_dim, w.n_kv_heads, w.n_q_heads
    nf = L // C
    if nf <= 2:
        S, cand, r = L, 0, 0
    else:
        cand = nf - 2
        r = min(w.top_chunks, cand)
        S = C + r * w.top_groups * g + (L - (nf - 1) * C)
    gpc = C // g
    return (cand * hkv * d * 2 + (r * gpc * hkv * d * 2 if w.top_groups < gpc else 0)
            + S * hkv * d * 2 * 2 + hq * d * 2 + hq * d * 4 + hq * 4)


DECODE_SOURCES = ("hga_common.cuh", "hga_attention.cuh", "hga_routed.cuh", "hga_decode.cuh")
PREFILL_SOURCES = ("hga_common.cuh", "hga_tcgen05.cuh", "hga_prefill_attn.cuh")
HISA_SOURCES = DECODE_SOURCES + ("hga_hisa.cuh",)


HISA_TOKENS = 2048  # tokens kept by the block-then-token decode (below the 2304 the two-level route keeps)


def hisa_bytes(L: int, k_tok: int = HISA_TOKENS, w=W64, reread: bool = False, logits: bool = False) -> int:
    """Algorithmic HBM bytes of one block-then-token decode query (all KV heads): candidate chunk
    summaries, K of every candidate token (the token step scores them; that covers the kept tokens' K),
    V of the kept tokens (K and V when every candidate is kept, the token step then being skipped), q,
    out and lse. What the kernels move beyond that: reread=True (hga_decode_hisa) adds the kept tokens'
    K a second time in the attention phase; logits=True (hga_decode_hisa_ws) adds the workspace
    traffic instead, the token step writing 8 fp32 logits per candidate and the attention reading
    those of the kept tokens."""
    C, d, hkv, hq = w.chunk, w.head_dim, w.n_kv_heads, w.n_q_heads
    nf = L // C
    if nf <= 2:
        cand, n_ct = 0, L
    else:
        cand = nf - 2
        n_ct = C + min(w.top_chunks, cand) * C + (L - (nf - 1) * C)
    kept = min(k_tok, n_ct)
    scored_k = n_ct if n_ct > k_tok else 0
    kept_rows = kept * (1 if scored_k else 2) + (kept if (scored_k and reread) else 0)
    lg = (scored_k + kept) * hkv * 8 * 4 if (scored_k and logits) else 0
    return (cand * hkv * d * 2 + scored_k * hkv * d * 2 + kept_rows * hkv * d * 2
            + hq * d * 2 + hq * d * 4 + hq * 4 + lg)


def kernel_source_hash(names=DECODE_SOURCES) -> str:
    """sha256 (first 16 hex) of the device-code files one kernel is built from."""
    import hashlib

    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "hierarchical_routed_sparse_build_b200", "csrc", n), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile="decode_64k_decode_kernel", names=DECODE_SOURCES):
    """DRAM bytes per launch from a committed ncu record (profiles/<profile>.json), if it was taken on the
    current sources (its source_hash equals kernel_source_hash(names)); None otherwise."""
    try:
        with open(os.path.join(ROOT, "profiles", profile + ".json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != kernel_source_hash(names):
        return None
    return int(rec["traffic_bytes_per_launch"])


def bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def prefill_flops(routed_total: int, n_pairs: int, w=synth.PREFILL_64K) -> int:
    """Useful QK^T + PV flops of one prefill: every (query, head) against its routed keys and
    its own causal prefix inside the block. routed_total = sum of routed counts over the
    n_pairs (block, KV head) pairs."""
    R = w.n_q_heads // w.n_kv_heads
    keys = w.block * routed_total + n_pairs * (w.block * (w.block + 1) // 2)
    return 4 * w.head_dim * R * keys


def run_prefill(dev, steps: int, warmup: int, cpu_seconds: float | None = None):
    """Time hga_prefill on the 2048-new-token, 63488-token-cache workload."""
    import torch

    import hierarchical_routed_sparse_build_b200 as hga

    w = synth.PREFILL_64K
    inp = synth.prefill_inputs(w)
    L0, T = inp.cache_len, w.n_new
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    k, v, q = dv(inp.k), dv(inp.v), dv(inp.q)
    lens = torch.tensor([L0], dtype=torch.int32, device=dev)
    kv = hga.make_kv(k, v, lens, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, max_len=k.shape[2], batch=1)
    p = hga.make_params(w.chunk, w.group, w.top_chunks, w.top_groups)
    nc = k.shape[2] // w.chunk
    cs = torch.zeros((1, w.n_kv_heads, nc, w.head_dim), dtype=torch.bfloat16, device=dev)
    gs = torch.zeros((1, w.n_kv_heads, nc, w.chunk // w.group, w.head_dim), dtype=torch.bfloat16, device=dev)
    hga.hga_build_summaries(kv, p, cs, gs)
    wsb = hga.hga_prefill_workspace_size(kv, w.n_q_heads, T, w.block, L0, p)
    ws = torch.zeros(wsb // 4, dtype=torch.int32, device=dev)
    nb = T // w.block
    # the workspace holds [blocks][KV heads][stride] routed positions, then one count per list
    stride = wsb // (4 * nb * w.n_kv_heads) - 1
    idx = ws[: nb * w.n_kv_heads * stride].view(nb, w.n_kv_heads, stride)
    n_idx = ws[nb * w.n_kv_heads * stride: nb * w.n_kv_heads * (stride + 1)].view(nb, w.n_kv_heads)
    out = torch.empty((T, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            flush.max()
            st[i].record(stream)
            fn()
            en[i].record(stream)
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in zip(st, en)])

    full = timed(lambda: hga.hga_prefill(q, w.n_q_heads, T, w.block, kv, L0, cs, gs, p, out, ws, wsb), steps)
    route = timed(lambda: hga.hga_route_blocks(q, w.n_q_heads, T, w.block, kv, L0, cs, gs, p, idx, stride,
                                               n_idx), steps)
    attend = timed(lambda: hga.hga_prefill_attend(q, w.n_q_heads, T, w.block, kv, L0, idx, stride, n_idx, p,
                                                  out), steps)
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in prefill: {bits}")
    fl = prefill_flops(int(n_idx.sum().item()), nb * w.n_kv_heads)
    burst, sustained, kind = bf16_peak()
    attn_tf = fl / (attend * 1e-3) / 1e12

    # growing history: block b routes over [0, 63488 + 64 b), earlier new blocks included
    gwsb = hga.hga_prefill_growing_workspace_size(kv, w.n_q_heads, T, w.block, L0, p)
    gws = torch.zeros(gwsb // 4, dtype=torch.int32, device=dev)
    gstride = gwsb // (4 * nb * w.n_kv_heads) - 1
    grow = timed(lambda: hga.hga_prefill_growing(q, w.n_q_heads, T, w.block, kv, L0, cs, gs, p, out, gws, gwsb),
                 steps)
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in growing prefill: {bits}")
    g_routed = int(gws[nb * w.n_kv_heads * gstride: nb * w.n_kv_heads * (gstride + 1)].sum().item())
    gfl = prefill_flops(g_routed, nb * w.n_kv_heads)
    return {
        "workload": "prefill_2048_on_63488: 2048 new tokens in 32 blocks of 64 on a 63488-token cache, 32 q / "
                    "4 KV heads, d 128, block-shared routing (C 128, g 16, top-32 + sink + local, top-4 groups) "
                    "+ own causal block (2304 routed keys + the causal prefix of the block per query); flops count "
                    "the useful QK^T and PV products",
        "tokens_per_s": round(T / (full * 1e-3), 1), "ms_per_step": round(full, 4),
        "route_ms": round(route, 4), "attend_ms": round(attend, 4),
        "flops_per_step": fl, "tflops_step": round(fl / (full * 1e-3) / 1e12, 1),
        "roofline": {"bound": "tensor", "kernel": "prefill_attn_kernel (tcgen05, TMEM accumulators)",
                     "achieved": round(attn_tf, 1), "peak": burst, "peak_kind": f"{kind} bf16 burst",
                     "unit": "TFLOP/s", "frac": round(attn_tf / burst, 4),
                     "frac_of_sustained": round(attn_tf / sustained, 4),
                     "traffic": profiled_traffic("prefill_64k_attn_kernel", PREFILL_SOURCES)},
        **({"cpu_baseline": oracle_prefill_baseline(inp, w, cpu_seconds)} if cpu_seconds else {}),
        "growing_history": {"what": "hga_prefill_growing: block b routes over its whole history "
                                    "[0, 63488 + 64 b), earlier blocks of the call included",
                            "ms_per_step": round(grow, 4), "tokens_per_s": round(T / (grow * 1e-3), 1),
                            "flops_per_step": gfl, "tflops_step": round(gfl / (grow * 1e-3) / 1e12, 1)},
    }


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle


def oracle_queries_per_s(inp, w, seconds: float, max_threads: int | None = None):
    """Time the oracle's decode (routing on prebuilt summaries + attention) on host cores."""
    import oracle

    R = w.n_q_heads // w.n_kv_heads
    B = len(inp.seq_lens)
    units = [(b, h) for b in range(min(B, 8)) for h in range(w.n_kv_heads)]
    prep = {}
    for (b, h) in units:
        L = int(inp.seq_lens[b])
        prep[(b, h)] = oracle.summaries(inp.k[b, h, :L], w.chunk, w.group)

    def one(u):
        b, h = u
        L = int(inp.seq_lens[b])
        cs, gs = prep[u]
        qh = inp.q[b, h * R:(h + 1) * R]
        tok = oracle.route(qh, cs, gs, L, w.chunk, w.group, w.top_chunks, w.top_groups)
        oracle.attend(qh, inp.k[b, h], inp.v[b, h], tok)

    threads = max_threads or os.cpu_count() or 1
    done = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        while time.perf_counter() - t0 < seconds:
            list(ex.map(one, units))
            done += len(units)
    dt = time.perf_counter() - t0
    queries = done / w.n_kv_heads
    return queries / dt, threads, f"{done} (sequence, KV head) decodes of 64K-token contexts " \
                                  f"({queries:.0f} queries) in {dt:.1f} s, summaries prebuilt"


def cpu_model() -> str:
    """The host CPU's model string (Linux /proc/cpuinfo), for the baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def oracle_rate(items, fn, seconds: float, threads: int | None = None):
    """Run fn over items (repeating the list) on host threads for about `seconds`;
    returns (items done per second, threads, items done, elapsed seconds)."""
    threads = threads or os.cpu_count() or 1
    done = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        while True:
            list(ex.map(fn, items))
            done += len(items)
            if time.perf_counter() - t0 >= seconds:
                break
    dt = time.perf_counter() - t0
    return done / dt, threads, done, dt


def oracle_decode_baseline(inp, w, seconds: float, contiguous=None) -> dict:
    """The oracle's decode (routing on prebuilt summaries, then attention) for every (sequence, KV head)
    of a decode input, on all host threads; queries/s (one query = all KV heads of one sequence)."""
    import oracle

    R = w.n_q_heads // w.n_kv_heads
    B = len(inp.seq_lens)
    prep = {}
    for b in range(B):
        L = int(inp.seq_lens[b])
        K, V = contiguous(b) if contiguous else (inp.k[b, :, :L], inp.v[b, :, :L])
        for h in range(w.n_kv_heads):
            Kh, Vh = np.ascontiguousarray(K[h]), np.ascontiguousarray(V[h])
            prep[(b, h)] = (Kh, Vh, oracle.summaries(Kh, w.chunk, w.group), L)

    def one(u):
        b, h = u
        Kh, Vh, (cs, gs), L = prep[u]
        qh = inp.q[b, h * R:(h + 1) * R]
        tok = oracle.route(qh, cs, gs, L, w.chunk, w.group, w.top_chunks, w.top_groups)
        oracle.attend(qh, Kh, Vh, tok)

    rate, threads, done, dt = oracle_rate(list(prep), one, seconds)
    return {"value": round(rate / w.n_kv_heads, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} (sequence, KV head) decodes of this input ({done / w.n_kv_heads:.0f} queries) in "
                      f"{dt:.1f} s, summaries prebuilt"}


def oracle_prefill_baseline(inp, w, seconds: float, pairs=((0, 0), (13, 1), (31, 3), (20, 2))) -> dict:
    """The oracle's prefill (block-max routing, then attention over the routed cache set plus the block's
    causal prefix) on a few (block, KV head) pairs of the same input; new tokens/s."""
    import oracle

    R = w.n_q_heads // w.n_kv_heads
    L0 = inp.cache_len
    sums = {h: oracle.summaries(np.ascontiguousarray(inp.k[0, h, :L0]), w.chunk, w.group) for h in range(w.n_kv_heads)}

    def one(pair):
        blk, h = pair
        qb = np.ascontiguousarray(inp.q[blk * w.block:(blk + 1) * w.block, h * R:(h + 1) * R])
        cs, gs = sums[h]
        tok = oracle.route(qb, cs, gs, L0, w.chunk, w.group, w.top_chunks, w.top_groups)
        oracle.prefill_block(qb, inp.k[0, h], inp.v[0, h], tok, P=L0 + w.block * blk)

    rate, threads, done, dt = oracle_rate(list(pairs), one, seconds)
    return {"value": round(rate * w.block / w.n_kv_heads, 1), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} (block of {w.block} queries, KV head) pairs of the 2048-on-63488 prefill in {dt:.1f} s "
                      "(summaries prebuilt); tokens/s = pairs/s x 64 / 4 KV heads"}


def cpu_baseline_record(inp, w, seconds: float, single_seconds: float = 3.0) -> dict:
    """The oracle on every host thread (the baseline value) and, on a short sample, on one thread."""
    v, cores, sample = oracle_queries_per_s(inp, w, seconds)
    v1, _, sample1 = oracle_queries_per_s(inp, w, single_seconds, max_threads=1)
    return {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model(), "single_thread": {"value": round(v1, 3), "unit": UNIT, "sample": sample1}}


# --------------------------------------------------------------------------- ranks


def max_over_ranks(x: float, dist, device) -> float:
    """Max of x over all ranks (device time of the slowest rank); x itself for one process."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: units every rank processed in every step over the slowest rank's time."""
    return units_per_rank * world * steps / (total_ms / 1e3)


# --------------------------------------------------------------------------- GPU arm


def run_summaries(hga, cache, timed, B: int, n: int = 5) -> dict:
    """Summary build over the whole cache (amortised over decode steps): K read once, chunk and group
    means written. Recorded as an error object if it fails."""
    try:
        times = timed(n, cache.build_summaries)
        st, bits = hga.hga_get_device_error()
        if st != 0:
            raise RuntimeError(f"device error bits {bits}")
        ms = statistics.median(times)
        w = W64
        nf = w.ctx_len // w.chunk
        per_head = w.ctx_len * w.head_dim * 2 + nf * w.head_dim * 2 * (1 + w.chunk // w.group)
        nbytes = B * w.n_kv_heads * per_head
        hbm, _ = peaks()
        return {"what": f"hga_build_summaries over {B} x 64K sequences (K read once; chunk and group means "
                        "written)", "us_per_call": round(ms * 1e3, 1), "alg_bytes": nbytes,
                "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)}
    except Exception as exc:  # recorded, so that the rest of the line is still printed
        return {"error": f"{type(exc).__name__}: {exc}"}


def run_paged_batch(hga, RoutedCache, dev, timed, n: int, cpu_seconds: float | None = None) -> dict:
    """The batched decode on a paged pool: 16 ragged sequences of 4K-64K tokens (seeded lengths), page =
    chunk = 128 tokens, shuffled page table, L2 flushed between steps. A failure here is recorded in the
    object rather than ending the run."""
    try:
        wp = synth.BATCHED_PAGED
        pin = synth.paged_inputs(wp)
        pc = RoutedCache(pin.k_pool, pin.v_pool, pin.seq_lens, chunk=wp.chunk, group=wp.group,
                         top_chunks=wp.top_chunks, top_groups=wp.top_groups, n_q_heads=wp.n_q_heads,
                         page_table=pin.page_table, device=dev)
        pc.build_summaries()
        pq = pc.q_tensor(pin.q)
        pout, plse = pc.out_buffers()
        for _ in range(3):
            pc.decode(pq, pout, plse)
        times = timed(n, lambda: pc.decode(pq, pout, plse))
        st, bits = hga.hga_get_device_error()
        if st != 0:
            raise RuntimeError(f"device error bits {bits}")
        step_ms = statistics.median(times)
        lens = [int(x) for x in pin.seq_lens]
        nbytes = sum(decode_bytes(L) for L in lens)
        hbm, _ = peaks()
        return {"what": "hga_decode on a paged pool: 16 sequences of seeded lengths in [4096, 65536], page = chunk = "
                        "128 tokens, shuffled page table",
                "lengths": {"min": min(lens), "max": max(lens), "total": sum(lens)},
                "us_per_step": round(step_ms * 1e3, 2), "queries_per_s": round(len(lens) / (step_ms * 1e-3)),
                "alg_bytes_per_step": nbytes, "GB_s": round(nbytes / (step_ms * 1e-3) / 1e9, 1),
                "frac_hbm": round(nbytes / (step_ms * 1e-3) / 1e9 / hbm, 4),
                **({"cpu_baseline": oracle_decode_baseline(pin, wp, cpu_seconds, contiguous=pin.contiguous)}
                   if cpu_seconds else {})}
    except Exception as exc:  # recorded, so that the rest of the line is still printed
        return {"error": f"{type(exc).__name__}: {exc}"}


def run_config(hga, RoutedCache, dev, timed, w, n: int, cpu_seconds: float | None) -> dict:
    """One decode configuration as its workload states it (batch 1), L2 flushed between steps, with the
    oracle timed on the same input beside it. A failure is recorded in the object."""
    try:
        inp = synth.decode_inputs(w)
        c = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=w.chunk, group=w.group, top_chunks=w.top_chunks,
                        top_groups=w.top_groups, n_q_heads=w.n_q_heads, device=dev)
        c.build_summaries()
        q = c.q_tensor(inp.q)
        out, lse = c.out_buffers()
        for _ in range(3):
            c.decode(q, out, lse)
        ms = statistics.median(timed(n, lambda: c.decode(q, out, lse)))
        st, bits = hga.hga_get_device_error()
        if st != 0:
            raise RuntimeError(f"device error bits {bits}")
        L = int(inp.seq_lens[0])
        nbytes = decode_bytes(L, w)
        hbm, _ = peaks()
        res = {"what": f"{w.name}: batch {len(inp.seq_lens)}, {w.n_q_heads} q / {w.n_kv_heads} KV heads, d {w.head_dim}, "
                       f"L {L}, chunk {w.chunk}, group {w.group}, top-{w.top_chunks} chunks + sink + local, "
                       f"top-{w.top_groups} groups; one fused decode launch per query",
               "us_per_query": round(ms * 1e3, 2), "queries_per_s": round(1.0 / (ms * 1e-3)),
               "alg_bytes_per_query": nbytes, "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 2),
               "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 5)}
        if cpu_seconds:
            res["cpu_baseline"] = oracle_decode_baseline(inp, w, cpu_seconds)
        return res
    except Exception as exc:  # recorded, so that the rest of the line is still printed
        return {"error": f"{type(exc).__name__}: {exc}"}


def run_gpu(args, rank: int, world: int, dist):
    import torch

    import hierarchical_routed_sparse_build_b200 as hga
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    if args.ctas:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, args.ctas)
    w = W64
    B = args.batch
    inp = synth.decode_inputs(w, lengths=[w.ctx_len] * B, replicas_of=min(B, args.distinct))
    cache = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=w.chunk, group=w.group, top_chunks=w.top_chunks,
                        top_groups=w.top_groups, n_q_heads=w.n_q_heads, device=dev)
    cache.build_summaries()
    q = cache.q_tensor(inp.q)
    out, lse = cache.out_buffers()
    stream = torch.cuda.current_stream()
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error after setup: {bits}")
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        cache.decode(q, out, lse)

    def timed(n, fn, per_step_flush=True):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            if per_step_flush:
                flush.max()
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        times = timed(args.steps, step)
        # keep sampling for at least a second of load
        t_end = time.time() + 1.0
        extra = 0
        while time.time() < t_end:
            timed(20, step)
            extra += 20
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in timed region: {bits}")
    total_ms = max_over_ranks(float(sum(times)), dist, dev)
    ms_per_step = total_ms / args.steps
    value = weak_scaling_rate(B, world, args.steps, total_ms)

    # end to end through the public API with host buffers: q copied in from pinned
    # host memory and out/lse copied back every step, double-buffered on a copy
    # stream so that step i+1's upload and step i's download run under decodes
    q_host = torch.from_numpy(inp.q.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    lse_host = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    q_dev = [torch.empty_like(q) for _ in range(2)]
    o_dev = [torch.empty_like(out) for _ in range(2)]
    l_dev = [torch.empty_like(lse) for _ in range(2)]
    copy = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    up_done, dec_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(n):
        """n end-to-end steps; returns their device time (ms) from the first upload to the last download."""
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.max()
        t_start.record(stream)
        copy.wait_event(t_start)
        with torch.cuda.stream(copy):
            q_dev[0].copy_(q_host, non_blocking=True)
            up_done[0].record(copy)
        for i in range(n):
            sl = i % 2
            if i + 1 < n:
                with torch.cuda.stream(copy):
                    if i >= 1:
                        copy.wait_event(dec_done[1 - sl])  # decode i-1 has read that q buffer
                    q_dev[1 - sl].copy_(q_host, non_blocking=True)
                    up_done[1 - sl].record(copy)
            stream.wait_event(up_done[sl])
            if i >= 2:
                stream.wait_event(down_done[sl])  # step i-2's outputs have left that buffer
            cache.decode(q_dev[sl], o_dev[sl], l_dev[sl])
            dec_done[sl].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(dec_done[sl])
                out_host[sl].copy_(o_dev[sl], non_blocking=True)
                lse_host[sl].copy_(l_dev[sl], non_blocking=True)
                down_done[sl].record(copy)
        stream.wait_stream(copy)
        t_end.record(stream)
        torch.cuda.synchronize()
        return t_start.elapsed_time(t_end)

    e2e_run(3)
    e2e_ms = max_over_ranks(e2e_run(args.steps), dist, dev)
    got = out_host[(args.steps - 1) % 2]
    if not torch.equal(got, out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-timed decode of the same queries")

    # batch-1 latency and the context-length sweep (same kernels, same cache)
    sweep = {}
    lens_saved = cache.seq_lens.clone()
    q1 = q[:1].contiguous()
    out1, lse1 = out[:1].contiguous(), lse[:1].contiguous()
    from hierarchical_routed_sparse_build_b200 import hga_decode, make_kv
    kv1 = make_kv(cache.k[:1], cache.v[:1], cache.seq_lens[:1], n_kv_heads=cache.n_kv_heads,
                  head_dim=cache.head_dim, max_len=cache.max_len, batch=1)
    cs1, gs1 = cache.chunk_sum[:1], cache.group_sum[:1]
    lat = timed(args.steps, lambda: hga_decode(q1, w.n_q_heads, kv1, cs1, gs1, cache.params, out1, lse1))
    hbm, peak_kind = peaks()
    cpu_s = args.cpu_point_seconds if (not args.no_cpu_baseline and world == 1) else None
    for L in SWEEP:
        cache.seq_lens.fill_(L)
        tl = timed(max(10, args.steps // 4), step)
        ms = statistics.median(tl)
        sweep[str(L)] = {"queries_per_s": round(B / (ms / 1e3)), "GB_s": round(B * decode_bytes(L) / (ms / 1e3) / 1e9, 1),
                         "frac_hbm": round(B * decode_bytes(L) / (ms / 1e3) / 1e9 / hbm, 4)}
        if cpu_s:
            # the same queries on the first two distinct sequences cut to length L
            sub = types.SimpleNamespace(q=inp.q[:2], k=inp.k[:2], v=inp.v[:2], seq_lens=np.full(2, L, np.int32))
            sweep[str(L)]["cpu_baseline"] = oracle_decode_baseline(sub, w, cpu_s)
    cache.seq_lens.copy_(lens_saved)
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in sweep: {bits}")

    # serving loop: append one token per sequence + fused decode, replayed from a CUDA
    # graph; the sequences start n_loop + warmup tokens short of 65536 and grow back to
    # it (the appended token is the query's own; its K/V overwrite the cache's last rows)
    n_loop = max(10, args.steps // 2)
    cache.seq_lens.fill_(w.ctx_len - n_loop - args.warmup)
    kn = torch.randn((B, w.n_kv_heads, w.head_dim), device=dev).to(torch.bfloat16)
    vn = torch.randn((B, w.n_kv_heads, w.head_dim), device=dev).to(torch.bfloat16)
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        cache.append(kn, vn)
        cache.decode(q, out, lse)
    for _ in range(args.warmup):
        graph.replay()
    loop_ms = timed(n_loop, graph.replay)
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the decode loop: {bits}")
    del graph
    cache.seq_lens.copy_(lens_saved)
    cache.build_summaries()
    loop_step = statistics.median(loop_ms)

    # block-then-token decode (HISA indexer variant) on the same cache: top-32 chunks,
    # then the top 2048 tokens of their 4352 candidates
    hisa_ms = timed(max(10, args.steps // 2),
                    lambda: cache.decode_hisa(q, HISA_TOKENS, out, lse))
    reread_ms = timed(max(10, args.steps // 2),
                      lambda: cache.decode_hisa(q, HISA_TOKENS, out, lse, logits_workspace=False))
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the block-then-token decode: {bits}")
    hisa_step = statistics.median(hisa_ms)
    reread_step = statistics.median(reread_ms)
    hbm_peak, _ = peaks()
    hisa = {"what": "hga_decode_hisa_ws: top-32 chunks by summary (plus first and last), then the top "
                    f"{HISA_TOKENS} of their tokens by the head-summed indexer score (the sum of per-head "
                    "logits the token step keeps in a workspace), exact attention over them reading only V; "
                    f"{B} x 64K sequences",
            "us_per_step": round(hisa_step * 1e3, 2), "queries_per_s": round(B / (hisa_step * 1e-3)),
            "alg_bytes_per_query": hisa_bytes(w.ctx_len),
            "moved_bytes_per_query": hisa_bytes(w.ctx_len, logits=True),
            "k_reread": {"what": "hga_decode_hisa (no workspace: the attention reads the kept tokens' K again)",
                         "us_per_step": round(reread_step * 1e3, 2),
                         "moved_bytes_per_query": hisa_bytes(w.ctx_len, reread=True)},
            "GB_s": round(B * hisa_bytes(w.ctx_len) / (hisa_step * 1e-3) / 1e9, 1),
            "frac_hbm": round(B * hisa_bytes(w.ctx_len) / (hisa_step * 1e-3) / 1e9 / hbm_peak, 4),
            "traffic": (lambda t: None if t is None else t * B // 64)(
                profiled_traffic("hisa_64k_hisa_decode_kernel", HISA_SOURCES))}

    # host-resident K/V (the pages' placement): 8 of the sequences in pinned, mapped host
    # memory, summaries in HBM; the decode kernel reads only the routed rows over the host link
    Bh = min(B, 8)
    kh = torch.from_numpy(inp.k[:Bh].view(np.int16)).view(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(inp.v[:Bh].view(np.int16)).view(torch.bfloat16).pin_memory()
    kvh = hga.make_kv(hga.hga_host_kv_pointer(kh), hga.hga_host_kv_pointer(vh), cache.seq_lens[:Bh],
                      n_kv_heads=cache.n_kv_heads, head_dim=cache.head_dim, max_len=cache.max_len, batch=Bh)
    qh, outh, lseh = q[:Bh].contiguous(), out[:Bh].contiguous(), lse[:Bh].contiguous()
    csh, gsh = cache.chunk_sum[:Bh], cache.group_sum[:Bh]
    host_ms = timed(max(5, args.steps // 10),
                    lambda: hga.hga_decode(qh, w.n_q_heads, kvh, csh, gsh, cache.params, outh, lseh))
    st, bits = hga.hga_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the host-resident decode: {bits}")
    host_step = statistics.median(host_ms)
    routed_kv = Bh * w.n_kv_heads * 2304 * 2 * w.head_dim * 2  # K and V rows read over the link
    host_kv = {"what": f"decode of {Bh} 64K sequences whose K/V live in pinned host memory "
                       "(hga_host_kv_pointer), summaries in HBM: only the routed rows cross the host link",
               "us_per_step": round(host_step * 1e3, 1), "queries_per_s": round(Bh / (host_step * 1e-3)),
               "link_GB_s": round(routed_kv / (host_step * 1e-3) / 1e9, 1),
               "routed_kv_bytes_per_step": routed_kv}
    del kh, vh
    decode_loop = {"what": "hga_append + hga_decode captured in one CUDA graph, replayed per step "
                           f"({n_loop} timed steps after {args.warmup}, lengths growing to {w.ctx_len}, "
                           "L2 flushed between steps)",
                   "us_per_step": round(loop_step * 1e3, 2), "queries_per_s": round(B / (loop_step * 1e-3)),
                   "gpu_launches_per_step": 3}

    alg = B * decode_bytes(w.ctx_len)
    mean_launch_s = statistics.mean(times) / 1e3
    achieved = alg / mean_launch_s / 1e9
    srt = sorted(times)
    pct = lambda p: srt[min(len(srt) - 1, int(round(p / 100 * (len(srt) - 1))))]
    prefill = None if args.no_prefill else run_prefill(dev, max(5, args.steps // 10), args.warmup, cpu_s)
    paged = run_paged_batch(hga, RoutedCache, dev, timed, max(10, args.steps // 2), cpu_s)
    configs = {w_.name: run_config(hga, RoutedCache, dev, timed, w_, max(10, args.steps // 2), cpu_s)
               for w_ in (synth.TINY_DECODE_4K, synth.DECODE_16K)}
    summaries = run_summaries(hga, cache, timed, B)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"decode_64k: {B} independent sequences x 65536-token bf16 K/V cache per GPU, "
                               "32 q heads / 4 KV heads / d 128, chunk 128, group 16, top-32 chunks + sink + "
                               "local, top-4 groups (2304 routed tokens per KV head, 3.5%)",
                   "batch_per_gpu": B, "ctx_len": w.ctx_len, "distinct_sequences": min(B, args.distinct),
                   "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
                   "l2": "flushed between steps (256 MiB read, outside the timed events)",
                   "ctas_per_head": args.ctas or "auto"},
        "roofline": {"bound": "hbm", "kernel": "decode_kernel<128> (fused routing + attention, one launch per step)",
                     "achieved": round(achieved, 1), "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4),
                     "traffic": args.traffic if args.traffic is not None else
                     (profiled_traffic() if B == 64 else None),
                     "alg_bytes_per_query": decode_bytes(w.ctx_len), "alg_bytes_per_launch": alg},
        "e2e": {"value": round(weak_scaling_rate(B, world, args.steps, e2e_ms), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(q_host.numel() * 2),
                "d2h_bytes_per_step": int(out_host[0].numel() * 4 + lse_host[0].numel() * 4),
                "how": "RoutedCache.decode per step; q uploaded from pinned host memory and out/lse downloaded "
                       "every step on a second stream, double-buffered (step i+1's upload and step i's download "
                       "overlap decode i); timed from the first upload to the last download"},
        "clocks": clocks.summary(),
        "gpu_launches": args.steps,
        "latency_ms": {"p50": round(pct(50), 5), "p95": round(pct(95), 5), "p99": round(pct(99), 5)},
        "batch1_latency_us": round(statistics.median(lat) * 1e3, 2),
        "sweep": sweep,
        "decode_loop_graph": decode_loop,
        "host_resident_kv": host_kv,
        "block_then_token": hisa,
        "paged_batch": paged,
        "configs": configs,
        "summaries": summaries,
        "prefill": prefill,
    }
    return res, inp, w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--batch", type=int, default=64, help="64K-token sequences per GPU")
    ap.add_argument("--distinct", type=int, default=8, help="distinct generated sequences (rest replicate)")
    ap.add_argument("--ctas", type=int, default=0, help="CTAs per (sequence, KV head); 0 = automatic")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--cpu-point-seconds", type=float, default=2.0,
                    help="oracle seconds beside each configuration, sweep point, the paged batch and prefill")
    ap.add_argument("--traffic", type=float, default=None, help="ncu dram bytes per launch, if measured")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill measurement")
    ap.add_argument("--prefill-only", action="store_true", help="time only the prefill workload (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.prefill_only:
        import torch

        print(json.dumps({"prefill": run_prefill(torch.device("cuda", 0), args.steps, args.warmup)}), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        w = W64
        inp = synth.decode_inputs(w, lengths=[w.ctx_len] * 8)
        per = []
        for _ in range(args.warmup):
            oracle_queries_per_s(inp, w, 0.5)
        for _ in range(args.steps):
            v, cores, sample = oracle_queries_per_s(inp, w, args.cpu_seconds / max(args.steps, 1))
            per.append(v)
        value = statistics.mean(per)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / value, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "decode_64k (same shapes and routing as our arm), CPU oracle on 8 sequences",
                       "batch_per_gpu": 8, "ctx_len": w.ctx_len},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        res, inp, w = run_gpu(args, rank, world, dist)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                res["cpu_baseline"] = cpu_baseline_record(inp, w, args.cpu_seconds)
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
