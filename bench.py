#!/usr/bin/env python
"""Benchmark of one MHA2MLA decode step over the latent KV cache.

A step is the serving-loop decode step for one batch: `mla_append` writes each
sequence's new token (latent c_kv + rotated RoPE key dims) at position L_b-1, then
`mla_decode` attends each sequence's new query over its L_b cached tokens (query
absorption, split-K latent attention, split merge + W_uv).  Metric: cached tokens per
second, sum_b L_b / step time.  Pair selection and SVDjoint run once at conversion
and are timed separately (`conversion_s`).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        python bench.py --impl reference ...   (the float64 CPU oracle, timed on host cores)
Multi-GPU (torchrun, one process per GPU): every rank runs an independent replica of
the workload (the path has no cross-sequence exchange); value = tokens of all ranks /
max-over-ranks time.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode cached tokens/s (batch×ctx per step) and % of B200 HBM peak"
UNIT = "cached tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
PER_WORKLOADS = ("llama2_7b_ragged_bf16", "llama2_7b_int4", "llama2_7b_int4_r128", "llama2_7b_int2")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama2_7b_bf16")
    ap.add_argument("--kernel", type=int, default=0,
                    help="decode kernel: 0 auto, 1 CUDA-core, 2 tcgen05 (token rows), 3 tcgen05 (head rows)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--separate-calls", action="store_true",
                    help="time the step as mla_append + mla_decode instead of one mla_decode_step")
    ap.add_argument("--prefill-only", action="store_true",
                    help="print only the chunked-prefill figure (64 queries per sequence) of the workload")
    ap.add_argument("--no-per-workload", dest="per_workload", action="store_false",
                    help="measure only --workload (default: also the ragged and int4 workloads at N=1)")
    return ap.parse_args()


def workload(name):
    from workloads import get
    try:
        return get(int(name))
    except ValueError:
        return get(name)


def wl_config(wl, lens):
    return {"workload": wl.name, "batch": wl.batch,
            "ctx": wl.ctx if wl.ctx is not None else f"ragged U[{wl.ctx_range[0]},{wl.ctx_range[1]}]",
            "cached_tokens_per_step": int(np.sum(lens)), "hidden": wl.hidden, "heads": wl.n_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "r_pairs": wl.r_pairs, "d_c": wl.d_c,
            "latent_cache": ("int4 g32 + fp16 scales" + (f", {wl.resid}-token bf16 residual window" if wl.resid else "")
                             if wl.cache == "int4_g32" else
                             "int2 g32 + fp16 scales" if wl.cache == "int2_g32" else wl.dtype),
            "step": "mla_decode_step: append of the B new tokens + decode of the B queries"}


# ------------------------------------------------------------------ oracle (CPU) timing
def oracle_decode_sample(wl, n_tokens, rounds, seconds_cap=None):
    """Time the float64 oracle's decode (unabsorbed form) of sequence 0's query over its
    first n_tokens cached tokens (all heads).  Weights come from the oracle's own
    conversion of a reduced-hidden copy of the layer: the decode cost does not depend on
    the hidden size (it reads the cache, W_uk and W_uv only)."""
    import oracle as O
    from workloads import generate as gen
    small = wl.with_(hidden=min(wl.hidden, 512), t_cal=256)
    w = gen.layer_weights(small)
    qc, kc = gen.calib_activations(small, w)
    conv = O.convert(w, qc, kc, small, cast=lambda a: gen.cast(a, small.dtype))
    theta = O.rope_theta(wl.head_dim, wl.rope_base)
    x = gen.context_tokens(small, 0, n_tokens)
    c, kr = O.append(x, np.arange(n_tokens), conv["W_dkv"], conv["W_krope"], conv["pair_idx"], theta)
    kr = gen.cast(kr, wl.dtype)
    quant = {"int4_g32": (O.quant_int4_g32, O.dequant_int4_g32),
             "int2_g32": (O.quant_int2_g32, O.dequant_int2_g32)}.get(wl.cache)
    if quant:
        codes, scales = quant[0](c)
        plain = gen.cast(c, wl.dtype)
    else:
        c = gen.cast(c, wl.dtype)
    q = gen.decode_queries(small, w)[0]
    times = []
    t_start = time.perf_counter()
    for _ in range(rounds):
        t0 = time.perf_counter()
        cc = quant[1](codes, scales) if quant else c
        if quant and wl.resid:
            cc = O.residual_window(cc, plain, wl.resid)
        O.decode_unabsorbed(q, cc, kr, conv["W_uk"], conv["W_uv"], conv["pair_idx"], theta)
        times.append(time.perf_counter() - t0)
        if seconds_cap and time.perf_counter() - t_start > seconds_cap:
            break
    return times


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(args.workload)
    from workloads import generate as gen
    lens = gen.seq_lens(wl)
    # size each step so the whole warmup+steps run stays within about two minutes
    probe_tokens = min(int(lens[0]), 512)
    t = statistics.median(oracle_decode_sample(wl, probe_tokens, 3))
    per_tok = t / probe_tokens
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_tok = int(max(16, min(int(lens[0]), budget / per_tok)))
    times = oracle_decode_sample(wl, n_tok, args.warmup + args.steps)
    timed = times[args.warmup:] or times
    step_s = statistics.mean(timed)
    value = n_tok / step_s
    sample = (f"oracle decode (float64, unabsorbed) of sequence 0's query over its first {n_tok} "
              f"cached tokens, all {wl.n_heads} heads, per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": len(timed), "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generators)", "config": wl_config(wl, lens),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU helpers
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def code_sha1(path):
    """SHA-1 of a C++/CUDA source with // comments and blank lines removed, so an edit of
    comments alone keeps the recorded counters valid while any code change voids them."""
    lines = []
    with open(path) as f:
        for line in f:
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha1("\n".join(lines).encode()).hexdigest()


def measured_traffic(workload_name, kernel_used):
    """DRAM bytes (read + write) per launch of the tensor-core attention kernel, from the
    committed ncu summary, when that summary was taken on this workload and on the current
    kernel code (else None: the counters no longer describe the kernel)."""
    files = {2: ("decode_tc_traffic.txt", "decode_tc.cu"), 3: ("attn_tc_traffic.txt", "chunk_tc.cu")}
    if kernel_used not in files:
        return None
    path = os.path.join(ROOT, "profiles", files[kernel_used][0])
    src = os.path.join(ROOT, "mha_mla_latent_b200", "csrc", files[kernel_used][1])
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.startswith("#"):
                    k, v = line.strip().split("=", 1)
                    kv[k] = v
        sha = code_sha1(src)
        if kv.get("source_sha1") != sha:
            return None
        if "traffic_bytes." + workload_name in kv:   # one capture per workload
            return int(kv["traffic_bytes." + workload_name])
        if kv.get("workload") != workload_name:
            return None
        return int(kv["traffic_bytes"])
    except (OSError, KeyError, ValueError):
        return None


def measured_peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return FALLBACK_BF16_TFLOPS


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s pool figure)"


def replica_aggregate(local_ms, tokens_per_rank, world, device):
    """Whole-job timing of N independent replicas: the slowest rank's time of the timed
    region (an all-reduce MAX over the process group when world > 1) and the job's value,
    tokens of all ranks / that time.  Every rank calls it at the same point."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    return max_ms, tokens_per_rank * world / (max_ms * 1e-3)


class Bench:
    """One workload set up on one GPU: the converted plan, cache replicas that together
    exceed twice the L2, the step's inputs, and the measurements of one step."""

    def __init__(self, name, dev, kernel=0, fused=True):
        import torch
        import mha_mla_latent_b200 as mla
        from mha_mla_latent_b200.cache import LatentCache, workspace
        from mha_mla_latent_b200.convert import convert_layer, plan_from_converted
        from workloads import generate as gen

        self.mla, self.torch = mla, torch
        self.fused = fused
        wl = self.wl = workload(name)
        self.dev = dev
        cfg = self.cfg = mla.config_from_workload(wl)
        lens = self.lens = gen.seq_lens(wl)
        B = wl.batch
        # ---- conversion (once): GPU pair selection + device SVD
        t0 = time.perf_counter()
        w = gen.layer_weights(wl)
        q_cal, k_cal = gen.calib_activations(wl, w)
        conv = convert_layer(cfg, gen.to_torch(w["W_k"], wl.dtype, dev), gen.to_torch(w["W_v"], wl.dtype, dev),
                             gen.to_torch(q_cal, wl.dtype, dev), gen.to_torch(k_cal, wl.dtype, dev))
        self.plan = plan = plan_from_converted(cfg, conv)
        torch.cuda.synchronize()
        self.conversion_s = time.perf_counter() - t0

        # ---- caches: enough replicas that consecutive steps never hit L2 from the previous one
        per_tok = mla.mla_cache_bytes_per_token(cfg)
        cache_bytes = int(np.sum(lens)) * per_tok
        if wl.resid:   # + the window's ring rows (dtype) and their position tags
            cache_bytes += int(np.sum(np.minimum(lens, wl.resid))) * (wl.d_c * 2 + 4)
        self.cache_bytes = cache_bytes
        self.n_rep = n_rep = max(1, -(-2 * L2_BYTES // cache_bytes))
        T_cap = int(lens.max())
        T_cap += T_cap % 2
        self.caches = caches = [LatentCache(cfg, B, T_cap, dev) for _ in range(n_rep)]
        t0 = time.perf_counter()
        chunk = 16384
        for b in range(B):
            L = int(lens[b])
            ctx = gen.context_tokens(wl, b, L - 1)
            for s in range(0, L - 1, chunk):
                e = min(L - 1, s + chunk)
                xt = gen.to_torch(ctx[s:e], wl.dtype, dev)
                mla.mla_append(plan, xt, torch.full((e - s,), b, dtype=torch.int32, device=dev),
                               torch.arange(s, e, dtype=torch.int32, device=dev), caches[0].struct)
        torch.cuda.synchronize()
        for c in caches[1:]:
            for name_ in ("c_kv", "c_scales", "k_rope", "c_resid", "resid_pos"):
                src, dst = getattr(caches[0], name_), getattr(c, name_)
                if src is not None:
                    dst.copy_(src)
        self.prefill_s = time.perf_counter() - t0
        assert mla.mla_device_error(plan) == 0

        # ---- step inputs
        self.xd = gen.to_torch(gen.decode_tokens(wl), wl.dtype, dev)
        self.q = gen.to_torch(gen.decode_queries(wl, w), wl.dtype, dev)
        self.seq_idx = torch.arange(B, dtype=torch.int32, device=dev)
        self.pos = torch.tensor(lens - 1, dtype=torch.int32, device=dev)
        self.seq_lens = torch.tensor(lens, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.q)
        self.ws = workspace(plan, B, dev)
        self.stream = torch.cuda.current_stream(dev)

        # which split-K attention kernel runs (the library's automatic choice unless forced)
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, kernel)
        kernel_used = mla.mla_decode_kernel_choice(plan, caches[0].struct)
        self.kernel_used = kernel_used
        mla.mla_plan_set_option(plan, mla.MLA_OPT_DECODE_KERNEL, kernel_used)
        torch.cuda.synchronize()
        assert mla.mla_device_error(plan) == 0
        self.tokens = int(np.sum(lens))
        # fused step: append + absorb(+schedule) in one kernel, split-K attention, combine(+W_uv);
        # separate calls: append (+ the ring-slot claim), absorb, attention, combine
        self.launches_per_step = 3 if fused else 4 + (1 if wl.resid else 0)

    def step(self, i):
        c = self.caches[i % self.n_rep].struct
        if self.fused:   # one call: append of the B new tokens + decode of the B queries
            self.mla.mla_decode_step(self.plan, c, self.seq_lens, self.xd, self.q, self.out, self.ws,
                                     stream=self.stream)
        else:
            self.mla.mla_append(self.plan, self.xd, self.seq_idx, self.pos, c, stream=self.stream)
            self.mla.mla_decode(self.plan, c, self.seq_lens, self.q, self.out, self.ws, stream=self.stream)

    def timed_steps(self, K, world=1, sampler=None):
        """ms per step over K steps (device time, CUDA events on the launching stream), the
        clocks sampled during the region; nothing but the steps is enqueued inside it."""
        torch = self.torch
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if sampler:
            sampler.start()
        # keep the GPU under the same load for ~1.5 s before the timed region so that the
        # 100 ms clock samples cover the timed region and its steady state
        t_soak = time.perf_counter()
        i = 0
        while time.perf_counter() - t_soak < 1.5:
            self.step(i)
            i += 1
            if i % 64 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        start.record(self.stream)
        for i in range(K):
            self.step(i)
        end.record(self.stream)
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        dev_err = self.mla.mla_device_error(self.plan)
        if dev_err:
            raise RuntimeError(f"device error word {dev_err} after the timed region: result invalid")
        return start.elapsed_time(end) / K, clocks

    def kernel_times(self, K):
        """Average ms of each kernel of the step, from events the library records right
        around each launch on its stream (MLA_OPT_PROFILE_KERNELS).  The events keep the
        kernels from overlapping, so these run in a separate loop from the timed steps."""
        import ctypes
        torch, mla = self.torch, self.mla
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(K)]
        for row in ev:
            for e in row:
                e.record(self.stream)
        handles = [(ctypes.c_void_p * 8)(*[e.cuda_event for e in row]) for row in ev]
        torch.cuda.synchronize()
        for i in range(K):
            mla.mla_plan_set_option(self.plan, mla.MLA_OPT_PROFILE_KERNELS, ctypes.addressof(handles[i]))
            self.step(i)
        torch.cuda.synchronize()
        mla.mla_plan_set_option(self.plan, mla.MLA_OPT_PROFILE_KERNELS, 0)
        names = ("append", "absorb", "attention", "combine")
        if self.fused:   # the append runs inside the first kernel with the absorption
            names = (None, "append+absorb", "attention", "combine")
        return {n: statistics.mean(ev[i][2 * k].elapsed_time(ev[i][2 * k + 1]) for i in range(K))
                for k, n in enumerate(names) if n}

    def chunk_line(self, Q, K):
        """Many queries per sequence (chunked prefill): the newest Q tokens of every sequence
        attend causally over its cache in one mla_decode_chunk call, the chunk kernel sharing
        each cache tile among a unit's queries.  Times K whole calls (absorption, attention,
        merge) over the rotated cache replicas with CUDA events on the call's stream; the
        rates below are per whole call."""
        torch, mla, wl = self.torch, self.mla, self.wl
        B, H = wl.batch, wl.n_heads
        g = torch.Generator(device="cpu").manual_seed(1234)
        q = (torch.randn(B, Q, H, wl.head_dim, generator=g) * 0.5).to(self.q.dtype).to(self.dev)
        out = torch.empty_like(q)
        ws = torch.empty(mla.mla_decode_chunk_workspace_bytes(self.plan, B, Q), dtype=torch.uint8, device=self.dev)
        call = lambda i: mla.mla_decode_chunk(self.plan, self.caches[i % self.n_rep].struct, self.seq_lens, q, out, ws,
                                              stream=self.stream)
        for i in range(3):
            call(i)
        torch.cuda.synchronize()
        s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(self.stream)
        for i in range(K):
            call(i)
        e0.record(self.stream)
        torch.cuda.synchronize()
        call_ms = s0.elapsed_time(e0) / K
        assert mla.mla_device_error(self.plan) == 0
        qper = max(1, 128 // H)
        units = -(-Q // qper)
        lens = np.asarray(self.lens, dtype=np.int64)
        # per query: latent scores and values over d_c, RoPE scores over 2r, for every head
        flops = 0
        for L in lens:
            pos = np.arange(L - Q, L) + 1   # tokens each query sees
            flops += int(pos.sum()) * H * (4 * wl.d_c + 2 * 2 * wl.r_pairs)
        per_tok = self.cache_bytes / float(lens.sum())
        streamed = sum(float(L - Q + min(Q, (k + 1) * qper)) for L in lens for k in range(units)) * per_tok
        peak_tf = measured_peak_tflops()
        return {"queries_per_seq": Q, "q_tokens_per_s": B * Q / (call_ms * 1e-3), "call_ms": call_ms,
                "queries_per_unit": qper,
                "tensor": {"achieved_tflops": flops / (call_ms * 1e-3) / 1e12, "peak_tflops": peak_tf,
                           "frac": flops / (call_ms * 1e-3) / 1e12 / peak_tf, "flops": flops},
                "hbm": {"unique_cache_bytes": self.cache_bytes, "streamed_bytes": streamed,
                        "streamed_gbs": streamed / (call_ms * 1e-3) / 1e9,
                        "frac": streamed / (call_ms * 1e-3) / 1e9 / measured_peak_hbm()[0]},
                "steps": K}

    def decode_only_ms(self, K):
        torch = self.torch
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(self.stream)
        for i in range(K):
            self.mla.mla_decode(self.plan, self.caches[i % self.n_rep].struct, self.seq_lens, self.q, self.out,
                                self.ws, stream=self.stream)
        e2.record(self.stream)
        torch.cuda.synchronize()
        return s2.elapsed_time(e2) / K

    def e2e(self, E):
        """The same step end to end through one C-ABI call with host buffers
        (mla_decode_step_host): pinned host sequence lengths, x and q copied in and the
        output copied back inside the timed region, every step."""
        torch = self.torch
        lh = self.seq_lens.cpu().pin_memory()
        xh = self.xd.cpu().pin_memory()
        qh = self.q.cpu().pin_memory()
        oh = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        torch.cuda.synchronize()
        s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s3.record(self.stream)
        for i in range(E):
            self.mla.mla_decode_step_host(self.plan, self.caches[i % self.n_rep].struct, lh, xh, qh, oh, self.ws,
                                          stream=self.stream)
        e3.record(self.stream)
        torch.cuda.synchronize()
        h2d = sum(t.numel() * t.element_size() for t in (lh, xh, qh))
        d2h = oh.numel() * oh.element_size()
        return s3.elapsed_time(e3) / E, h2d, d2h

    def roofline(self, attention_ms, workload_name):
        peak, peak_src = measured_peak_hbm()
        achieved = self.cache_bytes / (attention_ms * 1e-3) / 1e9
        kernel_name = {2: "tcgen05 split-K latent attention, a token per softmax thread (decode_tc_kernel)",
                       3: "tcgen05 split-K latent attention, a head per softmax thread (attn_tc_kernel)"}.get(
                           self.kernel_used, "CUDA-core split-K latent attention (decode_simt_kernel)")
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": measured_traffic(workload_name, self.kernel_used), "kernel": kernel_name,
                "bytes_per_launch": self.cache_bytes, "avg_launch_ms": attention_ms, "peak_source": peak_src}

    def weight_bytes(self):
        wl = self.wl
        eb = 2 if wl.dtype == "bf16" else 4
        return wl.n_kv_heads * wl.d_c * (wl.head_dim - 2 * wl.r_pairs) * eb + wl.n_kv_heads * wl.d_c * wl.head_dim * eb

    def cpu_baseline(self, seconds_cap):
        n_tok = int(min(self.lens[0], 4096))
        times = oracle_decode_sample(self.wl, n_tok, 50, seconds_cap=seconds_cap)
        return {"value": n_tok / statistics.median(times), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                "sample": f"float64 oracle decode of one query (all {self.wl.n_heads} heads) over "
                          f"{n_tok} cached tokens, median of {len(times)} runs"}

    def close(self):
        self.plan.close()
        self.caches = None


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    from mha_mla_latent_b200 import build
    build.build()

    dev = torch.device("cuda", local)
    bn = Bench(args.workload, dev, args.kernel, fused=not args.separate_calls)
    wl, K = bn.wl, args.steps
    if args.prefill_only:
        if rank == 0:
            print(json.dumps({"workload": args.workload, "prefill_chunk": bn.chunk_line(64, max(3, min(K, 50)))}),
                  flush=True)
        bn.close()
        return 0
    for i in range(args.warmup):
        bn.step(i)
    torch.cuda.synchronize()

    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(vis.split(",")[local] if vis else local)
    local_ms, clocks = bn.timed_steps(K, world, sampler)
    ms_per_step, value = replica_aggregate(local_ms, bn.tokens, world, dev)
    kt = bn.kernel_times(K)
    decode_ms = bn.decode_only_ms(min(K, 1000))
    e2e_ms, h2d, d2h = bn.e2e(args.e2e_steps)
    _, e2e_value = replica_aggregate(e2e_ms, bn.tokens, world, dev)
    peak, _ = measured_peak_hbm()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype if wl.cache == "same" else f"bf16 ({wl.cache[:4]} latent cache)",
        "data": "synthetic (seeded generators; random-init layer of the named shape)",
        "config": dict(wl_config(wl, bn.lens), parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       l2=f"{bn.n_rep} cache replicas rotated per step "
                          f"({bn.n_rep * bn.cache_bytes / 2**20:.0f} MiB > 2x L2)"),
        "roofline": bn.roofline(kt["attention"], args.workload),
        "decode_only_ms": decode_ms,
        "decode_roofline_frac": (bn.cache_bytes + bn.weight_bytes()) / (decode_ms * 1e-3) / 1e9 / peak,
        "kernel_ms": kt,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": bn.launches_per_step * K,
        "clocks": clocks,
        "conversion_s": bn.conversion_s, "prefill_s": bn.prefill_s,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = bn.cpu_baseline(20.0)
    if world == 1 and args.per_workload:
        try:   # chunked prefill over the same caches: 64 new tokens per sequence
            line["prefill_chunk"] = bn.chunk_line(64, max(5, min(K, 50)))
        except Exception as e:   # shapes the chunk kernel does not take
            line["prefill_chunk"] = {"unavailable": str(e).splitlines()[0][:200]}
    bn.close()
    del bn
    torch.cuda.empty_cache()

    # the other Llama-2-7B-shaped workloads, measured in the same run on one GPU: the
    # ragged long-context batch, the int4 latent cache, and the int4 cache with its
    # 128-token residual window
    if world == 1 and args.per_workload:
        per = {}
        for name in PER_WORKLOADS:
            if name == args.workload:
                continue
            b2 = Bench(name, dev, args.kernel, fused=not args.separate_calls)
            Kw = max(20, min(K, 500))
            for i in range(args.warmup):
                b2.step(i)
            torch.cuda.synchronize()
            ms, ck = b2.timed_steps(Kw, 1, ClockSampler(vis.split(",")[local] if vis else local))
            kt2 = b2.kernel_times(Kw)
            dms = b2.decode_only_ms(Kw)
            entry = {"value": b2.tokens / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "steps": Kw,
                     "config": wl_config(b2.wl, b2.lens), "roofline": b2.roofline(kt2["attention"], name),
                     "decode_only_ms": dms,
                     "decode_roofline_frac": (b2.cache_bytes + b2.weight_bytes()) / (dms * 1e-3) / 1e9 / peak,
                     "kernel_ms": kt2, "clocks": ck}
            if not args.no_cpu_baseline:
                entry["cpu_baseline"] = b2.cpu_baseline(5.0)
            per[name] = entry
            b2.close()
            del b2
            torch.cuda.empty_cache()
        line["per_workload"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
