#!/usr/bin/env python
"""Benchmark of the hybrid GQA attention hot path on B200.

Step (the headline workload): prefill of one 4-layer group -- 3 sliding
layers and 1 full layer, batch 1, 32768 tokens, 16 query / 4 KV heads,
head_dim 256 -- into fresh KV caches (RoPE, masked GQA attention, sigmoid
gate, linear-cache and ring appends).  Inputs are seeded N(0,1) bf16 and
each layer's fused qkv rows (400 MB) are larger than L2, so no flush is
needed between steps.

The JSON line also carries:
  roofline      the full-layer prefill attention kernel, timed live with CUDA
                events around its launches, against the measured bf16 peak;
  e2e           the same metric through the C ABI from pinned host buffers,
                copies inside the timed region;
  decode        decode, batch 16, 131072-token full-layer cache and a full
                512-slot ring (head at a random offset): KV GB/s, % of HBM,
                tokens/s; decode_fp8 the same over e4m3 caches, decode_paged
                with the full-layer cache in 64-token pages scattered over a pool;
  prefill_128k  one full layer, 131072 tokens: TFLOP/s and % of peak;
  layer_prefill the 4-layer group as whole layers (projections + attention);
  decode_1m     36-layer decode at 1M tokens: tokens/s (and decode_1m_fp8
                over e4m3 caches);
  decode_1m_sharded (by default, every rank; --quick skips it) the same with the full
                layers' history spread over the ranks;
  chunked_prefill 262144 tokens in 8192-token chunks, 36 layers (and
                chunked_prefill_fp8 over e4m3 caches; these and the 1M decode
                are skipped with --quick);
  cpu_baseline  the fp64 oracle on a bounded sample of the same workload.

`--impl reference` times the oracle as the reference arm instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

SLIDING, FULL = 0, 1
H, KVH, D, W = 16, 4, 256, 512
GROUP_LAYERS = [SLIDING, SLIDING, SLIDING, FULL]   # layers 0..3 of the 3 + 1 pattern
T_MAIN = 32768
B_MAIN = 1
METRIC = "prefill attn TFLOP/s"
WORKLOAD = ("prefill of one 4-layer group (3 sliding + 1 full), batch 1, seq 32768, 16 Q / 4 KV heads, "
            "head_dim 256, bf16 N(0,1) inputs, seed 1")


def config_dict(n_gpus: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": WORKLOAD, "batch": B_MAIN, "seq_len": T_MAIN, "layers": "sliding, sliding, sliding, full",
            "parallelism": f"replicas x{n_gpus}",
            "l2": "no flush: each layer's inputs (400 MB) exceed the 126 MB L2"}


def targets_summary(extras: dict, roofline: dict) -> dict:
    """The two stated targets (128K full-layer prefill >= 60 % of the bf16 peak,
    1M-token decode >= 70 % of HBM) in a few numbers."""
    out = {"headline_full_kernel_frac": roofline.get("frac")}
    p = extras.get("prefill_128k")
    if p:
        out["prefill_128k"] = {"kernel_ms": p["kernel_ms"], "tflops": p["kernel_tflops"],
                               "frac_of_peak": p["frac_of_peak"], "target": 0.60}
    d = extras.get("decode_1m")
    if d:
        out["decode_1m"] = {"tokens_per_s": d["tokens_per_s"], "gb_per_s": d["kv_gb_per_s"],
                            "frac_of_hbm": d["frac_of_hbm"], "target": 0.70}
    d8 = extras.get("decode_1m_fp8")
    if d8:
        out["decode_1m_fp8"] = {"tokens_per_s": d8["tokens_per_s"], "frac_of_hbm": d8["frac_of_hbm"],
                                "frac_of_measured_copy": d8["frac_of_measured_copy"]}
    ds = extras.get("decode_1m_sharded")
    if ds:
        out["decode_1m_sharded"] = {"tokens_per_s": ds["tokens_per_s"], "frac_of_hbm_per_gpu": ds["frac_of_hbm_per_gpu"]}
    return out


def pairs(n: int, lt: int) -> int:
    if lt == FULL or n <= W:
        return n * (n + 1) // 2
    return W * (W + 1) // 2 + (n - W) * W


def flops(n: int, lt: int, heads: int = H) -> int:
    return pairs(n, lt) * heads * 4 * D


def layer_seed(base: int, i: int) -> int:
    return base + 7919 * i


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of the kernel as it was when its sources (comments aside) hashed to `sha`.
# Reported as roofline.traffic only while the sources are unchanged; otherwise null.
TRAFFIC = {
    "prefill_full_T32768": {"bytes": 2.2145e9, "sha": "cde85cf6e90e8bda",
                            "sources": ["prefill.cu", "common.cuh"]},
    "prefill_sliding_T32768": {"bytes": 0.6381e9, "sha": "cde85cf6e90e8bda",
                               "sources": ["prefill.cu", "common.cuh"]},
    # captured at 16 x 32768 tokens; decode streams each cached byte once, so
    # traffic scales with the tokens: x 8590491648 / 2147483648
    "decode_full_B16_L131072": {"bytes": 2.1600e9 * 8590491648 / 2147483648, "sha": "5a3b85a75e2593a5",
                                "sources": ["decode.cu", "common.cuh"]},
    "decode_fp8_full_B16_L131072": {"bytes": 1.1028e9 * 8590491648 / 2147483648, "sha": "5a3b85a75e2593a5",
                                    "sources": ["decode.cu", "common.cuh"]},
}


def kernel_sources_sha(files) -> str:
    """Hash of the kernel sources with comments and whitespace taken out (a comment
    edit leaves the kernel, and its traffic, as they were)."""
    import hashlib
    import re
    d = hashlib.sha256()
    for f in files:
        src = open(os.path.join(ROOT, "full_gqa_attention_partial_b200", "csrc", f), encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        d.update(" ".join(src.split()).encode())
    return d.hexdigest()[:16]


def traffic_of(name: str):
    t = TRAFFIC.get(name)
    if t is None or kernel_sources_sha(t["sources"]) != t["sha"]:
        return None
    return t["bytes"]


# ---------------------------------------------------------------------------
# plumbing: ranks, peaks, clocks
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cuda"

    def init(self, backend="nccl"):
        self.device = "cuda" if backend == "nccl" else "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            # a short timeout: ranks waiting on one that died end with an error
            limit_s = float(os.environ.get("HYB_PG_TIMEOUT_S", "120"))
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=limit_s))
            self.pg = dist
        if backend == "nccl" and torch.cuda.is_available():
            torch.cuda.set_device(self.local)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def aggregate(self, units_per_rank: float, ms_this_rank: float):
        """Whole-job throughput: every rank's units over the slowest rank's time.

        Returns (units per second, max ms).  Weak scaling: each rank processes
        the same per-rank work, so the job processed world * units_per_rank."""
        ms = self.max(ms_this_rank)
        return self.world * units_per_rank / (ms / 1e3), ms

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# Decode reads the cache and writes almost nothing, so a read stream can exceed the
# measured copy figure (read + write traffic of a device-to-device copy): decode
# fractions are taken against the ~8 TB/s HBM figure the targets are stated in,
# with the fraction of the measured copy rate beside it.
HBM_READ_GBS = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        j = json.load(open(p))
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class Clocks:
    """nvidia-smi sampling (every 200 ms) while the timed regions run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        # raw samples go to $HYB_BENCH_OUT (default: the system's temporary directory)
        import tempfile
        out_dir = os.environ.get("HYB_BENCH_OUT") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"hyb_clocks_rank{os.environ.get('RANK', '0')}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            sel = []
            try:
                uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
                sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
            except Exception:
                pass
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.4 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples_under_load": len(load), "power_w_max": pmax}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def make_layer_inputs(T: int, seed: int):
    from full_gqa_attention_partial_b200 import synth
    return synth.prefill_inputs(B_MAIN, T, seed=seed, device="cuda")


def bench_main(hyb, args, dist: Dist, peaks):
    layers = [make_layer_inputs(T_MAIN, layer_seed(1, i)) for i in range(len(GROUP_LAYERS))]
    n_steps = args.warmup + args.steps
    caches = [[hyb.KVCache(lt, B_MAIN, capacity=T_MAIN) for lt in GROUP_LAYERS] for _ in range(n_steps)]
    ws_bytes = max(hyb.hyb_attn_prefill_workspace_size(lt, B_MAIN, T_MAIN, True) for lt in GROUP_LAYERS)
    ws = hyb.alloc_workspace(ws_bytes)
    outs = [torch.empty(B_MAIN, T_MAIN, H, D, dtype=torch.bfloat16, device="cuda") for _ in GROUP_LAYERS]
    step_flops = sum(flops(T_MAIN, lt) for lt in GROUP_LAYERS)

    def step(i):
        for li, lt in enumerate(GROUP_LAYERS):
            x = layers[li]
            hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, lt, out=outs[li],
                                 cache=caches[i][li], workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    dist.barrier()
    torch.cuda.synchronize()
    l0 = hyb.hyb_launch_count()
    timer = hyb.KernelTimer(args.steps * len(GROUP_LAYERS))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with timer:
        ev0.record()
        for i in range(args.steps):
            step(args.warmup + i)
        ev1.record()
    torch.cuda.synchronize()
    dist.barrier()
    launches = hyb.hyb_launch_count() - l0
    rate, ms = dist.aggregate(args.steps * step_flops, ev0.elapsed_time(ev1))
    assert hyb.hyb_device_error() == 0
    kt = timer.times_ms()
    per_layer = {li: kt[li::len(GROUP_LAYERS)] for li in range(len(GROUP_LAYERS))}
    full_ms = statistics.mean(per_layer[3])
    slide_ms = statistics.mean(t for li in range(3) for t in per_layer[li])
    # The timed region is well under a second: the full-layer kernel is compared
    # with the burst bf16 figure; the fraction of the sustained (seconds-long,
    # power-capped) figure is reported beside it.
    peak = peaks["bf16_tflops"]
    achieved = flops(T_MAIN, FULL) / (full_ms / 1e3) / 1e12
    kernel_share = sum(kt) / (ms / 1.0) if ms > 0 else None
    res = {
        "value": rate / 1e12,
        "ms_per_step": ms / args.steps,
        "gpu_launches": launches,
        "roofline": {
            "bound": "tensor", "kernel": "prefill_kernel<FULL> (tcgen05)", "achieved": achieved,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peaks['source']} bf16 burst",
            "timed_region_s": ms / 1e3,
            "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
            "sustained_peak": peaks["bf16_tflops_sustained"],
            "algorithmic_flops_per_launch": flops(T_MAIN, FULL),
            "avg_launch_ms": full_ms, "launches": len(per_layer[3]),
            "first_last_launch_ms": [per_layer[3][0], per_layer[3][-1]],
            "traffic": traffic_of("prefill_full_T32768"),
            "sliding_kernel": {"avg_launch_ms": slide_ms,
                               "achieved": flops(T_MAIN, SLIDING) / (slide_ms / 1e3) / 1e12,
                               "frac": flops(T_MAIN, SLIDING) / (slide_ms / 1e3) / 1e12 / peak,
                               "traffic": traffic_of("prefill_sliding_T32768")},
            "attention_kernels_share_of_step": kernel_share,
        },
    }
    # ---- e2e: pinned host inputs -> device -> library -> host ----
    # Three streams: host-to-device copies of the next layer's inputs and the
    # device-to-host copy of the previous layer's output overlap the attention
    # of the current layer (two input buffers, one output buffer per layer).
    host_in = [{k: layers[li][k].cpu().pin_memory() for k in ("qkv", "gate")} for li in range(len(GROUP_LAYERS))]
    host_out = [torch.empty(B_MAIN, T_MAIN, H, D, dtype=torch.bfloat16).pin_memory() for _ in GROUP_LAYERS]
    dev_qkv = [torch.empty_like(layers[0]["qkv"]) for _ in range(2)]
    dev_gate = [torch.empty_like(layers[0]["gate"]) for _ in range(2)]
    e2e_caches = [[hyb.KVCache(lt, B_MAIN, capacity=T_MAIN) for lt in GROUP_LAYERS] for _ in range(n_steps)]
    qkv_views = [(x[..., :4096].unflatten(-1, (H, D)), x[..., 4096:5120].unflatten(-1, (KVH, D)),
                  x[..., 5120:].unflatten(-1, (KVH, D))) for x in dev_qkv]
    h2d = sum(t.numel() * t.element_size() for hi in host_in for t in hi.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in GROUP_LAYERS]
    out_free = [torch.cuda.Event() for _ in GROUP_LAYERS]
    n_layer_calls = [0]

    def e2e_step(i):
        for li, lt in enumerate(GROUP_LAYERS):
            n = n_layer_calls[0]
            buf = n % 2
            with torch.cuda.stream(s_in):
                if n >= 2:
                    s_in.wait_event(in_free[buf])
                dev_qkv[buf].copy_(host_in[li]["qkv"], non_blocking=True)
                dev_gate[buf].copy_(host_in[li]["gate"], non_blocking=True)
                in_ready[buf].record(s_in)
            comp.wait_event(in_ready[buf])
            if n >= len(GROUP_LAYERS):
                comp.wait_event(out_free[li])
            q, k, v = qkv_views[buf]
            hyb.hyb_attn_prefill(q, k, v, dev_gate[buf], None, lt, out=outs[li], cache=e2e_caches[i][li], workspace=ws)
            in_free[buf].record(comp)
            out_ready[li].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[li])
                host_out[li].copy_(outs[li], non_blocking=True)
                out_free[li].record(s_out)
            n_layer_calls[0] += 1

    def drain():   # the compute stream waits for every copy issued so far
        for li in range(len(GROUP_LAYERS)):
            comp.wait_event(out_free[li])
        for b in range(2):
            ev = torch.cuda.Event()
            ev.record(s_in)
            comp.wait_event(ev)

    for i in range(args.warmup):
        e2e_step(i)
    drain()
    torch.cuda.synchronize()
    dist.barrier()
    ev0.record()
    for i in range(args.steps):
        e2e_step(args.warmup + i)
    drain()
    ev1.record()
    torch.cuda.synchronize()
    e2e_rate, e2e_ms = dist.aggregate(args.steps * step_flops, ev0.elapsed_time(ev1))
    res["e2e"] = {"value": e2e_rate / 1e12, "unit": "TFLOP/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps}
    del caches, e2e_caches, host_in, host_out
    return res, layers


def bench_prefill_128k(hyb, args, peaks):
    T = 131072
    x = make_layer_inputs(T, layer_seed(1, 3))
    ws = hyb.alloc_workspace(hyb.hyb_attn_prefill_workspace_size(FULL, 1, T, False))
    out = torch.empty(1, T, H, D, dtype=torch.bfloat16, device="cuda")
    n = 3
    hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], FULL, out=out, workspace=ws)
    torch.cuda.synchronize()
    timer = hyb.KernelTimer(n)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with timer:
        ev0.record()
        for _ in range(n):
            hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], FULL, out=out, workspace=ws)
        ev1.record()
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    call_ms = ev0.elapsed_time(ev1) / n
    k_ms = statistics.mean(timer.times_ms())
    f = flops(T, FULL)
    peak = peaks["bf16_tflops"]
    return {"workload": "one full layer, B=1, T=131072", "tflop": f / 1e12,
            "kernel_ms": k_ms, "call_ms": call_ms, "kernel_tflops": f / (k_ms / 1e3) / 1e12,
            "frac_of_peak": f / (k_ms / 1e3) / 1e12 / peak, "peak": peak, "launches": n,
            "frac_of_sustained_peak": f / (k_ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"]}


def bench_layer(hyb, args, peaks):
    """The 3-sliding + 1-full group as whole layers (projections included),
    T=32768, into fresh caches: hyb_attn_layer_prefill per layer."""
    T = T_MAIN
    hidden = make_layer_inputs(T, layer_seed(1, 0))["qkv"][..., :2560].contiguous()
    g = torch.Generator(device="cuda").manual_seed(77)
    w = [((torch.randn(6144, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16),
          (torch.randn(16, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16),
          (torch.randn(2560, 4096, generator=g, device="cuda") / 4096 ** 0.5).to(torch.bfloat16))
         for _ in GROUP_LAYERS]
    out = torch.empty(1, T, 2560, dtype=torch.bfloat16, device="cuda")
    ws = hyb.alloc_workspace(max(hyb.hyb_attn_layer_prefill_workspace_size(lt, 1, T, True) for lt in GROUP_LAYERS))
    n = 3
    caches = [[hyb.KVCache(lt, 1, capacity=T) for lt in GROUP_LAYERS] for _ in range(n + 1)]

    def step(i):
        for li, lt in enumerate(GROUP_LAYERS):
            hyb.hyb_attn_layer_prefill(hidden, *w[li], None, lt, out=out, cache=caches[i][li], workspace=ws)

    step(0)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(n):
        step(1 + i)
    ev1.record()
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    ms = ev0.elapsed_time(ev1) / n
    attn = sum(flops(T, lt) for lt in GROUP_LAYERS)
    proj = len(GROUP_LAYERS) * 2 * T * 2560 * (6144 + 16 + 4096)
    return {"workload": "3+1 group as whole layers (projections, synthetic weights), B=1, T=32768",
            "ms_per_step": ms, "tflop_per_step": (attn + proj) / 1e12, "projection_tflop": proj / 1e12,
            "tflops": (attn + proj) / (ms / 1e3) / 1e12,
            "frac_of_peak": (attn + proj) / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]}


def fill_full_cache(hyb, B: int, L: int, cap: int, seed: int, fp8: bool = False):
    """Full-layer cache holding L random tokens (keys taken as already rotated)."""
    from full_gqa_attention_partial_b200 import synth
    c = hyb.KVCache(FULL, B, capacity=cap, kv_dtype=hyb.KV_FP8 if fp8 else hyb.KV_BF16)
    if fp8:
        synth.fill_cache_fp8_(c.k, c.v, c.k_scale, c.v_scale, L, seed)
    else:
        synth.fill_cache_randn_(c.k, c.v, L, seed)
    c.len.fill_(L)
    return c


def fill_ring_cache(hyb, B: int, L: int, seed: int, head0: int, fp8: bool = False):
    """A 512-slot ring in the state it has after L tokens: token i at slot (head0 + i) % 512."""
    from full_gqa_attention_partial_b200 import synth
    c = hyb.KVCache(SLIDING, B, head0=[head0] * B, kv_dtype=hyb.KV_FP8 if fp8 else hyb.KV_BF16)
    if fp8:
        synth.fill_cache_fp8_(c.k, c.v, c.k_scale, c.v_scale, W, seed)
    else:
        synth.fill_cache_randn_(c.k, c.v, W, seed)
    idx = torch.arange(max(0, L - W), L, dtype=torch.int64, device="cuda")
    tag = torch.full((W,), -1, dtype=torch.int32, device="cuda")
    tag[(head0 + idx) % W] = idx.to(torch.int32)
    c.tag.copy_(tag.expand(B, W))
    c.len.fill_(L)
    c.head.fill_((head0 + L) % W)
    return c


# KV bytes decode streams per cached token per layer: K and V of 4 heads
KV_TOKEN_BYTES = {False: 4096, True: 2 * 4 * 256 + 2 * 4 * 4}   # bf16; FP8 codes + fp32 row scales


def fill_paged_cache(hyb, B: int, L: int, page: int, max_pages: int, seed: int, fp8: bool = False):
    """Paged full-layer cache: each sequence's pages are scattered over a pool
    of B x max_pages pages by a seeded permutation, L random tokens each."""
    from full_gqa_attention_partial_b200 import synth
    n_pages = B * max_pages
    g = torch.Generator().manual_seed(seed)
    table = torch.randperm(n_pages, generator=g).view(B, max_pages).to(torch.int32).cuda()
    c = hyb.KVCache(FULL, B, kv_dtype=hyb.KV_FP8 if fp8 else hyb.KV_BF16, page_size=page, n_pages=n_pages,
                    block_table=table)
    if fp8:
        synth.fill_cache_fp8_(c.k, c.v, c.k_scale, c.v_scale, page, seed)
    else:
        synth.fill_cache_randn_(c.k, c.v, page, seed)
    c.len.fill_(L)
    return c


def bench_decode(hyb, args, peaks, fp8: bool = False, page: int = 0):
    from full_gqa_attention_partial_b200 import synth
    B, L = 16, 131072
    n_steps = args.warmup + args.steps
    cap = L + n_steps + 1
    cap += (-cap) % 4
    if page:
        cap += (-cap) % page
    r = synth.ring_offset(2)
    full = fill_paged_cache(hyb, B, L, page, cap // page, seed=2, fp8=fp8) if page else \
        fill_full_cache(hyb, B, L, cap, seed=2, fp8=fp8)
    ring = fill_ring_cache(hyb, B, L, seed=3, head0=r, fp8=fp8)
    qs = [synth.decode_query(B, seed=1000 + i, device="cuda") for i in range(n_steps)]
    ws = hyb.alloc_workspace(max(hyb.hyb_attn_decode_workspace_size(FULL, B, cap),
                                 hyb.hyb_attn_decode_workspace_size(SLIDING, B, W)))
    out = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")

    def step(i):
        x = qs[i]
        hyb.hyb_kv_append(full, x["k"], x["v"])
        hyb.hyb_attn_decode(x["q"], x["gate"], full, max_len=cap, out=out, workspace=ws)
        hyb.hyb_kv_append(ring, x["k"], x["v"])
        hyb.hyb_attn_decode(x["q"], x["gate"], ring, max_len=W, out=out, workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    timer = hyb.KernelTimer(2 * args.steps)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with timer:
        ev0.record()
        for i in range(args.steps):
            step(args.warmup + i)
        ev1.record()
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    ms = ev0.elapsed_time(ev1) / args.steps
    kt = timer.times_ms()
    full_ms = statistics.mean(kt[0::2])
    ring_ms = statistics.mean(kt[1::2])
    # KV bytes read per step: every cached token's K and V of 4 heads (4096 B per token per layer)
    lens = [L + args.warmup + i + 1 for i in range(args.steps)]
    tb = KV_TOKEN_BYTES[fp8]
    full_bytes = statistics.mean(B * n * tb for n in lens)
    ring_bytes = B * W * tb
    achieved = full_bytes / (full_ms / 1e3) / 1e9
    step_gbs = (full_bytes + ring_bytes) / (ms / 1e3) / 1e9
    return {
        "workload": f"B=16, full cache 131072 + ring (head {r})" + (", FP8" if fp8 else "")
                    + (f", {page}-token pages" if page else ""),
        "tokens_per_s": B / (ms / 1e3), "ms_per_step": ms,
        "kv_gb_per_s": step_gbs, "frac_of_hbm": step_gbs / HBM_READ_GBS,
        "frac_of_measured_copy": step_gbs / peaks["hbm_gbs"],
        "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<FULL, FP8>" if fp8 else "decode_split_kernel<FULL>",
                     "achieved": achieved, "peak": HBM_READ_GBS, "unit": "GB/s", "frac": achieved / HBM_READ_GBS,
                     "frac_of_measured_copy": achieved / peaks["hbm_gbs"],
                     "bytes_per_launch": full_bytes, "avg_launch_ms": full_ms,
                     "traffic": None if page else
                     traffic_of("decode_fp8_full_B16_L131072" if fp8 else "decode_full_B16_L131072")},
        "sliding_kernel": {"avg_launch_ms": ring_ms, "achieved_gbs": ring_bytes / (ring_ms / 1e3) / 1e9},
    }


def bench_layer_decode(hyb, args, peaks):
    """The 3-sliding + 1-full group as whole decode layers (q_k_v_proj with the
    gate rows, append, attention, o_proj), B=16 over 131072-token caches:
    hyb_attn_layer_decode per layer.  The projections' share is the step time
    minus that of the attention alone (append + decode) on caches in the same
    state; they read 52.5 MB of weights per layer, so they are HBM-bound."""
    from full_gqa_attention_partial_b200 import synth
    B, L = 16, 131072
    n = args.steps
    cap = L + 2 * (args.warmup + 1 + n) + 2
    cap += (-cap) % 4
    g = torch.Generator(device="cuda").manual_seed(78)
    w = [((torch.randn(6144, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16),
          (torch.randn(16, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16),
          (torch.randn(2560, 4096, generator=g, device="cuda") / 4096 ** 0.5).to(torch.bfloat16))
         for _ in GROUP_LAYERS]
    r = synth.ring_offset(4)
    caches = [fill_full_cache(hyb, B, L, cap, seed=40 + i) if lt == FULL else
              fill_ring_cache(hyb, B, L, seed=40 + i, head0=r) for i, lt in enumerate(GROUP_LAYERS)]
    hid = [(torch.randn(B, 2560, generator=g, device="cuda")).to(torch.bfloat16) for _ in range(args.warmup + 1)]
    qs = [synth.decode_query(B, seed=2000 + i, device="cuda") for i in range(args.warmup + 1)]
    ws = hyb.alloc_workspace(max(hyb.hyb_attn_layer_decode_workspace_size(lt, B, cap if lt == FULL else W)
                                 for lt in GROUP_LAYERS))
    out = torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda")
    aout = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")

    def layer_step(i):
        for li, lt in enumerate(GROUP_LAYERS):
            hyb.hyb_attn_layer_decode(hid[i], *w[li], caches[li], max_len=cap if lt == FULL else W, out=out,
                                      workspace=ws)

    def attn_step(i):
        x = qs[i]
        for li, lt in enumerate(GROUP_LAYERS):
            hyb.hyb_kv_append(caches[li], x["k"], x["v"])
            hyb.hyb_attn_decode(x["q"], x["gate"], caches[li], max_len=cap if lt == FULL else W, out=aout,
                                workspace=ws)

    def timed(fn):
        # one step captured as a CUDA graph and replayed (the caches' device-side
        # len / head move the append position), so host time is not in the number
        for i in range(args.warmup):
            fn(i)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            fn(args.warmup)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for i in range(n):
            graph.replay()
        ev1.record()
        torch.cuda.synchronize()
        assert hyb.hyb_device_error() == 0
        del graph
        return ev0.elapsed_time(ev1) / n

    ms = timed(layer_step)
    attn_ms = timed(attn_step)
    proj_ms = max(ms - attn_ms, 1e-6)
    # the projection kernels alone: q_k_v_proj and o_proj of the 4 layers through hyb_linear
    pq = torch.empty(B, 6144, dtype=torch.bfloat16, device="cuda")
    po = torch.empty(B, 2560, dtype=torch.bfloat16, device="cuda")
    xa = torch.randn(B, 4096, generator=g, device="cuda").to(torch.bfloat16)

    def proj_step(i):
        for li in range(len(GROUP_LAYERS)):
            hyb.hyb_linear(hid[0], w[li][0], out=pq)
            hyb.hyb_linear(xa, w[li][2], out=po)

    pk_ms = timed(proj_step)
    pk_bytes = len(GROUP_LAYERS) * 2 * (6144 * 2560 + 2560 * 4096)
    wbytes = len(GROUP_LAYERS) * 2 * 2560 * (6144 + 16 + 4096)
    kv = B * (L + args.warmup + 1 + n) * KV_TOKEN_BYTES[False] + 3 * B * W * KV_TOKEN_BYTES[False]
    del caches
    return {"workload": "3+1 group as whole decode layers (projections, synthetic weights), B=16, caches 131072",
            "ms_per_step": ms, "tokens_per_s": B / (ms / 1e3),
            "gb_per_s": (wbytes + kv) / (ms / 1e3) / 1e9, "frac_of_hbm": (wbytes + kv) / (ms / 1e3) / 1e9 / HBM_READ_GBS,
            "projections": {"ms_per_step": proj_ms, "weight_bytes": wbytes,
                            "weight_gb_per_s": wbytes / (proj_ms / 1e3) / 1e9,
                            "frac_of_hbm": wbytes / (proj_ms / 1e3) / 1e9 / HBM_READ_GBS,
                            "kernels_alone": {"ms_per_step": pk_ms, "weight_bytes": pk_bytes,
                                              "weight_gb_per_s": pk_bytes / (pk_ms / 1e3) / 1e9,
                                              "frac_of_hbm": pk_bytes / (pk_ms / 1e3) / 1e9 / HBM_READ_GBS}},
            "attention_ms_per_step": attn_ms}


def bench_decode_1m(hyb, args, peaks, fp8: bool = False):
    """36 layers (27 rings, 9 full caches of ~1M tokens), batch 1, 64 steps of append + decode.

    The step's 144 launches are captured once in a CUDA graph; each timed step
    copies its token's q / k / v / gate into the graph's input buffers and
    replays it (the caches' device-side len / head move the append position)."""
    from full_gqa_attention_partial_b200 import synth
    n_steps = 64
    L0 = (1 << 20) - n_steps
    cap = 1 << 20
    r = synth.ring_offset(3)
    fulls = [fill_full_cache(hyb, 1, L0, cap, seed=3 + 17 * i, fp8=fp8) for i in range(9)]
    rings = [fill_ring_cache(hyb, 1, L0, seed=5000 + i, head0=r, fp8=fp8) for i in range(27)]
    qs = [synth.decode_query(1, seed=9000 + i, device="cuda") for i in range(n_steps)]
    ws_full = hyb.alloc_workspace(hyb.hyb_attn_decode_workspace_size(FULL, 1, cap))
    ws_ring = hyb.alloc_workspace(hyb.hyb_attn_decode_workspace_size(SLIDING, 1, W))
    out = torch.empty(1, H, D, dtype=torch.bfloat16, device="cuda")
    x = {key: torch.empty_like(val) for key, val in qs[0].items()}   # the graph's inputs

    def step():
        fi = ri = 0
        for layer in range(36):
            lt = FULL if layer % 4 == 3 else SLIDING
            if lt == FULL:
                c, ws, ml = fulls[fi], ws_full, cap
                fi += 1
            else:
                c, ws, ml = rings[ri], ws_ring, W
                ri += 1
            hyb.hyb_kv_append(c, x["k"], x["v"])
            hyb.hyb_attn_decode(x["q"], x["gate"], c, max_len=ml, out=out, workspace=ws)

    # capture on a side stream; capturing launches nothing, so the caches are untouched
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record()
    for i in range(n_steps):
        for key in x:
            x[key].copy_(qs[i][key])
        graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    ms = ev0.elapsed_time(ev1) / n_steps
    del graph
    tb = KV_TOKEN_BYTES[fp8]
    kv = statistics.mean(9 * tb * (L0 + i + 1) + 27 * tb * W for i in range(n_steps))
    del fulls, rings
    return {"workload": "36 layers, 9 full caches ~1M + 27 rings, B=1, 64 steps" + (", FP8" if fp8 else ""),
            "tokens_per_s": 1e3 / ms, "ms_per_step": ms, "kv_gb_per_s": kv / (ms / 1e3) / 1e9,
            "frac_of_hbm": kv / (ms / 1e3) / 1e9 / HBM_READ_GBS,
            "frac_of_measured_copy": kv / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}


def bench_decode_1m_sharded(hyb, args, peaks, d):
    """The 36-layer 1M-token decode with each full layer's history spread over
    the ranks (seqshard.py): rank r holds tokens history_range(L0, N, r) of
    every full layer and the steps' tokens in round-robin blocks of 64; the
    27 rings are whole on every rank.  A step is 9 x (partial attention, one
    all-gather of 16 KB, merge) + 27 ring decodes on every rank."""
    from full_gqa_attention_partial_b200 import seqshard, synth
    n_steps = 64
    L0 = (1 << 20) - n_steps
    lo, hi = seqshard.history_range(L0, d.world, d.rank)
    own_steps = sum(1 for s in range(n_steps) if (s // 64) % d.world == d.rank)
    cap = hi - lo + own_steps
    cap += (-cap) % 64
    r = synth.ring_offset(3)
    fulls = [fill_full_cache(hyb, 1, hi - lo, cap, seed=3 + 17 * i + 1000 * d.rank) for i in range(9)]
    decs = [seqshard.SeqShardedDecoder(c, block=64) for c in fulls]
    rings = [fill_ring_cache(hyb, 1, L0, seed=5000 + i, head0=r) for i in range(27)]
    qs = [synth.decode_query(1, seed=9000 + i, device="cuda") for i in range(n_steps)]
    ws_ring = hyb.alloc_workspace(hyb.hyb_attn_decode_workspace_size(SLIDING, 1, W))
    out = torch.empty(1, H, D, dtype=torch.bfloat16, device="cuda")
    pos = [torch.full((1,), L0 + i, dtype=torch.int32, device="cuda") for i in range(n_steps)]

    def step(i):
        x = qs[i]
        fi = ri = 0
        for layer in range(36):
            if layer % 4 == 3:
                decs[fi].step(x["q"], x["k"], x["v"], x["gate"], pos[i], i)
                fi += 1
            else:
                c = rings[ri]
                ri += 1
                hyb.hyb_kv_append(c, x["k"], x["v"])
                hyb.hyb_attn_decode(x["q"], x["gate"], c, max_len=W, out=out, workspace=ws_ring)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    d.barrier()
    torch.cuda.synchronize()
    ev0.record()
    for i in range(n_steps):
        step(i)
    ev1.record()
    torch.cuda.synchronize()
    d.barrier()
    assert hyb.hyb_device_error() == 0
    ms = d.max(ev0.elapsed_time(ev1) / n_steps)
    kv = statistics.mean(9 * 4096 * (L0 + i + 1) + d.world * 27 * 4096 * W for i in range(n_steps))
    del fulls, rings, decs
    per_gpu = kv / (ms / 1e3) / 1e9 / d.world
    return {"workload": f"36 layers, 9 full caches ~1M over {d.world} GPU(s), 27 rings each, B=1, 64 steps",
            "tokens_per_s": 1e3 / ms, "ms_per_step": ms, "kv_gb_per_s": kv / (ms / 1e3) / 1e9,
            "frac_of_hbm_per_gpu": per_gpu / HBM_READ_GBS,
            # the step is bound by each GPU streaming its share of the caches
            "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": HBM_READ_GBS, "unit": "GB/s",
                         "frac": per_gpu / HBM_READ_GBS, "frac_of_measured_copy": per_gpu / peaks["hbm_gbs"],
                         "bytes_per_step_per_gpu": kv / d.world, "ms_per_step": ms}}


def bench_chunked(hyb, args, peaks, fp8: bool = False):
    """262144 tokens in 8192-token chunks through all 36 layers (9 full, 27 sliding), batch 1
    (fp8: every cache in e4m3, the full layers read in place by the attention kernel).

    Each chunk is appended to its layer's cache and attends over the cached
    context.  The 32 chunk inputs (seed 4 + c) are shared by the layers: the
    work does not depend on the values.
    """
    from full_gqa_attention_partial_b200 import synth
    total, C = 262144, 8192
    n_chunks = total // C
    xs = [synth.prefill_inputs(1, C, seed=4 + c, device="cuda", start=c * C) for c in range(n_chunks)]
    kvd = hyb.KV_FP8 if fp8 else hyb.KV_BF16
    fulls = [hyb.KVCache(FULL, 1, capacity=total, kv_dtype=kvd) for _ in range(9)]
    rings = [hyb.KVCache(SLIDING, 1, kv_dtype=kvd) for _ in range(27)]
    ws = hyb.alloc_workspace(max(hyb.hyb_attn_prefill_cache_workspace_size(c, C) for c in (fulls[0], rings[0])))
    out = torch.empty(1, C, H, D, dtype=torch.bfloat16, device="cuda")
    work = 9 * flops(total, FULL) + 27 * flops(total, SLIDING)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for c in range(n_chunks):
        x = xs[c]
        fi = ri = 0
        for layer in range(36):
            if layer % 4 == 3:
                cache, lt = fulls[fi], FULL
                fi += 1
            else:
                cache, lt = rings[ri], SLIDING
                ri += 1
            hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, lt, out=out, cache=cache, workspace=ws)
    ev1.record()
    torch.cuda.synchronize()
    assert hyb.hyb_device_error() == 0
    ms = ev0.elapsed_time(ev1)
    rate = work / (ms / 1e3) / 1e12
    # a run of seconds under the power cap: compared with the sustained (seconds-long) figure
    return {"workload": "262144 tokens in 8192-token chunks, 36 layers, B=1" + (", FP8 caches" if fp8 else ""),
            "workspace_bytes": int(ws.numel()), "pflop": work / 1e15, "ms": ms,
            "tflops": rate, "frac_of_peak": rate / peaks["bf16_tflops_sustained"],
            "peak_source": "sustained", "frac_of_burst_peak": rate / peaks["bf16_tflops"],
            "prefill_tokens_per_s": total / (ms / 1e3)}


# ---------------------------------------------------------------------------
# the oracle on the host: cpu_baseline and the reference arm
# ---------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(host_layers, rows_per_layer: int, seed: int):
    """Times the oracle on `rows_per_layer` query rows of each layer; returns (flops, seconds)."""
    import oracle as O
    rng = np.random.default_rng(seed)
    total_flops, total_s = 0, 0.0
    for li, lt in enumerate(GROUP_LAYERS):
        x = host_layers[li]
        T = x["q"].shape[1]
        rows = np.sort(rng.choice(T, size=rows_per_layer, replace=False))
        t0 = time.perf_counter()
        O.prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lt, rows=rows)
        total_s += time.perf_counter() - t0
        for t in rows:
            n_keys = t + 1 if lt == FULL else min(t + 1, W)
            total_flops += n_keys * H * 4 * D
    return total_flops, total_s


def host_copies(layers):
    out = []
    for x in layers:
        out.append({"q": x["q"].float().cpu().numpy(), "k": x["k"].float().cpu().numpy(),
                    "v": x["v"].float().cpu().numpy(), "gate": x["gate"].float().cpu().numpy(),
                    "pos": x["pos"].cpu().numpy()})
    return out


def cpu_baseline(layers, rows_per_layer: int):
    host = host_copies(layers)
    f, s = oracle_sample(host, rows_per_layer, seed=0)
    return {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows_per_layer} random rows x 16 heads per layer of the step, {s:.1f} s",
            "cpu_model": cpu_model()}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return None
    from full_gqa_attention_partial_b200 import synth
    layers = [synth.prefill_inputs(B_MAIN, T_MAIN, seed=layer_seed(1, i)) for i in range(len(GROUP_LAYERS))]
    host = host_copies(layers)
    rows = args.ref_rows
    for i in range(args.warmup):
        oracle_sample(host, rows, seed=100 + i)
    f_tot, s_tot = 0, 0.0
    for i in range(args.steps):
        f, s = oracle_sample(host, rows, seed=200 + i)
        f_tot += f
        s_tot += s
    value = f_tot / s_tot / 1e12
    sample = (f"each step: {rows} random query rows x 16 heads of each of the 4 layers at T=32768, "
              f"fp64 numpy oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_tot * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1) bf16 inputs, seeded", "config": config_dict(args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(hyb, args):
    """One kernel on a small configuration, for profiler captures: 1 warm-up + args.steps launches."""
    from full_gqa_attention_partial_b200 import synth
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.case in ("linear_qkv", "linear_decode"):
        # q_k_v_proj's shape: M = seq x batch rows (tiled GEMM), or M = batch rows (a decode
        # step: the few-row kernel, rated by the weight bytes it streams)
        M, N, K = (args.seq * args.batch if args.case == "linear_qkv" else args.batch), 6144, 2560
        g = torch.Generator(device="cuda").manual_seed(5)
        x = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
        w = (torch.randn(N, K, generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        fn = lambda: hyb.hyb_linear(x, w, out=y)
        work, unit = (2 * M * N * K, "TFLOP/s") if args.case == "linear_qkv" else (N * K * 2, "GB/s")
    elif args.case == "prefill_full_fp8":
        # a full layer's prefill of seq tokens into an empty FP8 cache (the length is reset
        # before each call, so every launch does the same work)
        T, B = args.seq, args.batch
        x = synth.prefill_inputs(B, T, seed=layer_seed(1, 3), device="cuda")
        c = hyb.KVCache(FULL, B, capacity=T + (-T) % 4, kv_dtype=hyb.KV_FP8)
        ws = hyb.alloc_workspace(hyb.hyb_attn_prefill_cache_workspace_size(c, T))
        out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")

        def fn():
            c.len.zero_()
            hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], FULL, out=out, cache=c, workspace=ws)
        work = B * flops(T, FULL)
        unit = "TFLOP/s"
    elif args.case.startswith("prefill"):
        lt = FULL if args.case == "prefill_full" else SLIDING
        T, B = args.seq, args.batch
        x = synth.prefill_inputs(B, T, seed=layer_seed(1, 3), device="cuda")
        ws = hyb.alloc_workspace(hyb.hyb_attn_prefill_workspace_size(lt, B, T, False))
        out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
        fn = lambda: hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lt, out=out, workspace=ws)
        work = B * flops(T, lt)
        unit = "TFLOP/s"
    else:
        lt = FULL if args.case.startswith("decode_full") else SLIDING
        fp8 = args.case.endswith("_fp8")
        B, L = args.batch, args.seq
        cap = L + args.steps + 2
        cap += (-cap) % 4
        c = fill_full_cache(hyb, B, L, cap, seed=2, fp8=fp8) if lt == FULL else fill_ring_cache(hyb, B, L, 3, 17, fp8=fp8)
        xq = synth.decode_query(B, seed=5, device="cuda")
        ml = cap if lt == FULL else W
        ws = hyb.alloc_workspace(hyb.hyb_attn_decode_workspace_size(lt, B, ml))
        out = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")
        fn = lambda: hyb.hyb_attn_decode(xq["q"], xq["gate"], c, max_len=ml, out=out, workspace=ws)
        work = B * min(L, cap if lt == FULL else W) * KV_TOKEN_BYTES[fp8]
        unit = "GB/s"
    fn()
    torch.cuda.synchronize()
    if args.case.startswith("linear"):   # one kernel per call: events around the calls
        ev0.record()
        for _ in range(args.steps):
            fn()
        ev1.record()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / args.steps
    else:
        timer = hyb.KernelTimer(args.steps)
        with timer:
            for _ in range(args.steps):
                fn()
        ms = statistics.mean(timer.times_ms())
    assert hyb.hyb_device_error() == 0
    rate = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"case": args.case, "batch": args.batch, "seq": args.seq, "kernel_ms": ms,
                      "rate": rate, "unit": unit, "work_per_launch": work}), flush=True)


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-1m", action="store_true", help="(default) run the 36-layer 1M-token decode workload")
    ap.add_argument("--chunked", action="store_true",
                    help="(default) run the 262144-token chunked prefill through 36 layers")
    ap.add_argument("--quick", action="store_true",
                    help="skip the long sub-benchmarks (1M-token decode, chunked prefill)")
    ap.add_argument("--no-extras", action="store_true", help="only the headline step (no sub-benchmarks)")
    ap.add_argument("--decode-sharded", action="store_true",
                    help="also run the 1M-token decode with the full layers' history spread over the ranks")
    ap.add_argument("--cpu-rows", type=int, default=24, help="oracle rows per layer for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=8, help="oracle rows per layer per reference step")
    ap.add_argument("--case", choices=["prefill_full", "prefill_sliding", "prefill_full_fp8", "decode_full",
                                       "decode_sliding", "decode_full_fp8", "decode_sliding_fp8", "linear_qkv",
                                       "linear_decode"],
                    default=None, help="time one kernel on a small configuration (profiling)")
    ap.add_argument("--seq", type=int, default=16384)
    ap.add_argument("--batch", type=int, default=1)
    args = ap.parse_args()
    args.decode_1m = args.chunked = not args.quick
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    dist = Dist()
    if args.impl == "reference":
        res = run_reference(args, dist)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    dist.init()
    import full_gqa_attention_partial_b200 as hyb
    hyb.load()
    if args.case:
        run_case(hyb, args)
        return
    peaks = load_peaks()
    clocks = Clocks()
    clocks.start()
    nvtx = torch.cuda.nvtx

    def run(name, fn, *a, **kw):   # each sub-benchmark inside its own NVTX range
        nvtx.range_push(name)
        try:
            return fn(*a, **kw)
        finally:
            nvtx.range_pop()

    main_res, layers = run("step: 4-layer group prefill", bench_main, hyb, args, dist, peaks)
    extras = {}
    if dist.world == 1 and not args.no_extras:
        extras["prefill_128k"] = run("prefill_128k", bench_prefill_128k, hyb, args, peaks)
        extras["layer_prefill"] = run("layer_prefill", bench_layer, hyb, args, peaks)
        extras["decode"] = run("decode", bench_decode, hyb, args, peaks)
        extras["decode_fp8"] = run("decode_fp8", bench_decode, hyb, args, peaks, fp8=True)
        extras["decode_paged"] = run("decode_paged", bench_decode, hyb, args, peaks, page=64)
        extras["layer_decode"] = run("layer_decode", bench_layer_decode, hyb, args, peaks)
        if args.decode_1m:
            extras["decode_1m"] = run("decode_1m", bench_decode_1m, hyb, args, peaks)
            torch.cuda.empty_cache()
            extras["decode_1m_fp8"] = run("decode_1m_fp8", bench_decode_1m, hyb, args, peaks, fp8=True)
        if args.chunked:
            extras["chunked_prefill"] = run("chunked_prefill", bench_chunked, hyb, args, peaks)
            torch.cuda.empty_cache()
            extras["chunked_prefill_fp8"] = run("chunked_prefill_fp8", bench_chunked, hyb, args, peaks, fp8=True)
    # the sequence-sharded 1M decode runs by default (with one rank: the partial + merge
    # path over the whole history; every rank takes part: it has collectives)
    if (args.decode_sharded or args.decode_1m or dist.world > 1) and not args.no_extras:
        torch.cuda.empty_cache()
        extras["decode_1m_sharded"] = run("decode_1m_sharded", bench_decode_1m_sharded, hyb, args, peaks, dist)
    clk = clocks.stop()
    roof = main_res["roofline"]
    targets = targets_summary(extras, roof)
    roof["north_star_targets"] = targets
    line = {
        "metric": METRIC, "value": main_res["value"], "unit": "TFLOP/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic N(0,1) bf16, seeded (no dataset on the pages for this path)",
        "config": config_dict(dist.world),
        "roofline": roof, "e2e": main_res["e2e"], "gpu_launches": main_res["gpu_launches"],
        "clocks": clk,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_extras:
        line["cpu_baseline"] = cpu_baseline(layers, args.cpu_rows)
    line.update(extras)
    line["north_star_targets"] = targets   # last: the end of the line carries the targets
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
