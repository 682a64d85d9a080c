"""Benchmark of the low-bit KV-cache hot path on B200.

Workload (the metric's configuration): a Llama-3.1-8B-shaped attention layer,
16 sequences x 32 query / 8 KV heads x head_dim 128, bf16 inputs, keys with 4
outlier channels (x20), keys and queries Hadamard-rotated, K and V INT4 in
groups of 128 (fp16 scale/zero), contiguous cache, context 8192. A step is
one decode step: quantize-append one new token per sequence, then split-K
decode attention over the whole packed cache (split-K pass + merge pass).
Steps run as episodes of 64 decode steps (context 8193..8256); after each
episode the sequence lengths are rewound to 8192 outside the timed region.

value  = algorithmic packed-KV bytes attended per step (codes + fp16
         scale/zero of every cached token, K and V) / device step time
e2e    = the same bytes / wall time of a step driven from pinned host buffers
         (the library's CUDA-graph step: staging copies, uploads, append,
         decode, download, host wait)
         (new K/V and q uploaded, output read back) through the C-ABI calls
roofline (dominant kernel = the split-K attention pass): packed bytes / its
         CUDA-event duration against the measured HBM copy bandwidth

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own replica (weak scaling); no collective
touches the data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn packed-KV GB/s (% of 8 TB/s HBM); quantize-append tokens/s"
WORKLOAD = ("llama8b_layer: 16 seqs x 32 q / 8 kv heads x d128, bf16 in, context 8192 + 64 decode "
            "steps of 1 token, INT4 g128 K and V with fp16 scale/zero, Hadamard(128) on K and Q, "
            "contiguous cache")
BATCH, HQ, HKV, D, CTX, EPISODE = 16, 32, 8, 128, 8192, 64
BYTES_PER_TOKEN_HEAD = 2 * (D * 4 // 8 + (D // 128) * 4)   # K + V: 64 B codes + 4 B scale/zero
NOMINAL_HBM_GBS = 8000.0
FLUSH_BYTES = 256 << 20


def flush_l2(buf):
    """Evict L2 between timed steps: write a buffer twice the size of L2, then
    read it back, so the timed work starts from a cold L2 that holds no dirty
    lines (a write alone would leave ~126 MB of them, whose write-back the next
    kernel's reads would pay for)."""
    buf.zero_()
    buf.amax()
# the timed split-K variant: the kernel template and the unit that instantiates it
DECODE_SRC = [os.path.join(ROOT, "bit_kv_cache_21_b200", "csrc", f)
              for f in ("kvq_decode_kernel.cuh", "kvq_decode_plain.cu", "kvq_decode.cu", "kvq_common.cuh",
                        "kvq_internal.h")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_splitk_llama8b_traffic.json")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_launch():
    """dram bytes per split-K launch from the committed ncu summary, or None
    when the kernel source changed since it was captured."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        if d.get("source_sha256_16") != source_hash(DECODE_SRC):
            return None
        return float(d["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ---------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(torch_device)
            h = None
            uuid = str(getattr(props, "uuid", ""))
            if uuid:
                for cand in (uuid if uuid.startswith("GPU-") else "GPU-" + uuid, uuid):
                    try:
                        h = pynvml.nvmlDeviceGetHandleByUUID(cand)
                        break
                    except Exception:
                        pass
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        names = [n for b, n in _REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def make_inputs(seed_offset, n_decode):
    """History for the prefill plus the tokens and queries of n_decode steps."""
    import workloads as W
    w = W.LLAMA8B_LAYER
    ks, vs, _ = W.kv_history(w, [CTX + n_decode] * BATCH, seed_offset=seed_offset)
    k = np.stack(ks)  # [B][T][H][D]
    v = np.stack(vs)
    qs = np.stack([W.queries(w, BATCH, seed_offset=seed_offset * 1000 + i) for i in range(n_decode)])
    return k, v, qs


def bf16(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import bit_kv_cache_21_b200 as K

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    k, v, qs = make_inputs(rank, EPISODE)

    cap = CTX + EPISODE + 64
    spec = K.CacheSpec(BATCH, HKV, bits_k=4, bits_v=4, group_k=128, group_v=128,
                       hadamard_block_k=128, capacity_tokens=cap)
    cache = K.KVCache(spec, device=dev)
    lens = torch.zeros(BATCH, dtype=torch.int32, device=dev)
    cu_pre = torch.arange(0, (BATCH + 1) * CTX, CTX, dtype=torch.int32, device=dev)
    k_pre = bf16(k[:, :CTX].reshape(-1, HKV, D)).to(dev)
    v_pre = bf16(v[:, :CTX].reshape(-1, HKV, D)).to(dev)

    # quantize-append throughput on the bulk prefill (16 x 8192 tokens): one
    # warm-up, then the mean of 5 (its 537 MB of input exceed L2)
    pre_ms = []
    for r in range(6):
        lens.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        K.quantize_append(cache.desc, k_pre, v_pre, cu_pre, lens)
        e1.record(stream)
        torch.cuda.synchronize()
        if r > 0:
            pre_ms.append(e0.elapsed_time(e1))
    del k_pre, v_pre
    append_ms = statistics.mean(pre_ms)
    n_tok = BATCH * CTX
    append_bytes = n_tok * HKV * 2 * (D * 2 + D // 2 + 4)   # bf16 in + packed out, K and V
    append_info = {"metric": "quantize-append tokens/s", "value": n_tok / (append_ms * 1e-3),
                   "unit": "tokens/s", "GBps": append_bytes / (append_ms * 1e-3) / 1e9,
                   "frac_of_hbm": append_bytes / (append_ms * 1e-3) / 1e9 / peaks()[0],
                   "workload": "bulk prefill 16 x 8192 tokens x 8 KV heads, K and V, INT4 g128, "
                               "Hadamard K", "ms": append_ms, "timed": len(pre_ms)}

    # per-step device inputs for the episode
    k_steps = [bf16(k[:, CTX + i]).to(dev) for i in range(EPISODE)]       # [B][H][D]
    v_steps = [bf16(v[:, CTX + i]).to(dev) for i in range(EPISODE)]
    q_steps = [bf16(qs[i]).to(dev) for i in range(EPISODE)]
    cu_one = torch.arange(0, BATCH + 1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    ws = torch.empty(K.decode_workspace_size(cache.desc, BATCH, HQ, cap), dtype=torch.uint8, device=dev)
    out = torch.empty((BATCH, HQ, D), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ctx_lens = torch.full((BATCH,), CTX, dtype=torch.int32, device=dev)

    def step(i, evs=None):
        j = i % EPISODE
        if j == 0:
            lens.copy_(ctx_lens)
        if evs:
            evs[0].record(stream)
        K.quantize_append(cache.desc, k_steps[j], v_steps[j], cu_one, lens)
        if evs:
            evs[1].record(stream)
        # split-K pass, then the merge pass (a programmatic dependent launch)
        K.decode_attention(cache.desc, q_steps[j], lens, cap, scale, out=out, workspace=ws)
        if evs:
            evs[2].record(stream)
        return CTX + j + 1   # tokens attended per sequence

    for i in range(args.warmup):
        flush_l2(flush)
        step(i)
    torch.cuda.synchronize()
    # start the timed episodes at a step boundary of the episode
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    tokens = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clocks:
        for i in range(args.steps):
            flush_l2(flush)
            tokens.append(step(i, evs[i]))
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    append1_ms = [e[0].elapsed_time(e[1]) for e in evs]

    # the dominant kernel alone, for its roofline: the split-K pass over the
    # cache as the last step left it, L2 flushed before each launch
    lens_now = lens.clone()
    split_bytes = float(lens_now.sum().item()) * HKV * BYTES_PER_TOKEN_HEAD
    split_ms = []
    for i in range(args.warmup + args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        K.decode_splitk(cache.desc, q_steps[0], lens_now, cap, scale, ws)
        e1.record(stream)
        if i >= args.warmup:
            split_ms.append((e0, e1))
    torch.cuda.synchronize()
    split_ms = [a.elapsed_time(b) for a, b in split_ms]
    total_ms = sum(step_ms)
    bytes_total = sum(t * BATCH * HKV * BYTES_PER_TOKEN_HEAD for t in tokens)
    assert cache.device_status() == 0, "device status %d" % cache.device_status()

    # end to end from pinned host buffers
    import torch.cuda
    # per slot one pinned buffer holding the step's k, v and q back to back,
    # so the step uploads them with one copy
    hk, hv, hq = [], [], []
    for i in range(EPISODE):
        parts = [bf16(k[:, CTX + i]), bf16(v[:, CTX + i]), bf16(qs[i])]
        buf = torch.empty(sum(t.nbytes for t in parts), dtype=torch.uint8).pin_memory()
        views, off = [], 0
        for t in parts:
            view = buf[off:off + t.nbytes].view(t.dtype).view(t.shape)
            view.copy_(t)
            views.append(view)
            off += t.nbytes
        hk.append(views[0])
        hv.append(views[1])
        hq.append(views[2])
    # the step as the library's CUDA-graph step, one per pinned input slot (a
    # server cycles through a ring of such slots): the timed region replays
    # it (H2D uploads, append, decode, D2H download) and waits for the output
    hout = torch.empty((BATCH, HQ, D), dtype=torch.float32).pin_memory()
    graph_steps = [K.DecodeStep(cache.desc, lens, cu_one, cap, scale, hk[j], hv[j], hq[j], out_host=hout,
                                workspace=ws) for j in range(EPISODE)]
    e2e_s, e2e_bytes = [], 0
    for i in range(args.warmup + args.steps):
        j = i % EPISODE
        if j == 0:
            lens.copy_(ctx_lens)
            for gs in graph_steps:   # the lengths were rewound (outside the timed region)
                gs.sync_lengths()
        flush_l2(flush)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        graph_steps[j].run()
        torch.cuda.synchronize()
        t1 = time.perf_counter()
        if i >= args.warmup:
            e2e_s.append(t1 - t0)
            e2e_bytes += (CTX + j + 1) * BATCH * HKV * BYTES_PER_TOKEN_HEAD
    # Where the end-to-end time goes, from a separate pass of the same steps
    # (events would perturb the timed one): device time of the graph replay
    # (copies + kernels) against the host's wall time around replay + wait.
    bd_wall, bd_dev = [], []
    n_bd = min(EPISODE, max(8, args.steps // 4))
    lens.copy_(ctx_lens)
    for gs in graph_steps:
        gs.sync_lengths()
    for j in range(n_bd):
        flush_l2(flush)
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        ea.record(stream)
        graph_steps[j].run()
        eb.record(stream)
        torch.cuda.synchronize()
        t1 = time.perf_counter()
        bd_wall.append((t1 - t0) * 1e6)
        bd_dev.append(ea.elapsed_time(eb) * 1e3)
    assert cache.device_status() == 0, "device status %d after the graph steps" % cache.device_status()
    kernels_us = statistics.mean(step_ms) * 1e3
    e2e_breakdown = {"steps": n_bd, "host_wall_us": statistics.mean(bd_wall),
                     "graph_device_us": statistics.mean(bd_dev), "kernels_device_us": kernels_us,
                     "copies_and_gaps_us": statistics.mean(bd_dev) - kernels_us,
                     "host_launch_and_wait_us": statistics.mean(bd_wall) - statistics.mean(bd_dev)}
    h2d = hk[0].numel() * 2 + hv[0].numel() * 2 + hq[0].numel() * 2
    d2h = hout.numel() * 4

    res = {"total_ms": total_ms, "bytes": bytes_total, "split_ms": split_ms, "attn_ms": attn_ms,
           "split_bytes": split_bytes,
           "append1_ms": append1_ms, "step_ms": step_ms, "clocks": clocks.summary(),
           "append": append_info, "e2e_s": sum(e2e_s), "e2e_bytes": e2e_bytes, "e2e_breakdown": e2e_breakdown,
           "h2d": h2d, "d2h": d2h, "tokens": tokens}
    return res


# ---------------------------------------------------------------------------
# XQuant rematerialization leg: 8 sequences x 16384 positions, hidden 4096,
# 8 KV heads / 32 query heads. One step = kvq_remat_kv over the whole context
# (dequantize X, tensor-core GEMM, RoPE) + decode attention over the bf16 K/V.
# ---------------------------------------------------------------------------
XQ_T, XQ_HIDDEN, XQ_H, XQ_HQ = 16384, 4096, 8, 32


def run_remat(args, dev):
    import torch
    import bit_kv_cache_21_b200 as K

    B, T, hidden, H = args.remat_batch, XQ_T, XQ_HIDDEN, XQ_H
    XH = hidden // D
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    cache = K.KVCache(K.CacheSpec(B, XH, bits_k=4, group_k=128, capacity_tokens=T, with_v=False),
                      device=dev)
    lens = torch.zeros(B, dtype=torch.int32, device=dev)
    for b in range(B):   # X ~ N(0, 1) bf16, one sequence at a time
        x = torch.randn((T, XH, D), generator=gen, device=dev).to(torch.bfloat16)
        cu = torch.zeros(B + 1, dtype=torch.int32, device=dev)
        cu[b + 1:] = T
        K.quantize_append(cache.desc, x, None, cu, lens)
        del x
    w = (torch.randn((2 * H * D, hidden), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    q = torch.randn((B, XQ_HQ, D), generator=gen, device=dev).to(torch.bfloat16)
    cos, sin = K.rope_tables(T, D, 500000.0, device=dev)
    k_out = torch.empty((B, H, T, D), dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    desc = K.bf16_cache_desc(k_out, v_out, status)
    full = torch.full((B,), T, dtype=torch.int32, device=dev)
    ws = torch.empty(K.decode_workspace_size(desc, B, XQ_HQ, T), dtype=torch.uint8, device=dev)
    out = torch.empty((B, XQ_HQ, D), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(D)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        K.remat_kv(cache.desc, w, H, cos, sin, B, T, k_out, v_out)
        if evs:
            evs[1].record(stream)
        K.decode_attention(desc, q, full, T, scale, out=out, workspace=ws)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.remat_steps)]
    with ClockSampler(dev) as remat_clocks:   # a GEMM under the 1 kW cap: the clock it ran at
        for i in range(args.remat_steps):
            flush_l2(flush)
            step(evs[i])
        torch.cuda.synchronize()
    assert cache.device_status() == 0 and int(status[0]) == 0
    remat_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # the fused path: remat GEMM with attention in its epilogue (K/V never stored)
    fws = torch.empty(int(K.lib().kvq_remat_attention_workspace_size(B, XQ_HQ, T)), dtype=torch.uint8,
                      device=dev)
    fout = torch.empty_like(out)
    fused_ms = []
    for i in range(args.warmup + args.remat_steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        K.remat_attention(cache.desc, w, H, cos, sin, B, T, q, scale, out=fout, workspace=fws)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            fused_ms.append(e0.elapsed_time(e1))
    assert cache.device_status() == 0
    fused_diff = float((fout - out).abs().max())
    fused = statistics.mean(fused_ms)
    flops = 2.0 * B * T * (2 * H * D) * hidden
    kv_bytes = 2.0 * B * H * T * D * 2
    peak_b, peak_s, kind = tensor_peaks()
    tflops = flops / (remat_ms * 1e-3) / 1e12
    return {"workload": "xquant: %d seqs x %d positions, hidden %d, X INT4 g128, W_k/W_v %dx%d "
                        "bf16, RoPE theta 500000, then GQA decode attention %d q / %d kv heads "
                        "over the bf16 K/V" % (B, T, hidden, hidden, H * D, XQ_HQ, H),
            "steps": args.remat_steps, "ms_per_step": remat_ms + attn_ms,
            "remat": {"kernel": "remat_kernel", "bound": "tensor", "ms": remat_ms,
                      "flops_per_launch": flops, "achieved": tflops, "unit": "TFLOP/s",
                      "peak": peak_b, "peak_kind": kind + " bf16 burst", "frac": tflops / peak_b,
                      "frac_of_sustained": tflops / peak_s},
            "attention_bf16": {"ms": attn_ms, "bytes": kv_bytes,
                               "GBps": kv_bytes / (attn_ms * 1e-3) / 1e9},
            "fused_remat_attention": {"kernel": "remat_kernel<FUSED> + remat_merge_kernel", "ms": fused,
                                      "achieved": flops / (fused * 1e-3) / 1e12, "unit": "TFLOP/s",
                                      "frac": flops / (fused * 1e-3) / 1e12 / peak_b,
                                      "speedup_vs_unfused": (remat_ms + attn_ms) / fused,
                                      "max_abs_diff_vs_unfused": fused_diff},
            "clocks": remat_clocks.summary(),
            "gpu_launches_per_step": 4}


# ---------------------------------------------------------------------------
# Other decode workloads (extra objects of the default line; --part selects one)
# ---------------------------------------------------------------------------
def _synthetic_kv(gen, n_tok, H, dev, torch, seed):
    """bf16 K (4 outlier channels x20, drawn as the workload recipe does) and
    V ~ N(0, 1), [n_tok][H][128]."""
    import workloads as W
    ch = torch.as_tensor(W.outlier_channels(W.rng(seed)), dtype=torch.long, device=dev)
    k = torch.randn((n_tok, H, D), generator=gen, device=dev)
    k[:, :, ch] *= 20.0
    v = torch.randn((n_tok, H, D), generator=gen, device=dev)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def _time_steps(torch, stream, flush, n_warm, n_steps, step):
    """Run n_warm + n_steps steps (L2 flushed before each), timing append and
    attention of the last n_steps with events. step(i, evs) records evs[0..2]."""
    evs = []
    for i in range(n_warm + n_steps):
        flush_l2(flush)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(i, e)
        if i >= n_warm:
            evs.append(e)
    torch.cuda.synchronize()
    app = [e[0].elapsed_time(e[1]) for e in evs]
    att = [e[1].elapsed_time(e[2]) for e in evs]
    return app, att


def run_long_int2(args, dev):
    """1 sequence at 131072 positions, 32 q / 8 KV heads, KIVI INT2: keys per
    channel in 128-token blocks, values per token in groups of 32, a 128-token
    bf16 window. A step appends one token and attends over the whole context."""
    import torch
    import bit_kv_cache_21_b200 as K
    H, HQ_, T_END, R = 8, 32, 131072, 128
    n_steps, n_warm = 40, 3
    T0 = T_END - (n_steps + n_warm)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    spec = K.CacheSpec(1, H, bits_k=2, bits_v=2, group_k=R, group_v=32, per_channel_k=True,
                       residual_len=R, capacity_tokens=T_END + R)
    cache = K.KVCache(spec, device=dev)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    k, v = _synthetic_kv(gen, T0, H, dev, torch, 3)
    K.quantize_append(cache.desc, k, v, torch.tensor([0, T0], dtype=torch.int32, device=dev), lens)
    del k, v
    ks, vs = _synthetic_kv(gen, n_steps + n_warm, H, dev, torch, 3)
    q = torch.randn((1, HQ_, D), generator=gen, device=dev).to(torch.bfloat16)
    cu_one = torch.tensor([0, 1], dtype=torch.int32, device=dev)
    ws = torch.empty(K.decode_workspace_size(cache.desc, 1, HQ_, T_END), dtype=torch.uint8, device=dev)
    out = torch.empty((1, HQ_, D), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(D)

    def step(i, e):
        e[0].record(stream)
        K.quantize_append(cache.desc, ks[i:i + 1], vs[i:i + 1], cu_one, lens)
        e[1].record(stream)
        K.decode_attention(cache.desc, q, lens, T_END, scale, out=out, workspace=ws)
        e[2].record(stream)

    app, att = _time_steps(torch, stream, flush, n_warm, n_steps, step)
    assert cache.device_status() == 0
    nbytes = []
    for i in range(n_warm, n_warm + n_steps):
        T = T0 + i + 1
        Tq = R * ((T - 1) // R)
        nbytes.append(H * (Tq * (32 + 32 + 16) + (Tq // R) * D * 4 + (T - Tq) * 2 * D * 2))
    mb = statistics.mean(nbytes)
    return {"workload": "long_int2: 1 seq, 32 q / 8 kv heads, context %d..%d, K INT2 per channel "
                        "(128-token blocks), V INT2 per token (g32), 128-token bf16 window"
                        % (T0 + n_warm + 1, T_END),
            "steps": n_steps, "bytes_per_step": mb,
            "append_ms": statistics.mean(app), "attention_ms": statistics.mean(att),
            "attention_GBps": mb / (statistics.mean(att) * 1e-3) / 1e9,
            "attention_frac_of_hbm": mb / (statistics.mean(att) * 1e-3) / 1e9 / peaks()[0],
            "step_GBps": mb / ((statistics.mean(app) + statistics.mean(att)) * 1e-3) / 1e9}


def run_long_int2_sharded(args, dev, rank, world):
    """The long_int2 cache split by token range over the ranks (one GPU each):
    rank r holds its run of 256-token blocks of the 131072-token sequence in
    its own KIVI INT2 cache. A step is the sharded decode: split-K and partial
    merge on every rank, one NCCL all-gather of the partials (130 floats per
    query head), the cross-rank merge. Strong scaling: the sequence is fixed,
    each rank reads 1/world of it. Time = max over ranks of the mean step."""
    import torch
    import bit_kv_cache_21_b200 as K
    from bit_kv_cache_21_b200.sharded import decode_attention_sharded, shard_token_range
    H, HQ_, T_END, R = 8, 32, 131072, 128
    n_steps, n_warm = 20, 3
    lo, hi = shard_token_range(T_END, world, rank, 256)
    T_loc = hi - lo
    cap = max(256, -(-T_loc // 256) * 256)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3 + rank)
    spec = K.CacheSpec(1, H, bits_k=2, bits_v=2, group_k=R, group_v=32, per_channel_k=True,
                       residual_len=R, capacity_tokens=cap)
    cache = K.KVCache(spec, device=dev)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    if T_loc:
        k, v = _synthetic_kv(gen, T_loc, H, dev, torch, 3)
        K.quantize_append(cache.desc, k, v, torch.tensor([0, T_loc], dtype=torch.int32, device=dev), lens)
        del k, v
    qgen = torch.Generator(device=dev)
    qgen.manual_seed(33)  # the same query on every rank
    q = torch.randn((1, HQ_, D), generator=qgen, device=dev).to(torch.bfloat16)
    ws = torch.empty(K.decode_workspace_size(cache.desc, 1, HQ_, cap), dtype=torch.uint8, device=dev)
    out = torch.empty((1, HQ_, D), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(D)
    times = []
    for i in range(n_warm + n_steps):
        flush_l2(flush)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        decode_attention_sharded(cache.desc, q, lens, cap, scale, out=out, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= n_warm:
            times.append(e0.elapsed_time(e1))
    assert cache.device_status() == 0
    Tq = R * ((T_loc - 1) // R) if T_loc else 0
    nbytes = H * (Tq * (32 + 32 + 16) + (Tq // R) * D * 4 + (T_loc - Tq) * 2 * D * 2)
    ms = statistics.mean(times)
    if world > 1:
        t = torch.tensor([ms, float(nbytes)], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t[:1], op=torch.distributed.ReduceOp.MAX)
        torch.distributed.all_reduce(t[1:], op=torch.distributed.ReduceOp.SUM)
        ms, nbytes = float(t[0]), float(t[1])
    return {"workload": "long_int2 sharded by token range over %d GPU(s): 1 seq x 131072 tokens, "
                        "32 q / 8 kv heads, KIVI INT2, 128-token bf16 window on each rank" % world,
            "steps": n_steps, "bytes_per_step": nbytes, "attention_ms": ms,
            "attention_GBps": nbytes / (ms * 1e-3) / 1e9}


def run_append_hybrid(args, dev):
    """Bulk append of the llama8b-layer prefill (16 x 8192 tokens x 8 KV heads,
    K and V, bf16, INT4 g128, Hadamard(128) on K, x20 outlier key channels),
    plain and with InnerQ's hybrid groups; the mean of 3 timed appends after
    one warm-up, CUDA events."""
    import torch
    import bit_kv_cache_21_b200 as K
    S, H, T = 16, 8, 8192
    gen = torch.Generator(device=dev)
    gen.manual_seed(2)
    k, v = _synthetic_kv(gen, S * T, H, dev, torch, 2)
    cu = torch.arange(0, (S + 1) * T, T, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    for hyb in (False, True):
        cache = K.KVCache(K.CacheSpec(S, H, bits_k=4, bits_v=4, group_k=128, group_v=128,
                                      hadamard_block_k=128, capacity_tokens=T, hybrid=hyb), device=dev)
        ms = []
        for rep in range(4):
            lens = torch.zeros(S, dtype=torch.int32, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            K.quantize_append(cache.desc, k, v, cu, lens)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep > 0:
                ms.append(e0.elapsed_time(e1))
        assert cache.device_status() == 0
        res["hybrid" if hyb else "plain"] = {"ms": statistics.mean(ms),
                                             "tokens_per_s": S * T / (statistics.mean(ms) * 1e-3)}
        del cache
    return {"workload": "bulk prefill 16 x 8192 tokens x 8 KV heads, K and V, bf16, INT4 g128, "
                        "Hadamard(128) K, plain and hybrid groups", **res}


def _sweep_setup(dev, seed=6):
    """Shared data of the accuracy/cost sweeps: 16 seqs x 8 KV heads (32 q
    heads) x 4096 tokens of the outlier-key recipe, bf16, and decode attention
    over the same tokens kept in bf16 (the library's bits-16 mode)."""
    import torch
    import bit_kv_cache_21_b200 as K
    S, H, HQ_, T = 16, 8, 32, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    k, v = _synthetic_kv(gen, S * T, H, dev, torch, seed)               # [S*T][H][D]
    q = torch.randn((S, HQ_, D), generator=gen, device=dev).to(torch.bfloat16)
    kb = k.view(S, T, H, D).permute(0, 2, 1, 3).contiguous()            # [S][H][T][D]
    vb = v.view(S, T, H, D).permute(0, 2, 1, 3).contiguous()
    lens_full = torch.full((S,), T, dtype=torch.int32, device=dev)
    cu = torch.arange(0, (S + 1) * T, T, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    ref = K.decode_attention(K.bf16_cache_desc(kb, vb), q, lens_full, T, scale).double()
    return dict(S=S, H=H, HQ=HQ_, T=T, k=k, v=v, q=q, lens_full=lens_full, cu=cu, scale=scale, ref=ref)


def _sweep_row(spec_kw, d, dev, bytes_per_token_head, n_rep=5):
    """Append the sweep's tokens into a fresh cache of `spec_kw`, then decode;
    mean times over n_rep repetitions after one warm-up (L2 flushed before
    each timed launch), and the error of the attention against bf16."""
    import torch
    import bit_kv_cache_21_b200 as K
    S, H, HQ_, T = d["S"], d["H"], d["HQ"], d["T"]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    cache = K.KVCache(K.CacheSpec(S, H, capacity_tokens=T, **spec_kw), device=dev)
    ws = torch.empty(K.decode_workspace_size(cache.desc, S, HQ_, T), dtype=torch.uint8, device=dev)
    out = torch.empty((S, HQ_, D), dtype=torch.float32, device=dev)
    app_ms, att_ms = [], []
    for rep in range(n_rep + 1):
        lens = torch.zeros(S, dtype=torch.int32, device=dev)
        flush_l2(flush)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        K.quantize_append(cache.desc, d["k"], d["v"], d["cu"], lens)
        e[1].record(stream)
        flush_l2(flush)
        e[2].record(stream)
        K.decode_attention(cache.desc, d["q"], d["lens_full"], T, d["scale"], out=out, workspace=ws)
        e[3].record(stream)
        torch.cuda.synchronize()
        if rep > 0:  # the first repetition warms up
            app_ms.append(e[0].elapsed_time(e[1]))
            att_ms.append(e[2].elapsed_time(e[3]))
    assert cache.device_status() == 0
    sym_fraction = None
    if spec_kw.get("hybrid"):
        # groups that took the symmetric grid store z = -2^(bits-1) s exactly
        n_sym = n_all = 0
        for t, bits in ((cache.k_sz, spec_kw["bits_k"]), (cache.v_sz, spec_kw["bits_v"])):
            sz = t.view(torch.float16).view(-1, 2).float()
            n_sym += int(((sz[:, 1] == -(1 << (bits - 1)) * sz[:, 0]) & (sz[:, 0] != 0)).sum())
            n_all += sz.shape[0]
        sym_fraction = n_sym / n_all
    diff = out.double() - d["ref"]
    row = {"attn_rel_l2": float(diff.norm() / d["ref"].norm()),
           "attn_max_abs": float(diff.abs().max()),
           "append_ms": statistics.mean(app_ms),
           "append_tokens_per_s": S * T / (statistics.mean(app_ms) * 1e-3),
           "decode_ms": statistics.mean(att_ms),
           "decode_GBps": S * H * T * bytes_per_token_head / (statistics.mean(att_ms) * 1e-3) / 1e9}
    if sym_fraction is not None:
        row["symmetric_group_fraction"] = sym_fraction
    del cache, ws
    return row


SWEEP_WORKLOAD = ("16 seqs x 8 kv / 32 q heads x 4096 tokens, bf16 K with 4 outlier channels x20; "
                  "error of decode attention against attention over the same tokens in bf16")


def run_rotation_sweep(args, dev):
    """Accuracy and cost of the key rotation: no rotation, block-diagonal
    Hadamard with blocks of 32, 64 and 128 channels, each with and without
    QuaRot's random signs, and the 128 block with a 64-token attention-sink
    window; INT4 g128 K and V."""
    import torch
    import workloads as W
    d = _sweep_setup(dev)
    signs = torch.from_numpy(W.hadamard_signs(6)).to(dev)
    rows = []
    configs = [(hb, sg, 0) for hb in (0, 32, 64, 128) for sg in ((False, True) if hb else (False,))]
    configs.append((128, False, 64))   # plus InnerQ's attention-sink window of 64 bf16 tokens
    for hb, use_signs, sink in configs:
        kw = dict(bits_k=4, bits_v=4, group_k=128, group_v=128, hadamard_block_k=hb,
                  hadamard_signs=signs if use_signs else None, sink_len=sink)
        row = {"hadamard_block": hb, "random_signs": use_signs, "sink_tokens": sink}
        row.update(_sweep_row(kw, d, dev, BYTES_PER_TOKEN_HEAD))
        rows.append(row)
    return {"workload": "rotation sweep: " + SWEEP_WORKLOAD + "; INT4 g128 K and V", "rows": rows}


def _layout_bytes(bits, per_channel, G, R):
    """Stored bytes of one tensor per (token, head): codes plus the share of
    the 4-byte (scale, zero) pairs (per token: D/G of them; per channel: D per
    R-token block)."""
    return D * bits // 8 + (D * 4 // R if per_channel else (D // G) * 4)


def run_grouping_sweep(args, dev):
    """Accuracy and cost of the grouping axes with a 128-token bf16 window, no
    rotation: token-wise groups for both tensors; KIVI's keys per channel with
    values per token; InnerQ's keys grouped along channels (per token) with
    values grouped along tokens (per channel); both per channel. INT4 with
    128-wide groups and INT2 with 32-wide token groups. The KIVI and InnerQ
    layouts also run with InnerQ's hybrid symmetric/asymmetric groups."""
    d = _sweep_setup(dev)
    R = 128
    rows = []
    for bits, G in ((4, 128), (2, 32)):
        for pk, pv, hyb, name in ((False, False, False, "token/token"),
                                  (True, False, False, "KIVI: channel/token"),
                                  (True, False, True, "KIVI: channel/token, hybrid"),
                                  (False, True, False, "InnerQ: token/channel"),
                                  (False, True, True, "InnerQ: token/channel, hybrid"),
                                  (True, True, False, "channel/channel")):
            kw = dict(bits_k=bits, bits_v=bits, group_k=R if pk else G, group_v=R if pv else G,
                      per_channel_k=pk, per_channel_v=pv, residual_len=R, hybrid=hyb)
            bph = _layout_bytes(bits, pk, G, R) + _layout_bytes(bits, pv, G, R)
            row = {"bits": bits, "token_group": G, "keys": "channel" if pk else "token",
                   "values": "channel" if pv else "token", "hybrid": hyb, "layout": name,
                   "bytes_per_token_head": bph}
            row.update(_sweep_row(kw, d, dev, bph))
            rows.append(row)
    return {"workload": "grouping sweep: " + SWEEP_WORKLOAD + "; residual window 128 bf16 tokens; "
                        "keys / values grouped per token or per channel (128-token blocks)",
            "rows": rows}


def run_paged_mix(args, dev):
    """64 sequences, lognormal lengths (median 4096, sigma 1, clipped to
    [1024, 32768]), 16-token pages, INT4 g128, Hadamard keys. A step appends a
    512-token chunk to 8 sequences and one token to the other 56, then attends
    over all 64; every 4 steps the lengths are rewound outside the timing."""
    import numpy as np
    import torch
    import bit_kv_cache_21_b200 as K
    import workloads as W
    H, HQ_, PS, EP = 8, 32, 16, 4
    n_steps, n_warm = 20, 4
    pre = W.paged_lengths(4)
    new = np.array([512] * 8 + [1] * 56)
    final = pre + EP * new
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    spec = K.CacheSpec(64, H, hadamard_block_k=128, paged=True, page_size=PS,
                       max_pages_per_seq=int(final.max()) // PS + 1,
                       num_pages=int(sum(final // PS + 1)))
    cache = K.KVCache(spec, device=dev)
    need = [(int(t) + PS - 1) // PS for t in final]
    free = np.random.default_rng(4).permutation(spec.num_pages)
    bt = np.full((64, spec.max_pages_per_seq), -1, np.int32)
    i0 = 0
    for s_, n in enumerate(need):
        bt[s_, :n] = free[i0:i0 + n]
        i0 += n
    cache.block_table.copy_(torch.from_numpy(bt))
    lens = torch.zeros(64, dtype=torch.int32, device=dev)
    cu_pre = torch.from_numpy(np.concatenate([[0], np.cumsum(pre)]).astype(np.int32)).to(dev)
    k, v = _synthetic_kv(gen, int(pre.sum()), H, dev, torch, 4)
    K.quantize_append(cache.desc, k, v, cu_pre, lens)
    del k, v
    pre_lens = lens.clone()
    n_new = int(new.sum())
    cu_new = torch.from_numpy(np.concatenate([[0], np.cumsum(new)]).astype(np.int32)).to(dev)
    step_kv = [_synthetic_kv(gen, n_new, H, dev, torch, 4) for _ in range(EP)]
    q = torch.randn((64, HQ_, D), generator=gen, device=dev).to(torch.bfloat16)
    max_len = int(final.max())
    ws = torch.empty(K.decode_workspace_size(cache.desc, 64, HQ_, max_len), dtype=torch.uint8, device=dev)
    out = torch.empty((64, HQ_, D), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(D)

    def step(i, e):
        j = i % EP
        if j == 0:
            lens.copy_(pre_lens)
        kk, vv = step_kv[j]
        e[0].record(stream)
        K.quantize_append(cache.desc, kk, vv, cu_new, lens)
        e[1].record(stream)
        K.decode_attention(cache.desc, q, lens, max_len, scale, out=out, workspace=ws)
        e[2].record(stream)

    app, att = _time_steps(torch, stream, flush, n_warm, n_steps, step)
    assert cache.device_status() == 0
    nbytes = [float(sum(pre + ((i % EP) + 1) * new)) * H * BYTES_PER_TOKEN_HEAD
              for i in range(n_warm, n_warm + n_steps)]
    mb = statistics.mean(nbytes)
    appended = n_new * H * 2 * (D * 2 + D // 2 + 4)
    return {"workload": "paged_mix: 64 seqs, lognormal lengths (median 4096, sigma 1) %d..%d tokens, "
                        "16-token pages, INT4 g128, Hadamard K; per step 8 x 512 + 56 x 1 appended"
                        % (int(pre.min()), int(final.max())),
            "steps": n_steps, "bytes_per_step": mb,
            "append_ms": statistics.mean(app), "append_tokens_per_s": n_new / (statistics.mean(app) * 1e-3),
            "append_GBps": appended / (statistics.mean(app) * 1e-3) / 1e9,
            "attention_ms": statistics.mean(att),
            "attention_GBps": mb / (statistics.mean(att) * 1e-3) / 1e9,
            "attention_frac_of_hbm": mb / (statistics.mean(att) * 1e-3) / 1e9 / peaks()[0],
            "step_GBps": mb / ((statistics.mean(app) + statistics.mean(att)) * 1e-3) / 1e9}


def cpu_units(n_units, seed=0):
    """Oracle-side cache state of n_units (sequence, KV head) units of the
    workload at context 8193: the oracle's own packed K/V and 4 queries."""
    import oracle
    import workloads as W
    T = CTX + 1
    g = W.rng(seed + 77)
    ch = W.outlier_channels(g)
    units = []
    for _ in range(n_units):
        kh = W.finish(W.keys(g, (T, D), ch), "bf16")
        vh = W.finish(W.normal(g, (T, D)), "bf16")
        q = W.finish(W.normal(g, (4, D)), "bf16")
        units.append((oracle.quantize_tokens(kh, 128, 128, 4), oracle.quantize_tokens(vh, 0, 128, 4), q))
    return units


def cpu_time(units, budget_s):
    """The oracle (float64, one thread) on whole units, cycling through them
    until budget_s of work: dequantize the unit's packed K and V, rotate the
    queries and attend. Returns (GB/s of packed bytes, units done, seconds)."""
    import oracle
    done, t_used, nbytes = 0, 0.0, 0
    while done == 0 or t_used < budget_s:
        (kc, ksz), (vc, vsz), q = units[done % len(units)]
        t0 = time.perf_counter()
        kd = oracle.dequant_tokens(kc, ksz, 128, 4)
        vd = oracle.dequant_tokens(vc, vsz, 128, 4)
        oracle.decode_attention_gqa(q, kd[None], vd[None], 1.0 / math.sqrt(D), rotate_q_block=128)
        t_used += time.perf_counter() - t0
        done += 1
        nbytes += kc.shape[0] * BYTES_PER_TOKEN_HEAD
    return nbytes / t_used / 1e9, done, t_used


_CPU_STATE = {}


def _cpu_worker_init(barrier, counter, n_units):
    """Spawned host process of the all-core oracle baseline: its own units,
    built once (seeded by the order the processes start in)."""
    with counter.get_lock():
        idx = counter.value
        counter.value += 1
    _CPU_STATE["barrier"] = barrier
    _CPU_STATE["units"] = cpu_units(n_units, seed=100 + idx)


def _cpu_worker(budget_s):
    """The oracle on this process's units for budget_s (at least one unit),
    started once every process has reached the barrier."""
    units = _CPU_STATE["units"]
    _CPU_STATE["barrier"].wait()
    t0 = time.perf_counter()
    gbs, done, secs = cpu_time(units, budget_s)
    t1 = time.perf_counter()
    return gbs * secs * 1e9, done, t0, t1   # packed bytes, units, wall interval


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_pool(n_units):
    """One spawned process per host core (spawned, not forked: the parent may
    hold a CUDA context). Each map over `cores` tasks runs one task per process:
    a process holds its task at the barrier until all have arrived."""
    import multiprocessing as mp
    n = cpu_cores()
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(n, timeout=600)
    counter = ctx.Value("i", 0)
    return ctx.Pool(n, initializer=_cpu_worker_init, initargs=(barrier, counter, n_units)), n


def cpu_time_all_cores(budget_s, n_units=2):
    """The oracle on every host core at once for about budget_s. Returns
    (total packed GB/s = bytes of all processes / wall time of the concurrent
    run, units done, wall seconds, cores)."""
    pool, n = cpu_pool(n_units)
    with pool:
        res = pool.map(_cpu_worker, [budget_s] * n, chunksize=1)
    nbytes = sum(r[0] for r in res)
    wall = max(r[3] for r in res) - min(r[2] for r in res)
    return nbytes / wall / 1e9, sum(r[1] for r in res), wall, n


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=640)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--part", default="all",
                    choices=["all", "decode", "remat", "long_int2", "paged_mix", "rotation_sweep",
                             "grouping_sweep", "long_int2_sharded", "append_hybrid"],
                    help="run one leg alone: decode (the metric's step), remat, long_int2, "
                         "paged_mix, rotation_sweep, grouping_sweep, long_int2_sharded or "
                         "append_hybrid (all but decode print their own line)")
    ap.add_argument("--remat-batch", type=int, default=8)
    ap.add_argument("--remat-steps", type=int, default=10)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The reference arm is the CPU oracle as it stands (the pages ship no
        # code), on every host core: one spawned process per core, each step
        # one (sequence, KV head) unit per process. Rank 0 alone runs it.
        if rank != 0:
            return
        pool, n = cpu_pool(1)
        vals, n_units, secs = [], 0, 0.0
        with pool:
            for i in range(args.warmup + args.steps):
                res = pool.map(_cpu_worker, [0.0] * n, chunksize=1)
                wall = max(r[3] for r in res) - min(r[2] for r in res)
                if i >= args.warmup:
                    vals.append(sum(r[0] for r in res) / wall / 1e9)
                    n_units += sum(r[1] for r in res)
                    secs += wall
        value = statistics.median(vals)
        sample = ("one (sequence, KV head) unit of the decode step at context 8193 per process per "
                  "step, %d processes (one per host core), %d steps, %d units (%.1f s of oracle work "
                  "wall): float64 dequantize + attention" % (n, args.steps, n_units, secs))
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": WORKLOAD},
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": n, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.part == "append_hybrid":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        leg = run_append_hybrid(args, dev)
        if rank == 0:
            print(json.dumps({"metric": "quantize-append tokens/s", "value": leg["hybrid"]["tokens_per_s"],
                              "unit": "tokens/s", "n_gpus": world, "higher_is_better": True,
                              "data": "synthetic", "config": {"workload": leg["workload"]},
                              args.part: leg}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.part == "long_int2_sharded":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        leg = run_long_int2_sharded(args, dev, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "decode-attn packed-KV GB/s (token-range sharded)",
                              "value": leg["attention_GBps"], "unit": "GB/s", "n_gpus": world,
                              "higher_is_better": True, "scaling": "strong", "data": "synthetic",
                              "config": {"workload": leg["workload"]}, args.part: leg}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.part in ("long_int2", "paged_mix"):
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        leg = (run_long_int2 if args.part == "long_int2" else run_paged_mix)(args, dev)
        if rank == 0:
            print(json.dumps({"metric": "decode-attn packed-KV GB/s", "value": leg["attention_GBps"],
                              "unit": "GB/s", "n_gpus": world, "higher_is_better": True,
                              "data": "synthetic", "config": {"workload": leg["workload"]},
                              args.part: leg}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.part in ("rotation_sweep", "grouping_sweep"):
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        rot = args.part == "rotation_sweep"
        sw = (run_rotation_sweep if rot else run_grouping_sweep)(args, dev)
        if rank == 0:
            print(json.dumps({"metric": "decode-attn error vs bf16 and cost per " +
                                        ("key rotation" if rot else "grouping layout"),
                              "n_gpus": world, "data": "synthetic",
                              "config": {"workload": sw["workload"]}, args.part: sw}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.part == "remat":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        rr = run_remat(args, dev)
        if rank == 0:
            print(json.dumps({"metric": "remat TFLOP/s (tensor cores)", "value": rr["remat"]["achieved"],
                              "unit": "TFLOP/s", "n_gpus": world, "higher_is_better": True,
                              "data": "synthetic", "dtype": "bf16 MMA, fp32 accumulate",
                              "config": {"workload": rr["workload"]}, "remat_leg": rr}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    res = run_ours(args, rank, world, local_rank)
    rr = run_remat(args, torch.device("cuda", local_rank)) if args.part == "all" else None
    li = run_long_int2(args, torch.device("cuda", local_rank)) if args.part == "all" else None
    pm = run_paged_mix(args, torch.device("cuda", local_rank)) if args.part == "all" else None
    sw = run_rotation_sweep(args, torch.device("cuda", local_rank)) if args.part == "all" else None
    gs = run_grouping_sweep(args, torch.device("cuda", local_rank)) if args.part == "all" else None

    # max over ranks of the device time; bytes summed over ranks
    total_ms, total_bytes, e2e_s, e2e_bytes = res["total_ms"], res["bytes"], res["e2e_s"], res["e2e_bytes"]
    if world > 1:
        t = torch.tensor([total_ms, e2e_s], dtype=torch.float64, device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        b = torch.tensor([float(total_bytes), float(e2e_bytes)], dtype=torch.float64, device="cuda")
        torch.distributed.all_reduce(b, op=torch.distributed.ReduceOp.SUM)
        total_ms, e2e_s = float(t[0]), float(t[1])
        total_bytes, e2e_bytes = float(b[0]), float(b[1])
    if rank == 0:
        hbm_peak, peak_kind = peaks()
        value = total_bytes / (total_ms * 1e-3) / 1e9
        split_mean_ms = statistics.mean(res["split_ms"])
        bytes_per_launch = res["split_bytes"]
        achieved = bytes_per_launch / (split_mean_ms * 1e-3) / 1e9
        traffic = traffic_per_launch()
        cpu_gbs, cpu_done, cpu_s = cpu_time(cpu_units(16), args.cpu_budget)
        all_gbs, all_done, all_s, n_cores = cpu_time_all_cores(args.cpu_budget)
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4 packed K/V, fp32 math", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": BATCH * world, "seq_len": CTX,
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": "flushed between steps (256 MiB write, then read back: cold, clean L2)",
                       "pct_of_8TBs": 100.0 * value / NOMINAL_HBM_GBS},
            "roofline": {"kernel": "decode_splitk_kernel", "bound": "hbm", "achieved": achieved,
                         "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": traffic,
                         "bytes_per_launch": bytes_per_launch, "ms_per_launch": split_mean_ms},
            "breakdown_ms": {"append": statistics.mean(res["append1_ms"]),
                             "attention_splitk_and_merge": statistics.mean(res["attn_ms"])},
            "append": res["append"],
            "cpu_baseline": {"value": all_gbs, "unit": "GB/s", "cores": n_cores, "kind": "oracle",
                             "sample": "%d (sequence, KV head) units of the decode step at context 8193 "
                                       "on %d host processes at once (%.1f s wall), each cycling over "
                                       "2 units of its own: float64 dequantize + attention"
                                       % (all_done, n_cores, all_s),
                             "single_thread": {"value": cpu_gbs, "unit": "GB/s", "cores": 1,
                                               "sample": "%d units cycling over 16 (%.1f s)"
                                                         % (cpu_done, cpu_s)}},
            "e2e": {"value": e2e_bytes / e2e_s / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                    "breakdown": res["e2e_breakdown"]},
            "gpu_launches": 4 * args.steps,   # append, advance lengths, split-K, merge
            "clocks": res["clocks"],
        }
        if rr is not None:
            line["xquant_remat"] = rr
        if li is not None:
            line["long_int2"] = li
        if pm is not None:
            line["paged_mix"] = pm
        if sw is not None:
            line["rotation_sweep"] = sw
        if gs is not None:
            line["grouping_sweep"] = gs
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
