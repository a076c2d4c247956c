"""Throughput of the Q4 paged KV-cache path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl q4kv|reference]

One step is one pass of the whole path over one batch of synthetic input:
for every layer, quantise all K/V tokens into the paged 4-bit pool (K
Walsh-Hadamard rotated), apply the workload's eviction / mixed-width steps,
then run split-K paged GQA decode attention for the batch.  The default
workload is the largest single-GPU configuration: the Qwen2.5-14B-shaped
eviction-masked cache (48 layers, 40 query / 8 KV heads, head_dim 128,
32 sessions x 16384 tokens, fp16 input, 60 % of slots remapped to the
sentinel), all 48 layers resident in HBM (~132 GB).

Printed (rank 0, one JSON line): value = algorithmic HBM bytes of the whole
step (quantise: read K/V, write codes + scale/zero; decode: read codes +
scale/zero + mask of every live block) / step time, in GB/s, summed over
ranks; the metric's parts (decode GB/s, its fraction of HBM and KV tokens/s;
quantise GB/s); per-kernel CUDA-event times; the roofline of the dominant
kernel and of both kernels; an end-to-end number through host buffers; the
CPU oracle on a bounded sample, on one thread and on all host cores.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Q4 paged decode-attn HBM GB/s (% of ~8 TB/s), KV tokens/s; quantize GB/s"

# The arithmetic the path computes in: the encoder is binary32 (rotation,
# group statistics, correctly rounded quotients) producing 4/8-bit codes with
# fp16 scale/zero; decode runs keys as u4/u8 codes x s8 query digits on int8
# MMAs (exact int32), values as fp16 MMAs with fp16 weights, both
# accumulating in fp32; softmax and merge in fp32.
DTYPE_LABEL = "int8 MMA (u4/u8 codes x s8 query digits, s32 acc) + fp16 MMA (f32 acc); encoder f32"


# ---------------------------------------------------------------------------
# workload description (shared by both arms)
# ---------------------------------------------------------------------------

def workload_by_name(name):
    from decode_attention_q4kv_b200 import workloads as W
    if name.startswith("sweep:"):
        _, b, c = name.split(":")
        return W.sweep_point(int(b), int(c))
    aliases = {"gemma": W.GEMMA3_12B, "tiny": W.TINY, "mixed": W.LLAMA31_8B_MIXED,
               "evict": W.QWEN25_14B_EVICT}
    if name in aliases:
        return aliases[name]
    return W.WORKLOADS[name]


def bytes_per_layer(w, fp8=False):
    """Algorithmic HBM bytes of one layer: (quantise, decode)."""
    in_elem = 2
    vec = w.head_dim
    ng = vec // 64
    n_tok = w.prefill_tokens or w.n_tokens
    q4_row = vec // 2 + ng * 4          # codes + (scale, zero) of one (token, head), one tensor
    q8_row = vec + ng * 4
    n_q8 = w.n_q8_blocks
    n_blocks = w.n_blocks
    frac8 = n_q8 / n_blocks if n_blocks else 0.0
    row = (1 - frac8) * q4_row + frac8 * q8_row
    if fp8:                              # the FP8 comparison cache: one byte per value, no params
        row = vec
    quant = n_tok * w.n_kv_heads * (2 * vec * in_elem + 2 * row)
    if w.q8_fraction and not fp8:
        quant += n_tok * w.n_kv_heads * vec * in_elem        # mean |K| pass reads K once more
    dec_tok = w.batch * w.ctx
    decode = dec_tok * w.n_kv_heads * 2 * row + n_blocks * 32 + w.batch * w.blocks_per_seq * 4
    decode += w.batch * w.n_q_heads * vec * (in_elem + 4)
    return quant, decode


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class ClockSampler:
    """Polls NVML during the timed region (SM clock, throttle reasons)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period_s=0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = None
            props = torch.cuda.get_device_properties(index)
            try:       # CUDA and NVML number devices differently: match by UUID
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:        # no NVML: report that instead of clocks
            self.nvml, self.error = None, repr(e)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def result(self):
        if not self.nvml:
            return {"error": self.error}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons)}


class Job:
    """All layers of one workload resident on one GPU, ready to step."""

    def __init__(self, w, device, rank=0, layers=None, fp8=False, decode_kernel=1):
        import torch

        import decode_attention_q4kv_b200 as q4
        from decode_attention_q4kv_b200 import workloads as W

        self.w, self.dev, self.torch, self.q4, self.W = w, device, torch, q4, W
        if isinstance(layers, (list, tuple)):
            layer_ids = list(layers)
        else:
            layer_ids = list(range(layers or w.layers))
        self.layer_ids = layer_ids
        self.n_layers = len(layer_ids)
        n_tok = w.prefill_tokens or w.n_tokens
        n_pool = max(w.n_blocks, n_tok // 256) if w.permuted_pool else w.n_blocks
        self.fp8 = fp8
        self.n_q8 = n_pool if fp8 else w.n_q8_blocks
        self.n_q4 = n_pool - self.n_q8
        self.layers = []
        for l in layer_ids:
            lid = rank_layer_id(l, rank)
            k, v = W.kv_tokens(w, lid, n_tok, device)
            q = W.query(w, lid, device)
            pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, self.n_q4, self.n_q8, k_rotated=not fp8,
                               device=device, fp8=fp8)
            self.layers.append(dict(k=k, v=v, q=q, pool=pool,
                                    out=torch.empty((w.batch, w.n_q_heads, w.head_dim),
                                                    dtype=torch.float16, device=device)))
        if w.permuted_pool:
            self.tables = W.permuted_tables(w).to(device)
            self.prefill_ids = torch.arange(n_tok // 256, dtype=torch.int32, device=device)
        else:
            self.tables = W.identity_tables(w).to(device)
            self.prefill_ids = None
        self.ids = self.tables.reshape(-1).contiguous()
        self.lens = W.seq_lens(w).to(device)
        self.evict = W.evicted_slot_ids(w, W.identity_tables(w)).to(device) if w.evict_fraction else None
        self.plan = q4.DecodePlan(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.blocks_per_seq)
        self.plan.c.kernel = decode_kernel
        self.ws = self.plan.workspace(device)
        if w.permuted_pool:
            # fill the whole pool once by tiling the quantised prefill (setup, not timed)
            for L in self.layers:
                L["pool"].quantize(L["k"], L["v"], self.prefill_ids)
                self._tile(L["pool"], n_tok // 256)
        self.quant_bytes, self.decode_bytes = bytes_per_layer(w, fp8)
        self.launches_per_layer = 1 + 1 + (1 if self.plan.n_splits > 1 else 0)
        if w.q8_fraction and not fp8:
            self.launches_per_layer += 3
        if self.evict is not None:
            self.launches_per_layer += 1

    def _tile(self, pool, n_src):
        names = ("k_codes8", "v_codes8") if self.fp8 else ("k_codes4", "v_codes4", "k_params4", "v_params4")
        for name in names:
            t = getattr(pool, name)
            for s in range(n_src, t.shape[0], n_src):
                e = min(s + n_src, t.shape[0])
                t[s:e].copy_(t[: e - s])

    def quantize_layer(self, L, mark=None):
        w, q4 = self.w, self.q4
        if w.q8_fraction and not self.fp8:
            am = q4.block_absmean(L["k"])
            ids = q4.mixed_block_ids(am, self.n_q8, 0, self.n_q4)
            L["ids"] = ids
            # sequence b's i-th chunk lives in block ids[b * nb + i]
            L["tables"] = ids.view(w.batch, w.blocks_per_seq)
        elif self.prefill_ids is not None:
            ids = self.prefill_ids
        else:
            ids = self.ids
        L["pool"].quantize(L["k"], L["v"], ids)
        if mark is not None:
            mark.record()   # the encoder's span ends here; the remap of evicted slots follows
        if self.evict is not None:
            L["pool"].invalidate(self.evict)

    @property
    def ids_per_layer(self):
        return [L.get("ids") for L in self.layers]

    @property
    def last_ids(self):
        return getattr(self, "_last_ids", None if not self.w.q8_fraction else self.layers[0].get("ids"))

    @last_ids.setter
    def last_ids(self, v):
        self._last_ids = v

    def decode_layer(self, L):
        self.q4.decode_attention(L["pool"], L["q"], L.get("tables", self.tables), self.lens,
                                 plan=self.plan, workspace=self.ws, out=L["out"])

    def append_setup(self):
        """One new token per sequence (seeded), written over each sequence's last slot."""
        torch, W, w = self.torch, self.W, self.w
        kn, vn = W.random_small(w.batch, w.n_kv_heads, w.head_dim, w.dtype, seed=w.seed + 77)
        self.k_new = kn.view(w.batch, 1, w.n_kv_heads, w.head_dim).to(self.dev)
        self.v_new = vn.view(w.batch, 1, w.n_kv_heads, w.head_dim).to(self.dev)
        self.lens_before = (self.lens - 1).contiguous()
        # algorithmic bytes of one append: K/V rows read, codes and params written
        vec = 2 * w.head_dim * 2 + 2 * (w.head_dim // 2 + 4 * (w.head_dim // 64))
        self.append_bytes = w.batch * w.n_kv_heads * vec

    def append_layer(self, L):
        L["pool"].append(self.k_new, self.v_new, L.get("tables", self.tables), self.lens_before)

    def append_decode_layer(self, L):
        """The generation step as one call (q4kv_append_decode)."""
        self.q4.append_decode(L["pool"], self.k_new, self.v_new, L["q"], L.get("tables", self.tables),
                              self.lens_before, plan=self.plan, workspace=self.ws, out=L["out"])

    def step(self, events=None):
        for L in self.layers:
            if events is not None:
                e0, eq, e1, e2 = events.pop()
                e0.record()
            self.quantize_layer(L, eq if events is not None else None)
            if events is not None:
                e1.record()
            self.decode_layer(L)
            if events is not None:
                e2.record()

    @property
    def bytes_per_step(self):
        return self.n_layers * (self.quant_bytes + self.decode_bytes)


# ---------------------------------------------------------------------------
# multi-rank plumbing (weak scaling: every rank runs its own replica)
# ---------------------------------------------------------------------------

def rank_layer_id(layer: int, rank: int) -> int:
    """Input stream of `layer` on `rank`: ranks draw disjoint data."""
    return layer + 1000 * rank


def reduce_max(value: float, device) -> float:
    """Max of `value` over all ranks of the default process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def check_world(gpus: int, world: int) -> None:
    """--gpus N must match the launch: one process per GPU (torchrun for N > 1)."""
    if gpus != world:
        sys.stderr.write(f"bench.py: --gpus {gpus} but WORLD_SIZE is {world}; launch N > 1 ranks with "
                         f"python -m torch.distributed.run --nproc-per-node {gpus} bench.py --gpus {gpus}\n")
        sys.exit(2)


def job_throughput(world: int, bytes_per_step: float, steps: int, elapsed_s: float) -> float:
    """Whole-job GB/s: every rank moved bytes_per_step per step; time = slowest rank."""
    return world * bytes_per_step * steps / elapsed_s / 1e9


# Files whose contents decide a kernel's DRAM traffic per launch: its own
# source, the shared device headers and the ABI header; for decode also the
# host code that picks the split count (the partials it writes depend on it).
_CSRC = os.path.join("decode_attention_q4kv_b200", "csrc")
KERNEL_SOURCES = {
    "quantize": ("quantize.cu", "encode.cuh", "async_copy.cuh", "q4kv_internal.cuh"),
    "decode": ("decode_tc.cu", "decode.cu", "api.cu", "encode.cuh", "async_copy.cuh", "q4kv_internal.cuh"),
}


def sources_digest(kernel=None):
    """Digest of one kernel's sources (KERNEL_SOURCES), or of every file under csrc/."""
    names = KERNEL_SOURCES[kernel] if kernel else sorted(os.listdir(os.path.join(ROOT, _CSRC)))
    paths = [os.path.join(ROOT, _CSRC, n) for n in names]
    if kernel:
        paths.append(os.path.join(ROOT, "include", "q4kv.h"))
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel_key, launches_scale=1.0):
    """DRAM bytes per launch from the committed ncu summary, if that kernel's sources still match."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except OSError:
        return None
    ent = t.get(kernel_key)
    if not ent or ent.get("sources") != sources_digest(kernel_key.split(":")[0]):
        return None
    return ent["dram_bytes_per_launch"] * launches_scale


def measured_peak(key, fallback):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = json.load(f).get(key)
        if v:
            return float(v), "measured"
    except OSError:
        pass
    return fallback, "fallback"


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    check_world(args.gpus, world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w = workload_by_name(args.workload)
    job = Job(w, dev, rank, args.layers, fp8=args.fp8, decode_kernel=args.decode_kernel)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        job.step()
    torch.cuda.synchronize()

    # timed region: K steps, events around every quantise and decode launch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
          for _ in range(args.steps * job.n_layers)]
    todo = list(reversed(ev))
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for _ in range(args.steps):
            job.step(todo)
        stop.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed = reduce_max(start.elapsed_time(stop) / 1e3, dev)
    q_ms = statistics.mean(a.elapsed_time(b) for a, b, _, _ in ev)
    inv_ms = statistics.mean(b.elapsed_time(c) for _, b, c, _ in ev)   # remap of evicted slots (0 if none)
    d_ms = statistics.mean(b.elapsed_time(c) for _, _, b, c in ev)

    # decode alone over all layers, cold (each layer's pool untouched for a full sweep)
    reps = max(3, min(20, args.steps))
    cold = []
    for _ in range(reps):
        for L in job.layers:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            job.decode_layer(L)
            b.record()
            cold.append((a, b))
    torch.cuda.synchronize()
    d_cold_ms = statistics.median(a.elapsed_time(b) for a, b in cold)

    # generation step: append one new token per sequence (over its last slot), then decode
    job.append_setup()
    gen = []
    for _ in range(reps):
        for L in job.layers:
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record()
            job.append_layer(L)
            b.record()
            job.decode_layer(L)
            c.record()
            gen.append((a, b, c))
    torch.cuda.synchronize()
    app_ms = statistics.median(a.elapsed_time(b) for a, b, _ in gen)
    sep_ms = statistics.median(a.elapsed_time(c) for a, _, c in gen)
    fused = []
    for _ in range(reps):
        for L in job.layers:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            job.append_decode_layer(L)
            b.record()
            fused.append((a, b))
    torch.cuda.synchronize()
    gen_ms = statistics.median(a.elapsed_time(b) for a, b in fused)

    paging = measure_paging(job, dev, reps, d_cold_ms)
    card = measure_card(job, dev, reps) if not args.fp8 else None
    # 2-bit blocks are read by plan kernel 1 only
    q2mix = measure_q2mix(job, dev, reps) if not args.fp8 and args.decode_kernel == 1 else None

    e2e = run_e2e(job, args, dev, world) if not args.no_e2e else None
    if world > 1:
        dist.barrier()

    if rank == 0:
        peak, peak_src = measured_peak("hbm_gbs", 6650.0)
        q_gbps = job.quant_bytes / (q_ms * 1e-3) / 1e9
        d_gbps = job.decode_bytes / (d_ms * 1e-3) / 1e9
        d_cold_gbps = job.decode_bytes / (d_cold_ms * 1e-3) / 1e9
        kv_tok = w.batch * w.ctx * w.n_kv_heads
        dominant = "quantize" if q_ms >= d_ms else "decode"
        roofs = {
            "quantize": dict(bound="hbm", achieved=round(q_gbps, 1), peak=peak, unit="GB/s",
                             frac=round(q_gbps / peak, 4),
                             traffic=traffic_for(f"quantize:{w.name}"),
                             kernel="quantize_kernel", algorithmic_bytes_per_launch=job.quant_bytes,
                             us_per_launch=round(q_ms * 1e3, 2),
                             peak_source=f"{peak_src} hbm_gbs (burst copy)"),
            "decode": dict(bound="hbm", achieved=round(d_cold_gbps, 1), peak=peak, unit="GB/s",
                           frac=round(d_cold_gbps / peak, 4),
                           traffic=traffic_for(f"decode:{w.name}"),
                           kernel="decode_tc_kernel + merge_kernel",
                           algorithmic_bytes_per_launch=job.decode_bytes,
                           us_per_launch=round(d_cold_ms * 1e3, 2),
                           peak_source=f"{peak_src} hbm_gbs (burst copy)"),
        }
        roof = roofs[dominant]
        value = job_throughput(world, job.bytes_per_step, args.steps, elapsed)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_LABEL, "data": "synthetic",
            "metric_parts": {"decode_gbps": round(d_cold_gbps, 1),
                             "decode_frac_of_hbm": round(d_cold_gbps / peak, 4),
                             "kv_tokens_per_s": round(kv_tok / (d_cold_ms * 1e-3), 1),
                             "quantize_gbps": round(q_gbps, 1),
                             "quantize_frac_of_hbm": round(q_gbps / peak, 4),
                             "hbm_peak_gbps": peak, "hbm_peak_source": peak_src},
            "config": {"workload": w.name, "layers": job.n_layers, "batch": w.batch, "ctx": w.ctx,
                       "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                       "input_dtype": w.dtype, "storage": ("fp8 e4m3 codes (the comparison cache), no scale, 256-token blocks" if args.fp8 else
                                   "int4 codes, group 64, fp16 scale+zero, 256-token blocks"),
                       "q8_fraction": 0.0 if args.fp8 else w.q8_fraction, "evict_fraction": w.evict_fraction,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "decode_splits": job.plan.n_splits, "decode_kernel": args.decode_kernel,
                       "l2": "step inputs larger than L2 (%.1f GB)" % (job.bytes_per_step / 1e9)},
            "kernels": {
                "quantize": {"gbps": round(q_gbps, 1), "us_per_launch": round(q_ms * 1e3, 2),
                             "bytes_per_launch": job.quant_bytes},
                "invalidate": {"us_per_launch_in_step": round(inv_ms * 1e3, 2),
                               "slots_per_launch": 0 if job.evict is None else int(job.evict.numel()),
                               "note": "remap of the evicted slots after each layer's encode (evicted workload only)"},
                "decode": {"gbps_in_step": round(d_gbps, 1), "us_per_launch_in_step": round(d_ms * 1e3, 2),
                           "gbps_cold": round(d_cold_gbps, 1), "us_per_launch_cold": round(d_cold_ms * 1e3, 2),
                           "bytes_per_launch": job.decode_bytes,
                           "kv_tokens_per_s": round(kv_tok / (d_cold_ms * 1e-3), 1),
                           "frac_cold": round(d_cold_gbps / peak, 4)},
                "append": {"us_per_launch": round(app_ms * 1e3, 2), "tokens_per_launch": w.batch,
                           "bytes_per_launch": job.append_bytes,
                           "append_then_decode_us": round(gen_ms * 1e3, 2),
                           "append_then_decode_separate_us": round(sep_ms * 1e3, 2),
                           "note": "one new token per sequence written over its last slot, then decode over "
                                   "the grown cache: append_then_decode_us = q4kv_append_decode (one decode launch "
                                   "that encodes the new rows itself), _separate_us = the two calls back to back"},
                "paging": paging,
                "card": card,
                "q2mix": q2mix,
            },
            "roofline": roof,
            "roofline_kernels": roofs,
            "gpu_launches": job.launches_per_layer * job.n_layers * args.steps,
            "clocks": clk.result(),
        }
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline and not args.fp8:   # the oracle leg times the Q4 path
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_q2mix(job, dev, reps):
    """Three code widths in one paged pool: the first layer's blocks coded
    8-bit (the quarter with the highest mean |K|), 2-bit (the quarter with
    the lowest) and 4-bit (the rest) -- a fixed synthetic policy standing in
    for QKVShare's learned width controller, which gives no distribution.
    Times the encoder over the whole layer and decode over the mixed pool
    with the bench's own plan; algorithmic bytes count each block at its width."""
    import torch
    import decode_attention_q4kv_b200 as q4
    w = job.w
    if w.permuted_pool:
        return None
    L = job.layers[0]
    k, v = L["k"], L["v"]
    nb, hkv, d = w.n_blocks, w.n_kv_heads, w.head_dim
    am = q4.block_absmean(k)
    order = torch.argsort(am, descending=True, stable=True)
    ranks = torch.empty_like(order)
    ranks[order] = torch.arange(nb, device=dev)
    n8, n2 = nb // 4, nb // 4
    n4 = nb - n8 - n2
    ids = torch.where(ranks < n8, n4 + ranks,
                      torch.where(ranks >= nb - n2, n4 + n8 + ranks - (nb - n2), ranks - n8)).to(torch.int32)
    pool = q4.Q4KVPool(hkv, d, n4, n8, device=dev, n_q2_blocks=n2)
    tables = ids.view(w.batch, w.blocks_per_seq)
    ng = d // 64
    row = {4: d // 2 + 4 * ng, 8: d + 4 * ng, 2: d // 4 + 4 * ng}
    code_bytes = 256 * hkv * 2 * (n4 * row[4] + n8 * row[8] + n2 * row[2])
    q_bytes = w.n_tokens * hkv * 2 * d * 2 + code_bytes
    d_bytes = code_bytes + nb * 32 + w.batch * w.blocks_per_seq * 4 + w.batch * w.n_q_heads * d * (2 + 4)

    def timed(fn):
        out = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            out.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in out)

    q_ms = timed(lambda: pool.quantize(k, v, ids))
    dec = lambda: q4.decode_attention(pool, L["q"], tables, job.lens, plan=job.plan, workspace=job.ws, out=L["out"])
    dec()
    d_ms = timed(dec)
    assert pool.read_device_error() == 0
    return {"blocks": {"8": n8, "4": n4, "2": n2}, "bits_per_value": round(8 * code_bytes / (2 * nb * 256 * hkv * d), 3),
            "quantize_us": round(q_ms * 1e3, 1), "quantize_gbps": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
            "decode_us": round(d_ms * 1e3, 2), "decode_gbps": round(d_bytes / (d_ms * 1e-3) / 1e9, 1),
            "decode_bytes": d_bytes,
            "note": "first layer, blocks 8-bit (top quarter by mean |K|), 2-bit (bottom quarter), 4-bit (rest); "
                    "decode repeated on one layer (L2 may hold part of it)"}


def measure_card(job, dev, reps):
    """Per-token mixed widths {2, 4, 8, FP16} (the synthetic mix of
    workloads.CARD_WIDTH_MIX): encode the first layer's tokens into one card
    and rebuild fp16 K/V from it.  Algorithmic bytes: encode reads K/V and
    writes the card; decode reads the card and writes K/V."""
    import torch
    import decode_attention_q4kv_b200 as q4
    from decode_attention_q4kv_b200 import workloads as W
    L = job.layers[0]
    k, v = L["k"], L["v"]
    n, hkv, d = k.shape
    widths = W.token_widths(n, job.w.seed, device=dev)
    card = q4.card_encode(k, v, widths)
    torch.cuda.synchronize()
    payload = int(card[32:40].cpu().numpy().view("<i8")[0])
    card_bytes = 64 + (n + 15) // 16 * 16 + (8 * (n + 1) + 15) // 16 * 16 + payload
    kv_bytes = 2 * n * hkv * d * k.element_size()

    def timed(fn):
        out = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            out.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in out)

    enc_ms = timed(lambda: q4.card_encode(k, v, widths))
    dec_ms = timed(lambda: q4.card_decode(card, n, hkv, d, out_dtype=torch.float16))
    counts = {int(w_): int((widths == w_).sum()) for w_ in (2, 4, 8, 16)}
    return {"tokens": n, "width_counts": counts, "card_bytes": card_bytes,
            "bits_per_value": round(8 * payload / (2 * n * hkv * d), 3),
            "encode_us": round(enc_ms * 1e3, 1), "encode_gbps": round((kv_bytes + card_bytes) / (enc_ms * 1e-3) / 1e9, 1),
            "decode_us": round(dec_ms * 1e3, 1), "decode_gbps": round((kv_bytes + card_bytes) / (dec_ms * 1e-3) / 1e9, 1),
            "note": "card = per-token widths {2,4,8,FP16}; decode rebuilds fp16 K/V"}


def measure_paging(job, dev, reps, decode_ms):
    """Block images of the first layer's whole pool to and from pinned host
    memory: the export and import kernels alone, the copy engine moving the
    same bytes (reference), and the import on a second stream beside a decode
    of the same layer (the import targets a second pool, so decode reads
    unchanged blocks)."""
    import torch
    import decode_attention_q4kv_b200 as q4
    L = job.layers[0]
    pool = L["pool"]
    nb = pool.n_blocks
    ids = torch.arange(nb, dtype=torch.int32, device=dev)
    stride = pool.image_stride()
    images = torch.empty((nb, stride), dtype=torch.uint8, pin_memory=True)
    moved = pool.nbytes() + 16 * nb                       # every block's sections + its header
    other = q4.Q4KVPool(pool.n_kv_heads, pool.head_dim, pool.n_q4_blocks, pool.n_q8_blocks,
                        k_rotated=pool.k_rotated, device=dev, fp8=pool.fp8)
    flat = images.view(-1)
    dev_buf = torch.empty(flat.numel(), dtype=torch.uint8, device=dev)

    def timed(fn):
        out = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            out.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in out)

    host_ids = ids.cpu()
    h2d_ms = timed(lambda: dev_buf.copy_(flat, non_blocking=True))
    d2h_ms = timed(lambda: flat.copy_(dev_buf, non_blocking=True))
    s_dec, s_copy = torch.cuda.Stream(), torch.cuda.Stream()

    def beside(import_ids, move=None):
        # The GPU first spins ~50 us in a gate kernel while the host enqueues
        # the decode and the import on their streams, so both start together
        # and neither span includes the host's own launch time.  move: another
        # transfer in place of the import (a plain pinned copy, as reference).
        spans = []
        for _ in range(reps):
            torch.cuda._sleep(100000)
            go = torch.cuda.Event()
            go.record()
            s_dec.wait_event(go)
            s_copy.wait_event(go)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(s_dec)
            with torch.cuda.stream(s_dec):
                job.decode_layer(L)
            e[1].record(s_dec)
            e[2].record(s_copy)
            with torch.cuda.stream(s_copy):
                if move is None:
                    other.import_blocks(images, import_ids)
                else:
                    move()
            e[3].record(s_copy)
            spans.append(e)
        torch.cuda.synchronize()
        return (round(statistics.median(a.elapsed_time(b) for a, b, _, _ in spans) * 1e3, 2),
                round(statistics.median(c.elapsed_time(d) for _, _, c, d in spans) * 1e3, 1))

    gbps = lambda ms: round(moved / (ms * 1e-3) / 1e9, 2)
    out = {"blocks": nb, "bytes": moved, "image_stride": stride,
           "copy_engine_h2d_gbps": round(flat.numel() / (h2d_ms * 1e-3) / 1e9, 2),
           "copy_engine_d2h_gbps": round(flat.numel() / (d2h_ms * 1e-3) / 1e9, 2),
           "decode_us_alone": round(decode_ms * 1e3, 2),
           "decode_us_beside_plain_h2d": beside(None, lambda: dev_buf.copy_(flat, non_blocking=True))[0]}
    for tag, the_ids in (("kernel", ids), ("copy_engine", host_ids)):
        exp_ms = timed(lambda: pool.export_blocks(the_ids, images))
        imp_ms = timed(lambda: other.import_blocks(images, the_ids))
        dec_b, imp_b = beside(the_ids)
        out[tag] = {"export_gbps": gbps(exp_ms), "export_us": round(exp_ms * 1e3, 1),
                    "import_gbps": gbps(imp_ms), "import_us": round(imp_ms * 1e3, 1),
                    "decode_us_beside_import": dec_b, "import_us_beside_decode": imp_b}
    out["note"] = ("pinned host images of the first layer's whole pool; kernel = device block ids, one "
                   "launch reading/writing host memory; copy_engine = host block ids, strided copies, no SM")
    return out


def run_e2e(job, args, dev, world):
    """Same metric through the public API from pinned host buffers, copies timed."""
    import torch

    w = job.w
    n_ring = min(2, job.n_layers)
    host = []
    for i in range(n_ring):
        L = job.layers[i]
        host.append(dict(k=L["k"].cpu().pin_memory(), v=L["v"].cpu().pin_memory(),
                         q=L["q"].cpu().pin_memory(),
                         out=torch.empty(L["out"].shape, dtype=L["out"].dtype).pin_memory()))
    steps = max(1, min(args.steps, 5))

    def one_step():
        for li, L in enumerate(job.layers):
            H = host[li % n_ring]
            L["k"].copy_(H["k"], non_blocking=True)
            L["v"].copy_(H["v"], non_blocking=True)
            L["q"].copy_(H["q"], non_blocking=True)
            job.quantize_layer(L)
            job.decode_layer(L)
            H["out"].copy_(L["out"], non_blocking=True)

    one_step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        one_step()
    b.record()
    torch.cuda.synchronize()
    el = reduce_max(a.elapsed_time(b) / 1e3, dev)
    L0 = job.layers[0]
    h2d = job.n_layers * sum(L0[x].numel() * L0[x].element_size() for x in ("k", "v", "q"))
    d2h = job.n_layers * L0["out"].numel() * L0["out"].element_size()
    return {"value": round(job_throughput(world, job.bytes_per_step, steps, el), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "inputs copied from pinned host memory and the fp16 output read back, per layer, inside the timed region"}


# ---------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

_LAYER_CACHE = {}


def _layer_inputs(w, layer):
    """Host K/V/q of one layer (drawing them is slower than the sample; the
    last layer drawn is kept, so successive KV-head slices reuse it)."""
    from decode_attention_q4kv_b200 import workloads as W
    key = (w.name, layer)
    if key not in _LAYER_CACHE:
        _LAYER_CACHE.clear()
        n_tok = w.prefill_tokens or w.n_tokens
        k, v = W.kv_tokens(w, layer, n_tok, "cpu")
        _LAYER_CACHE[key] = (k, v, W.query(w, layer, "cpu"))
    return _LAYER_CACHE[key]


def oracle_sample(w, kv_heads=1, layer=0, head=0):
    """One bounded sample: one layer, KV heads [head, head + kv_heads), all
    sessions, on the host.

    Quantises every token of those heads and decodes every query head that
    reads them, with the oracle as it stands.  Returns (seconds, algorithmic
    bytes of the sample); drawing the inputs is not timed.
    """
    import numpy as np
    import torch

    from decode_attention_q4kv_b200 import workloads as W
    from oracle import q4kv_oracle as O

    n_tok = w.prefill_tokens or w.n_tokens
    k, v, q = _layer_inputs(w, layer)
    k, v = k[:, head:head + kv_heads].contiguous(), v[:, head:head + kv_heads].contiguous()
    g = w.gqa
    q = q[:, head * g:(head + kv_heads) * g].contiguous()

    def host(t):
        if t.dtype == torch.float16:
            return t.numpy(), "fp16"
        return t.view(torch.int16).numpy().view(np.uint16), "bf16"

    kh, dt = host(k)
    vh, _ = host(v)
    qh, _ = host(q)
    nb = w.n_blocks
    n_q8 = w.n_q8_blocks
    t0 = time.perf_counter()
    if w.q8_fraction:
        ids = O.mixed_block_ids(O.block_absmean(kh, dt), n_q8, 0, nb - n_q8)
    else:
        ids = np.arange(-(-n_tok // 256))
    pool = O.OraclePool(kv_heads, w.head_dim, nb - n_q8, n_q8)
    pool.quantize_blocks(kh, vh, dt, ids)
    if w.evict_fraction:
        tabs = W.identity_tables(w)
        slots = W.evicted_slot_ids(w, tabs)
        pool.invalidate_slots(slots.tolist())
    tables = np.asarray(ids, np.int64).reshape(w.batch, -1) if not w.permuted_pool else \
        (W.permuted_tables(w).numpy() % (n_tok // 256))
    O.decode_attention(pool, qh, dt, tables, [w.ctx] * w.batch)
    secs = time.perf_counter() - t0
    frac = kv_heads / w.n_kv_heads
    qb, db = bytes_per_layer(w)
    return secs, (qb + db) * frac


def host_cores() -> int:
    """Cores this process may run on (its affinity mask), else the machine's count."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _oracle_samples_1t(w, slices):
    """oracle_sample of each (layer, head) slice in turn on one thread (a
    worker of the all-cores leg)."""
    from threadpoolctl import threadpool_limits
    secs = nbytes = 0.0
    with threadpool_limits(limits=1):
        for layer, head in slices:
            s, b = oracle_sample(w, kv_heads=1, layer=layer, head=head)
            secs += s
            nbytes += b
    return secs, nbytes


def _worker_ready(w, layer):
    """Imports and the worker's input layer, paid before the timed region."""
    from oracle import q4kv_oracle  # noqa: F401
    _layer_inputs(w, layer)
    return True


def cpu_baseline_all_cores(w, workers, per_worker=1):
    """The oracle, unchanged, on `workers` processes at once: each quantises and
    decodes its own one-KV-head slice of a different layer on one thread.
    Value = the slices' algorithmic bytes / wall time from submission to the
    last result (the pool is started and warmed first).  Workers are spawned,
    not forked, because this process has initialised CUDA."""
    import concurrent.futures as cf
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
        # every worker draws the same layer; each then takes other KV heads
        for f in [ex.submit(_worker_ready, w, 0) for _ in range(workers)]:
            f.result()
        t0 = time.perf_counter()
        futs = [ex.submit(_oracle_samples_1t, w, [(0, (per_worker * i + j) % w.n_kv_heads)
                                                   for j in range(per_worker)])
                for i in range(workers)]
        nbytes = sum(f.result()[1] for f in futs)
        wall = time.perf_counter() - t0
    return nbytes / wall / 1e9, wall


def all_cores_workers(w, cores):
    """Worker count for the all-cores leg: every core, bounded by host memory
    (each worker draws one layer's K/V in fp32 before slicing one head)."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 16 << 30
    n_tok = w.prefill_tokens or w.n_tokens
    per_worker = 8 * n_tok * w.n_kv_heads * w.head_dim + (1 << 30)
    return max(1, min(cores, int(0.6 * avail // per_worker)))


def cpu_baseline(w, target_s=15.0, all_cores=True):
    """The oracle on a bounded sample: one-KV-head slices of successive layers
    until ~target_s on one thread; then the same slices on all host cores."""
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        total_s, total_b, n = 0.0, 0.0, 0
        while total_s < target_s and n < 4 * w.n_kv_heads:
            s2, b2 = oracle_sample(w, kv_heads=1, layer=n // w.n_kv_heads, head=n % w.n_kv_heads)
            total_s += s2
            total_b += b2
            n += 1
    cores = host_cores()
    out = {"value": round(total_b / total_s / 1e9, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "host_cores": cores,
           "sample": f"{n} x (one KV head of {w.n_kv_heads} of a layer: quantise all "
                     f"{w.prefill_tokens or w.n_tokens} tokens + decode the {w.gqa} query heads "
                     f"of all {w.batch} sessions); numpy/BLAS limited to 1 thread",
           "seconds": round(total_s, 2)}
    if all_cores and cores > 1:
        workers = all_cores_workers(w, cores)
        per_worker = max(1, min(16, round(5.0 / max(total_s / n, 1e-3))))   # ~5 s per worker
        try:
            v, wall = cpu_baseline_all_cores(w, workers, per_worker)
            out["all_cores"] = {"value": round(v, 5), "unit": "GB/s", "cores": workers,
                                "sample": f"{workers} processes (spawned) at once, each {per_worker} "
                                          f"slice(s) as above on one thread",
                                "seconds": round(wall, 2)}
        except Exception as e:          # reported, not fatal: the GPU line stands without it
            out["all_cores"] = {"error": repr(e)[:200]}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits

    w = workload_by_name(args.workload)
    with threadpool_limits(limits=1):
        hkv = w.n_kv_heads
        for i in range(args.warmup):
            oracle_sample(w, kv_heads=1, layer=i // hkv, head=i % hkv)
        secs, nbytes = 0.0, 0.0
        for i in range(args.warmup, args.warmup + args.steps):
            s, b = oracle_sample(w, kv_heads=1, layer=i // hkv, head=i % hkv)
            secs += s
            nbytes += b
    value = nbytes / secs / 1e9
    line = {"metric": METRIC, "value": round(value, 5), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "layers": w.layers, "batch": w.batch, "ctx": w.ctx,
                       "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                       "input_dtype": w.dtype},
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "host_cores": host_cores(),
                             "sample": "each step: one KV head of a layer (all tokens quantised, "
                                       "its query heads decoded), numpy/BLAS limited to 1 thread"},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="q4kv", choices=["q4kv", "reference"])
    ap.add_argument("--workload", default="evict",
                    help="evict (default: Qwen2.5-14B shape, 32 x 16384, 60%% evicted), gemma, mixed, tiny, "
                         "or sweep:B:C")
    ap.add_argument("--decode-kernel", type=int, default=1, choices=[0, 1],
                    help="decode variant: 1 tensor-core pipeline (default), 0 CUDA-core kernel")
    ap.add_argument("--fp8", action="store_true",
                    help="run the same workload on the FP8 (E4M3) comparison cache instead of Q4")
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)      # timing rule: at least 3 untimed steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
