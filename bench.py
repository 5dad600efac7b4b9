"""Benchmark of the packed-KV-cache per-layer step on B200.

One step = one pass of the whole hot path for one layer of the pages-scale
workload (B=1, 12 heads x 128, 6,240-token blocks, 40-block compressed pool,
top-16, 27,872-key context):
  select (query pooling + block scoring + top-k) -> attend -> append the
  finished block (evicts the oldest compressed block) -> temporal RoPE shift
  of the sink by 4 frames.
Inputs are resident in HBM; L2 is flushed between timed steps, outside the
step's events: a 256 MB buffer is written (twice the 126 MB L2), then another
256 MB buffer is read, so that the L2 holds only clean lines of that buffer
and the timed step does not pay the write-back of the flush's dirty lines.
The metric is packed-cache attention TFLOP/s (attention FLOPs of the step /
step time) and the per-layer step latency; the roofline line is the
attention kernel's own time.

The same JSON line carries, under "configs", the other workloads of the
path, each timed with CUDA events (L2 flushed between iterations) and with
its own roofline: the 30-layer block of 4 denoising steps at CFG batch 2
(selection at the first step, reused by the others; append and sink shift
of every layer after the block), the dense 748,800-key layer, and the
batch-2 stress layers with a 1,000-block pool (scoring, top-k and the RoPE
shift of every cached key: the HBM-bound kernels; attention with 16 and 64
routed blocks; and the streaming scorer of the allocation-free selection,
which reads the whole compressed pool).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--configs all|none|c2,c3,c4]

For N > 1 run under torchrun: every rank runs an independent replica (its
own cache and stream of blocks, no data-path collective), time = max over
ranks, value = the ranks' total work / that time.  The extra configs run on
rank 0 only, after the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# library kernels per step besides the selection's and the attention's:
# copy_runs + kmean (append with a compressed copy); rope_shift is added when
# a block was evicted
LAUNCHES_PER_STEP_BASE = 2


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    """(rank, world, local_rank) from torchrun's environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def reduce_max(x: float, device=None) -> float:
    """Maximum of x over all ranks (x itself on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def rank_seed(base: int, rank: int) -> int:
    """Each replica draws its own blocks."""
    return base + 7919 * rank


# ---------------------------------------------------------------- head sharding

def head_shard(H: int, world: int, rank: int):
    """Heads [lo, hi) of this rank: contiguous ranges whose sizes differ by at
    most one (the first H mod world ranks take one more)."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def select_head_sharded(cache, layer, Q, scores, heads_total, reduce_sum, route_scores_only, route_given):
    """The selection of a layer whose heads are spread over ranks (one
    exchange): this rank scores the live blocks on its own heads, divided by
    the total head count (a partial of the all-head score), the partials are
    summed across ranks (reduce_sum, in place), and every rank takes the same
    top-k of the sum with the method's ranking rule."""
    cache.select_mid_ex(layer, Q, policy=route_scores_only, heads_total=heads_total, scores_out=scores)
    reduce_sum(scores)
    cache.select_mid_ex(layer, None, policy=route_given, scores_in=scores)


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_flops(B, H, Lq, Lk, D=128) -> float:
    """QK^T and PV: 2 multiply-adds per (query, key, dim), 2 FLOP each."""
    return 4.0 * B * H * Lq * Lk * D


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every
    ~2 ms by NVML in a host thread (so that even a 20 ms timed region holds
    several samples), or by ``nvidia-smi -lms 100`` if NVML is unavailable.
    The GPU is found by its UUID: NVML numbers every GPU of the machine,
    CUDA only the visible ones."""

    INTERVAL_S = 0.002
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.rows = []          # (host time, sm MHz, max sm MHz, [reason names])
        self.thread = None
        self.stop_flag = False
        self.proc = None
        self.path = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)

    def start(self):
        try:
            nv, h = self._nvml_handle()
        except Exception:
            nv = None
        if nv is not None:
            import threading
            self.source = "nvml"

            def loop():
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                while not self.stop_flag:
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((time.time(), float(sm), float(mx), reason_names(bits)))
                    except Exception:
                        pass
                    time.sleep(self.INTERVAL_S)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        try:
            self.source = "nvidia-smi"
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.device_index)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            self.source = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            self.thread = None
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            with open(self.path) as f:
                self.rows = parse_smi_rows(f.readlines())
            os.unlink(self.path)
            self.proc = None

    def window(self, t0: float | None = None, t1: float | None = None):
        """Summary of the samples taken between host times t0 and t1."""
        s = summarize_rows(self.rows, t0, t1)
        if s is not None:
            s["source"] = self.source
        return s

    def window_at_least(self, t0: float, t1: float, n: int = 3):
        """The same, widened around [t0, t1] until it holds n samples."""
        s = summarize_rows_at_least(self.rows, t0, t1, n)
        if s is not None:
            s["source"] = self.source
        return s


REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}


def reason_names(bits: int) -> list:
    """Names of the clock-event reasons set in an NVML reasons bitmask (the
    ones that decide whether a timed run is kept)."""
    return sorted(name for name, b in REASON_BITS.items() if bits & b)


def parse_smi_rows(lines):
    """nvidia-smi CSV rows (the ClockSampler fields, no header, no units) ->
    (host time or None, sm MHz or None, max MHz or None, [active reasons])."""
    import datetime
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    rows = []
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            ts = None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        reasons = [names[i] for i in range(4) if parts[5 + i].lower().startswith("active")]
        rows.append((ts, num(parts[1]), num(parts[2]), reasons))
    return rows


def summarize_rows(rows, t0: float | None = None, t1: float | None = None):
    """Median SM clock, max clock and active reasons of the sample rows whose
    time lies in [t0, t1]; None if no row qualifies."""
    sel = [r for r in rows if t0 is None or r[0] is None or t0 <= r[0] <= t1]
    if not sel:
        return None
    sm = [r[1] for r in sel if r[1] is not None]
    mx = [r[2] for r in sel if r[2] is not None]
    reasons = sorted({x for r in sel for x in r[3]})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(sel)}


def summarize_rows_at_least(rows, t0: float, t1: float, n: int = 3, max_pad_s: float = 5.0):
    """summarize_rows over [t0, t1], widened symmetrically (10 ms, doubling,
    at most max_pad_s each side) until it holds at least n samples: a timed
    region of a few tens of ms can fall between two samples of the host
    thread.  The record says which window it covers ("window_s") and how far
    past the timed region it reaches ("pad_s")."""
    pad = 0.0
    s = summarize_rows(rows, t0, t1)
    while (s is None or s["samples"] < n) and pad < max_pad_s:
        pad = min(max_pad_s, 0.01 if pad == 0.0 else 2 * pad)
        s = summarize_rows(rows, t0 - pad, t1 + pad)
    if s is not None:
        s["window_s"] = round(t1 - t0 + 2 * pad, 3)
        s["pad_s"] = pad
    return s


def summarize_clocks(lines, t0: float | None = None, t1: float | None = None):
    """summarize_rows over nvidia-smi CSV lines."""
    return summarize_rows(parse_smi_rows(lines), t0, t1)


def traffic_for(kernel_src: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent:
        return None
    with open(kernel_src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    return ent.get("dram_bytes_per_launch") if ent.get("source_sha") == h else None


# ---------------------------------------------------------------- the GPU arm

class L2Flush:
    """Evicts the L2 between timed iterations: writes a 256 MB buffer, then
    reads another 256 MB buffer, so the lines left in L2 are clean ones of
    a buffer no kernel under test touches."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(32 << 20, dtype=torch.int64, device=dev)

    def __call__(self, i):
        self.w.fill_(i & 0xFF)
        self.r.sum()


SUSTAINED_AFTER_MS = 500.0   # timed regions at least this long are compared with the sustained peak


def roofline(kernel: str, bound: str, amount: float, ms: float, peaks: dict, peak_src: str,
             sustained: bool = False, traffic=None) -> dict:
    """Roofline record: `amount` algorithmic bytes (bound "hbm") or FLOPs
    (bound "tensor") per launch over `ms` milliseconds, against the measured
    HBM copy bandwidth or bf16 dense throughput (burst for a kernel timed by
    itself, sustained for one timed inside a long run)."""
    if bound == "hbm":
        ach = amount / (ms * 1e-3) / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        unit, label = "GB/s", "HBM copy"
    else:
        ach = amount / (ms * 1e-3) / 1e12
        key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
        unit, label = "TFLOP/s", "bf16 dense " + ("(sustained)" if sustained else "(burst)")
    return {"kernel": kernel, "bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": unit,
            "frac": round(ach / peak, 4), "peak_source": f"{peak_src} {label}",
            ("algorithmic_bytes" if bound == "hbm" else "algorithmic_flop"): amount, "ms": round(ms, 4),
            "traffic": traffic}


def timed_ms(fn, iters, flush, stream):
    """Median device time (ms) of fn over `iters` calls, L2 flushed before
    each, CUDA events on the launching stream."""
    import torch
    ts = []
    for i in range(iters):
        flush(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def fill_cache(pf, wl, d, dev, layers=1, sink_rope_in_attention=False):
    """A cache holding d's sink, mid pool and recent blocks in every layer."""
    cache = pf.PackedKVCache(pf.config_for(wl, layers=layers, sink_rope_in_attention=sink_rope_in_attention),
                             device=dev)
    for l in range(layers):
        for s_ in range(wl.sink_blocks):
            cache.append_block(l, d["sink_K"][:, s_].contiguous(), d["sink_V"][:, s_].contiguous())
        if wl.pool_blocks:
            cache.load_mid(l, d["mid_K"].contiguous(), d["mid_V"].contiguous())
        for r in range(wl.recent_blocks):
            cache.append_block(l, d["recent_K"][:, r].contiguous(), d["recent_V"][:, r].contiguous(),
                               d["recent_Kc"][:, r].contiguous(), d["recent_Vc"][:, r].contiguous())
    return cache


def measure_stress(pf, synth, dev, flush, stream, peaks, src, iters) -> dict:
    """The batch-2 stress layers (1,000-block compressed pool): selection,
    the RoPE shift of every cached key and of the sink, attention with 16 and
    64 routed blocks, and the allocation-free selection streaming the pool."""
    import torch
    out = {}
    for name in ("stress16", "stress64"):
        wl = synth.WORKLOADS[name]
        d = synth.make_layer(wl, synth.nominal_seed(list(synth.WORKLOADS).index(name)), device=dev)
        cache = fill_cache(pf, wl, d, dev)
        B, H, D, n, nc, P = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c, wl.pool_blocks
        row = H * D * 2
        r = {}
        if name == "stress16":
            ms = timed_ms(lambda: cache.select_mid(0, d["Q"]), iters, flush, stream)
            # reads: the queries (bf16) and every live block's cached mean key (fp32)
            r["select"] = roofline("qsum_slab_kernel + score_cached_kernel", "hbm", B * n * row + B * P * H * D * 4, ms,
                                   peaks, src)
            info = cache.info(0)
            sel = torch.empty((B, wl.n_top), dtype=torch.int32, device=dev)
            ms = timed_ms(lambda: pf.pf_select_mid_static(d["Q"], B, n, H, info["pool_k"], info["pool_slots"], nc,
                                                          info["mid_head"], P, wl.n_top, sel),
                          iters, flush, stream)
            # reads: the queries and every live block's n_c compressed keys
            r["select_streaming"] = roofline("qpool_kernel + score_kernel", "hbm", B * n * row + B * P * nc * row,
                                             ms, peaks, src)
            parts = pf.PART_SINK | pf.PART_MID | pf.PART_RECENT
            rows = B * (wl.sink_blocks * n + P * nc + wl.recent_blocks * (n + nc))
            ms = timed_ms(lambda: cache.rope_shift(0, parts, 4), iters, flush, stream)
            # 22 rotary pairs = 88 bytes read and 88 written per (key, head)
            r["rope_shift_all"] = roofline("rope_shift_kernel", "hbm", rows * H * 176, ms, peaks, src)
            ms = timed_ms(lambda: cache.rope_shift(0, pf.PART_SINK, 4), iters, flush, stream)
            r["rope_shift_sink"] = roofline("rope_shift_kernel", "hbm", B * wl.sink_blocks * n * H * 176, ms,
                                            peaks, src)
        cache.select_mid(0, d["Q"])
        O = torch.empty_like(d["Q"])
        Lk = cache.info(0)["context_tokens"]
        ms = timed_ms(lambda: cache.attend(0, d["Q"], d["K_cur"], d["V_cur"], O), iters, flush, stream)
        r["attend"] = roofline("attend_kernel + tail_merge_kernel", "tensor", attention_flops(B, H, n, Lk, D), ms, peaks, src)
        r["context_tokens"] = Lk
        cache.poll_device_error()
        out[name] = r
        del cache, d, O
        torch.cuda.empty_cache()
    return out


def measure_dense(pf, synth, dev, flush, stream, peaks, src, iters) -> dict:
    """The dense layer: 6,240 queries over 748,800 full-resolution keys."""
    import torch
    wl = synth.WORKLOADS["dense"]
    d = synth.make_layer(wl, synth.nominal_seed(list(synth.WORKLOADS).index("dense")), device=dev)
    cache = fill_cache(pf, wl, d, dev)
    O = torch.empty_like(d["Q"])
    Lk = cache.info(0)["context_tokens"]
    ms = timed_ms(lambda: cache.attend(0, d["Q"], d["K_cur"], d["V_cur"], O), iters, flush, stream)
    r = {"context_tokens": Lk,
         "attend": roofline("attend_kernel + tail_merge_kernel", "tensor", attention_flops(wl.batch, wl.heads, wl.n, Lk), ms, peaks, src)}
    cache.poll_device_error()
    del cache, d, O
    torch.cuda.empty_cache()
    return r


def measure_block(pf, synth, dev, flush, stream, peaks, src, blocks=3) -> dict:
    """One generated block of the 30-layer model at CFG batch 2 (cond +
    uncond): 4 denoising steps x 30 layers of pf_attend_step (selection at
    the first step, reused by the other three), then pf_finish_block (append
    the block to every layer, evict the oldest compressed block, shift every
    sink).  116-block pool per layer."""
    import torch
    wl = synth.WORKLOADS["step30"].replace(batch=2)
    L, S = wl.layers, 4
    B, H, D, n, nc = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c
    cache = pf.PackedKVCache(pf.config_for(wl, layers=L), device=dev)
    blk = synth.make_block(wl, 77, dev)
    pool = synth.bf16_normal((B, wl.pool_blocks, nc, H, D), 78, dev)
    for l in range(L):
        for _ in range(wl.sink_blocks):
            cache.append_block(l, blk["K"], blk["V"])
        cache.load_mid(l, pool, pool)
        cache.append_block(l, blk["K"], blk["V"], blk["Kc"], blk["Vc"])
    del pool
    Qs = [synth.bf16_normal((B, n, H, D), 100 + l, dev) for l in range(L)]
    Ks = [synth.bf16_normal((B, n, H, D), 200 + l, dev) for l in range(L)]
    Vs = [synth.bf16_normal((B, n, H, D), 300 + l, dev) for l in range(L)]
    Kcs = [synth.bf16_normal((B, nc, H, D), 400 + l, dev) for l in range(L)]
    O = torch.empty_like(Qs[0])

    def block():
        for step in range(S):
            for l in range(L):
                cache.attend_step(l, step, Qs[l], Ks[l], Vs[l], O)
        cache.finish_block(Ks, Vs, Kcs, Kcs)

    block()
    ms = timed_ms(block, blocks, flush, stream)
    att_launches = pf.attend_launches(cache.cfg, cache.info(0), torch.cuda.get_device_properties(dev).multi_processor_count)
    Lk = cache.info(0)["context_tokens"]
    flops = L * S * attention_flops(B, H, n, Lk, D)
    cache.poll_device_error()
    r = {"ms_per_block": round(ms, 3), "layer_step_ms": round(ms / (L * S), 4), "context_tokens": Lk,
         "attention_flop_per_block": flops,
         # attend (and its tail merge) per layer and step; the selection's two
         # kernels per layer at step 0; copy + key mean per layer's append; one
         # shift launch for all sinks
         "launches_per_block": L * S * att_launches + 2 * L + 2 * L + 1,
         "attend_block": roofline("attend_kernel + tail_merge_kernel (whole block: selection, appends and shifts included)", "tensor",
                                  flops, ms, peaks, src, sustained=True)}
    del cache, Qs, Ks, Vs, Kcs, O, blk
    torch.cuda.empty_cache()
    return r


def measure_configs(which, pf, synth, dev, flush, stream, peaks, src, iters) -> dict:
    """The workloads beside the headline, keyed by the configuration they stand for."""
    out = {}
    if "c2" in which:
        out["c2_block_30_layers_4_steps_cfg2"] = measure_block(pf, synth, dev, flush, stream, peaks, src)
    if "c3" in which:
        out["c3_dense_748800_keys"] = measure_dense(pf, synth, dev, flush, stream, peaks, src, max(3, iters // 4))
    if "c4" in which:
        out.update({f"c4_{k}": v for k, v in measure_stress(pf, synth, dev, flush, stream, peaks, src, iters).items()})
    return out


def run_gpu(args):
    import torch

    import synth
    from packed_kv_cache_b200 import build as pfbuild
    pfbuild.build()
    import packed_kv_cache_b200 as pf

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init("nccl")
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[WORKLOAD]
    H_all = wl.heads
    sharded = args.shard == "heads"
    base_seed = synth.nominal_seed(list(synth.WORKLOADS).index(WORKLOAD))
    if sharded:
        # one layer spread over the ranks by heads: every rank draws the same
        # layer and keeps its own heads
        lo, hi = head_shard(H_all, world, rank)
        if hi <= lo:
            raise SystemExit(f"--shard heads needs at most {H_all} ranks")
        seed = base_seed
        full = synth.make_layer(wl, seed, device=dev)
        d = {k: (v[..., lo:hi, :].contiguous() if torch.is_tensor(v) and v.dim() >= 4 else v)
             for k, v in full.items()}
        del full
        wl = wl.replace(heads=hi - lo)
    else:
        seed = rank_seed(base_seed, rank)
        d = synth.make_layer(wl, seed, device=dev)
    B, H, D, n, nc = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c
    stream = torch.cuda.current_stream(dev)

    cache = fill_cache(pf, wl, d, dev)
    # the current block's inputs (resident); its compressed copy for the append
    Q, Kn, Vn = d["Q"], d["K_cur"], d["V_cur"]
    Kcn = synth.bf16_normal((B, nc, H, D), seed + 1, dev)
    Vcn = synth.bf16_normal((B, nc, H, D), seed + 2, dev)
    O = torch.empty_like(Q)
    info0 = cache.info(0)
    # the pool is full at every step (each append evicts one block): the
    # attention's launch count is the same for every step
    att_launches = pf.attend_launches(cache.cfg, info0, torch.cuda.get_device_properties(dev).multi_processor_count)
    Lk = info0["context_tokens"]
    flops = attention_flops(B, H, n, Lk, D)              # this rank's heads
    # [B, live blocks] partial (then summed) block scores of the sharded selection;
    # the pool stays full from step to step (each append evicts one block)
    scores = torch.zeros((B, max(1, info0["mid_count"])), dtype=torch.float32, device=dev)
    import torch.distributed as dist

    def all_reduce_sum(t):
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.SUM)

    def select(q):
        if sharded:   # scores on this rank's heads (2 launches), then the top-k of the summed scores (1)
            select_head_sharded(cache, 0, q, scores, H_all, all_reduce_sum, pf.ROUTE_SCORES_ONLY, pf.ROUTE_GIVEN)
            return 3
        cache.select_mid(0, q)   # query sums, then scores and top-k
        return 2

    def step(q, k, v, kc, vc, out, att_events=None):
        nl = select(q)
        if att_events is not None:
            att_events[0].record(stream)
        cache.attend(0, q, k, v, out)
        if att_events is not None:
            att_events[1].record(stream)
        ev = cache.append_block(0, k, v, kc, vc)
        if ev:
            cache.rope_shift(0, pf.PART_SINK, ev * wl.block_frames)
        return LAUNCHES_PER_STEP_BASE + nl + att_launches + (1 if ev else 0)

    clocks = ClockSampler(local)
    clocks.start()
    t_run0 = time.time()
    flush = L2Flush(dev)
    for i in range(args.warmup):
        flush(i)
        step(Q, Kn, Vn, Kcn, Vcn, O)
    torch.cuda.synchronize(dev)
    cache.poll_device_error()
    assert cache.info(0)["context_tokens"] == Lk

    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    ev_att = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier()
    t_start = time.time()
    launches = 0
    for i in range(args.steps):
        flush(i + 7)
        ev_step[i][0].record(stream)
        launches += step(Q, Kn, Vn, Kcn, Vcn, O, ev_att[i])
        ev_step[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t_end = time.time()
    barrier()
    cache.poll_device_error()
    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    att_ms = [a.elapsed_time(b) for a, b in ev_att]
    total_ms = reduce_max(sum(step_ms), dev)
    att_mean_ms = reduce_max(statistics.mean(att_ms), dev)
    ms_per_step = total_ms / args.steps
    # whole-job work: every rank's heads (sharded: one layer; replicas: one layer each)
    job_flops = attention_flops(B, H_all, n, Lk, D) if sharded else world * flops
    value = args.steps * job_flops / (total_ms * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers.  Each step's
    # inputs come from pinned host memory and its output goes back to pinned
    # host memory; the copies run on their own streams (host-to-device and
    # device-to-host engines), double-buffered, so that step i+1's inputs and
    # step i-1's output move while step i computes.  The timed region runs
    # from before the first input copy to after the last output copy.
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    hin = tuple(pin(t) for t in (Q, Kn, Vn, Kcn, Vcn))
    hO = [torch.empty(O.shape, dtype=O.dtype, pin_memory=True) for _ in range(2)]
    din = [tuple(torch.empty_like(t) for t in (Q, Kn, Vn, Kcn, Vcn)) for _ in range(2)]
    dO = [torch.empty_like(O) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = hO[0].numel() * hO[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(nsteps, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)

        def copy_in(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[b])        # step i-2 no longer reads these buffers
                for dst, src in zip(din[b], hin):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)

        copy_in(0)
        for i in range(nsteps):
            b = i % 2
            if i + 1 < nsteps:
                copy_in(i + 1)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])           # step i-2's output has left dO[b]
            step(*din[b], dO[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                hO[b].copy_(dO[b], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)
        if e_end is not None:
            e_end.record(stream)

    e2e_run(args.warmup)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    e2e_value = args.steps * job_flops / (e2e_ms * 1e-3) / 1e12
    cache.poll_device_error()
    cache.close()
    del cache, din, dO, hin, hO
    torch.cuda.empty_cache()

    peaks, peak_src = load_peaks()
    configs = {}
    if rank == 0 and args.configs != "none":
        which = {"c2", "c3", "c4"} if args.configs == "all" else set(args.configs.split(","))
        configs = measure_configs(which, pf, synth, dev, flush, stream, peaks, peak_src, max(args.steps, 5))
    t_run1 = time.time()
    clocks.stop()
    # a timed region of SUSTAINED_AFTER_MS or more runs at the power cap's
    # clock: the sustained bf16 peak is its denominator, the burst one below
    att = roofline("attend_kernel + tail_merge_kernel", "tensor", flops, att_mean_ms, peaks, peak_src,
                   sustained=total_ms >= SUSTAINED_AFTER_MS,
                   traffic=traffic_for(os.path.join(ROOT, "packed_kv_cache_b200", "csrc", "attend.cu"), WORKLOAD))
    line = {
        "metric": "packed-cache attention TFLOP/s (per-layer step)",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": ("one layer, pages scale: B=1, H=12, d_h=128, block 4x30x52 (n=6240), "
                         "compressed 182 tokens/block, pool 40, top-16, context 27872 keys; "
                         "step = select + attend + append(evict) + sink RoPE shift"),
            "context_tokens": Lk,
            "attention_flop_per_step": job_flops,
            "l2": "flushed between steps (256 MB write, then 256 MB read of another buffer), outside the step events",
            "parallelism": (f"heads sharded x{world} ({H} of {H_all} heads on this rank; NCCL all-reduce of the "
                            f"[B, P] partial block scores before the top-k)" if sharded else
                            f"replicas x{world} (independent streams, no collective)"),
        },
        "attention_ms": round(att_mean_ms, 4),
        "roofline": att,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / args.steps, 4)},
        "gpu_launches": launches,
        "clocks": clocks.window_at_least(t_start, t_end),
        "clocks_run": clocks.window(t_run0, t_run1),
        "configs": configs,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:   # the oracle's timing: one process only
        line["cpu_baseline"] = cpu_baseline({k: v for k, v in d.items()}, wl, budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------- the oracle on host cores

def oracle_step(d, wl, rows, heads=None):
    """One bounded sample of the step on the CPU oracle: selection over the
    whole pool, the sink shift, and attention for ``rows`` query rows; with
    ``heads`` = (lo, hi), every part restricted to those heads (the inputs are
    sliced before the oracle sees them)."""
    import numpy as np

    import oracle
    if heads is not None:
        lo, hi = heads
        d = {k: (v[..., lo:hi, :] if hasattr(v, "dim") and v.dim() >= 4 else v) for k, v in d.items()}
    S = oracle.select_scores(d["Q"], d["mid_K"])
    sel = oracle.select_topk(S, wl.n_top)
    B, D = wl.batch, wl.head_dim
    H = d["Q"].shape[2]
    sinkK = oracle.rope_shift(d["sink_K"].reshape(B, -1, H, D), wl.block_frames)
    parts = [(sinkK, d["sink_V"].reshape(B, -1, H, D))]
    mK = [oracle.to_f64(d["mid_K"][b, sel[b]]).reshape(-1, H, D) for b in range(B)]
    mV = [oracle.to_f64(d["mid_V"][b, sel[b]]).reshape(-1, H, D) for b in range(B)]
    parts.append((np.stack(mK), np.stack(mV)))
    parts.append((d["recent_K"].reshape(B, -1, H, D), d["recent_V"].reshape(B, -1, H, D)))
    parts.append((d["K_cur"], d["V_cur"]))
    oracle.attend(d["Q"], parts, rows=rows)
    Lk = sum(p[0].shape[1] for p in parts)
    return attention_flops(B, H, len(rows), Lk, D)


def cpu_model() -> str | None:
    """The host CPU's model name (Linux), recorded beside the oracle's timing."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(d, wl, budget_s=15.0):
    import numpy as np
    dc = {k: (v.cpu() if hasattr(v, "cpu") else v) for k, v in d.items()}
    # two short calibrations separate the fixed cost (selection over the
    # pool, sink shift) from the per-query-row cost of the attention sample
    times = []
    for nr in (16, 256):
        rows = np.linspace(0, wl.n - 1, nr).astype(np.int64)
        t0 = time.perf_counter()
        oracle_step(dc, wl, rows)
        times.append(time.perf_counter() - t0)
    per_row = max((times[1] - times[0]) / 240, 1e-6)
    fixed = max(times[0] - 16 * per_row, 0.0)
    nrows = int(min(wl.n, max(16, (0.9 * budget_s - fixed) / per_row)))
    rows = np.linspace(0, wl.n - 1, nrows).astype(np.int64)
    t0 = time.perf_counter()
    fl = oracle_step(dc, wl, rows)
    dt = time.perf_counter() - t0
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "cpu": cpu_model(), "kind": "oracle",
            "sample": (f"selection over the whole 40-block pool, sink RoPE shift, and attention of "
                       f"{nrows} of 6240 query rows x 12 heads over the 27872-key context, float64 numpy; "
                       f"{dt:.1f} s"), "seconds": round(dt, 2)}


def run_reference(args):
    import numpy as np

    import synth
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = synth.WORKLOADS[WORKLOAD]
    d = synth.make_layer(wl, synth.nominal_seed(list(synth.WORKLOADS).index(WORKLOAD)))

    def sample_rows(nr):
        return np.linspace(0, wl.n - 1, nr).astype(np.int64)

    if args.ref_rows:
        nh, nr = wl.heads, args.ref_rows
    else:
        # size the per-step sample so that the warm-up and timed steps fit in
        # --ref-seconds whatever --steps is: start from one head and 16 query
        # rows, then double the heads (up to all of them), else the rows, as
        # long as one measured step of the larger sample still fits
        def step_seconds(nh, nr):
            t0 = time.perf_counter()
            oracle_step(d, wl, sample_rows(nr), (0, nh))
            return time.perf_counter() - t0

        per_step = args.ref_seconds / (args.steps + args.warmup)
        nh, nr = 1, 16
        t = step_seconds(nh, nr)
        while t < per_step:
            for cand in ((min(wl.heads, 2 * nh), nr), (nh, min(wl.n, 2 * nr))):
                if cand == (nh, nr):
                    continue
                tc = step_seconds(*cand)
                if tc <= per_step:
                    (nh, nr), t = cand, tc
                    break
            else:
                break
    rows = sample_rows(nr)
    heads = (0, nh)
    for _ in range(args.warmup):
        oracle_step(d, wl, rows, heads)
    t0 = time.perf_counter()
    fl = 0.0
    for _ in range(args.steps):
        fl += oracle_step(d, wl, rows, heads)
    dt = time.perf_counter() - t0
    v = fl / dt / 1e12
    line = {
        "impl": "reference",
        "metric": "packed-cache attention TFLOP/s (per-layer step)",
        "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": ("one layer, pages scale: B=1, H=12, d_h=128, n=6240, pool 40x182, "
                                "top-16, context 27872 keys; oracle sample per step"),
                   "rows_per_step": int(nr), "heads_per_step": int(nh)},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(), "cpu": cpu_model(), "kind": "oracle",
                         "sample": f"per step, on {nh} of {wl.heads} heads: selection over the whole pool, "
                                   f"sink shift, attention of {nr} of {wl.n} query rows over the "
                                   f"27872-key context; float64 numpy"},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- configs only

def run_suite(args):
    """The extra configurations alone (no headline), one JSON line each."""
    import torch

    import synth
    from packed_kv_cache_b200 import build as pfbuild
    pfbuild.build()
    import packed_kv_cache_b200 as pf

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, src = load_peaks()
    which = {"c2", "c3", "c4"} if args.configs in ("all", "none") else set(args.configs.split(","))
    clocks = ClockSampler(0)
    clocks.start()
    out = measure_configs(which, pf, synth, dev, L2Flush(dev), stream, peaks, src, max(args.steps, 5))
    clocks.stop()
    for k, v in out.items():
        print(json.dumps({"config": k, **v}), flush=True)
    print(json.dumps({"clocks": clocks.window()}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="reference arm: query rows per step on all heads (default: sized to --ref-seconds)")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: host seconds for the warm-up and timed steps together")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default="all",
                    help="workloads measured beside the headline: all, none, or a comma list of c2 (30-layer "
                         "block, 4 denoising steps, CFG batch 2), c3 (dense layer), c4 (stress layers)")
    ap.add_argument("--suite", action="store_true",
                    help="only the --configs workloads, one JSON line each (no headline)")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="heads: one layer spread over the ranks by heads (strong scaling; one NCCL all-reduce "
                         "of the partial block scores per step); none: independent replicas (weak scaling)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.suite:
        run_suite(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
