"""Benchmark: paged decode attention on B200 -- decode tokens/s and KV GB/s.

One step = one decode-attention call of the whole hot path (split planning,
paged block gather, K/V tile streaming, scores, online softmax, P V, split
partials, log-sum-exp combine) over one batch of synthetic inputs resident in
HBM.  Default (headline) workload: the largest single-GPU shape of the
head-sharing sweep, MHA with B=32, H_q=H_kv=32, d=128, T=32768, bf16, 64-token
blocks, random-permutation block table (a 16 GiB cache, far larger than L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl native|reference] [--no-per-config]

Timing: W warm-up steps, then blocks of exactly K steps, each bracketed by a
barrier and a device synchronisation and timed with CUDA events on the
launching stream; blocks repeat until about --min-seconds of timed work has
run (so the clock sampler sees the region) and the median block is reported.
The line also carries `per_config`: every other workload of the benchmark
plan timed the same way (kernel and step time, algorithmic bytes, fraction of
the measured HBM peak).

N > 1 runs under torch.distributed.run, one rank per GPU, each rank with its
own batch (weak scaling; ranks share nothing on the data path -- the only
collectives are the timing barrier and the max-over-ranks reduction).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

L2_BYTES = 126 * 2 ** 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
# Sources of each main kernel: a committed DRAM-traffic figure is used only
# while the hash of these files matches the one recorded with it.
KERNEL_SOURCES = {
    "gqa_split_kernel": ["decode_attention_kv_paged_b200/csrc/gqa_decode.cuh",
                         "decode_attention_kv_paged_b200/csrc/plan.cuh",
                         "decode_attention_kv_paged_b200/csrc/common.cuh"],
    "gqa_tc128_kernel": ["decode_attention_kv_paged_b200/csrc/gqa_tc128.cu",
                         "decode_attention_kv_paged_b200/csrc/tc_common.cuh",
                         "decode_attention_kv_paged_b200/csrc/plan.cuh",
                         "decode_attention_kv_paged_b200/csrc/common.cuh"],
    "gqa_tc_kernel": ["decode_attention_kv_paged_b200/csrc/gqa_tc.cu",
                      "decode_attention_kv_paged_b200/csrc/tc_common.cuh",
                      "decode_attention_kv_paged_b200/csrc/plan.cuh",
                      "decode_attention_kv_paged_b200/csrc/common.cuh"],
    "mla_decode_kernel": ["decode_attention_kv_paged_b200/csrc/mla_decode.cu",
                          "decode_attention_kv_paged_b200/csrc/tc_common.cuh",
                          "decode_attention_kv_paged_b200/csrc/plan.cuh",
                          "decode_attention_kv_paged_b200/csrc/common.cuh"],
}

WORKLOAD_ALIASES = {
    "llama3_8b": W.LLAMA3_8B.name,
    "tiny": W.TINY.name,
    "ragged_full": W.RAGGED_FULL.name,
    "ragged_window": W.RAGGED_WINDOW.name,
    "ragged_window_sink": W.RAGGED_WINDOW_SINK.name,
    "ragged_window_ring": W.RAGGED_WINDOW_RING.name,
    "ragged_window_global": W.RAGGED_WINDOW_GLOBAL.name,
    "llama3_8b_fp8": W.LLAMA3_8B_FP8.name,
    "mla": W.MLA_DSV2.name,
    "mla_fp8": W.MLA_DSV2_FP8.name,
}


HEADLINE = W.sweep_config(32, 32).name


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=HEADLINE,
                    help="headline (default: the largest sweep shape) | llama3_8b | tiny | "
                         "ragged_full | ragged_window | ragged_window_sink | ragged_window_ring "
                         "| ragged_window_global | llama3_8b_fp8 | mla | a sweep name such as "
                         "sweep_bf16_B8_Hq32_Hkv8_d128_T32768")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="repeat K-step blocks until this much timed work has run")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true",
                    help="skip the oracle CPU baseline (profiling runs)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def workload(name):
    if name == "headline":
        name = HEADLINE
    return W.WORKLOADS[WORKLOAD_ALIASES.get(name, name)]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return j, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_hash(kind):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel, wl_name):
    """dram bytes per launch of `kernel` on `wl_name` from the committed ncu
    capture, if the kernel's sources are unchanged since it was taken; else
    None."""
    return traffic_entry(kernel, wl_name)[0]


def traffic_entry(kernel, wl_name):
    """(dram bytes per launch or None, note).  A capture taken on a smaller
    case of the same shape is scaled to a full launch by the units processed
    (its entry records the factor).  The note says why the figure is missing:
    no capture of this kernel on this workload, or a capture of other
    sources of the kernel."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, f"no ncu capture of {kernel}"
    with open(TRAFFIC_FILE) as f:
        j = json.load(f)
    e = j.get(wl_name)
    if not e or e.get("kernel") != kernel:
        return None, f"no ncu capture of {kernel} on this workload"
    if e.get("kernel_hash") != kernel_hash(kernel):
        return None, (f"the ncu capture of {kernel} on this workload "
                      f"({e.get('dram_bytes_per_launch', 0) / 1e6:.1f} MB per launch) was "
                      "taken on other sources of the kernel")
    return e.get("dram_bytes_per_launch"), None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock and throttle-reason samples every 50 ms; the summary
    keeps the samples taken inside the marked timed windows."""
    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.windows = []

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def mark(self, t0, t1):
        """Record a timed window (host wall-clock seconds)."""
        self.windows.append((t0, t1))

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
        return False

    def summary(self):
        import datetime
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[1]), float(parts[2]), parts))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if any(t0 <= r[0] <= t1 for t0, t1 in self.windows)]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for *_, parts in use:
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use),
                "power_w_max": max((float(r[3][3]) for r in use
                                    if r[3][3].replace(".", "", 1).isdigit()), default=None),
                "samples": len(use), "samples_in_timed_region": len(inside),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank scalar over all ranks (timing only; NCCL on GPUs,
    gloo on CPU)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg_seed, rank):
    """Each rank draws its own batch (weak scaling: per-GPU work is fixed)."""
    return cfg_seed + 1000 * rank


def whole_job_tokens_per_s(world, batch, steps, ms_max):
    """Decode tokens/s of the whole job: all ranks' sequences over the
    slowest rank's time."""
    return world * batch * steps / (ms_max / 1e3)


# --------------------------------------------------------------- helpers
def visible_keys(T, window, sink):
    """Keys a decode query of a sequence with T cached tokens sees: the window
    [T - window, T) (all of [0, T) without one) plus the first `sink`."""
    if T <= 0:
        return 0
    lo = max(0, T - window) if window > 0 else 0
    return T - lo + min(sink, lo)


def visible_tiles(T, window, sink):
    """64-token blocks holding at least one visible key."""
    if T <= 0:
        return 0
    lo = max(0, T - window) if window > 0 else 0
    w0, w1 = lo // 64, (T - 1) // 64 + 1
    a = min((sink + 63) // 64, w1)
    return w1 if a >= w0 else a + w1 - w0


def _global_set(row):
    """The positions a global-position row holds (ascending run, -1 pads)."""
    out, prev = [], -1
    for p in row:
        if p <= prev:
            break
        out.append(p)
        prev = p
    return out


def visible_keys_global(T, window, row):
    """visible_keys with an explicit global set: the window, the global
    positions before it, or every key when the query (T - 1) is global."""
    G = [p for p in _global_set(row) if p < T]
    if T <= 0:
        return 0
    if window <= 0 or T - 1 in G:
        return T
    lo = max(0, T - window)
    return T - lo + sum(1 for p in G if p < lo)


def visible_tiles_global(T, window, row):
    if T <= 0:
        return 0
    G = [p for p in _global_set(row) if p < T]
    w1 = (T - 1) // 64 + 1
    if window <= 0 or T - 1 in G:
        return w1
    w0 = max(0, T - window) // 64
    return len({p // 64 for p in G if p // 64 < w0}) + w1 - w0


def kv_row_bytes(cfg):
    """Cache bytes of one (token, KV head) row, K and V together: 2 d s, or
    2 (d + 4) for the fp8 cache (one byte per element plus a fp32 row scale)."""
    if cfg.kv_fp8:
        return 2 * (cfg.d + 4)
    return 2 * cfg.d * (torch.finfo(cfg.dtype).bits // 8)


def algorithmic_bytes_gqa(inp):
    """K+V bytes of visible keys (both caches) + q + out."""
    cfg = inp.cfg
    s = torch.finfo(cfg.dtype).bits // 8
    vis = 0
    rows = inp.global_pos.tolist() if inp.global_pos is not None else None
    for b, T in enumerate(inp.seq_list):
        vis += (visible_keys_global(T, inp.window, rows[b]) if rows
                else visible_keys(T, inp.window, cfg.sink))
    kv = vis * cfg.H_kv * kv_row_bytes(cfg)
    qo = 2 * cfg.B * cfg.H_q * cfg.d * s
    return kv, kv + qo


def tile_bytes_gqa(inp):
    """Bytes the kernel reads in whole 64-token tiles (incl. edge over-read)."""
    cfg = inp.cfg
    s = torch.finfo(cfg.dtype).bits // 8
    blocks = 0
    rows = inp.global_pos.tolist() if inp.global_pos is not None else None
    for b, T in enumerate(inp.seq_list):
        blocks += (visible_tiles_global(T, inp.window, rows[b]) if rows
                   else visible_tiles(T, inp.window, cfg.sink))
    return blocks * 64 * cfg.H_kv * kv_row_bytes(cfg)


def algorithmic_bytes_mla(inp):
    """Latent rows of the visible keys (bf16, or fp8 codes plus a fp32 row
    scale) + q + out."""
    cfg = inp.cfg
    row = (cfg.d_c + cfg.d_r + 4) if cfg.kv_fp8 else (cfg.d_c + cfg.d_r) * 2
    lat = sum(inp.seq_list) * row
    qo = cfg.B * cfg.H * (2 * cfg.d_c + cfg.d_r) * 2
    return lat, lat + qo


def mla_flops(inp):
    cfg = inp.cfg
    return sum(inp.seq_list) * cfg.H * 2 * (2 * cfg.d_c + cfg.d_r)


# ------------------------------------------------------------ native arm
def kernel_name(attn, cfg):
    """The main kernel a decode call of this workload launches."""
    if isinstance(cfg, W.MLAConfig):
        return "mla_decode_kernel"
    _, _, path = attn.gqa_config(cfg.B, cfg.H_q, cfg.H_kv, cfg.d,
                                 "fp8" if cfg.kv_fp8 else cfg.dtype)
    return {0: "gqa_split_kernel", 1: "gqa_tc128_kernel", 2: "gqa_tc_kernel"}[path]


def launches_per_step(kernel):
    """Library kernels one decode call launches: the CUDA-core split kernel
    combines its own splits; the tensor-core and MLA paths add a combine."""
    return 1 if kernel == "gqa_split_kernel" else 2


class Problem:
    """Device-resident inputs of one workload and the decode call over them.
    Caches smaller than 8x the L2 are replicated and rotated so consecutive
    steps never find the previous step's cache in L2."""

    def __init__(self, attn, cfg, dev, seed):
        self.attn, self.cfg = attn, cfg
        self.is_mla = isinstance(cfg, W.MLAConfig)
        make = W.make_mla_inputs if self.is_mla else W.make_gqa_inputs
        base = make(cfg, device=dev, seed=seed)
        if self.is_mla:
            self.kv_bytes, self.alg_bytes = algorithmic_bytes_mla(base)
            cache = base.latent_cache.numel() * base.latent_cache.element_size()
            if base.latent_scale is not None:
                cache += base.latent_scale.numel() * 4
        else:
            self.kv_bytes, self.alg_bytes = algorithmic_bytes_gqa(base)
            cache = 2 * base.k_cache.numel() * base.k_cache.element_size()
            if base.k_scale is not None:
                cache += 2 * base.k_scale.numel() * 4
        self.reps = 1 if cache >= 8 * L2_BYTES else min(64, max(2, math.ceil(3 * L2_BYTES / cache)))
        self.cache_bytes = cache
        self.inputs = [base] + [make(cfg, device=dev, seed=seed + r) for r in range(1, self.reps)]
        self.outs = [torch.empty_like(i.q_lat if self.is_mla else i.q) for i in self.inputs]
        self.base = base
        if self.reps * cache > 2 * L2_BYTES:
            self.l2 = (f"inputs larger than L2: {self.reps} cache replica(s) of "
                       f"{cache / 2**20:.0f} MiB, rotated")
        else:
            self.l2 = (f"L2-resident: {self.reps} replicas of {cache / 2**10:.0f} KiB "
                       "(launch-bound case)")

    def step(self, i):
        attn, cfg = self.attn, self.cfg
        x, out = self.inputs[i % self.reps], self.outs[i % self.reps]
        if self.is_mla and cfg.kv_fp8:
            attn.decode_mla_fp8(x.q_lat, x.q_rope, x.latent_cache, x.latent_scale, x.seq_lens,
                                x.block_table, x.scale, out=out)
        elif self.is_mla:
            attn.decode_mla(x.q_lat, x.q_rope, x.latent_cache, x.seq_lens, x.block_table,
                            x.scale, out=out)
        elif cfg.kv_fp8:
            attn.decode_gqa_fp8(x.q, x.k_cache, x.v_cache, x.k_scale, x.v_scale, x.seq_lens,
                                x.block_table, x.scale, window=x.window, sink_tokens=cfg.sink,
                                ring_blocks=cfg.ring, out=out)
        else:
            attn.decode_gqa_ext(x.q, x.k_cache, x.v_cache, x.seq_lens, x.block_table, x.scale,
                                window=x.window, sink_tokens=cfg.sink, ring_blocks=cfg.ring,
                                out=out, global_pos=x.global_pos)


def time_blocks(attn, step, K, warmup, min_s, world, clk=None, max_blocks=200):
    """W warm-up steps, then blocks of exactly K steps, each between a barrier
    and a device synchronisation, timed with CUDA events on the launching
    stream, repeated until min_s seconds of (slowest-rank) timed work; every
    rank takes the same number of blocks (the stop test uses the max over
    ranks).  These blocks run the decode calls exactly as a caller would
    (nothing recorded between a call's kernels, so a tensor-core path's
    combine launch overlaps its main kernel).  Then a few more K-step blocks
    with the library recording events around each call's main kernel give
    that kernel's own duration."""
    for i in range(max(warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    if attn.last_error() != attn.OK:
        raise SystemExit("device error during warm-up")
    n = max(warmup, 3)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)

    def block(prof):
        nonlocal n
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.time()
        if prof is not None:
            prof.__enter__()
        ev0.record()
        for i in range(K):
            step(n + i)
        ev1.record()
        if prof is not None:
            prof.__exit__(None, None, None)
        torch.cuda.synchronize()
        barrier(world)
        t1 = time.time()
        if clk is not None:
            clk.mark(t0, t1)
        n += K
        return max_over_ranks(ev0.elapsed_time(ev1), world)

    block_ms = []
    total = 0.0
    while True:
        ms = block(None)
        block_ms.append(ms)
        total += ms / 1e3
        if total >= min_s or len(block_ms) >= max_blocks:
            break
    kern_ms = []
    prof_blocks = max(1, min(5, math.ceil(0.2 / max(statistics.median(block_ms) / 1e3, 1e-6))))
    for _ in range(prof_blocks):
        prof = attn.ProfileEvents(K)
        block(prof)
        kern_ms.extend(prof.times_ms(K))
    if attn.last_error() != attn.OK:
        raise SystemExit("device error during the timed region")
    return {"block_ms": block_ms, "prof_blocks": prof_blocks,
            "ms_per_step": statistics.median(block_ms) / K,
            "kernel_ms_avg": max_over_ranks(sum(kern_ms) / len(kern_ms), world),
            "kernel_ms_median": max_over_ranks(statistics.median(kern_ms), world)}


def roofline_entry(prob, kernel, kern_ms, pk):
    """Fraction of the binding roofline of the dominant kernel: HBM bytes for
    the GQA family; for MLA the tighter of HBM bytes and tensor-core FLOPs."""
    cfg = prob.cfg
    t = kern_ms / 1e3
    roof = None
    if prob.is_mla:
        flops = mla_flops(prob.base)
        t_hbm = prob.alg_bytes / (pk["hbm_gbs"] * 1e9)
        t_tc = flops / (pk.get("bf16_tflops", 1590.0) * 1e12)
        if t_tc > t_hbm:
            roof = {"bound": "tensor", "achieved": flops / t / 1e12,
                    "peak": pk.get("bf16_tflops"), "unit": "TFLOP/s"}
    if roof is None:
        roof = {"bound": "hbm", "achieved": prob.alg_bytes / t / 1e9, "peak": pk["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = kernel
    roof["kernel_ms_avg"] = kern_ms
    roof["algorithmic_bytes_per_launch"] = prob.alg_bytes
    roof["traffic"], note = traffic_entry(kernel, cfg.name)
    if note:
        roof["traffic_note"] = note
    if prob.is_mla:
        roof["flops_per_launch"] = mla_flops(prob.base)
        roof["tensor_frac"] = (mla_flops(prob.base) / t / 1e12) / pk.get("bf16_tflops", 1590.0)
        roof["hbm_frac"] = (prob.alg_bytes / t / 1e9) / pk["hbm_gbs"]
    return roof


def config_entry(attn, cfg, dev, seed, K, warmup, min_s, pk, clk=None):
    """Time one workload (one rank) and describe it for `per_config`."""
    prob = Problem(attn, cfg, dev, seed)
    r = time_blocks(attn, prob.step, K, warmup, min_s, 1, clk=clk, max_blocks=50)
    kernel = kernel_name(attn, cfg)
    roof = roofline_entry(prob, kernel, r["kernel_ms_avg"], pk)
    e = {"workload": cfg.name, "kernel": kernel,
         "kernel_us": r["kernel_ms_avg"] * 1e3, "step_us": r["ms_per_step"] * 1e3,
         "algorithmic_bytes": prob.alg_bytes, "kv_bytes": prob.kv_bytes,
         "tokens_per_s": cfg.B / (r["ms_per_step"] / 1e3),
         "kernel_gbs": prob.alg_bytes / (r["kernel_ms_avg"] / 1e3) / 1e9,
         "frac_of_measured_hbm": prob.alg_bytes / (r["kernel_ms_avg"] / 1e3) / 1e9
         / pk["hbm_gbs"],
         "frac_of_8tbs_spec": prob.alg_bytes / (r["kernel_ms_avg"] / 1e3) / 1e9 / 8000.0,
         "bound": roof["bound"], "frac": roof["frac"], "traffic": roof["traffic"],
         "steps_timed": K * len(r["block_ms"]), "l2": prob.l2}
    if "traffic_note" in roof:
        e["traffic_note"] = roof["traffic_note"]
    if prob.is_mla:
        e["tensor_frac"] = roof["tensor_frac"]
        e["flops"] = roof["flops_per_launch"]
        if not cfg.kv_fp8:
            e["mla_absorb"] = mla_absorb_timing(attn, cfg, dev, seed)
    else:
        e["tile_overread_bytes"] = tile_bytes_gqa(prob.base) - prob.kv_bytes
    del prob
    torch.cuda.empty_cache()
    return e


# Every workload of the benchmark plan, by what it is (the headline excluded
# at run time): the tiny fp32 case, the Llama-3-8B shape, the nine points of
# the head-sharing sweep, the ragged 24/4/256 shape full and with w=4096, the
# DeepSeek-V2 MLA shape; then the window/global/ring and fp8-cache variants.
PER_CONFIG = [W.TINY, W.LLAMA3_8B, *W.SWEEP, W.RAGGED_FULL, W.RAGGED_WINDOW, W.MLA_DSV2,
              W.LLAMA3_8B_FP8, W.MQA_B8_FP8, W.MLA_DSV2_FP8, W.RAGGED_WINDOW_SINK,
              W.RAGGED_WINDOW_RING,
              W.RAGGED_WINDOW_GLOBAL]


def run_native(args, rank, world, local):
    import decode_attention_kv_paged_b200 as attn
    attn.load()
    cfg = workload(args.workload)
    dev = torch.device("cuda", local)
    pk, pk_kind = peaks()
    K = args.steps
    prob = Problem(attn, cfg, dev, rank_seed(cfg.seed, rank))
    with ClockSampler(local) as clk:
        r = time_blocks(attn, prob.step, K, args.warmup, args.min_seconds, world, clk=clk)
    kernel = kernel_name(attn, cfg)
    roof = roofline_entry(prob, kernel, r["kernel_ms_avg"], pk)
    roof["peak_source"] = pk_kind
    ms = r["ms_per_step"]
    B = cfg.B
    kv_gbs = world * prob.kv_bytes / (ms / 1e3) / 1e9
    line = {
        "metric": "decode tokens/s and KV-cache read GB/s (% of B200 HBM peak), 1 GPU",
        "value": whole_job_tokens_per_s(world, B, 1, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("fp8e4m3 cache, bf16 q/out, f32 accumulate" if getattr(cfg, "kv_fp8", False)
                  else "bf16" if cfg.dtype == torch.bfloat16 else "f32"),
        "data": "synthetic (seeded N(0,1) q/K/V, random-permutation block table)",
        "config": {"workload": cfg.name, "global_batch": B * world,
                   "seq_len": getattr(cfg, "T", None) or max(prob.base.seq_list),
                   "parallelism": f"dp{world} (independent batches, no collective)",
                   "l2": prob.l2},
        "timing": {"blocks": len(r["block_ms"]), "steps_per_block": K,
                   "kernel_event_blocks": r["prof_blocks"],
                   "ms_per_step_median_block": ms,
                   "ms_per_step_min_block": min(r["block_ms"]) / K,
                   "ms_per_step_max_block": max(r["block_ms"]) / K,
                   "kernel_ms_median": r["kernel_ms_median"]},
        "kv_gbs": kv_gbs,
        "kv_frac_of_peak": kv_gbs / world / pk["hbm_gbs"],
        "kv_frac_of_8tbs_spec": kv_gbs / world / 8000.0,
        "roofline": roof,
        "gpu_launches": launches_per_step(kernel) * K * len(r["block_ms"]),
        "gpu_launches_per_step": launches_per_step(kernel),
        "clocks": clk.summary(),
    }
    if not prob.is_mla:
        line["tile_overread_bytes_per_step"] = tile_bytes_gqa(prob.base) - prob.kv_bytes
    e2e_input = prob.inputs[0]
    del prob
    if not args.no_e2e:
        line["e2e"] = e2e_native(attn, cfg, e2e_input, isinstance(cfg, W.MLAConfig), K, world,
                                 dev)
    del e2e_input
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_config:
        entries = []
        with ClockSampler(local) as pclk:
            for c in PER_CONFIG:
                if c.name == cfg.name:
                    continue
                entries.append(config_entry(attn, c, dev, c.seed, K, args.warmup, 0.05, pk,
                                            clk=pclk))
        line["per_config"] = {"peak_gbs": pk["hbm_gbs"], "peak_source": pk_kind,
                              "clocks": pclk.summary(), "entries": entries}
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, isinstance(cfg, W.MLAConfig), args.cpu_seconds)
    return line


def mla_absorb_timing(attn, cfg, dev, seed, iters=16):
    """Time of the products either side of the absorbed decode at this shape
    (q_c (U^K)^T before, z U^V after), per call; each streams the per-head
    weights (H x d_c x 128 bf16) once.  `*_us`: device time per call, from a
    CUDA graph of `iters` back-to-back calls (the entry points allocate
    nothing, so they capture); `*_api_us`: the same calls issued from Python
    one by one (host overhead included)."""
    # Eight weight sets (8 x 2 x 16.8 MB, more than the L2) used in turn, so
    # each call streams its weights from HBM as a decode step would.
    ws = [W.make_mla_absorb_inputs(cfg, device=dev, seed=seed + r) for r in range(8)]
    w = ws[0]
    z = torch.empty((cfg.B, cfg.H, cfg.d_c), dtype=torch.bfloat16, device=dev).normal_()
    q_out = torch.empty((cfg.B, cfg.H, cfg.d_c), dtype=torch.bfloat16, device=dev)
    o_out = torch.empty((cfg.B, cfg.H, w.U_V.shape[2]), dtype=torch.bfloat16, device=dev)
    out = {}
    it = [0]

    def nxt():
        it[0] += 1
        return ws[it[0] % len(ws)]

    for name, fn in (("absorb_q", lambda: attn.mla_absorb_q(w.q_c, nxt().U_K, out=q_out)),
                     ("project_out", lambda: attn.mla_project_out(z, nxt().U_V, out=o_out))):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name + "_api_us"] = e0.elapsed_time(e1) * 1e3 / iters
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(iters):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(5):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        out[name + "_us"] = e0.elapsed_time(e1) * 1e3 / (5 * iters)
        del g
    wbytes = cfg.H * cfg.d_c * 128 * 2
    out["weight_bytes_each"] = wbytes
    out["absorb_q_gbs"] = wbytes / (out["absorb_q_us"] * 1e-6) / 1e9
    out["project_out_gbs"] = wbytes / (out["project_out_us"] * 1e-6) / 1e9
    out["note"] = ("device time per call from a CUDA graph of back-to-back calls cycling over "
                   "8 weight sets (larger than L2); *_api_us issue the calls from Python one by one")
    return out


def e2e_native(attn, cfg, x, is_mla, K, world, dev):
    """The same metric through the public API with host buffers: each step
    copies the new token's q (and K/V or latent row) from pinned host memory,
    appends it to the paged cache at position T-1, runs decode attention and
    reads the output back to the host."""
    B = cfg.B
    g = torch.Generator().manual_seed(7)
    if is_mla:
        width = cfg.d_c + cfg.d_r
        h_q = W.randn((B, cfg.H, cfg.d_c), g, torch.bfloat16).pin_memory()
        h_r = W.randn((B, cfg.H, cfg.d_r), g, torch.bfloat16).pin_memory()
        h_lat = W.randn((B, width), g, torch.bfloat16).pin_memory()
        h_out = torch.empty((B, cfg.H, cfg.d_c), dtype=torch.bfloat16).pin_memory()
        d_q, d_r, d_lat = (torch.empty_like(t, device=dev) for t in (h_q, h_r, h_lat))
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_r, h_lat))
    else:
        h_q = W.randn((B, cfg.H_q, cfg.d), g, cfg.dtype).pin_memory()
        h_k = W.randn((B, cfg.H_kv, cfg.d), g, cfg.dtype).pin_memory()
        h_v = W.randn((B, cfg.H_kv, cfg.d), g, cfg.dtype).pin_memory()
        h_out = torch.empty_like(h_q).pin_memory()
        d_q, d_k, d_v = (torch.empty_like(t, device=dev) for t in (h_q, h_k, h_v))
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v))
    d2h = h_out.numel() * h_out.element_size()
    pos = (x.seq_lens - 1).clamp(min=0).contiguous()
    d_out = torch.empty_like(h_out, device=dev)

    def step():
        d_q.copy_(h_q, non_blocking=True)
        if is_mla:
            d_r.copy_(h_r, non_blocking=True)
            d_lat.copy_(h_lat, non_blocking=True)
            if cfg.kv_fp8:
                attn.kv_append_mla_fp8(d_lat, x.latent_cache, x.latent_scale, pos,
                                       x.block_table)
                attn.decode_mla_fp8(d_q, d_r, x.latent_cache, x.latent_scale, x.seq_lens,
                                    x.block_table, x.scale, out=d_out)
            else:
                attn.kv_append_mla(d_lat, x.latent_cache, pos, x.block_table)
                attn.decode_mla(d_q, d_r, x.latent_cache, x.seq_lens, x.block_table,
                                x.scale, out=d_out)
        else:
            d_k.copy_(h_k, non_blocking=True)
            d_v.copy_(h_v, non_blocking=True)
            vis = dict(window=x.window, sink_tokens=cfg.sink, ring_blocks=cfg.ring)
            if cfg.kv_fp8:
                attn.kv_append_fp8(d_k, d_v, x.k_cache, x.v_cache, x.k_scale, x.v_scale, pos,
                                   x.block_table, **vis)
                attn.decode_gqa_fp8(d_q, x.k_cache, x.v_cache, x.k_scale, x.v_scale,
                                    x.seq_lens, x.block_table, x.scale, out=d_out, **vis)
            else:
                attn.kv_append_ext(d_k, d_v, x.k_cache, x.v_cache, pos, x.block_table, **vis)
                attn.decode_gqa_ext(d_q, x.k_cache, x.v_cache, x.seq_lens, x.block_table,
                                    x.scale, out=d_out, global_pos=x.global_pos, **vis)
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    # Host round trip per step: the host has each step's output in hand
    # before it issues the next step's copies (a decode loop's latency).
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(K):
        step()
        stream.synchronize()
    t1 = time.perf_counter()
    barrier(world)
    ms = max_over_ranks((t1 - t0) * 1e3, world)
    # The same steps issued back to back without a host wait in between.
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(K):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms_pipe = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": world * B * K / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / K,
            "pipelined_tokens_per_s": world * B * K / (ms_pipe / 1e3),
            "pipelined_ms_per_step": ms_pipe / K,
            "note": "step = H2D of the new token's q/K/V from pinned host memory + kv_append "
                    "+ decode + D2H of the output, and the host waits for the output before "
                    "the next step (wall clock, max over ranks); pipelined_* issue the same "
                    "steps without the host wait (CUDA events)"}


# ------------------------------------------------------------- oracle arm
def _oracle_problem(cfg, is_mla, seqs, seed):
    """Host-resident inputs of the first `seqs` sequences of the workload."""
    if is_mla:
        sub = W.MLAConfig(cfg.name, B=seqs, H=cfg.H, d_c=cfg.d_c, d_r=cfg.d_r,
                          T=cfg.T, seed=seed, kv_fp8=cfg.kv_fp8)
        return W.make_mla_inputs(sub)
    lens = None
    if cfg.ragged:
        g = torch.Generator().manual_seed(cfg.seed)
        lens = W.draw_seq_lens(cfg, g)[:seqs]
    sub = W.GQAConfig(cfg.name, B=seqs, H_q=cfg.H_q, H_kv=cfg.H_kv, d=cfg.d,
                      seq_lens=lens, T=cfg.T, dtype=cfg.dtype, window=cfg.window,
                      sink=cfg.sink, ring=cfg.ring, kv_fp8=cfg.kv_fp8,
                      contiguous=cfg.contiguous, seed=seed, n_global=cfg.n_global)
    return W.make_gqa_inputs(sub)


def _oracle_call(orc, x, is_mla):
    if is_mla and x.cfg.kv_fp8:
        lat = orc.dequantize_e4m3(x.latent_cache.numpy(), x.latent_scale.numpy())
        return orc.decode_mla(x.q_lat.double().numpy(), x.q_rope.double().numpy(), lat,
                              x.seq_lens, x.block_table, x.scale)
    if is_mla:
        return orc.decode_mla(x.q_lat, x.q_rope, x.latent_cache, x.seq_lens,
                              x.block_table, x.scale)
    if x.cfg.kv_fp8:
        k = orc.dequantize_e4m3(x.k_cache.numpy(), x.k_scale.numpy())
        v = orc.dequantize_e4m3(x.v_cache.numpy(), x.v_scale.numpy())
        return orc.decode_gqa_vis(x.q.double().numpy(), k, v, x.seq_lens, x.block_table,
                                  x.scale, window=x.window, sink=x.cfg.sink, ring=x.cfg.ring)
    return orc.decode_gqa_vis(x.q, x.k_cache, x.v_cache, x.seq_lens, x.block_table,
                              x.scale, window=x.window, sink=x.cfg.sink, ring=x.cfg.ring,
                              global_pos=x.global_pos)


def _pick_sample(cfg, is_mla, orc, target_s):
    """Sequences per oracle call sized to ~target_s of CPU time."""
    x = _oracle_problem(cfg, is_mla, 1, cfg.seed)
    t0 = time.perf_counter()
    _oracle_call(orc, x, is_mla)
    one = max(time.perf_counter() - t0, 1e-4)
    return max(1, min(cfg.B, int(target_s / one))), one


def cpu_baseline(cfg, is_mla, target_s):
    import oracle as orc
    cores = os.cpu_count() or 1
    orc.set_threads(cores)
    n, _ = _pick_sample(cfg, is_mla, orc, target_s)
    x = _oracle_problem(cfg, is_mla, n, cfg.seed)
    # Repeat the pass until about target_s seconds of CPU work have run.
    passes, t0 = 0, time.perf_counter()
    while True:
        _oracle_call(orc, x, is_mla)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or passes >= 100000:
            break
    return {"value": n * passes / dt, "unit": "tokens/s", "cores": orc.get_threads(),
            "kind": "oracle",
            "sample": f"{n} of the workload's {cfg.B} sequences (fp64 C oracle, "
                      f"OpenMP), {passes} pass(es), {dt:.1f} s"}


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle as it stands, on the host cores."""
    if rank != 0:
        return None
    import oracle as orc
    cfg = workload(args.workload)
    is_mla = isinstance(cfg, W.MLAConfig)
    cores = os.cpu_count() or 1
    orc.set_threads(cores)
    # bound the whole run to a few minutes: each step ~ budget / (K + W)
    per_step = max(0.2, min(3.0, 150.0 / max(1, args.steps + args.warmup)))
    n, _ = _pick_sample(cfg, is_mla, orc, per_step)
    x = _oracle_problem(cfg, is_mla, n, cfg.seed)
    for _ in range(max(args.warmup, 3) if per_step < 1 else 1):
        _oracle_call(orc, x, is_mla)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_call(orc, x, is_mla)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = (f"{n} of {cfg.B} sequences per step (fp64 C oracle, OpenMP over "
              f"{orc.get_threads()} threads)")
    return {
        "impl": "reference",
        "metric": "decode tokens/s and KV-cache read GB/s (% of B200 HBM peak), 1 GPU",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (same seeded recipe)",
        "config": {"workload": cfg.name, "global_batch": cfg.B},
        "cpu_baseline": {"value": value, "unit": "tokens/s",
                         "cores": orc.get_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        line = run_native(args, rank, world, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
