"""Benchmark of the attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step is one pass of the whole hot path over one batch of synthetic
input: the fused causal forward pass on the long-prefill workload
(B=1, H=32, N=16384, d=128, bf16) followed by paged decode on the
paged-decode workload (64 sequences, H=32, d=128, KV lengths uniform in
[1024, 32768], 256-token pages).  Inputs are resident in HBM before the timed
region; both working sets are larger than the 126 MB L2 (384 MB and ~17.7 GB),
so no flush runs between steps.

Printed: one JSON line (rank 0).  `value` is forward TFLOP/s (FLOPs counted as
4*B*H*N^2*d, halved for causal) from CUDA events around the forward launches;
`decode` carries the paged-decode GB/s (algorithmic K/V + q + o + table bytes).
With N GPUs (torchrun, one process per GPU) every rank runs an independent
replica of the step ("replicas only": the path has no exchange step); times
are the max over ranks and `value` counts the work of all ranks.

--impl reference times the fp64 CPU oracle as it stands, on a bounded sample
of the same workload, on this machine's host cores (rank 0 only).
"""
import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from attn_fwd_04_b200 import workloads as W  # noqa: E402

METRIC = "attn fwd TFLOPS & % of BF16 tensor peak; paged-decode HBM GB/s (1×B200)"
FWD = W.LONG_PREFILL
DEC = W.PAGED_DECODE
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0, "sustained_sm_mhz": 1300.0}


# ---------------------------------------------------------------------------
# helpers shared by both arms
# ---------------------------------------------------------------------------
def fwd_flops(w=FWD) -> float:
    f = 4.0 * w.B * w.H * w.N * w.N * w.d
    return f / 2 if w.causal else f


def decode_bytes(seq_lens, H, d, B, H_kv=None) -> float:
    """Algorithmic bytes of one decode launch: every cached K and V element
    once (H_kv heads, default H), q and o (H heads), the page table and the
    lengths."""
    Hk = H if H_kv is None else H_kv
    tokens = float(sum(int(x) for x in seq_lens))
    pages = float(sum((int(x) + 255) // 256 for x in seq_lens))
    return tokens * Hk * d * 2 * 2 + 2 * B * H * d * 2 + pages * 4 + B * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        cl = j.get("clocks_under_load") or {}
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j["bf16_tflops_sustained"]),
                "sm_max_mhz": float(j.get("sm_max_mhz") or FALLBACK_PEAKS["sm_max_mhz"]),
                "sustained_sm_mhz": float(cl.get("sm_mhz_median") or
                                          FALLBACK_PEAKS["sustained_sm_mhz"]),
                "source": "measured"}
    except Exception:
        d = dict(FALLBACK_PEAKS)
        d["source"] = "fallback"
        return d


def tensor_peak_regime(peaks, clocks, region_ms):
    """Which measured GEMM peak a forward timing is compared with.

    The pool's cuBLAS figures were taken in two regimes: a burst at the full
    SM clock (bf16_tflops) and a seconds-long loop held at the 1000 W power
    cap (bf16_tflops_sustained).  A timed region during which the power cap
    was active (sw_power_cap among the reasons sampled inside it) is in the
    sustained regime, one without it in the burst regime.  Without a reason
    list, the median SM clock decides (nearer the burst GEMM's full clock or
    the sustained GEMM's median); without clock samples, the region's length
    (under 2 s: burst).  Returns (regime, peak TFLOP/s, reason)."""
    hi, lo = peaks["sm_max_mhz"], peaks["sustained_sm_mhz"]
    clocks = clocks or {}
    sm_mhz = clocks.get("sm_mhz")
    reasons = clocks.get("reasons")
    if sm_mhz is not None and isinstance(reasons, list):
        burst = "sw_power_cap" not in reasons
        why = (f"power cap {'not ' if burst else ''}active during the timed region "
               f"(median SM clock {sm_mhz:.0f} MHz)")
    elif sm_mhz is not None:
        burst = sm_mhz >= 0.5 * (hi + lo)
        why = (f"median SM clock {sm_mhz:.0f} MHz during the timed region, against "
               f"{hi:.0f} (burst GEMM) and {lo:.0f} (sustained GEMM)")
    else:
        burst = region_ms < 2000.0
        why = f"no clock samples; timed region {region_ms / 1e3:.2f} s long"
    if burst:
        return "burst", peaks["bf16_tflops"], why
    return "sustained", peaks["bf16_tflops_sustained"], why


def kernel_source_sha(files):
    """Hash of the kernel's code: the files with their comments and white
    space removed, so that a comment edit does not mark a capture stale."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "attn_fwd_04_b200", "csrc", f), encoding="utf-8") as fh:
            code = re.sub(r"/\*.*?\*/", " ", fh.read(), flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, sha: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic_per_launch.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = dict(x.split("=", 1) for x in line.split() if "=" in x)
        if parts.get("kernel") == kernel and parts.get("src_sha") == sha:
            try:
                return float(parts["dram_bytes"])
            except (KeyError, ValueError):
                return None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling around the timed region.

    A reader thread stamps every sample with the host's monotonic clock when
    it arrives, so that the samples taken while the timed region ran (between
    mark_start() and mark_end(), the host enqueueing the region right after
    the first mark and waiting for it to finish before the second) can be told
    apart from those taken before and after it."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except Exception:
            self.proc = None
            return

        def reader():
            for line in self.proc.stdout:
                self.lines.append((time.monotonic(), line))

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    @classmethod
    def parse(cls, stamped, t0=None, t1=None):
        """Summary of (time, csv line) samples: the median SM clock, max clock,
        the throttle reasons seen, over the samples inside [t0, t1] (all when
        no sample falls inside)."""
        rows = []
        for t, line in stamped:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm, smax = float(f[1]), float(f[2])
            except ValueError:
                continue
            try:
                pw = float(f[3])
            except ValueError:
                pw = None
            rows.append((t, sm, smax, pw, [n for n, v in zip(cls.REASONS, f[5:9])
                                             if v.lower() == "active"]))
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        use = inside if inside else rows
        sm = [r[1] for r in use]
        pw = [r[3] for r in use if r[3] is not None]
        reasons = sorted({n for r in use for n in r[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in use) if use else None,
                "samples": len(use), "samples_in_timed_region": len(inside),
                "window": "timed region" if inside else "around the timed region (none inside)",
                "reasons": reasons,
                "power_w_median": statistics.median(pw) if pw else None}

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(2 * self.period_ms / 1e3)  # let the last in-region sample arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        return self.parse(list(self.lines), self.t0, self.t1)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def reduce_max(values, world):
    """Element-wise max of a list of floats over ranks."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def job_rate(world: int, work_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the work every rank did (ranks are replicas of
    the same step) over the slowest rank's time, in work units per second."""
    return world * work_per_rank_step * steps / (max_ms * 1e-3)


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle samples (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_rows_sample(slices, target_s: float, seed: int, causal: bool = True):
    """Time the oracle on seeded random query rows of one-head problems,
    growing the sample until it has run about target_s seconds.  `slices` are
    (q, k, v) fp64 arrays [1, 1, L, d], converted once outside the timing.
    FLOPs are counted like the GPU numbers: 4*L*d per row, halved when
    causal.  Returns (TFLOP/s, rows, seconds)."""
    import oracle
    g = torch.Generator().manual_seed(seed)
    done_flops, done_rows, spent, count = 0.0, 0, 0.0, 32
    while spent < target_s:
        for qh, kh, vh in slices:
            L, d = qh.shape[2], qh.shape[3]
            rows = sorted(set(torch.randint(0, L, (count,), generator=g).tolist()))
            t0 = time.perf_counter()
            oracle.attention(qh, kh, vh, causal, 1 / math.sqrt(d), rows=rows)
            spent += time.perf_counter() - t0
            done_rows += len(rows)
            done_flops += len(rows) * 4.0 * L * d / (2 if causal else 1)
        count = min(count * 2, 4096)
    return done_flops / spent / 1e12, done_rows, spent


def _f64_slice(t):
    import numpy as np
    return np.ascontiguousarray(t.double().cpu().numpy())[None, None]


def oracle_fwd_sample(q, k, v, target_s: float, seed: int, n_heads: int = 2):
    """The oracle on seeded random rows of `n_heads` seeded heads of the
    long-prefill workload (q, k, v [1, H, N, d]) -> (TFLOP/s, rows, seconds)."""
    H = q.shape[1]
    g = torch.Generator().manual_seed(seed)
    heads = torch.randperm(H, generator=g)[:n_heads].tolist()
    slices = [tuple(_f64_slice(t[0, h]) for t in (q, k, v)) for h in heads]
    return oracle_rows_sample(slices, target_s, seed + 1, FWD.causal)


def oracle_other_workloads(target_s: float):
    """The oracle on the batched, variable-length and 128K-context forward
    workloads: seeded random rows of two seeded (sequence, head) problems of
    each, about target_s seconds apiece.  For the 128K context the full
    launch's oracle time is extrapolated from the sampled rate by FLOPs."""
    out = {}
    for w in (W.BATCHED, W.CTX128K):
        q, k, v = W.fwd_inputs(w, device="cuda")[:3]
        g = torch.Generator().manual_seed(w.seed)
        picks = [(int(torch.randint(0, w.B, (1,), generator=g)),
                  int(torch.randint(0, w.H, (1,), generator=g))) for _ in range(2)]
        slices = [tuple(_f64_slice(t[b, h]) for t in (q, k, v)) for b, h in picks]
        del q, k, v
        tf, rows, secs = oracle_rows_sample(slices, target_s, w.seed, w.causal)
        d = {"value": tf, "unit": "TFLOP/s",
             "sample": f"{rows} seeded random rows of (sequence, head) {picks}, {secs:.1f} s"}
        if w is W.CTX128K:
            d["extrapolated_full_launch_s"] = fwd_flops(w) / (tf * 1e12)
            d["note"] = "full-launch time extrapolated from the sampled rate by FLOPs"
        out[w.name] = d
    w = W.BATCHED_VARLEN
    q, k, v, cu = W.varlen_workload_inputs(w, device="cuda")
    g = torch.Generator().manual_seed(w.seed)
    picks = [(int(torch.randint(0, w.B, (1,), generator=g)),
              int(torch.randint(0, w.H, (1,), generator=g))) for _ in range(2)]
    slices = [tuple(_f64_slice(t[int(cu[b]):int(cu[b + 1]), h]) for t in (q, k, v))
              for b, h in picks]
    del q, k, v
    tf, rows, secs = oracle_rows_sample(slices, target_s, w.seed, w.causal)
    out[w.name] = {"value": tf, "unit": "TFLOP/s",
                   "sample": f"{rows} seeded random rows of (sequence, head) {picks} "
                             f"(lengths {[int(cu[b + 1] - cu[b]) for b, _ in picks]}), "
                             f"{secs:.1f} s"}
    torch.cuda.empty_cache()
    return out


def oracle_decode_sample(cache: W.PagedCache, target_s: float):
    """Time the oracle's paged decode on whole sequences of the decode
    workload (shortest first) for about target_s seconds -> GB/s."""
    import oracle
    lens = cache.seq_lens.tolist()
    order = sorted(range(len(lens)), key=lambda b: lens[b])
    H, d = cache.q.shape[1], cache.q.shape[2]
    spent, nbytes, seqs = 0.0, 0.0, 0
    for b in order:
        off = sum(cache.pages_per_seq[:b])
        n = cache.pages_per_seq[b]
        idx = cache.page_table[off:off + n].long().to(cache.k_pages.device)
        kp = cache.k_pages.index_select(0, idx).cpu()
        vp = cache.v_pages.index_select(0, idx).cpu()
        t0 = time.perf_counter()
        oracle.decode_paged(cache.q[b:b + 1].cpu(), kp, vp, torch.arange(n, dtype=torch.int32),
                            cache.seq_lens[b:b + 1].cpu(), cache.page_size)
        spent += time.perf_counter() - t0
        nbytes += decode_bytes([lens[b]], H, d, 1)
        seqs += 1
        if spent >= target_s:
            break
    return nbytes / spent / 1e9, seqs, spent


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------
# grouped-query variants of the long-prefill and paged-decode workloads:
# 32 query heads over 8 K/V heads (groups of 4)
GQA_HKV = 8


def secondary_workloads(fa, stream, steps: int = 5, warmup: int = 3):
    """Throughput on the other workloads (tiny, batched, variable-length, 128K
    context; the grouped-query forward and decode), timed with CUDA events,
    each after a 0.5 s idle pause; reported beside the headline number, not
    part of the timed step."""
    out = {}

    def timed(fn, flops, name, extra=None, n=steps):
        # every workload starts from an idle GPU, so that none inherits the
        # power-capped clock of the one before it
        torch.cuda.synchronize()
        time.sleep(0.5)
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if fa.fa_get_device_error() != fa.FA_OK:
            raise RuntimeError(f"device error on {name}")
        ms = e0.elapsed_time(e1) / n
        d = {"ms_per_launch": ms, "tflops": flops / (ms * 1e-3) / 1e12,
             "pct_of_2250": 100 * flops / (ms * 1e-3) / 1e12 / DATASHEET_BF16_TFLOPS}
        d.update(extra or {})
        out[name] = d

    # the headline forward alone in a short burst after an idle pause: the
    # power controller has not yet brought the clock down (the headline value
    # is the sustained rate of the long timed region)
    q, k, v = W.fwd_inputs(FWD, device="cuda")[:3]
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    timed(lambda: fa.fa_fwd(q, k, v, FWD.causal, 1 / math.sqrt(FWD.d), o=o, lse=lse,
                            stream=stream),
          fwd_flops(FWD), FWD.name + "_burst20", {"what": "20 launches after 0.5 s idle"}, n=20)
    del q, k, v, o, lse
    for w in (W.TINY_CAUSAL, W.BATCHED, W.CTX128K):
        q, k, v = W.fwd_inputs(w, device="cuda")[:3]
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        sc = 1 / math.sqrt(w.d)
        timed(lambda: fa.fa_fwd(q, k, v, w.causal, sc, o=o, lse=lse, stream=stream),
              fwd_flops(w), w.name)
        del q, k, v, o, lse
    w = W.BATCHED_VARLEN
    q, k, v, cu = W.varlen_workload_inputs(w, device="cuda")
    lens = (cu[1:] - cu[:-1]).tolist()
    cud = cu.cuda()
    o = torch.empty_like(q)
    lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=q.device)
    flops = sum(4.0 * w.H * L * L * w.d / (2 if w.causal else 1) for L in lens)
    sc = 1 / math.sqrt(w.d)
    timed(lambda: fa.fa_fwd_varlen(q, k, v, cud, max(lens), w.causal, sc, o=o, lse=lse,
                                   stream=stream),
          flops, w.name, {"lengths": lens})
    del q, k, v, cu, cud, o, lse
    # grouped-query forward: long-prefill shape, 8 K/V heads
    w = FWD
    q, k, v = W.gqa_fwd_inputs(w.B, w.H, GQA_HKV, w.N, w.d, seed=21, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    timed(lambda: fa.fa_fwd_gqa(q, k, v, True, 1 / math.sqrt(w.d), o=o, lse=lse, stream=stream),
          fwd_flops(w), f"gqa_long_prefill_fwd_b1_h32_hkv{GQA_HKV}_n16384_d128_causal")
    del q, k, v, o, lse
    # rotary embedding fused into the forward pass: the long-prefill workload
    q, k, v = W.fwd_inputs(w, device="cuda")
    rc, rs = W.rope_tables(w.N, w.d, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    timed(lambda: fa.fa_fwd_rope(q, k, v, rc, rs, True, 1 / math.sqrt(w.d), o=o, lse=lse,
                                 stream=stream),
          fwd_flops(w), f"rope_{w.name}")
    del q, k, v, o, lse, rc, rs
    # backward pass on the long-prefill workload: five products per tile
    # against the forward pass's two, so 2.5x its FLOPs
    q, k, v = W.fwd_inputs(w, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, True, 1 / math.sqrt(w.d))
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    timed(lambda: fa.fa_bwd(q, k, v, o, lse, g, True, 1 / math.sqrt(w.d), dq=dq, dk=dk, dv=dv,
                            stream=stream),
          2.5 * fwd_flops(w), f"bwd_{w.name}")
    del q, k, v, o, lse, g, dq, dk, dv
    # backward pass with 8 K/V heads (each CTA walks the tiles of 4 query heads)
    q, k, v = W.gqa_fwd_inputs(w.B, w.H, GQA_HKV, w.N, w.d, seed=21, device="cuda")
    o, lse = fa.fa_fwd_gqa(q, k, v, True, 1 / math.sqrt(w.d))
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    timed(lambda: fa.fa_bwd_gqa(q, k, v, o, lse, g, True, 1 / math.sqrt(w.d), dq=dq, dk=dk,
                                dv=dv, stream=stream),
          2.5 * fwd_flops(w), f"bwd_gqa_long_prefill_b1_h32_hkv{GQA_HKV}_n16384_d128_causal")
    del q, k, v, o, lse, g, dq, dk, dv
    # backward pass over the variable-length workload's packed sequences
    wv = W.BATCHED_VARLEN
    q, k, v, cu = W.varlen_workload_inputs(wv, device="cuda")
    lens = (cu[1:] - cu[:-1]).tolist()
    cud = cu.cuda()
    o, lse = fa.fa_fwd_varlen(q, k, v, cud, max(lens), wv.causal, 1 / math.sqrt(wv.d))
    g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(8),
                    device="cuda").to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    vflops = sum(4.0 * wv.H * L * L * wv.d / (2 if wv.causal else 1) for L in lens)
    timed(lambda: fa.fa_bwd_varlen(q, k, v, o, lse, g, cud, max(lens), wv.causal,
                                   1 / math.sqrt(wv.d), dq=dq, dk=dk, dv=dv, stream=stream),
          2.5 * vflops, f"bwd_{wv.name}")
    del q, k, v, cu, cud, o, lse, g, dq, dk, dv
    # grouped-query paged decode: the decode workload's lengths with 8, 2 and
    # 1 K/V heads (the last two: the evenly split chunk stream)
    lengths = W.varlen_lengths(DEC.B, DEC.len_lo, DEC.len_hi, DEC.seed)
    for h_kv in (GQA_HKV, 2, 1):
        c = W.paged_inputs(DEC.B, DEC.H, DEC.d, lengths, DEC.seed, DEC.page_size, device="cuda",
                           H_kv=h_kv)
        pt, sl = c.page_table.cuda(), c.seq_lens.cuda()
        do = torch.empty_like(c.q)
        nbytes = decode_bytes(lengths, DEC.H, DEC.d, DEC.B, H_kv=h_kv)
        name = f"gqa_paged_decode_b64_h32_hkv{h_kv}_d128_len1024to32768_page256"
        timed(lambda: fa.fa_decode_paged_gqa(c.q, c.k_pages, c.v_pages, pt, sl, DEC.page_size,
                                             o=do, stream=stream), 0.0, name)
        ms = out[name]["ms_per_launch"]
        out[name] = {"ms_per_launch": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                     "bytes_per_launch": nbytes}
        del c, pt, sl, do
    # paged prefill: 1024 new queries per sequence after 1024..8192 cached
    # tokens, K/V read through the page table; FLOPs count every attended
    # (query, key) pair (4*d per pair and head)
    w = W.PAGED_PREFILL
    cache, q, cu = W.prefill_workload_inputs(w, device="cuda")
    pt, sl, cud = cache.page_table.cuda(), cache.seq_lens.cuda(), cu.cuda()
    o = torch.empty_like(q)
    lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=q.device)
    pairs = sum(w.q_len * (int(L) - w.q_len) + w.q_len * (w.q_len + 1) // 2
                for L in cache.seq_lens.tolist())
    timed(lambda: fa.fa_prefill_paged(q, cache.k_pages, cache.v_pages, pt, sl, cud, w.q_len,
                                      w.causal, 1 / math.sqrt(w.d), o=o, lse=lse, stream=stream),
          4.0 * w.d * w.H * pairs, w.name, {"context_after": cache.seq_lens.tolist()})
    del cache, q, cu, pt, sl, cud, o, lse
    torch.cuda.empty_cache()
    return out


def decode_cache(batch: int, h_kv: int) -> W.PagedCache:
    if batch >= DEC.B and h_kv == DEC.H:
        return W.decode_workload_inputs(DEC, device="cuda")
    lengths = W.varlen_lengths(DEC.B, DEC.len_lo, DEC.len_hi, DEC.seed)[:batch]
    return W.paged_inputs(len(lengths), DEC.H, DEC.d, lengths, DEC.seed, DEC.page_size,
                          device="cuda", H_kv=h_kv)


def run_single_path(args, local):
    """Profiling aid (--only prefill / rope / bwd / batched / varlen /
    bwd_varlen): the paged-prefill workload, the RoPE forward pass or the
    backward pass on the long-prefill workload, the forward pass on the
    batched or the variable-length prefill workload, or the backward pass on
    the latter, alone, timed with CUDA events; prints its own short JSON
    line."""
    import attn_fwd_04_b200 as fa
    torch.cuda.set_device(local)
    stream = torch.cuda.current_stream()
    if args.only == "bwd":
        w = FWD
        q, k, v = W.fwd_inputs(w, device="cuda")
        o, lse = fa.fa_fwd(q, k, v, True, 1 / math.sqrt(w.d), stream=stream)
        g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                        device="cuda").to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        flops = 2.5 * fwd_flops(w)
        name = f"bwd_{w.name}"

        def fn():
            fa.fa_bwd(q, k, v, o, lse, g, True, 1 / math.sqrt(w.d), dq=dq, dk=dk, dv=dv,
                      stream=stream)
    elif args.only == "batched":
        w = W.BATCHED
        q, k, v = W.fwd_inputs(w, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        flops = fwd_flops(w)
        name = w.name

        def fn():
            fa.fa_fwd(q, k, v, w.causal, 1 / math.sqrt(w.d), o=o, lse=lse, stream=stream)
    elif args.only == "varlen":
        w = W.BATCHED_VARLEN
        q, k, v, cu = W.varlen_workload_inputs(w, device="cuda")
        lens = (cu[1:] - cu[:-1]).tolist()
        cud = cu.cuda()
        o = torch.empty_like(q)
        lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=q.device)
        flops = sum(4.0 * w.H * L * L * w.d / (2 if w.causal else 1) for L in lens)
        name = w.name

        def fn():
            fa.fa_fwd_varlen(q, k, v, cud, max(lens), w.causal, 1 / math.sqrt(w.d), o=o, lse=lse,
                             stream=stream)
    elif args.only == "bwd_varlen":
        w = W.BATCHED_VARLEN
        q, k, v, cu = W.varlen_workload_inputs(w, device="cuda")
        lens = (cu[1:] - cu[:-1]).tolist()
        cud = cu.cuda()
        o, lse = fa.fa_fwd_varlen(q, k, v, cud, max(lens), w.causal, 1 / math.sqrt(w.d),
                                  stream=stream)
        g = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(8),
                        device="cuda").to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        flops = 2.5 * sum(4.0 * w.H * L * L * w.d / (2 if w.causal else 1) for L in lens)
        name = f"bwd_{w.name}"

        def fn():
            fa.fa_bwd_varlen(q, k, v, o, lse, g, cud, max(lens), w.causal, 1 / math.sqrt(w.d),
                             dq=dq, dk=dk, dv=dv, stream=stream)
    elif args.only == "prefill":
        w = W.PAGED_PREFILL
        cache, q, cu = W.prefill_workload_inputs(w, device="cuda")
        pt, sl, cud = cache.page_table.cuda(), cache.seq_lens.cuda(), cu.cuda()
        o = torch.empty_like(q)
        lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=q.device)
        pairs = sum(w.q_len * (int(L) - w.q_len) + w.q_len * (w.q_len + 1) // 2
                    for L in cache.seq_lens.tolist())
        flops = 4.0 * w.d * w.H * pairs
        name = w.name

        def fn():
            fa.fa_prefill_paged(q, cache.k_pages, cache.v_pages, pt, sl, cud, w.q_len, w.causal,
                                1 / math.sqrt(w.d), o=o, lse=lse, stream=stream)
    else:
        w = FWD
        q, k, v = W.fwd_inputs(w, device="cuda")
        rc, rs = W.rope_tables(w.N, w.d, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        flops = fwd_flops(w)
        name = f"rope_{w.name}"

        def fn():
            fa.fa_fwd_rope(q, k, v, rc, rs, True, 1 / math.sqrt(w.d), o=o, lse=lse, stream=stream)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("device error")
    ms = e0.elapsed_time(e1) / args.steps
    return {"workload": name, "ms_per_launch": ms, "tflops": flops / (ms * 1e-3) / 1e12,
            "steps": args.steps, "warmup": args.warmup}


def run_native(args, world, rank, local):
    import attn_fwd_04_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()
    do_fwd = args.only in ("all", "fwd")
    do_dec = args.only in ("all", "decode")

    scale = 1 / math.sqrt(FWD.d)
    if do_fwd:
        q, k, v = W.fwd_inputs(FWD, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty((FWD.B, FWD.H, FWD.N), dtype=torch.float32, device=dev)
    if do_dec:
        cache = decode_cache(args.decode_batch, args.decode_hkv)
        h_kv = int(cache.k_pages.shape[1])
        dpt, dsl = cache.page_table.to(dev), cache.seq_lens.to(dev)
        do = torch.empty_like(cache.q)
    torch.cuda.synchronize()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if do_fwd:
            fa.fa_fwd(q, k, v, FWD.causal, scale, o=o, lse=lse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if do_dec and h_kv == DEC.H:
            fa.fa_decode_paged(cache.q, cache.k_pages, cache.v_pages, dpt, dsl, DEC.page_size,
                               o=do, stream=stream)
        elif do_dec:
            fa.fa_decode_paged_gqa(cache.q, cache.k_pages, cache.v_pages, dpt, dsl,
                                   DEC.page_size, o=do, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("device error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first reading
    sampler.mark_start()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier(world)
    clocks = sampler.stop()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("device error during the timed steps")

    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = t_start.elapsed_time(t_end)
    fwd_sum, dec_sum, total_ms = reduce_max([sum(fwd_ms), sum(dec_ms), total_ms], world)

    flops = fwd_flops()
    fwd_tflops = job_rate(world, flops, args.steps, fwd_sum) / 1e12 if do_fwd else None
    per_launch_tf = flops / (fwd_sum / args.steps * 1e-3) / 1e12 if do_fwd else None
    if do_dec:
        dbytes = decode_bytes(cache.seq_lens.tolist(), DEC.H, DEC.d, cache.q.shape[0],
                              H_kv=h_kv)
        dec_gbs = job_rate(world, dbytes, args.steps, dec_sum) / 1e9
        per_launch_gbs = dbytes / (dec_sum / args.steps * 1e-3) / 1e9

    # ---- end to end through the public API, host buffers ------------------
    # Every step copies its q, k, v from pinned host memory, runs fa_fwd and
    # copies o and lse back.  Two sets of device buffers and three streams let
    # step i+1's host-to-device copies run while step i computes and its
    # results travel back (PCIe is full duplex); events order each buffer's
    # reuse.
    e2e = None
    if do_fwd and not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 8))
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        dbuf = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(o),
                 torch.empty_like(lse)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def e2e_step(i):
            b = i & 1
            dq2, dk2, dv2, do2, dl2 = dbuf[b]
            if used[b]:
                s_in.wait_event(comp_done[b])      # step i-2 has read this buffer's inputs
                stream.wait_event(out_done[b])     # and its outputs have gone back
            with torch.cuda.stream(s_in):
                dq2.copy_(hq, non_blocking=True)
                dk2.copy_(hk, non_blocking=True)
                dv2.copy_(hv, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            fa.fa_fwd(dq2, dk2, dv2, FWD.causal, scale, o=do2, lse=dl2, stream=stream)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                ho[b].copy_(do2, non_blocking=True)
                hl[b].copy_(dl2, non_blocking=True)
                out_done[b].record(s_out)
            used[b] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record(s_in)
        s_in.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        s_out.wait_event(out_done[0])
        s_out.wait_event(out_done[1])
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier(world)
        (e2e_ms,) = reduce_max([e0.elapsed_time(e1)], world)
        # the results that came back are the device pass's, bit for bit
        last = (e2e_steps - 1) & 1
        if not (torch.equal(ho[last], o.cpu()) and torch.equal(hl[last], lse.cpu())):
            raise RuntimeError("end-to-end outputs differ from the device-resident pass")
        e2e = {"value": job_rate(world, flops, e2e_steps, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv)),
               "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size() +
                                     hl[0].numel() * hl[0].element_size(),
               "steps": e2e_steps,
               "what": "fa_fwd through the Python binding; every step copies q/k/v from pinned "
                       "host memory and o/lse back inside the timed region, two steps in "
                       "flight (copies in, compute and copies out on three streams)"}

    secondary = None
    if do_fwd and not args.no_secondary:
        secondary = secondary_workloads(fa, stream)

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and do_fwd:
        import oracle
        tf, rows, secs = oracle_fwd_sample(q, k, v, args.cpu_seconds, seed=2)
        cpu_baseline = {"value": tf, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                        "kind": "oracle",
                        "sample": f"{rows} seeded random query rows of two seeded heads of the "
                                  f"long-prefill workload, {secs:.1f} s, FLOPs counted like "
                                  f"the GPU number (2*N*d per causal row)"}
        if do_dec:
            gbs, seqs, dsecs = oracle_decode_sample(cache, args.cpu_seconds / 2)
            cpu_baseline["decode"] = {"value": gbs, "unit": "GB/s",
                                      "sample": f"{seqs} whole sequences (shortest first) of "
                                                f"the paged-decode workload, {dsecs:.1f} s"}
        if not args.no_secondary:
            cpu_baseline["other_workloads"] = oracle_other_workloads(args.cpu_seconds / 3)
        cpu_baseline["cpu_model"] = cpu_model()

    if rank != 0:
        return None
    fwd_sha = kernel_source_sha(["fwd_sm100.cu", "fa_ptx.cuh", "fa_internal.h"])
    dec_sha = kernel_source_sha(["decode_sm100.cu", "fa_ptx.cuh", "fa_internal.h"])
    # the forward's tensor peak is the measured GEMM figure of the regime the
    # timed region ran in (burst at full clock, or sustained at the power cap)
    regime, peak_tf, regime_why = tensor_peak_regime(peaks, clocks, total_ms)
    out = {
        "metric": METRIC,
        "value": fwd_tflops if do_fwd else dec_gbs,
        "unit": "TFLOP/s" if do_fwd else "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded torch.randn, N(0,1) bf16; lengths uniform; shuffled page pool)",
        "config": {
            "workload": " + ".join(([FWD.name] if do_fwd else []) + ([DEC.name] if do_dec else [])),
            "l2": "inputs larger than L2 (fwd 384 MiB, decode ~17.7 GB); no flush",
            "parallelism": f"replicas x{world}",
        },
        "gpu_launches": args.steps * ((1 if do_fwd else 0) + (3 if do_dec else 0)),
        "clocks": clocks,
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "other_workloads": secondary,
    }
    if do_fwd:
        out["config"]["fwd"] = {"B": FWD.B, "H": FWD.H, "N": FWD.N, "d": FWD.d,
                                "causal": FWD.causal, "scale": scale, "seed": FWD.seed}
        out["pct_of_bf16_peak"] = {
            "datasheet_2250": 100 * per_launch_tf / DATASHEET_BF16_TFLOPS,
            "measured_burst": 100 * per_launch_tf / peaks["bf16_tflops"],
            "measured_sustained": 100 * per_launch_tf / peaks["bf16_tflops_sustained"]}
        out["fwd_ms_per_launch"] = fwd_sum / args.steps
        sm_ghz = (clocks.get("sm_mhz") or 0) / 1e3
        out["roofline"] = {"bound": "tensor", "kernel": "fa_fwd_kernel", "achieved": per_launch_tf,
                           "peak": peak_tf, "unit": "TFLOP/s", "frac": per_launch_tf / peak_tf,
                           "regime": regime,
                           "peak_source": f"{peaks['source']} bf16 {regime} GEMM peak ({regime_why})",
                           "timed_region_s": total_ms / 1e3,
                           "tflops_per_sm_ghz": per_launch_tf / sm_ghz if sm_ghz else None,
                           "traffic": recorded_traffic("fa_fwd_kernel", fwd_sha),
                           "algorithmic_flops_per_launch": flops}
    if do_dec:
        out["config"]["decode"] = {"B": int(cache.q.shape[0]), "H": DEC.H, "H_kv": h_kv,
                                   "d": DEC.d,
                                   "page_size": DEC.page_size,
                                   "len_range": [DEC.len_lo, DEC.len_hi], "seed": DEC.seed,
                                   "tokens": int(cache.seq_lens.sum())}
        out["decode"] = {"value": dec_gbs, "unit": "GB/s", "ms_per_launch": dec_sum / args.steps,
                         "bytes_per_launch": dbytes,
                         "pct_of_hbm": {"datasheet_8000": 100 * per_launch_gbs / 8000.0,
                                        "measured": 100 * per_launch_gbs / peaks["hbm_gbs"]}}
        dec_kernel = "fa_decode_split_kernel" if h_kv == DEC.H else "fa_decode_gqa_kernel"
        out["roofline_decode"] = {
            "bound": "hbm", "kernel": f"{dec_kernel} (+plan, merge)",
            "achieved": per_launch_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": per_launch_gbs / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} copy",
            "traffic": recorded_traffic(dec_kernel, dec_sha),
            "algorithmic_bytes_per_launch": dbytes}
    # each kernel's share of the step's device time (CUDA events); the one with
    # the larger share is the step's dominant kernel
    if do_fwd and do_dec and fwd_sum + dec_sum > 0:
        shares = {"roofline": fwd_sum / (fwd_sum + dec_sum),
                  "roofline_decode": dec_sum / (fwd_sum + dec_sum)}
        top = max(shares, key=shares.get)
        for key, share in shares.items():
            out[key]["share_of_step"] = share
            out[key]["dominant"] = key == top
    return out


# ---------------------------------------------------------------------------
# reference arm: the oracle, timed as it stands
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    # inputs on the host (the oracle is CPU code); same seeded recipe, drawn on
    # the CPU generator so no GPU is needed for this arm
    q, k, v = W.fwd_inputs(FWD, device="cpu")
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        oracle_fwd_sample(q, k, v, per_step, seed=100 + i)
    tfs, rows_total, secs_total = [], 0, 0.0
    for i in range(args.steps):
        tf, rows, secs = oracle_fwd_sample(q, k, v, per_step, seed=200 + i)
        tfs.append(tf)
        rows_total += rows
        secs_total += secs
    per_row = (4.0 * FWD.N * FWD.d) / (2 if FWD.causal else 1)
    value = rows_total * per_row / secs_total / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * secs_total / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded recipe as the native arm, drawn on the CPU)",
        "config": {"workload": FWD.name, "fwd": {"B": FWD.B, "H": FWD.H, "N": FWD.N, "d": FWD.d,
                                                 "causal": FWD.causal, "seed": FWD.seed},
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows_total} seeded random query rows over {args.steps} "
                                   f"steps of ~{per_step:.1f} s each"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the forward pass on the other workloads")
    ap.add_argument("--only", choices=["all", "fwd", "decode", "prefill", "rope", "bwd", "batched",
                                       "varlen", "bwd_varlen"],
                    default="all",
                    help="profiling aid: run one entry point only (the JSON line then "
                         "reports that part alone)")
    ap.add_argument("--decode-hkv", type=int, default=DEC.H,
                    help="K/V heads of the decode cache (fewer than 32 runs the grouped-query "
                         "decode)")
    ap.add_argument("--decode-batch", type=int, default=DEC.B,
                    help="profiling aid: decode over the first B sequences only")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "native":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # CPU only: rank 0 runs the oracle, any other rank exits at once
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, world, int(os.environ.get("RANK", "0")))
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.only in ("prefill", "rope", "bwd", "batched", "varlen", "bwd_varlen"):
        print(json.dumps(run_single_path(args, int(os.environ.get("LOCAL_RANK", "0")))),
              flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        out = run_native(args, world, rank, local)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
