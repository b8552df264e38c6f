"""Benchmark: absorbed-MLA split-KV decode step on B200.

A step is one pass of the decode hot path (steps A2-A9) over one batch, inputs
resident in HBM, through the call a user makes for that shape:

* FP8 cache and at most one (64-row group, request) pair per SM: the single
  launch mla_decode_fused.  It cuts every request into S equal page ranges, S
  as large as one wave of CTAs allows (148 at batch 1, 9 at batch 16 on 148
  SMs), and merges the partials after a grid barrier in the same kernel.
* otherwise mla_decode_partial followed by mla_combine, with the workload's
  own split count.

The two-kernel step with the workload's split count (64 at batch 1, 32 at
batch 16) is timed as well for every workload and reported under
"two_kernel".  The FP8 cache itself is produced once per run by
mla_quantize_fp8 (step A1), which is timed on its own under "quantize".

Default workload: batch 1, q_len 1, 64 heads, 128K context, FP8 E4M3 paged
KV (page 64, shuffled block table).  The other four workloads are measured in
the same run, each under its own key: "tiny" (batch 1, 16 heads, 1024 tokens,
bf16), "batch16" (batch 16 at 128K, FP8), "ragged_b32_bf16" (batch 32, 128
heads, ragged lengths, bf16) and "verify_q4_256k" (batch 8, q_len 4 causal,
256K, FP8; tensor-bound, so its roofline is against the bf16 tensor peak).
L2 is flushed (a 256 MiB write) before every timed step, outside the timed
events, so the 75.5 MB batch-1 cache is read from HBM.

value = KV bytes read per step (sum_b L_b * 576) over all ranks / step time,
in GB/s; ms_per_step is the device time of one step (max over ranks).
With --gpus N > 1 every rank runs its own replica of the workload (the
batch's requests are independent; no collective on the data path) and the
timing is the max over ranks.

--impl reference times the CPU oracle (the only reference implementation
available) on a bounded sample of the same workload.
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
sys.path.insert(0, ROOT)

METRIC = "MLA decode µs/step and KV-read HBM GB/s (% of peak) at 128K ctx, batch 1/16"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def load_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, "measured" | "fallback")."""
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"mla_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


KERNEL_SOURCES = {
    "decode_fp8_kernel": ["decode_fp8.cu", "ptx.cuh", "kernels.cuh"],
    "decode_bf16_kernel": ["decode_bf16.cu", "ptx.cuh", "kernels.cuh"],
}


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from profiles/traffic.txt, if it was measured on
    the kernel sources as they are now (SHA-256 match), else None."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(here, "mla_split_kv_absorbed_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    try:
        with open(os.path.join(here, "profiles", "traffic.txt")) as fh:
            for line in fh:
                parts = line.split()
                if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel \
                        and parts[1] == workload and parts[2] == h.hexdigest():
                    return int(parts[3])
    except OSError:
        pass
    return None


def setup_workload(name, device):
    import torch
    import mla_split_kv_absorbed_b200 as m
    from mla_split_kv_absorbed_b200 import workloads as wl
    w = wl.make(name, device=device)
    if w.spec.kv_dtype == "fp8":
        kv = torch.empty(w.kv_pool.shape, dtype=torch.uint8, device=device)
        m.mla_quantize_fp8(w.kv_pool, kv, w.inv_scale)
    else:
        kv = w.kv_pool
    torch.cuda.synchronize()
    return w, kv


def time_quantize(w, kv, reps=5):
    """Step A1 over the whole pool: GB/s of (2 + 1) bytes per element."""
    import torch
    import mla_split_kv_absorbed_b200 as m
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    n = w.kv_pool.numel()
    times = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        m.mla_quantize_fp8(w.kv_pool, kv, w.inv_scale)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    t = min(times[1:]) if len(times) > 1 else times[0]
    return {"elements": n, "us": t * 1e6, "gbs": 3.0 * n / t / 1e9}


def run_steps(w, kv, steps, warmup, flush_bytes=256 << 20):
    """Time `steps` decode steps (partial + combine) with an L2 flush before each.

    Returns per-step total device times and per-step partial-kernel times (s).
    The totals come from steps bracketed by two events only, so nothing sits
    between the two kernels on the stream (the merge kernel is a programmatic
    dependent launch of the partial kernel); the partial-kernel times come from
    a second set of steps with an event between the two kernels."""
    import torch
    import mla_split_kv_absorbed_b200 as m
    stream = torch.cuda.current_stream()
    part_o, part_lse = m.alloc_partials(w.B, w.q_len, w.H, w.max_splits)
    out = torch.empty((w.B, w.q_len, w.H, 512), dtype=torch.bfloat16, device="cuda")
    out_lse = torch.empty((w.B, w.q_len, w.H), dtype=torch.float32, device="cuda")
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(e_start=None, e_mid=None, e_end=None):
        if e_start is not None:
            e_start.record(stream)
        m.mla_decode_partial(w.q_nope, w.q_rope, kv, w.kv_scale, w.block_table, w.seq_lens,
                             w.num_splits, w.max_splits, w.softmax_scale, part_o, part_lse, err,
                             stream)
        if e_mid is not None:
            e_mid.record(stream)
        m.mla_combine(part_o, part_lse, w.num_splits, w.max_splits, out, out_lse, stream)
        if e_end is not None:
            e_end.record(stream)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    tot_ev = [(ev(), ev()) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step(tot_ev[i][0], None, tot_ev[i][1])
    par_ev = [(ev(), ev()) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step(par_ev[i][0], par_ev[i][1], None)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    total = [a.elapsed_time(b) * 1e-3 for a, b in tot_ev]
    partial = [a.elapsed_time(b) * 1e-3 for a, b in par_ev]
    return total, partial


def run_single_launch(w, kv, steps, warmup, flush_bytes=256 << 20):
    """Per-step device times of the single-launch decode (mla_decode_fused),
    L2 flushed before each step, and its split count; None when the shape has
    no single launch (bf16 cache, or more row groups x requests than SMs)."""
    import torch
    import mla_split_kv_absorbed_b200 as m
    if w.spec.kv_dtype != "fp8":
        return None
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    S = m.mla_fused_splits(w.B, w.q_len, w.H, sms)
    if S < 1:
        return None
    stream = torch.cuda.current_stream()
    ws_buf = m.alloc_fused_workspace(w.B, w.q_len, w.H)
    out = torch.empty((w.B, w.q_len, w.H, 512), dtype=torch.bfloat16, device="cuda")
    out_lse = torch.empty((w.B, w.q_len, w.H), dtype=torch.float32, device="cuda")
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        m.mla_decode_fused(w.q_nope, w.q_rope, kv, w.kv_scale, w.block_table, w.seq_lens,
                           w.softmax_scale, ws_buf, out, out_lse, err, stream)
    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    return [a.elapsed_time(b) * 1e-3 for a, b in evs], S


def run_e2e(w, kv, steps, warmup, fused):
    """Same step through the public API with host buffers: per step, one
    pinned-host -> device copy of the step's inputs (queries, seq_lens, block
    table, and num_splits for the two-kernel step, packed by HostStaging), the
    decode call, and one device -> host copy of O and LSE; for the single
    launch the three are one CUDA graph (DecodeGraph), replayed every step.
    The KV cache stays resident in HBM, as in serving."""
    import torch
    import mla_split_kv_absorbed_b200 as m
    stream = torch.cuda.current_stream()
    st = m.HostStaging(w.B, w.q_len, w.H, w.block_table.shape[1], with_num_splits=not fused)
    for name in st.host:
        st.host[name].copy_(getattr(w, name).cpu())
    if fused:
        graph = m.DecodeGraph(st, kv, w.kv_scale, w.softmax_scale)
    else:
        part = m.alloc_partials(w.B, w.q_len, w.H, w.max_splits)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    d = st.dev

    def step():
        if fused:
            graph.replay(stream)
            return
        st.upload(stream)
        m.decode(d["q_nope"], d["q_rope"], kv, w.kv_scale, d["block_table"], d["seq_lens"],
                 d["num_splits"], w.max_splits, w.softmax_scale, out=st.out,
                 out_lse=st.out_lse, workspace=part)
        st.download(stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    return statistics.median(times), st.in_bytes, st.out_bytes


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_rows_rate(w, codes, budget_s, threads):
    """Oracle decode of whole query rows on `threads` cores for about budget_s:
    (rows done, seconds, projected seconds for a full step)."""
    import numpy as np
    import oracle
    from mla_split_kv_absorbed_b200 import workloads as wl
    qn, qr = wl.bf16_bits(w.q_nope), wl.bf16_bits(w.q_rope)
    bt, sl = w.block_table.cpu().numpy(), w.seq_lens.cpu().numpy()
    R = w.B * w.q_len * w.H
    oracle.set_num_threads(threads)
    rows_done, t_used, batch = 0, 0.0, threads
    while t_used < budget_s and rows_done < R:
        rows = np.arange(rows_done, min(R, rows_done + batch), dtype=np.int64)
        t0 = time.perf_counter()
        oracle.decode_rows(qn, qr, codes, w.kv_scale, bt, sl, w.q_len, w.H, w.softmax_scale, rows)
        t_used += time.perf_counter() - t0
        rows_done += rows.size
    return rows_done, t_used, t_used * R / rows_done


def cpu_baseline(w, kv_codes_host, budget_s=12.0):
    """The oracle, as it stands, on a bounded sample: whole query rows of the
    workload (all tokens of the row), as many as fit in about budget_s on all
    host cores; the projected full-step time gives the same GB/s metric.  Also
    on one core for the tiny and batch-1 workloads, and the quantiser."""
    import numpy as np
    import oracle
    from mla_split_kv_absorbed_b200 import workloads as wl
    all_threads = os.cpu_count() or 1
    oracle.set_num_threads(all_threads)
    threads = oracle.num_threads()
    R = w.B * w.q_len * w.H
    rows_done, t_used, t_step = _oracle_rows_rate(w, kv_codes_host, budget_s, threads)
    one_core = {}
    tiny = wl.make("tiny")
    r1, t1, ts1 = _oracle_rows_rate(tiny, host_codes(tiny, None), 2.0, 1)
    one_core["tiny"] = {"value": tiny.kv_bytes / ts1 / 1e9, "unit": "GB/s", "us_per_step": ts1 * 1e6,
                        "sample": f"{r1} of {tiny.B * tiny.H} rows, {t1:.2f} s"}
    r2, t2, ts2 = _oracle_rows_rate(w, kv_codes_host, 4.0, 1)
    one_core[w.spec.name] = {"value": w.kv_bytes / ts2 / 1e9, "unit": "GB/s", "s_per_step": ts2,
                             "sample": f"{r2} of {R} rows, {t2:.2f} s"}
    oracle.set_num_threads(all_threads)
    # quantiser: step A1 over the first 16M values of the pool, GB/s of 3 B/element
    x = wl.bf16_bits(w.kv_pool).reshape(-1)[: 1 << 24]
    t0 = time.perf_counter()
    oracle.quantize(x, w.inv_scale)
    tq = time.perf_counter() - t0
    return {"value": w.kv_bytes / t_step / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{rows_done} of {R} query rows (all {int(w.seq_lens.max())} tokens each), "
                      f"{t_used:.1f} s, projected to a full step ({t_step:.1f} s)",
            "one_core": one_core,
            "quantize": {"value": 3.0 * x.size / tq / 1e9, "unit": "GB/s", "cores": threads,
                         "elements": int(x.size), "s": tq}}


def host_codes(w, kv):
    """FP8 codes for the oracle, produced by the oracle's own quantiser."""
    import oracle
    from mla_split_kv_absorbed_b200 import workloads as wl
    if w.spec.kv_dtype == "fp8":
        return oracle.quantize(wl.bf16_bits(w.kv_pool), w.inv_scale)
    return wl.bf16_bits(w.kv_pool)


def pct(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(q * len(xs)))]


def flops_per_step(w):
    """Algorithmic flops of one step: 2 (576 + 512) per visible token per query row."""
    sl = w.seq_lens.cpu().tolist()
    tok_rows = sum(w.H * (L - w.q_len + 1 + q) for L in sl for q in range(w.q_len))
    return 2 * (576 + 512) * tok_rows


def roofline_of(w, name, t_kernel, peak_hbm, peak_tflops, kernel):
    """Roofline of the dominant kernel over its launch time: KV bytes against
    the HBM peak, or, for the q_len-4 verify, MMA flops against the tensor peak."""
    if w.q_len > 1:
        fl = flops_per_step(w)
        return {"bound": "tensor", "achieved": fl / t_kernel / 1e12, "peak": peak_tflops,
                "unit": "TFLOP/s", "frac": fl / t_kernel / 1e12 / peak_tflops,
                "algorithmic_flops": fl, "kernel": kernel, "kernel_us": t_kernel * 1e6}
    return {"bound": "hbm", "achieved": w.kv_bytes / t_kernel / 1e9, "peak": peak_hbm,
            "unit": "GB/s", "frac": w.kv_bytes / t_kernel / 1e9 / peak_hbm,
            "traffic": recorded_traffic(kernel, name), "algorithmic_bytes": w.kv_bytes,
            "kernel": kernel, "kernel_us": t_kernel * 1e6}


def two_kernel_summary(w, tot, par, ws, peak_hbm):
    """The two-kernel step (partial + combine) with the workload's split count."""
    t = max_over_ranks(statistics.median(tot), ws)
    tp = max_over_ranks(statistics.median(par), ws)
    return {"api": "mla_decode_partial + mla_combine", "num_splits": w.max_splits,
            "us_per_step": t * 1e6, "us_p10": pct(tot, 0.1) * 1e6, "us_p90": pct(tot, 0.9) * 1e6,
            "kv_gbs": w.kv_bytes / t / 1e9, "frac_of_peak": w.kv_bytes / t / 1e9 / peak_hbm,
            "partial_us": tp * 1e6, "partial_p10": pct(par, 0.1) * 1e6,
            "partial_p90": pct(par, 0.9) * 1e6, "partial_gbs": w.kv_bytes / tp / 1e9}


def measure(name, steps, warmup, peak_hbm, peak_tflops, ws):
    """One workload: the step through its own call (single launch where the
    shape has one), the two-kernel step with the workload's split count, and
    the dominant kernel's roofline."""
    import torch
    w, kv = setup_workload(name, "cuda")
    if w.spec.splits == "by_length":
        # the library's own split rule gives the same counts as the workload
        import mla_split_kv_absorbed_b200 as m
        chosen = m.mla_choose_splits(w.seq_lens.cpu(), 148, 64)
        assert torch.equal(chosen, w.num_splits.cpu()), "mla_choose_splits disagrees with the workload"
    single = run_single_launch(w, kv, steps, warmup)
    tot, par = run_steps(w, kv, steps, warmup)
    two = two_kernel_summary(w, tot, par, ws, peak_hbm)
    kernel = "decode_fp8_kernel" if w.spec.kv_dtype == "fp8" else "decode_bf16_kernel"
    res = {"workload": name, "B": w.B, "q_len": w.q_len, "H": w.H, "kv": w.spec.kv_dtype,
           "kv_bytes_per_step": w.kv_bytes, "steps": steps}
    if single is not None:
        times, S = single
        t = max_over_ranks(statistics.median(times), ws)
        res.update({"api": "mla_decode_fused", "num_splits": S, "us_per_step": t * 1e6,
                    "us_p10": pct(times, 0.1) * 1e6, "us_p90": pct(times, 0.9) * 1e6})
        res["roofline"] = roofline_of(w, name, t, peak_hbm, peak_tflops, kernel)
    else:
        t = two["us_per_step"] * 1e-6
        res.update({"api": two["api"], "num_splits": w.max_splits, "us_per_step": two["us_per_step"],
                    "us_p10": two["us_p10"], "us_p90": two["us_p90"]})
        res["roofline"] = roofline_of(w, name, two["partial_us"] * 1e-6, peak_hbm, peak_tflops,
                                      kernel)
    res["kv_gbs"] = w.kv_bytes / t / 1e9
    res["frac_of_peak"] = w.kv_bytes / t / 1e9 / peak_hbm
    res["two_kernel"] = two
    del kv, w
    torch.cuda.empty_cache()
    return res


def dist_setup(backend="nccl"):
    """One process per GPU (torchrun env); `gloo` is for the CPU tests."""
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(x, ws, device="cuda"):
    """Slowest rank's time: every timed number is the max over ranks."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank, t_step_max, ws):
    """Whole-job KV GB/s: every replica reads its own bytes in the slowest time."""
    return ws * bytes_per_rank / t_step_max / 1e9


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


EXTRA_WORKLOADS = [
    ("tiny", "tiny"),                              # B1 H16 L1024 bf16, 4 splits
    ("batch16", "b16_128k_fp8"),                   # B16 H64 L128K FP8, 32 splits
    ("ragged_b32_bf16", "b32_ragged_bf16"),        # B32 H128 ragged bf16, splits by length
    ("verify_q4_256k", "verify_q4_256k_fp8"),      # B8 q_len 4 H64 L256K FP8, 64 splits
]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="b1_128k_fp8")
    ap.add_argument("--no-extra", action="store_true", help="time only the main workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        return reference_arm(args)

    import torch
    ws, rank, local = dist_setup()
    peak, peak_tf, peak_kind = load_peaks()

    w, kv = setup_workload(args.workload, "cuda")
    quant = time_quantize(w, kv) if w.spec.kv_dtype == "fp8" else None
    import mla_split_kv_absorbed_b200 as m
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    fused = w.spec.kv_dtype == "fp8" and m.mla_fused_splits(w.B, w.q_len, w.H, sms) >= 1

    # the timed region: K steps through the workload's own call
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = time.perf_counter()
        if fused:
            times, S = run_single_launch(w, kv, args.steps, args.warmup)
            t_kernel_list = times
        else:
            times, t_kernel_list = run_steps(w, kv, args.steps, args.warmup)
            S = w.max_splits
        wall = time.perf_counter() - t0
    torch.cuda.synchronize()
    barrier(ws)
    t_step = max_over_ranks(statistics.median(times), ws)
    t_kernel = max_over_ranks(statistics.median(t_kernel_list), ws)
    value = job_gbs(w.kv_bytes, t_step, ws)

    # the two-kernel step with the workload's own split count, for context
    if fused:
        tot, par = run_steps(w, kv, args.steps, args.warmup)
    else:
        tot, par = times, t_kernel_list
    two = two_kernel_summary(w, tot, par, ws, peak)

    e2e_t, h2d, d2h = run_e2e(w, kv, max(5, args.steps // 2), args.warmup, fused)
    e2e_t = max_over_ranks(e2e_t, ws)

    extra = {}
    if not args.no_extra:
        with ClockSampler(local) as clk_x:
            for key, name in EXTRA_WORKLOADS:
                if name != args.workload:
                    extra[key] = measure(name, args.steps, args.warmup, peak, peak_tf, ws)
        extra["clocks_extra"] = clk_x.summary()

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, host_codes(w, kv))

    kernel_name = "decode_fp8_kernel" if w.spec.kv_dtype == "fp8" else "decode_bf16_kernel"
    roof = roofline_of(w, args.workload, t_kernel, peak, peak_tf, kernel_name)
    roof.update({"kernel_p10": pct(t_kernel_list, 0.1) * 1e6,
                 "kernel_p90": pct(t_kernel_list, 0.9) * 1e6, "peak_kind": peak_kind,
                 "launch": "the whole step (single launch)" if fused else
                           "the partial kernel of the two-kernel step"})
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step * 1e3,
        "us_per_step": t_step * 1e6,
        "us_p10": pct(times, 0.1) * 1e6,
        "us_p90": pct(times, 0.9) * 1e6,
        "frac_of_peak": w.kv_bytes / t_step / 1e9 / peak,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if w.spec.kv_dtype == "fp8" else "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "q_len": w.q_len, "H": w.H,
                   "seq_len": int(w.seq_lens.max().item()), "kv": w.spec.kv_dtype, "page": 64,
                   "kv_bytes_per_step": w.kv_bytes,
                   "api": "mla_decode_fused" if fused else "mla_decode_partial + mla_combine",
                   "num_splits": S, "workload_num_splits": w.max_splits,
                   "l2": "flushed before every timed step (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{ws}"},
        "roofline": roof,
        "e2e": {"value": ws * w.kv_bytes / e2e_t / 1e9, "unit": "GB/s", "us_per_step": e2e_t * 1e6,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (1 if fused else 2) * args.steps,
        "clocks": clk.summary(),
        "timed_wall_s": wall,
        "two_kernel": two,
    }
    if quant is not None:
        line["quantize"] = quant
    line.update(extra)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def reference_arm(args):
    """The oracle timed as the reference implementation (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from mla_split_kv_absorbed_b200 import workloads as wl
    w = wl.make(args.workload, device="cpu")
    codes = host_codes(w, None)
    qn, qr = wl.bf16_bits(w.q_nope), wl.bf16_bits(w.q_rope)
    bt, sl = w.block_table.numpy(), w.seq_lens.numpy()
    R = w.B * w.q_len * w.H
    threads = oracle.num_threads()
    rows_per_step = threads
    for _ in range(args.warmup):
        oracle.decode_rows(qn, qr, codes, w.kv_scale, bt, sl, w.q_len, w.H, w.softmax_scale,
                           np.arange(min(rows_per_step, R), dtype=np.int64))
    times = []
    for i in range(args.steps):
        rows = (np.arange(rows_per_step, dtype=np.int64) + i * rows_per_step) % R
        t0 = time.perf_counter()
        oracle.decode_rows(qn, qr, codes, w.kv_scale, bt, sl, w.q_len, w.H, w.softmax_scale, rows)
        times.append((time.perf_counter() - t0) * R / rows_per_step)
    t_step = statistics.median(times)
    value = w.kv_bytes / t_step / 1e9
    sample = f"{rows_per_step} of {R} query rows per step (all tokens), projected to a full step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "q_len": w.q_len, "H": w.H,
                   "seq_len": int(sl.max()), "kv": w.spec.kv_dtype, "page": 64,
                   "kv_bytes_per_step": w.kv_bytes, "api": "oracle (fp64, unsplit)",
                   "workload_num_splits": w.max_splits},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    main()
