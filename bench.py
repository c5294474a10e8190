#!/usr/bin/env python
"""Benchmark of the paged decode step on one node (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config opt13b]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

A step is one decode round of the whole hot path for one batch of running
sequences, through the library's decode-step runtime (``pkv_decode_step``):
host block-table update with copy-on-write, one table upload, block copy,
append of the new K/V rows, paged decode attention and the split-context
merge.  The metric is KV GB/s: sum over the batch of context_len x 2 x H_kv x d
x bytes (the bytes attention must read), per second, in 10^9 B/s.

Inputs: the workload's shapes (``workloads.CONFIGS``), K/V histories drawn on
the GPU from a seeded torch generator and written through ``kv_append``.  The
pool holds ``--replicas`` independent batches of the workload (by default
enough that the distinct KV cycled between two reads of one batch is at least
three times the 126 MB L2); step k runs batch k mod replicas, so contexts grow
by only steps/replicas tokens during the run and every step streams its
batch's KV from HBM.  Multi-GPU: each rank runs its own pool and batches (weak
scaling, no collective on the data path); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
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

import workloads as wl  # noqa: E402

METRIC = "paged decode KV GB/s (% of B200 HBM peak); attended tokens/sec at 1 GPU"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=12)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="opt13b", choices=sorted(wl.CONFIGS))
    ap.add_argument("--block-size", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per batch (0: the workload's own); for small profiling runs")
    ap.add_argument("--variant", default="b", choices=["a", "b"])
    ap.add_argument("--replicas", type=int, default=0,
                    help="replica batches in the pool (0: enough that the cycled distinct KV "
                         "is at least 3x the L2)")
    ap.add_argument("--e2e-steps", type=int, default=0, help="default: steps // 3")
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--kernel", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-records", action="store_true",
                    help="skip the Llama-2-70B GQA and FP8 (MHA bs 16 and 4, GQA) records "
                         "measured after the OPT-13B headline")
    ap.add_argument("--mode", choices=["decode", "prefill", "swap"], default="decode",
                    help="prefill: the prompt phase of the workload's batch (every history "
                         "attended causally as one prompt); swap: one sequence's blocks out to "
                         "pinned host memory and back, per block size")
    return ap.parse_args()


def config_of(args) -> wl.Config:
    cfg = wl.CONFIGS[args.config]
    if args.block_size:
        cfg = cfg.with_block_size(args.block_size)
    if args.batch:
        cfg = dataclasses.replace(cfg, batch=args.batch)
    return cfg


# DRAM traffic of the decode kernel per launch, as a multiple of its
# algorithmic KV bytes, from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) of the same workload with one replica batch.  Valid
# only while the kernel's sources hash to the recorded value, else the bench
# reports null.
TRAFFIC = {
    # (config, block size, kernel): (dram bytes / algorithmic bytes, sha256 of its sources)
    # 605.3 MB algorithmic, 612.7 MB read + written
    ("opt13b", 16, "decode_simt2_kernel"):
        (1.0123, "3d500856b22f29f4b5587277bc162b747071c43be02490f014a82dffad3bbe4e"),
    # 287.0 MB, 293.0 MB
    ("llama2_70b", 16, "decode_tc_kernel"):
        (1.0206, "41088eff1f3e70d27c0838ec828e7bc4b6fb816a0c73fc2f08446899f6ee67fb"),
    # 1,346.1 MB, 1,359.6 MB
    ("fp8", 16, "decode_tc_kernel"):
        (1.0100, "41088eff1f3e70d27c0838ec828e7bc4b6fb816a0c73fc2f08446899f6ee67fb"),
    # 1,346.1 MB, 1,351.7 MB
    ("fp8", 4, "decode_tc_kernel"):
        (1.0041, "41088eff1f3e70d27c0838ec828e7bc4b6fb816a0c73fc2f08446899f6ee67fb"),
    # 143.5 MB, 148.8 MB
    ("fp8_gqa", 16, "decode_tc_kernel"):
        (1.0370, "41088eff1f3e70d27c0838ec828e7bc4b6fb816a0c73fc2f08446899f6ee67fb"),
    # 8.3 MB, 3.0 MB (the samples of one prompt share its blocks; the re-reads
    # within a launch hit L2)
    ("falcon7b", 16, "decode_lean_kernel"):
        (0.3593, "ce148d142c0abfb12978045714de63ba937c3f19448974ab10a4b1c96d8c6e00"),
}
KERNEL_SOURCES = {
    "decode_lean_kernel": ("decode_lean.cu", "tc_common.cuh", "kernels_common.cuh"),
    "decode_tc_kernel": ("decode_tc.cu", "tc_common.cuh", "kernels_common.cuh"),
    "decode_simt2_kernel": ("decode_simt2.cu", "kernels_common.cuh"),
    "decode_simt_kernel": ("decode_simt.cu", "kernels_common.cuh"),
}


def kernel_sources_sha(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(ROOT, "pagedattention_decode_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_per_launch(cfg: wl.Config, kernel: str, algorithmic_bytes: float):
    entry = TRAFFIC.get((cfg.name, cfg.block_size, kernel))
    if entry is None or entry[1] != kernel_sources_sha(kernel):
        return None
    return int(entry[0] * algorithmic_bytes)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, polled)
# ---------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(torch_device)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                sm = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                self.samples.append((sm, self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_sm, "reasons": [], "samples": 0}
        sms = [s for s, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        return {"sm_mhz": float(statistics.median(sms)), "sm_max_mhz": int(self.max_sm),
                "reasons": [n for b, n in REASONS.items() if bits & b and b != 0x1],
                "samples": len(sms)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(cfg: wl.Config, target_bytes: float, seed: int = 0):
    """The first sequences of the workload whose KV bytes reach target_bytes,
    admitted into a fresh oracle (set-up, not timed)."""
    from oracle.engine import DecodeOracle
    lens = wl.history_lengths(cfg, seed, "b")
    per = cfg.samples_per_prompt
    seqs, tot = [], 0
    for i in range(cfg.batch):
        n = int(lens[i // per]) if per > 1 else int(lens[i])
        seqs.append(i)
        tot += (n + 1) * cfg.kv_bytes_per_token
        if tot >= target_bytes:
            break
    nb = sum(-(-(int(lens[i // per] if per > 1 else lens[i]) + 64) // cfg.block_size) + 2
             for i in seqs)
    ks = vs = 1.0
    if cfg.kv_dtype == "fp8":
        ks, vs = wl.fp8_scales_for(cfg, seed, [lens[i] for i in seqs], steps=1)
    orc = DecodeOracle(nb, cfg.block_size, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype, ks, vs,
                       order=wl.free_order(nb, seed, cfg.permute))
    for i in seqs:
        src = i // per if per > 1 else i
        n = int(lens[src])
        k, v = wl.history_kv(cfg, seed, src, n)
        orc.admit(i, wl.round_to(k, cfg.q_dtype), wl.round_to(v, cfg.q_dtype), cfg.q_dtype)
    return orc, seqs


def oracle_step(orc, cfg, seqs, step):
    q, k, v = [], [], []
    for s in seqs:
        a, b, c = wl.step_qkv(cfg, 0, s, step)
        q.append(a), k.append(b), v.append(c)
    q = wl.round_to(np.stack(q), cfg.q_dtype)
    k = wl.round_to(np.stack(k), cfg.q_dtype)
    v = wl.round_to(np.stack(v), cfg.q_dtype)
    t0 = time.perf_counter()
    orc.step(seqs, q, k, v, cfg.q_dtype, cfg.scale)
    dt = time.perf_counter() - t0
    nbytes = sum(orc.bm.lengths[s] for s in seqs) * cfg.kv_bytes_per_token
    return dt, nbytes


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(cfg: wl.Config, budget_s: float) -> dict:
    """The oracle as it stands on a bounded sample of the workload: one warm-up
    step, then oracle decode steps (append then attend) until the budget is
    spent; GB/s over the same byte definition."""
    orc, seqs = oracle_sample(cfg, target_bytes=64e6)
    oracle_step(orc, cfg, seqs, 0)
    times, nbytes = [], []
    t_end = time.perf_counter() + budget_s
    step = 1
    while time.perf_counter() < t_end and step < 200:
        dt, nb = oracle_step(orc, cfg, seqs, step)
        times.append(dt)
        nbytes.append(nb)
        step += 1
    gbs = sum(nbytes) / sum(times) / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{len(seqs)} of {cfg.batch} sequences of the workload, {len(times)} "
                      f"decode steps (append + fp64 attention), median step "
                      f"{statistics.median(times) * 1e3:.1f} ms"}


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = config_of(args)
    # per step a bounded sample sized so that the whole run stays within minutes
    orc, seqs = oracle_sample(cfg, target_bytes=24e6)
    for s in range(args.warmup):
        oracle_step(orc, cfg, seqs, s)
    times, nbytes = [], []
    for s in range(args.steps):
        dt, nb = oracle_step(orc, cfg, seqs, args.warmup + s)
        times.append(dt)
        nbytes.append(nb)
    tot = sum(times)
    gbs = sum(nbytes) / tot / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.description, "sample_sequences": len(seqs)},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{len(seqs)} of {cfg.batch} sequences per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
L2_BYTES = 126e6


def distinct_kv_bytes(cfg: wl.Config, seed: int = 0) -> float:
    """KV bytes of one batch's distinct cached tokens (shared prompt blocks once)."""
    return float(wl.history_lengths(cfg, seed, "b").sum()) * cfg.kv_bytes_per_token


def auto_replicas(cfg: wl.Config) -> int:
    """Replica batches such that the KV cycled through between two reads of the
    same batch is at least 3x the L2: every step's KV then comes from HBM."""
    return int(min(512, max(8, -(-3 * L2_BYTES // distinct_kv_bytes(cfg)))))


def build_batches(cfg: wl.Config, pk, torch, replicas: int, growth: int, seed: int):
    """One pool holding `replicas` independent batches of the workload.
    Returns (pool, [seq ids per batch], [context lengths per batch])."""
    B = cfg.batch
    per = cfg.samples_per_prompt
    lens = [wl.history_lengths(cfg, seed + r, "b") for r in range(replicas)]
    if per > 1:
        nb = sum(int(sum(-(-int(n) // cfg.block_size) for n in l)) + B * (growth // cfg.block_size + 3)
                 for l in lens)
    else:
        nb = sum(wl.pool_blocks(cfg, l, growth) for l in lens)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[cfg.q_dtype]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed * 7919 + 17)
    # draw every history first (the FP8 scale is amax / 448 over all of it)
    hist = []
    for r in range(replicas):
        n_rows = int(sum(lens[r]))
        k = torch.randn((n_rows, cfg.n_kv_heads, cfg.head_dim), generator=gen, device="cuda",
                        dtype=torch.float32).to(dt)
        v = torch.randn((n_rows, cfg.n_kv_heads, cfg.head_dim), generator=gen, device="cuda",
                        dtype=torch.float32).to(dt)
        hist.append((k, v))
    ks = vs = 1.0
    if cfg.kv_dtype == "fp8":
        ks = wl.fp8_scale(max(float(k.abs().max()) for k, _ in hist) * 1.05)
        vs = wl.fp8_scale(max(float(v.abs().max()) for _, v in hist) * 1.05)
    pool = pk.kv_pool_create(nb, cfg.block_size, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype, ks, vs)
    pk.bt_reset(pool, wl.free_order(nb, seed, cfg.permute))
    groups, ctx = [], []
    for r in range(replicas):
        k, v = hist[r]
        ids = []
        slots = []
        row = 0
        if per > 1:
            for p_i, n in enumerate(lens[r]):
                sid = r * B + p_i * per
                slots.append(pk.bt_alloc(pool, sid, int(n)))
                rows = np.arange(row, row + int(n))
                row += int(n)
                ids.append(sid)
                for c in range(1, per):
                    pk.bt_fork(pool, sid, sid + c)
                    ids.append(sid + c)
            c_r = np.repeat(lens[r], per).astype(np.int64)
        else:
            for i, n in enumerate(lens[r]):
                sid = r * B + i
                slots.append(pk.bt_alloc(pool, sid, int(n)))
                ids.append(sid)
            c_r = lens[r].astype(np.int64).copy()
        s = torch.from_numpy(np.concatenate(slots)).cuda()
        pk.kv_append(pool, s, k, v)
        groups.append(np.asarray(sorted(ids), dtype=np.int64))
        ctx.append(c_r)
    del hist
    torch.cuda.synchronize()
    assert pk.pkv_device_error(pool) == 0
    return pool, groups, ctx


def profile_stride(R: int) -> int:
    """Every how many timed rounds one is profiled: the smallest stride >= 3
    coprime with the number of replica batches, so that the profiled rounds
    visit every batch in turn instead of a fixed subset."""
    p = 3
    while math.gcd(p, R) != 1:
        p += 1
    return p


def measure_decode(cfg: wl.Config, pk, torch, pd, K: int, W: int, E: int, R: int,
                   partition: int, kernel: int, rank: int, local: int) -> dict:
    """One workload through the decode-step runtime: K timed rounds after R
    priming and W warm-up rounds, then E end-to-end rounds through the
    host-buffer call.  Returns this rank's raw measurements."""
    growth = -(-(R + K + W + E) // R) + 2
    pool, groups, ctx = build_batches(cfg, pk, torch, R, growth, seed=1000 * rank)
    B = cfg.batch
    max_ctx = max(int(c.max()) for c in ctx) + growth
    max_blocks = -(-max_ctx // cfg.block_size) + 2
    step = pk.Step(pool, B, max_blocks, cfg.n_q_heads, cfg.q_dtype, partition, kernel,
                   max_seqs=B * R)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[cfg.q_dtype]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4242 + rank)
    n_sets = 16
    q = torch.randn((n_sets, B, cfg.n_q_heads, cfg.head_dim), generator=gen, device="cuda").to(dt)
    kn = torch.randn((n_sets, B, cfg.n_kv_heads, cfg.head_dim), generator=gen, device="cuda").to(dt)
    vn = torch.randn((n_sets, B, cfg.n_kv_heads, cfg.head_dim), generator=gen, device="cuda").to(dt)
    out = torch.empty((B, cfg.n_q_heads, cfg.head_dim), dtype=dt, device="cuda")
    b_tok = cfg.kv_bytes_per_token
    scale = cfg.scale

    # device pointers resolved once: the timed loop is the C call per round
    stream_ptr = int(torch.cuda.current_stream().cuda_stream)
    qp = [int(q[i].data_ptr()) for i in range(n_sets)]
    kp = [int(kn[i].data_ptr()) for i in range(n_sets)]
    vp = [int(vn[i].data_ptr()) for i in range(n_sets)]
    outp = int(out.data_ptr())
    ctx_sum = [int(c.sum()) for c in ctx]
    n_per = [len(c) for c in ctx]

    def run_step(k):
        r = k % R
        i = k % n_sets
        step.run_raw(groups[r], qp[i], kp[i], vp[i], scale, outp, stream_ptr)
        ctx_sum[r] += n_per[r]
        ctx[r] += 1
        return ctx_sum[r], step.last_launches

    # priming (setup, untimed): one round per replica batch makes its block
    # tables resident on the device; then the W warm-up rounds
    for k in range(R + W):
        run_step(k)
    torch.cuda.synchronize()
    pd.barrier()

    # every prof_every-th timed round records CUDA events around its launches
    # on the launch stream; prof_every is coprime with R, so the profiled
    # rounds walk through all replica batches
    prof_every = profile_stride(R)
    pk.pkv_step_profile(step, K, prof_every)
    clocks = ClockSampler(local)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks.start()
    torch.cuda.synchronize()
    ev0.record()
    tokens = 0
    launches = 0
    step_bytes = []
    for k in range(R + W, R + W + K):
        t, nl = run_step(k)
        tokens += t
        launches += nl
        step_bytes.append(t * b_tok)
    ev1.record()
    torch.cuda.synchronize()
    clocks.stop()
    pd.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    kernel_used = step.last_kernel
    pro_ms, dec_ms, merge_ms = pk.pkv_step_profile_read(step, K)
    pk.pkv_step_profile(step, 0)
    prof_ks = list(range(0, K, prof_every))[: len(dec_ms)]
    prof_bytes = [step_bytes[k] for k in prof_ks]
    prof_batches = sorted({(R + W + k) % R for k in prof_ks})

    # end to end through the C ABI's host-buffer call (pkv_decode_step_host):
    # per round the new q/k/v come from pinned host memory and the output is
    # back in host memory when the call returns (a serving loop needs it
    # before the next round); q | k | v packed in one pinned buffer, so the
    # call moves them in one copy
    hqkv = torch.cat([t[0].flatten() for t in (q, kn, vn)]).cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=dt).pin_memory()
    esz = hqkv.element_size()
    base = int(hqkv.data_ptr())
    hp = [base, base + q[0].numel() * esz, base + (q[0].numel() + kn[0].numel()) * esz,
          int(hout.data_ptr())]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e2e_bytes = 0
    e2e_round_ms = []
    e0.record()
    for k in range(R + W + K, R + W + K + E):
        r = k % R
        ctx[r] += 1
        t0 = time.perf_counter()
        step.run_host_raw(groups[r], hp[0], hp[1], hp[2], scale, hp[3], stream_ptr)
        e2e_round_ms.append((time.perf_counter() - t0) * 1e3)
        e2e_bytes += int(ctx[r].sum()) * b_tok
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    bits = pk.pkv_device_error(pool)
    if bits:
        raise SystemExit(f"device error bits {bits:#x} on {cfg.name}")
    # KV memory actually storing tokens ("KV 缓存与分页注意力" §块表): slots
    # holding tokens over slots the blocks reserve, against reserving the
    # longest possible sequence up front (§先占好最长的位置)
    st = pk.bt_stats(pool)
    max_len = (cfg.lengths[2] if cfg.lengths[0] != "fixed" else cfg.lengths[1]) + growth
    n_seqs = st["num_seqs"]
    utilisation = {
        "paged": round(st["stored_slots"] / max(1, st["used_blocks"] * cfg.block_size), 5),
        "per_sequence": round(st["logical_tokens"] / max(1, st["table_slots"]), 5),
        "max_length_reservation": round(st["logical_tokens"] / max(1, n_seqs * max_len), 5),
        "max_length": int(max_len),
    }
    res = {
        "elapsed_ms": elapsed_ms, "tokens": tokens, "bytes": tokens * b_tok,
        "launches": launches, "step_bytes": step_bytes,
        "e2e_ms": e2e_ms, "e2e_bytes": e2e_bytes, "e2e_rounds": E,
        "e2e_round_ms_median": float(statistics.median(e2e_round_ms)),
        "h2d": hqkv.numel() * esz, "d2h": hout.numel() * hout.element_size(),
        "kernel": pk.KERNEL_NAMES.get(kernel_used, "unknown"),
        "prof_every": prof_every, "prof_bytes": [int(x) for x in prof_bytes],
        "prof_batches": sorted(prof_batches),
        "dec_ms": [float(x) for x in dec_ms], "merge_ms": [float(x) for x in merge_ms],
        "pro_ms": [float(x) for x in pro_ms],
        "utilisation": utilisation, "clocks": clocks.summary(), "R": R,
        "pool_blocks": pool.num_blocks,
    }
    step.close()
    pool.close()
    del q, kn, vn, out
    torch.cuda.empty_cache()
    return res


def roofline_of(cfg: wl.Config, m: dict, peak: float, peak_kind: str) -> dict:
    """The decode kernel against the HBM roofline, from the profiled rounds:
    achieved = profiled_bytes / (profiled_launches x decode_ms_mean)."""
    n = len(m["dec_ms"])
    dec_total = float(np.sum(m["dec_ms"]))
    pbytes = int(np.sum(m["prof_bytes"]))
    achieved = pbytes / (dec_total / 1e3) / 1e9
    return {
        "bound": "hbm",
        "kernel": m["kernel"],
        "achieved": round(achieved, 2),
        "peak": peak,
        "peak_kind": peak_kind,
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": traffic_per_launch(cfg, m["kernel"], float(np.mean(m["step_bytes"]))),
        "algorithmic_bytes_per_launch": int(np.mean(m["step_bytes"])),
        "profiled_bytes": pbytes,
        "profiled_launches": n,
        "profiled_batches": m["prof_batches"],
        "decode_ms_mean": round(dec_total / max(n, 1), 6),
        "merge_ms_mean": round(float(np.mean(m["merge_ms"])), 6),
        "prologue_ms_mean": round(float(np.mean(m["pro_ms"])), 6),
        "profile_note": f"one timed round in {m['prof_every']} (a stride coprime with the "
                        f"{m['R']} replica batches) records CUDA events on the launch stream "
                        "around its kernels, which run without programmatic dependent launch "
                        "in those rounds; achieved = profiled_bytes / profiled_launches / "
                        "decode_ms_mean",
    }


def e2e_of(m: dict) -> dict:
    return {
        "value": round(m["e2e_bytes"] / (m["e2e_ms"] / 1e3) / 1e9, 2),
        "unit": "GB/s",
        "api": "pkv_decode_step_host (pinned host q/k/v in, output back in host memory)",
        "h2d_bytes_per_step": int(m["h2d"]),
        "d2h_bytes_per_step": int(m["d2h"]),
        "steps": m["e2e_rounds"],
        "ms_per_step": round(m["e2e_ms"] / m["e2e_rounds"], 5),
        "host_ms_per_step_median": round(m["e2e_round_ms_median"], 5),
    }


# workloads measured after the headline in the same process (one GPU):
# (record name, config, block size or 0 for the config's own)
SUB_RECORDS = (("llama2_70b_gqa_bf16", "llama2_70b", 0),
               ("fp8_bs16", "fp8", 16),
               ("fp8_bs4", "fp8", 4),
               ("fp8_gqa", "fp8_gqa", 0))


def run_ours(args) -> None:
    import torch

    import pagedattention_decode_02_b200 as pk
    from pagedattention_decode_02_b200 import dist as pd

    rank, world, local = pd.rank_world()
    torch.cuda.set_device(local)
    pd.init("nccl", timeout_s=120, device=torch.device("cuda", local))

    cfg = config_of(args)
    K, W = args.steps, args.warmup
    E = args.e2e_steps or max(K // 3, 40)
    R = args.replicas if args.replicas > 0 else auto_replicas(cfg)
    m = measure_decode(cfg, pk, torch, pd, K, W, E, R, args.partition, args.kernel, rank, local)
    tokens = m["tokens"]

    # time = max over ranks, work = sum over ranks (no data-path collective)
    (elapsed_ms, e2e_ms), (total_bytes, tokens_all, e2e_all, launches_all) = pd.reduce_run(
        [m["elapsed_ms"], m["e2e_ms"]], [m["bytes"], tokens, m["e2e_bytes"], m["launches"]],
        device="cuda")

    subs = {}
    if world == 1 and not args.no_sub_records and args.config == "opt13b" and not args.block_size:
        Ks = max(K, 60)
        for name, cname, bs in SUB_RECORDS:
            c = wl.CONFIGS[cname]
            if bs:
                c = c.with_block_size(bs)
            sm = measure_decode(c, pk, torch, pd, Ks, max(W, 3), max(Ks // 3, 40),
                                auto_replicas(c), 0, 0, rank, local)
            subs[name] = sm

    if rank == 0:
        value = total_bytes / (elapsed_ms / 1e3) / 1e9
        peak, peak_kind = peaks()
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": W,
            "ms_per_step": round(elapsed_ms / K, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": cfg.kv_dtype,
            "data": "synthetic (seeded torch.randn K/V/q; lengths from workloads.py)",
            "config": {
                "workload": cfg.description,
                "batch": cfg.batch, "n_q_heads": cfg.n_q_heads, "n_kv_heads": cfg.n_kv_heads,
                "head_dim": cfg.head_dim, "block_size": cfg.block_size,
                "mean_context": round(tokens / K / cfg.batch, 1),
                "replica_batches_in_pool": m["R"],
                "priming": "one untimed round per replica batch before the warm-up (uploads "
                           "its block tables to the device)",
                "pool_blocks": m["pool_blocks"],
                "l2": f"no flush: {m['R']} replica batches cycled, "
                      f"{m['R'] * distinct_kv_bytes(cfg) / 1e6:.0f} MB of distinct KV between "
                      "two reads of one batch (> 3 x 126 MB L2); attended KV per step "
                      f"{np.mean(m['step_bytes']) / 1e6:.0f} MB",
                "parallelism": f"dp{world}",
            },
            "attended_tokens_per_s": round(tokens_all / (elapsed_ms / 1e3), 1),
            "seq_tokens_heads_per_s": round(tokens_all * cfg.n_q_heads / (elapsed_ms / 1e3), 1),
            "pct_of_nominal_8tbs": round(100 * value / NOMINAL_HBM_GBS / world, 2),
            "roofline": roofline_of(cfg, m, peak, peak_kind),
            "e2e": dict(e2e_of(m), value=round(e2e_all / (e2e_ms / 1e3) / 1e9, 2),
                        ms_per_step=round(e2e_ms / m["e2e_rounds"], 5)),
            "kv_utilisation": m["utilisation"],
            "gpu_launches": int(launches_all),
            "clocks": m["clocks"],
        }
        if subs:
            recs = {}
            for name, sm in subs.items():
                c = wl.CONFIGS[dict((n, cn) for n, cn, _ in SUB_RECORDS)[name]]
                bs = dict((n, b) for n, _, b in SUB_RECORDS)[name]
                if bs:
                    c = c.with_block_size(bs)
                v = sm["bytes"] / (sm["elapsed_ms"] / 1e3) / 1e9
                recs[name] = {
                    "workload": c.description + (f" (block size {bs})" if bs else ""),
                    "value": round(v, 2), "unit": "GB/s",
                    "steps": len(sm["step_bytes"]),
                    "ms_per_step": round(sm["elapsed_ms"] / len(sm["step_bytes"]), 5),
                    "pct_of_nominal_8tbs": round(100 * v / NOMINAL_HBM_GBS, 2),
                    "attended_tokens_per_s": round(sm["tokens"] / (sm["elapsed_ms"] / 1e3), 1),
                    "replica_batches_in_pool": sm["R"],
                    "roofline": roofline_of(c, sm, peak, peak_kind),
                    "e2e": e2e_of(sm),
                    "kv_utilisation": sm["utilisation"],
                    "gpu_launches": int(sm["launches"]),
                    "clocks": sm["clocks"],
                }
            line["sub_records"] = recs
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget)
        print(json.dumps(line), flush=True)
    pd.finish()


def peak_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def run_prefill(args) -> None:
    """Prompt phase ("KV 缓存与分页注意力" §一次写一个词元: a whole prompt at once)
    of one batch of the workload: every sequence's history is its prompt, its
    keys and values already in the pool, attended causally through the block
    table.  FLOPs count the unmasked (query, key) pairs: 4 d per pair per
    query head."""
    import torch

    import pagedattention_decode_02_b200 as pk

    torch.cuda.set_device(0)
    cfg = config_of(args)
    K, W = args.steps, args.warmup
    pool, groups, ctx = build_batches(cfg, pk, torch, 1, 0, seed=0)
    seqs, lens = groups[0], ctx[0]
    max_blocks = max(pk.bt_num_blocks(pool, int(s)) for s in seqs)
    tables, lens_i32, _ = pk.bt_export(pool, seqs, max_blocks)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16}[cfg.q_dtype]
    rows = int(lens.sum())
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    q = torch.randn((rows, cfg.n_q_heads, cfg.head_dim), generator=gen, device="cuda").to(dt)
    out = torch.empty_like(q)
    starts = torch.from_numpy(np.concatenate([[0], np.cumsum(lens_i32)]).astype(np.int32)).cuda()
    t_tab = torch.from_numpy(tables).cuda()
    t_len = torch.from_numpy(lens_i32).cuda()
    max_q = int(lens_i32.max())
    pairs = float(np.sum(lens.astype(np.float64) * (lens + 1) / 2))
    flops = 4.0 * cfg.head_dim * cfg.n_q_heads * pairs
    kv_bytes = float(lens.sum()) * cfg.kv_bytes_per_token

    def call(kernel=pk.PKV_PREFILL_AUTO):
        pk.paged_prefill_attention(pool, q, starts, t_tab, t_len, cfg.scale, max_q_len=max_q,
                                   out=out, kernel=kernel)

    def timed(kernel, sampler=None):
        for _ in range(W):
            call(kernel)
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        if sampler:
            sampler.start()
        ev0.record()
        for _ in range(K):
            call(kernel)
        ev1.record()
        torch.cuda.synchronize()
        if sampler:
            sampler.stop()
        return ev0.elapsed_time(ev1) / K

    # the warp-level mma.sync kernel, timed first as the baseline
    ms_legacy = timed(pk.PKV_PREFILL_MMA_SYNC)
    clocks = ClockSampler(0)
    ms = timed(pk.PKV_PREFILL_AUTO, clocks)
    # end to end: the prompt's queries from pinned host memory, the output back
    hq = q.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=dt).pin_memory()
    E = max(3, K // 3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record()
    for _ in range(E):
        q.copy_(hq, non_blocking=True)
        call()
        hout.copy_(out, non_blocking=True)
        stream.synchronize()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E
    if pk.pkv_device_error(pool):
        raise SystemExit("device error")
    peak, kind = peak_tflops()
    achieved = flops / (ms / 1e3) / 1e12
    line = {
        "metric": "paged prefill attention TFLOP/s (causal, unmasked query-key pairs)",
        "value": round(achieved, 2),
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.q_dtype,
        "data": "synthetic (seeded torch.randn q/K/V; lengths from workloads.py)",
        "config": {"workload": "prompt phase of " + cfg.description, "rows": rows,
                   "mean_prompt": round(float(lens.mean()), 1),
                   "l2": f"no flush: each call reads {kv_bytes / 1e6:.0f} MB of K/V "
                         "and writes the output; the K/V of one (sequence, head) is re-read "
                         "by its row tiles from L2"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": None, "kernel": "prefill_tc05_kernel",
                     "flops_per_launch": flops,
                     "note": "tcgen05.mma (M 128) with tensor-memory accumulators; FLOPs count "
                             "4 d per unmasked (query, key) pair and query head"},
        "baseline_mma_sync": {"kernel": "prefill_tc_kernel", "ms_per_step": round(ms_legacy, 5),
                              "value": round(flops / (ms_legacy / 1e3) / 1e12, 2),
                              "unit": "TFLOP/s",
                              "frac": round(flops / (ms_legacy / 1e3) / 1e12 / peak, 4)},
        "e2e": {"value": round(flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(hq.numel() * hq.element_size()),
                "d2h_bytes_per_step": int(hout.numel() * hout.element_size()),
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": K,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def run_swap(args) -> None:
    """Preemption by swapping ("KV 缓存与分页注意力" §放不下的时候: the blocks go
    to CPU memory and come back when the sequence's turn comes): one sequence
    of the workload's shape (2,048 tokens) swapped out to pinned host buffers
    and back in, for every block size 1 .. 64; bytes moved per second each
    way.  The page reports that swapping is slower for small blocks."""
    import torch

    import pagedattention_decode_02_b200 as pk

    torch.cuda.set_device(0)
    cfg = config_of(args)
    K, W = args.steps, args.warmup
    n_tok = 2048
    res = {}
    stream = torch.cuda.current_stream()
    for bs in (1, 2, 4, 8, 16, 32, 64):
        nb = -(-n_tok // bs) + 4
        pool = pk.kv_pool_create(nb, bs, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype)
        kb, vb = pool.device_buffers()
        kb.copy_(torch.randint(0, 120, kb.shape, dtype=torch.uint8, device="cuda"))
        vb.copy_(torch.randint(0, 120, vb.shape, dtype=torch.uint8, device="cuda"))
        blk = pk.block_bytes(pool)
        n_blocks = -(-n_tok // bs)
        hk = torch.empty(n_blocks * blk, dtype=torch.uint8).pin_memory()
        hv = torch.empty(n_blocks * blk, dtype=torch.uint8).pin_memory()
        pk.bt_alloc(pool, 0, n_tok)
        t_out = t_in = 0.0
        for i in range(W + K):
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
            pk.kv_swap_out(pool, 0, hk, hv, stream=stream)
            e1.record()
            pk.kv_swap_in(pool, 0, hk, hv, n_tok, stream=stream)
            e2.record()
            torch.cuda.synchronize()
            if i >= W:
                t_out += e0.elapsed_time(e1)
                t_in += e1.elapsed_time(e2)
        moved = 2.0 * n_blocks * blk
        res[str(bs)] = {"bytes": int(moved), "out_gbs": round(moved * K / (t_out / 1e3) / 1e9, 2),
                        "in_gbs": round(moved * K / (t_in / 1e3) / 1e9, 2),
                        "out_us": round(t_out / K * 1e3, 2), "in_us": round(t_in / K * 1e3, 2)}
        if pk.pkv_device_error(pool):
            raise SystemExit("device error")
        pool.close()
    best = max(v["in_gbs"] for v in res.values())
    print(json.dumps({
        "metric": "KV swap GB/s per block size (device <-> pinned host, one 2048-token sequence)",
        "value": res["16"]["in_gbs"], "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": W,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.kv_dtype,
        "data": "synthetic (random pool bytes)",
        "config": {"workload": f"one {n_tok}-token sequence of {cfg.description}",
                   "per_block_size": res, "best_in_gbs": best},
        "gpu_launches": 2 * K,
    }), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "prefill":
        run_prefill(args)
    elif args.mode == "swap":
        run_swap(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
