#!/usr/bin/env python
"""Benchmark of the CKDA hot path on B200: prints ONE JSON line (rank 0).

Default workload: the KDA-layer prefill -- B=4, H=16, T=4096, d_k=d_v=128,
chunk 64, bf16 q/k/v, fp32 gates -- through ``ckda_fwd_chunked``.  A step is
one chunked forward over that batch; ``value`` is whole-job tokens/s (tokens
= B*T positions, each with all H heads).  The recurrent decode step (B=256,
H=32, d=128, bf16, 1024 steps) is measured in the same run and reported under
``decode``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch under torchrun: every rank runs an independent replica on
its own seeded batch (weak scaling; the path has no cross-unit exchange), the
time is the max over ranks and ``value`` sums all ranks' tokens.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# workload constants (KDA-layer prefill)
B, T, H, D, CHUNK = 4, 4096, 16, 128, 64
DEC_B, DEC_H, DEC_STEPS = 256, 32, 1024

# algorithmic counts per token-head (d = 128, C = 64).  The scope table's
# figure counts o in the input precision (bf16): q, k, v, o bf16 + alpha fp32 +
# beta fp32 = 1540 B.  The bench stores o in fp32 (the precision the parity
# bounds are checked at), which moves 256 B more per token-head: both are
# reported, the first as the roofline's `achieved`.
BYTES_PER_TOKEN_HEAD = 4 * D * 2 + D * 4 + 4                  # 1540: q,k,v,o bf16 + alpha + beta
BYTES_PER_TOKEN_HEAD_F32_OUT = 3 * D * 2 + D * 4 + 4 + D * 4  # 1796: o in fp32
# gate-extreme packed workload (fp32 q, k, v, alpha, out; beta)
VARLEN_BYTES_PER_TOKEN_HEAD = 4 * D * 4 + 4 + D * 4           # 2564
STRICT_FLOPS_PER_TOKEN_HEAD = 6 * CHUNK * D + 6 * D * D + CHUNK * CHUNK // 3
DENSE_FLOPS_PER_TOKEN_HEAD = 12 * CHUNK * D + 6 * D * D
DEC_BYTES_PER_HEAD_STEP = 2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 4
# Gated DeltaNet-2 forward: q, k, v bf16 + alpha, b (d_k) and w (d_v) fp32 + out fp32
GDN2_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 4 + D * 4 + D * 4 + D * 4
# SFDA forward: q, k, v bf16 + alpha and theta (d_k / 2 each) fp32 + beta + out fp32
SFDA_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + 2 * (D // 2) * 4 + 4 + D * 4
# backward: q, k, v bf16 + alpha, beta, dO fp32 in; dq, dk, dalpha, dv fp32 + dbeta out
BWD_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 4 + 4 + D * 4 + 3 * D * 4 + D * 4 + 4

SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
# fp32 CUDA-core roof of the kernels that run on FFMA (the fp32-faithful
# forward, the backward): 128 fp32 lanes per SM, one FMA (2 flops) per lane
# per clock, at the B200's maximum SM clock of 1965 MHz.
FP32_LANES_PER_SM = 128
SM_MAX_MHZ = 1965.0
# backward: one recompute of the state step (S' = Diag(a) S, r = S'^T k,
# S' + k u^T: 5 d^2) and the adjoint step (dq, q do^T, dS^T k, dS u + S' dr,
# k dr^T, rowsum(dS' . S), Diag(a) dS': 15 d^2) per token-head
BWD_FLOPS_PER_TOKEN_HEAD = 20 * D * D


def fp32_alu_peak_tflops(torch, dev):
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * FP32_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12, sms


def alu_roofline(flops, ms, peak, sms, what):
    achieved = flops / (ms / 1e3) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "flops_per_launch": flops,
            "peak_basis": f"{sms} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 flops x "
                          f"{SM_MAX_MHZ:.0f} MHz (FFMA)",
            "flops": what}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20, help="0 skips the end-to-end leg")
    ap.add_argument("--decode-steps", type=int, default=DEC_STEPS,
                    help="decode steps timed (inputs for all of them are pre-generated)")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward sub-measure")
    ap.add_argument("--no-long", action="store_true",
                    help="skip the long-context prefill sub-measure (B=1, T=65536, H=32)")
    ap.add_argument("--no-sfda", action="store_true",
                    help="skip the SFDA (phase-decay gates) sub-measure")
    ap.add_argument("--no-gdn2", action="store_true",
                    help="skip the Gated DeltaNet-2 forward measurement")
    ap.add_argument("--no-tiny", action="store_true",
                    help="skip the tiny fp32 workload's latency sub-measure")
    ap.add_argument("--no-varlen", action="store_true",
                    help="skip the gate-extreme packed fp32 workload's sub-measure")
    ap.add_argument("--batch", type=int, default=B,
                    help="sequences of the prefill workload (smaller values make a case small "
                         "enough for a full ncu capture; the bench line is quoted at 4)")
    ap.add_argument("--json-out", default=None)
    return ap.parse_args()


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seeds(rank: int):
    """Seeds of the two rotating input sets of a rank: every replica draws its
    own batch (weak scaling, no shared data)."""
    return [1000 * rank + i for i in range(2)]


def max_over_ranks(x: float, ws: int, device="cpu") -> float:
    """Max of a per-rank time over all ranks (the job is as slow as its slowest rank)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, ws: int, seconds_per_step: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return ws * units_per_rank / seconds_per_step


def _emit(obj, args, rank):
    if rank != 0:
        return
    line = json.dumps(obj)
    print(line, flush=True)
    if args.json_out:
        with open(args.json_out, "w") as f:
            f.write(line + "\n")


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi while running.

    ``start`` returns once the first sample has been written (nvidia-smi can
    take a second to come up), ``mark`` notes where the timed region begins,
    and ``stop`` reports the samples taken from that mark on.  ``count``
    gives how many there are so far, so that a timed region too short for
    several samples can be followed by untimed repetitions of the same work
    until there are enough (``soak_steps`` in the record)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.tmp = None
        self.first = 0
        self.soak_steps = 0

    def _lines(self):
        try:
            with open(self.tmp.name) as f:
                return [ln for ln in f.read().splitlines() if ln.count(",") >= 7]
        except OSError:
            return []

    def count(self) -> int:
        return max(0, len(self._lines()) - self.first) if self.proc is not None else 0

    def mark(self):
        if self.proc is not None:
            self.first = len(self._lines())

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return self
        t0 = time.perf_counter()
        while not self._lines() and time.perf_counter() - t0 < 10.0 and self.proc.poll() is None:
            time.sleep(0.05)
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        lines = self._lines()[self.first:]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.tmp.name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons),
                "soak_steps": self.soak_steps}


# ------------------------------------------------------------ reference ---

def _oracle_sample(n_units, seed=0):
    """A bounded sample of the workload for the CPU oracle: n (b, h) units of
    full length T, drawn exactly like the GPU inputs."""
    from delta_rule_linear_ckda_b200 import inputs

    nb = max(1, min(B, n_units))
    case = inputs.kda_prefill(seed=seed, device="cpu", B=nb, T=T, H=H, d=D)
    hsel = max(1, min(H, math.ceil(n_units / nb)))
    return case, nb, hsel


def _time_oracle(n_units, threads):
    import oracle

    case, nb, hsel = _oracle_sample(n_units)
    q, k, v, a, b = (x[:, :, :hsel].contiguous() for x in (case.q, case.k, case.v, case.alpha, case.beta))
    t0 = time.perf_counter()
    oracle.forward(q, k, v, a, b, n_threads=threads)
    dt = time.perf_counter() - t0
    token_heads = nb * hsel * T
    return dt, token_heads, nb * hsel


def cpu_baseline(target_s=10.0):
    """The oracle on all host threads over the whole workload (all B*H units),
    repeated until about ``target_s`` seconds of wall time have been spent."""
    import oracle

    threads = oracle.default_threads()
    total_dt, total_th, reps = 0.0, 0, 0
    while total_dt < target_s and reps < 50:
        dt, th, u = _time_oracle(B * H, threads)
        total_dt += dt
        total_th += th
        reps += 1
    tokens_per_s = total_th / total_dt / H  # token-heads/s per position with all H heads
    return {"value": tokens_per_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"the whole kda_prefill batch ({B * H} (b,h) units x T={T}) x {reps} "
                      f"passes, {total_dt:.1f} s wall, fp64 sequential loop"}


def run_reference(args, ws, rank):
    if rank != 0:
        return
    import oracle

    threads = oracle.default_threads()
    dt1, _, _ = _time_oracle(1, 1)
    # each step: a bounded sample of whole (b, h) units, sized so that the
    # whole run stays near 100 s of oracle time (at most 1 s per step)
    step_s = min(1.0, 100.0 / max(1, args.steps + args.warmup))
    n_units = int(max(1, min(B * H, step_s * threads / max(dt1, 1e-6))))
    for _ in range(args.warmup):
        _time_oracle(n_units, threads)
    total_dt, total_th = 0.0, 0
    for _ in range(args.steps):
        dt, th, u = _time_oracle(n_units, threads)
        total_dt += dt
        total_th += th
    value = total_th / total_dt / H
    obj = {"metric": "CKDA fwd tokens/s (KDA-layer prefill T=4096, H=16, d=128)",
           "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1000.0 * total_dt / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference",
           "config": {"workload": f"kda_prefill B={B} H={H} T={T} d={D} C={CHUNK} bf16 inputs",
                      "sample_units_per_step": n_units, "parallelism": "host threads"},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": f"{n_units} (b,h) units x T={T} per step"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    _emit(obj, args, rank)


# ------------------------------------------------------------------ ours ---

# sources of the forward's kernels: a committed DRAM-traffic figure is used
# only while these are unchanged
FWD_KERNEL_SOURCES = ("fwd_tc.cu", "sm100.cuh", "common.cuh")


def _kernel_src_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "delta_rule_linear_ckda_b200", "csrc")
    for fn in FWD_KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_from_profile():
    """DRAM bytes per launch from a committed ncu summary, if it matches the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    if d.get("src_hash") != _kernel_src_hash():
        return None, d.get("src_hash")
    return d.get("fwd_dram_bytes_per_launch"), d.get("src_hash")


def run_ours(args, ws, rank, local):
    import torch
    import torch.distributed as dist

    import delta_rule_linear_ckda_b200 as ck
    from delta_rule_linear_ckda_b200 import _lib, inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if ws > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    hbm_peak, tc_peak, tc_peak_sus, peak_src = _peaks()

    def barrier():
        if ws > 1:
            dist.barrier()

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, ws, dev)

    # two input sets (each ~0.4 GB > 126 MB L2), rotated so no step finds its
    # inputs in L2
    sets = [inputs.kda_prefill(seed=sd, device=dev, B=B) for sd in rank_seeds(rank)]
    out = torch.empty(sets[0].v.shape, dtype=torch.float32, device=dev)
    S_final = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    path = ck.fwd_path(B, T, H, D, D, CHUNK, torch.bfloat16, torch.float32)
    variants = {}
    for kind, off in (("gdn2", args.no_gdn2), ("sfda", args.no_sfda)):
        if not off:
            variants[kind] = _run_variant(kind, ck, torch, inputs, rank, dev, stream, barrier,
                                          max_ranks, ws, hbm_peak)
    if not args.no_long:
        variants["long_prefill"] = _run_long(ck, torch, inputs, rank, dev, stream, barrier,
                                             max_ranks, ws, hbm_peak)
    if not args.no_bwd:
        variants["bwd"] = _run_bwd(ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws,
                                   hbm_peak)
    wsbuf = torch.empty(max(1, ck.workspace_bytes(B, T, H, D, D, CHUNK)), dtype=torch.uint8,
                        device=dev)
    two_phase = path == "tcgen05"

    def step(i):
        # One forward over the batch through the public call (on the
        # tensor-core path: the factor kernel, then the carry kernel).
        c = sets[i % 2]
        ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, chunk=CHUNK, out=out, S_final=S_final,
                       workspace=wsbuf)

    def split_step(i, mid):
        # The same two kernels issued as the two ABI phases, so an event
        # between them times each kernel (a separate loop: events between
        # the kernels cost the loop about 2 %).
        c = sets[i % 2]
        ck.fwd_factors(c.q, c.k, c.v, c.alpha, c.beta, chunk=CHUNK, workspace=wsbuf)
        mid.record(stream)
        ck.fwd_carry(wsbuf, c.v, B, T, H, D, D, chunk=CHUNK, out=out, S_final=S_final)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id).start() if rank == 0 else None

    K = args.steps
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark()
    wall0 = time.perf_counter()
    ev0.record(stream)
    for i in range(K):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    wall = time.perf_counter() - wall0
    if sampler:
        # a region too short for 5 samples: the same steps again, untimed,
        # until the sampler has seen 5 (at most 3 s)
        t_soak = time.perf_counter()
        while (sampler.count() < 5 and sampler.proc is not None
               and time.perf_counter() - t_soak < 3.0):
            for j in range(8):
                step(j)
            sampler.soak_steps += 8
            torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_ranks(ev0.elapsed_time(ev1))
    ms_per_step = elapsed_ms / K
    # the forward's kernels run back to back in the timed region, so the
    # forward's (the kernel pair's) average duration is the step time
    kern_ms = ms_per_step
    kernels = None
    if two_phase:
        KS = min(K, 50)
        ks = [torch.cuda.Event(enable_timing=True) for _ in range(KS)]
        km = [torch.cuda.Event(enable_timing=True) for _ in range(KS)]
        ke = [torch.cuda.Event(enable_timing=True) for _ in range(KS)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(KS):
            ks[i].record(stream)
            split_step(i, km[i])
            ke[i].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        f_ms = max_ranks(statistics.mean(ks[i].elapsed_time(km[i]) for i in range(KS)))
        c_ms = max_ranks(statistics.mean(km[i].elapsed_time(ke[i]) for i in range(KS)))
        kernels = {"factor_kernel": {"ms": f_ms, "share": f_ms / (f_ms + c_ms),
                                     "workspace_bytes_written": wsbuf.numel()},
                   "carry_kernel": {"ms": c_ms, "share": c_ms / (f_ms + c_ms)},
                   "timing": f"{KS} forwards issued as the two ABI phases with an event "
                             "before, between and after the kernels"}
    tokens = B * T
    value = whole_job_rate(tokens, ws, ms_per_step / 1e3)

    token_heads = B * T * H
    alg_bytes = token_heads * BYTES_PER_TOKEN_HEAD + B * H * D * D * 4
    alg_bytes_f32_out = token_heads * BYTES_PER_TOKEN_HEAD_F32_OUT + B * H * D * D * 4
    strict_flops = token_heads * STRICT_FLOPS_PER_TOKEN_HEAD
    dense_flops = token_heads * DENSE_FLOPS_PER_TOKEN_HEAD
    achieved_gbs = alg_bytes / (kern_ms / 1e3) / 1e9
    achieved_gbs_f32_out = alg_bytes_f32_out / (kern_ms / 1e3) / 1e9
    tflops_strict = strict_flops / (kern_ms / 1e3) / 1e12
    tflops_dense = dense_flops / (kern_ms / 1e3) / 1e12
    traffic, _ = _traffic_from_profile()

    # ---- end to end: host (pinned) buffers through the public API --------
    e2e = None
    if args.e2e_steps > 0:
        e2e = _run_e2e(args, ck, torch, sets[0], out, S_final, stream, barrier, max_ranks,
                       ws, tokens, dev, wsbuf)

    # ---- decode step (B=256, H=32, d=128, bf16), 1024 steps --------------
    decode = None
    if not args.no_decode:
        decode = _run_decode(args, ck, torch, inputs, rank, dev, stream, barrier, max_ranks,
                             ws, hbm_peak)
    # ---- the two fp32 workloads: tiny (latency) and gate-extreme varlen --
    if not args.no_tiny:
        variants["tiny"] = _run_tiny(ck, torch, inputs, rank, dev, stream, barrier, max_ranks)
    if not args.no_varlen:
        variants["varlen"] = _run_varlen(ck, torch, inputs, rank, dev, stream, barrier,
                                         max_ranks, ws, hbm_peak)
    extra_roof = {"achieved_fp32_out_bytes": achieved_gbs_f32_out,
                  "frac_fp32_out_bytes": achieved_gbs_f32_out / hbm_peak,
                  "algorithmic_bytes_fp32_out": alg_bytes_f32_out}
    _finish(args, ws, rank, value, K, ms_per_step, alg_bytes, achieved_gbs, hbm_peak, traffic,
            peak_src, kern_ms, tflops_strict, tflops_dense, tc_peak, e2e, clocks, wall, decode,
            _lib.LIB_PATH, path, kernels, variants, extra_roof)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def _run_e2e(args, ck, torch, c, out, S_final, stream, barrier, max_ranks, ws, tokens, dev, wsbuf):
    """End to end through the public API with host buffers: every step copies its
    inputs from pinned host memory, runs the forward and copies out and S_final
    back.  Steps are pipelined on three streams with double-buffered device
    tensors: the copies of step i + 1 in (and of step i - 1 out) overlap the
    forward of step i, as a serving loop would run them."""
    host = {n: getattr(c, n).cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta")}
    dbuf = [{n: torch.empty_like(getattr(c, n)) for n in host} for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    sfs = [S_final, torch.empty_like(S_final)]
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    sf_h = [torch.empty(S_final.shape, dtype=S_final.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size() + sf_h[0].numel() * sf_h[0].element_size()
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    issued = [0]

    def e2e_step():
        i = issued[0]
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[b])  # the forward of step i - 2 has read these inputs
            for n, t in host.items():
                dbuf[b][n].copy_(t, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])  # step i - 2's results have left these buffers
        d = dbuf[b]
        ck.fwd_chunked(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=CHUNK, out=outs[b],
                       S_final=sfs[b], workspace=wsbuf)
        ev_cmp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            out_h[b].copy_(outs[b], non_blocking=True)
            sf_h[b].copy_(sfs[b], non_blocking=True)
            ev_out[b].record(s_out)
        issued[0] += 1

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    E = max(1, args.e2e_steps)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(s_in)
    for _ in range(E):
        e2e_step()
    ev1.record(s_out)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_ranks(ev0.elapsed_time(ev1)) / E
    e2e_value = ws * tokens / (e2e_ms / 1e3)
    return {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "pipelined": "H2D, forward and D2H on three streams, double-buffered"}


def _run_variant(kind, ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws, hbm_peak,
                 steps=20):
    """A variant's forward at the bench sizes (bf16 q/k/v, fp32 gates and
    output); two rotating input sets.  kind "gdn2": Gated DeltaNet-2 (erase and
    write gates); kind "sfda": SFDA (phase-decay gates)."""
    if kind == "gdn2":
        sets = [inputs.gdn2_prefill(B, T, H, D, D, dtype=torch.bfloat16, chunk=CHUNK,
                                    seed=3000 + 10 * rank + i, device=dev) for i in range(2)]
    else:
        sets = [inputs.sfda_prefill(B, T, H, D, D, dtype=torch.bfloat16, chunk=CHUNK,
                                    seed=4000 + 10 * rank + i, device=dev) for i in range(2)]
    out = torch.empty(sets[0].v.shape, dtype=torch.float32, device=dev)
    S_final = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    wsbuf = torch.empty(max(1, ck.workspace_bytes(B, T, H, D, D, CHUNK)), dtype=torch.uint8,
                        device=dev)

    def step(i):
        c = sets[i % 2]
        if kind == "gdn2":
            ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], chunk=CHUNK,
                                out=out, S_final=S_final, workspace=wsbuf)
        else:
            ck.sfda_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["theta"], c.beta, chunk=CHUNK,
                                out=out, S_final=S_final, workspace=wsbuf)

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for i in range(steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_ranks(ev0.elapsed_time(ev1)) / steps
    per_th = GDN2_BYTES_PER_TOKEN_HEAD if kind == "gdn2" else SFDA_BYTES_PER_TOKEN_HEAD
    nbytes = B * T * H * per_th + B * H * D * D * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    del sets
    if kind == "gdn2":
        path = ck.fwd_path(B, T, H, D, D, CHUNK, torch.bfloat16, torch.float32)
        what = f"gdn2_prefill B={B} H={H} T={T} d={D} C={CHUNK} bf16 q/k/v, fp32 alpha/b/w"
    else:
        path = ck.fwd_path(B, T, H, D, D, CHUNK, torch.bfloat16, torch.float32)
        what = (f"sfda_prefill B={B} H={H} T={T} d={D} C={CHUNK} bf16 q/k/v, fp32 "
                f"alpha/theta (d/2 pairs)/beta")
    return {"workload": f"{what}, fp32 out ({path} kernels)",
            "ms_per_step": ms, "tokens_per_s": ws * B * T / (ms / 1e3),
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "hbm_frac_of_measured": gbs / hbm_peak,
            "gpu_launches": steps * (2 if path == "tcgen05" else 1)}


def _run_long(ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws, hbm_peak, steps=10):
    """The long-context prefill (B=1, T=65536, H=32, d=128, bf16 q/k/v, S0 read,
    S_final stored): the forward's two kernels timed apart, as in the main step."""
    Bl, Tl, Hl = 1, 65536, 32
    c = inputs.long_prefill(seed=6000 + rank, device=dev, T=Tl, H=Hl, d=D)
    out = torch.empty(c.v.shape, dtype=torch.float32, device=dev)
    S_final = torch.empty((Bl, Hl, D, D), dtype=torch.float32, device=dev)
    wsb = torch.empty(ck.workspace_bytes(Bl, Tl, Hl, D, D, CHUNK), dtype=torch.uint8, device=dev)

    def step(mid=None):
        ck.fwd_factors(c.q, c.k, c.v, c.alpha, c.beta, chunk=CHUNK, workspace=wsb)
        if mid is not None:
            mid.record(stream)
        ck.fwd_carry(wsb, c.v, Bl, Tl, Hl, D, D, S0=c.S0, chunk=CHUNK, out=out, S_final=S_final)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    km = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(steps):
        ks[i].record(stream)
        step(km[i])
        ke[i].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    f_ms = max_ranks(statistics.mean(ks[i].elapsed_time(km[i]) for i in range(steps)))
    c_ms = max_ranks(statistics.mean(km[i].elapsed_time(ke[i]) for i in range(steps)))
    # the forward through the public call, back to back
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, chunk=CHUNK, out=out,
                       S_final=S_final, workspace=wsb)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_ranks(e0.elapsed_time(e1)) / steps
    # the same forward as a chunk-parallel scan over G segments per sequence
    scan = {}
    for G in (2, 4):
        wss = torch.empty(ck.scan_workspace_bytes(Bl, Tl, Hl, D, D, G), dtype=torch.uint8,
                          device=dev)
        for _ in range(2):
            ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, G, S0=c.S0, out=out,
                                S_final=S_final, workspace=wss)
        torch.cuda.synchronize(dev)
        assert ck.device_status(dev) == 0
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(5):
            ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, G, S0=c.S0, out=out,
                                S_final=S_final, workspace=wss)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        scan[f"segments_{G}"] = {"ms_per_step": max_ranks(e0.elapsed_time(e1)) / 5,
                                 "gpu_launches_per_step": 4}
        del wss
    th = Bl * Tl * Hl
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    nbytes = th * BYTES_PER_TOKEN_HEAD + 2 * Bl * Hl * D * D * 4  # + S0 read, S_final written
    nbytes32 = th * BYTES_PER_TOKEN_HEAD_F32_OUT + 2 * Bl * Hl * D * D * 4
    return {"workload": f"long_prefill B={Bl} H={Hl} T={Tl} d={D} C={CHUNK} bf16 q/k/v, fp32 "
                        "gates and out, S0 read, S_final stored (tcgen05 kernels)",
            "ms_per_step": ms, "tokens_per_s": ws * Bl * Tl / (ms / 1e3),
            "achieved_gbs_fp32_out_bytes": nbytes32 / (ms / 1e3) / 1e9,
            "kernels": {"factor_kernel_ms": f_ms, "carry_kernel_ms": c_ms,
                        "carry_ctas": Hl * Bl * (4 if 2 * (2 * Hl * Bl) <= n_sm else 2),
                        "carry_columns_per_cta": 32 if 2 * (2 * Hl * Bl) <= n_sm else 64},
            "chunk_parallel_scan": scan,
            "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
            "hbm_frac_of_measured": nbytes / (ms / 1e3) / 1e9 / hbm_peak,
            "gpu_launches": 2 * steps}


def _run_tiny(ck, torch, inputs, rank, dev, stream, barrier, max_ranks, calls=200):
    """Latency of the tiny fp32 workload (B=1, H=2, T=64, d=16, C=16): one
    forward call per step, timed eagerly through the Python API and replayed
    from a CUDA graph of the same calls."""
    c = inputs.tiny(seed=rank, device=dev)
    out = torch.empty(c.v.shape, dtype=torch.float32, device=dev)
    S_final = torch.empty((1, 2, 16, 16), dtype=torch.float32, device=dev)

    def call():
        ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, chunk=c.chunk, out=out, S_final=S_final)

    for _ in range(5):
        call()
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(calls):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    eager_us = 1e3 * max_ranks(e0.elapsed_time(e1)) / calls
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(calls):
            call()
    torch.cuda.synchronize(dev)
    barrier()
    e0.record(stream)
    gr.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    graph_us = 1e3 * max_ranks(e0.elapsed_time(e1)) / calls
    del gr
    return {"workload": "tiny B=1 H=2 T=64 d=16 C=16 fp32 (alpha ~ U[-1,1], beta ~ U[0,2])",
            "kernel": ck.fwd_path(1, 64, 2, 16, 16, 16, torch.float32, torch.float32),
            "us_per_call_eager": eager_us, "us_per_call_graph": graph_us,
            "tokens_per_s_graph": 64 / (graph_us / 1e6), "bound": "launch latency",
            "gpu_launches_per_call": 1}


def _run_varlen(ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws, hbm_peak,
                steps=10):
    """The gate-extreme packed workload (64 sequences, L ~ U[128, 4096], H=16,
    d=128, fp32 q/k/v; near-zero gates then orthogonal transitions; S0 = 0,
    S_final stored): ms per forward and GB/s of its algorithmic bytes (2564
    B per token-head plus S_final), inputs larger than L2."""
    c = inputs.varlen(seed=rank, device=dev)
    Tt = c.q.shape[1]
    N = c.n_seqs
    out = torch.empty(c.v.shape, dtype=torch.float32, device=dev)
    S_final = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)

    def call():
        ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, cu_seqlens=c.cu_seqlens, chunk=CHUNK,
                       out=out, S_final=S_final)

    for _ in range(2):
        call()
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_ranks(e0.elapsed_time(e1)) / steps
    nbytes = Tt * H * VARLEN_BYTES_PER_TOKEN_HEAD + N * H * D * D * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    peak, sms = fp32_alu_peak_tflops(torch, dev)
    roof = alu_roofline(Tt * H * STRICT_FLOPS_PER_TOKEN_HEAD, ms, peak, sms,
                        "strict chunk flops per token-head (6 C d + 6 d^2 + C^2 / 3) x token-heads")
    return {"workload": f"varlen N={N} L~U[128,4096] (T_total={Tt}) H={H} d={D} C={CHUNK} fp32, "
                        "gate extremes, S0=0, S_final stored",
            "kernel": ck.fwd_path(N, Tt, H, D, D, CHUNK, torch.float32, torch.float32,
                                  varlen=True),
            "ms_per_step": ms, "tokens_per_s": ws * Tt / (ms / 1e3),
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "hbm_frac_of_measured": gbs / hbm_peak,
            "hbm_floor_ms_at_measured": nbytes / (hbm_peak * 1e9) * 1e3,
            "roofline": roof, "alu_floor_ms": roof["flops_per_launch"] / (peak * 1e12) * 1e3,
            "steps": steps, "gpu_launches": steps}


def _run_bwd(ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws, hbm_peak, steps=5):
    """Backward at the bench sizes (bf16 q/k/v, fp32 gates and dO, fp32
    gradients, no S0 / dS_final); inputs larger than L2, one set."""
    c = inputs.kda_prefill(seed=5000 + rank, device=dev, B=B)
    g = torch.Generator(device=dev).manual_seed(5100 + rank)
    dO = torch.randn(c.v.shape, generator=g, device=dev)
    grads = {"dq": torch.empty(c.q.shape, dtype=torch.float32, device=dev),
             "dk": torch.empty(c.k.shape, dtype=torch.float32, device=dev),
             "dv": torch.empty(c.v.shape, dtype=torch.float32, device=dev),
             "dalpha": torch.empty(c.alpha.shape, dtype=torch.float32, device=dev),
             "dbeta": torch.empty(c.beta.shape, dtype=torch.float32, device=dev)}
    wsb = torch.empty(ck.bwd_workspace_bytes(B, T, H, D, D), dtype=torch.uint8, device=dev)

    def step():
        ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO, grads=grads, want_dS0=False,
                       workspace=wsb)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    assert ck.device_status(dev) == 0
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_ranks(ev0.elapsed_time(ev1)) / steps
    nbytes = B * T * H * BWD_BYTES_PER_TOKEN_HEAD
    gbs = nbytes / (ms / 1e3) / 1e9
    peak, sms = fp32_alu_peak_tflops(torch, dev)
    roof = alu_roofline(B * T * H * BWD_FLOPS_PER_TOKEN_HEAD, ms, peak, sms,
                        "per-token adjoint with one state recompute, 20 d^2 per token-head")
    return {"workload": f"kda_prefill backward B={B} H={H} T={T} d={D}: bf16 q/k/v, fp32 "
                        "alpha/beta/dO, fp32 gradients (fp32 CUDA-core kernel, clusters of "
                        f"{D // 32} CTAs per (sequence, head))",
            "ms_per_step": ms, "tokens_per_s": ws * B * T / (ms / 1e3),
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "hbm_frac_of_measured": gbs / hbm_peak, "workspace_bytes": wsb.numel(),
            "roofline": roof, "gpu_launches": steps}


def _run_decode(args, ck, torch, inputs, rank, dev, stream, barrier, max_ranks, ws, hbm_peak):
    """Decode steps through the public API, timed twice over the same steps:
    eagerly (one Python call per step, as a plain loop issues them) and as a
    CUDA graph of those calls replayed once (the kernels back to back, as a
    serving loop under graphs runs them).  ``ms_per_step`` is the graph
    figure; ``ms_per_step_eager`` the eager one."""
    steps = max(1, args.decode_steps)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    dc = inputs.decode(seed=2000 + rank, device=dev, B=DEC_B, H=DEC_H, d=D, steps=steps + 8)
    S = dc.S0.clone()
    dout = torch.empty((DEC_B, DEC_H, D), dtype=torch.float32, device=dev)

    def timed(issue, n):
        torch.cuda.synchronize(dev)
        barrier()
        ev0.record(stream)
        issue()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        eager = max_ranks(ev0.elapsed_time(ev1)) / n
        gr = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(gr):
                issue()
            ok = 1.0
        except Exception:
            ok = 0.0
        torch.cuda.synchronize(dev)
        ok = -max_ranks(-ok)  # every rank's capture succeeded
        barrier()
        ev0.record(stream)
        if ok:
            gr.replay()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        graph = max_ranks(ev0.elapsed_time(ev1)) / n
        del gr
        return (graph if ok else eager), eager, ("cuda_graph" if ok else "eager")

    def kda_steps():
        for t in range(8, 8 + steps):
            ck.decode_step(dc.q[t], dc.k[t], dc.v[t], dc.alpha[t], dc.beta[t], S, out=dout)

    for t in range(8):
        ck.decode_step(dc.q[t], dc.k[t], dc.v[t], dc.alpha[t], dc.beta[t], S, out=dout)
    dec_ms, dec_eager, how = timed(kda_steps, steps)
    dbytes = DEC_B * DEC_H * DEC_BYTES_PER_HEAD_STEP
    dgbs = dbytes / (dec_ms / 1e3) / 1e9
    decode = {"workload": f"decode B={DEC_B} H={DEC_H} d={D} bf16 q/k/v, fp32 out, "
                          f"{steps} steps",
              "ms_per_step": dec_ms, "ms_per_step_eager": dec_eager, "timing": how,
              "tokens_per_s": ws * DEC_B / (dec_ms / 1e3),
              "achieved_gbs": dgbs, "hbm_frac_of_measured": dgbs / hbm_peak,
              "hbm_frac_of_spec_8tbs": dgbs / SPEC_HBM_GBS,
              "bytes_per_step": dbytes, "gpu_launches": steps}
    # the two gate variants' decode steps on the same tokens and state size,
    # 64 steps each after 4 warm-up steps
    vs = min(64, steps)
    g = torch.Generator(device=dev).manual_seed(2100 + rank)
    u = lambda *shape: torch.rand(*shape, generator=g, device=dev)  # noqa: E731
    bvar = {"gdn2": (u(vs + 4, DEC_B, DEC_H, D), u(vs + 4, DEC_B, DEC_H, D)),
            "sfda": (u(vs + 4, DEC_B, DEC_H, D // 2),
                     (2 * u(vs + 4, DEC_B, DEC_H, D // 2) - 1) * 3.141592653589793)}
    # bytes per head-step beyond the state: q, k, v bf16, out fp32, and the gates
    gate_bytes = {"gdn2": D * 4 + D * 4 + D * 4, "sfda": 2 * (D // 2) * 4 + 4}
    for kind, (g1, g2) in bvar.items():
        def one(t):
            if kind == "gdn2":
                ck.gdn2_decode_step(dc.q[t], dc.k[t], dc.v[t], dc.alpha[t], g1[t], g2[t], S,
                                    out=dout)
            else:
                ck.sfda_decode_step(dc.q[t], dc.k[t], dc.v[t], g1[t], g2[t], dc.beta[t], S,
                                    out=dout)

        def var_steps():
            for t in range(4, 4 + vs):
                one(t)
        for t in range(4):
            one(t)
        ms, eager, how = timed(var_steps, vs)
        nb = DEC_B * DEC_H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + gate_bytes[kind])
        decode[kind] = {"ms_per_step": ms, "ms_per_step_eager": eager, "timing": how,
                        "tokens_per_s": ws * DEC_B / (ms / 1e3),
                        "achieved_gbs": nb / (ms / 1e3) / 1e9,
                        "hbm_frac_of_measured": nb / (ms / 1e3) / 1e9 / hbm_peak,
                        "bytes_per_step": nb, "steps": vs, "gpu_launches": vs}
    del dc, S, bvar
    return decode


def _finish(args, ws, rank, value, K, ms_per_step, alg_bytes, achieved_gbs, hbm_peak, traffic,
            peak_src, kern_ms, tflops_strict, tflops_dense, tc_peak, e2e, clocks, wall, decode,
            lib_path, path, kernels=None, variants=None, extra_roof=None):
    # `dtype` names the workload's input precision (bf16 q/k/v); the
    # arithmetic is in `compute`: tcgen05 MMAs on fp16 operands with fp32
    # accumulation and fp32 state, or fp32 FFMA on CUDA cores
    dtype = "bf16"
    obj = {
        "metric": "CKDA fwd tokens/s (KDA-layer prefill T=4096, H=16, d=128)",
        "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "compute": {"kernel": path, "mma_operands": "f16" if path == "tcgen05" else None,
                    "accumulate": "f32", "state": "f32", "inputs": "bf16 q/k/v, f32 gates"},
        "config": {"workload": f"kda_prefill B={B} H={H} T={T} d_k=d_v={D} C={CHUNK} "
                               "bf16 q/k/v, fp32 alpha/beta, fp32 out, S0=0, S_final stored",
                   "global_batch": ws * B, "seq_len": T, "heads": H, "head_dim": D,
                   "chunk": CHUNK, "parallelism": f"replicas x{ws} (no data-path collective)",
                   "l2": "inputs larger than L2: two rotating 0.40 GB input sets"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                     "peak_source": f"{peak_src} hbm_gbs (burst copy)",
                     "algorithmic_bytes_per_launch": alg_bytes, "kernel_ms": kern_ms,
                     "bytes_per_token_head": BYTES_PER_TOKEN_HEAD,
                     "scope": "the chunked forward: factor kernel + carry kernel, one pair per "
                              "step; bytes are the scope table's algorithmic bytes (q, k, v, o "
                              "bf16, alpha, beta fp32, S_final); the fp32-output accounting "
                              "(the output the bench actually stores) is beside it",
                     **(extra_roof or {})},
        "kernels": kernels,
        "tensor": {"strict_tflops": tflops_strict, "dense_block_tflops": tflops_dense,
                   "frac_strict_of_measured": tflops_strict / tc_peak,
                   "frac_dense_of_measured": tflops_dense / tc_peak,
                   "frac_strict_of_spec": tflops_strict / SPEC_BF16_TFLOPS,
                   "frac_dense_of_spec": tflops_dense / SPEC_BF16_TFLOPS,
                   "measured_bf16_tflops": tc_peak},
        "e2e": e2e,
        "gpu_launches": 2 * K if path == "tcgen05" else K,
        "clocks": clocks,
        "wall_s_timed_region": wall,
        "lib": os.path.relpath(lib_path, ROOT),
    }
    if decode is not None:
        obj["decode"] = decode
    for kind, res in (variants or {}).items():
        obj[kind] = res
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        obj["cpu_baseline"] = cpu_baseline()
    _emit(obj, args, rank)


def main():
    global B
    args = _args()
    B = args.batch
    ws, rank, local = _dist()
    if args.impl == "reference":
        run_reference(args, ws, rank)
        return
    run_ours(args, ws, rank, local)


if __name__ == "__main__":
    main()
