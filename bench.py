"""Benchmark of the top-k sparse FlashAttention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sfa|reference]

One step = one pass of the whole hot path on seeded synthetic inputs already resident in
HBM: the whole public sfa_fwd call on the long-context NSA prefill workload (lengths
[65536, 32768], Hq = Hkv = 4, d128, block 64, top-16 with init 1 / local 2: the largest
single-GPU configuration, which also runs the block-major schedule and its partial merge),
followed by the whole sfa_decode call on the paged top-k decode workload (B32, Hq32/Hkv8,
d128, L ~ U[16384, 131072], page 256, 2048 tokens per (sequence, kv head)).  L2 is flushed
(256 MiB write) before every step, outside the kernel events.

The JSON line's value is the prefill's effective TFLOP/s (4*d flops per kept query-key pair
per query head, the pairs counted exactly from the selections); the decode figure (gathered
K+V bytes per second) is reported beside it.  The other prefill configurations (tiny, varlen
NSA, dense window) are timed beside the step under "prefill_configs", each as its whole
public call.  Under torchrun each rank runs its own instance of the workload (independent
problems, no collective; weak scaling) and the time is the max over ranks.  --impl reference
times the fp64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sfa_workloads as W  # noqa: E402

METRIC = "sparse-attn fwd effective TFLOP/s & decode gathered-KV GB/s, 1×B200"
PREFILL_NAMES = {
    1: "tiny_256_d64: 1 x 256 tokens, Hq4/Hkv1, d64, bs32, topk4 (block 0 + own block)",
    2: "nsa_varlen_16k: lens [8192,4096,2048,2048], Hq16/Hkv4, d128, bs64, topk16 (init1, local2)",
    3: "dense_window_1k_4k: B2, sq1024/sk4096, Hq32/Hkv8, d128, causal, window (1024,0), all 17 touched blocks",
    4: "nsa_long_96k: lens [65536,32768], Hq4/Hkv4, d128, bs64, topk16 (init1, local2)",
}
PREFILL_CONFIGS = {1: W.config1, 2: W.config2, 3: W.config3, 4: W.config4}
DECODE_NAME = "paged_topk_decode_b32: B32, Hq32/Hkv8, d128, L~U[16384,131072], page256, 2048 tok/(b,hk)"
# the decode cases the profiling parts put in its place
DECODE_PART_NAMES = {"all": DECODE_NAME,
                     "prefill": "tiny decode: B2, Hq32/Hkv8, d128, L~U[1024,2048], page256, 256 tok/(b,hk)",
                     "decode-small": "paged_topk_decode_b32 with L~U[4096,16384]"}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the dominant kernel of
# each stage, from one `ncu` capture of that kernel on its workload.  A figure holds only for the
# kernel sources it was taken on: the digest of those files must match, else the bench reports null.
TRAFFIC = {
    # the six kernels of one call on nsa_long_96k (prep, plan, scatter, query-major, block-major, merge)
    "prefill_c4": {"files": ["sfa_fwd_pipe_kernel.cu", "sfa_fwd_inv_kernel.cu", "sfa_prep.cu", "sfa_device.cuh"],
                   "sha256": "2c5060e737605c2773b8d36dde669c8833f4615aad99b892c2e733003c06c81b",
                   "bytes": 3969697536},
    # the one kernel of a call on nsa_varlen_16k (the fused query-major kernel)
    "prefill_c2": {"files": ["sfa_fwd_pipe_kernel.cu", "sfa_device.cuh"],
                   "sha256": "f8b1585aed8bcf23a6056420f9d897e21a56bccd284f10646aaf0fb216cf7a05",
                   "bytes": 138302208},
    # one launch on paged_topk_decode_b32
    "decode_split_kernel": {"files": ["sfa_decode_kernel.cu", "sfa_device.cuh"],
                            "sha256": "3c37939e4121865544ad7821a99c3ea8855117df49a3588bb15bf558a99db3f4",
                            "bytes": 271037696},
}


def source_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "sparse_flashattention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def kernel_traffic(kernel):
    t = TRAFFIC.get(kernel)
    if not t or t["sha256"] is None:
        return None
    return t["bytes"] if source_digest(t["files"]) == t["sha256"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kept_per_token(c):
    """Kept keys of every (query token, kv head), int64 (total_q, Hkv): the keys of every distinct
    block id of the token's selection that is a block of its sequence, inside the causal / window
    mask.  Counted on the host from the selection as given (duplicates, -1 and out-of-range ids
    dropped)."""
    out = np.zeros((c.total_q, c.Hkv), np.int64)
    for b in range(c.batch):
        q0, q1 = int(c.cu_q[b]), int(c.cu_q[b + 1])
        sq, sk = q1 - q0, int(c.cu_k[b + 1] - c.cu_k[b])
        if sq == 0:
            continue
        nblk = (sk + c.bs - 1) // c.bs
        i = np.arange(sq, dtype=np.int64)
        lo = np.zeros(sq, np.int64)
        hi = np.full(sq, sk - 1, np.int64)
        if c.causal:
            hi = np.minimum(hi, i + sk - sq)
        if c.wr >= 0:
            hi = np.minimum(hi, i + sk - sq + c.wr)
        if c.wl >= 0:
            lo = np.maximum(lo, i + sk - sq - c.wl)
        s = np.sort(np.asarray(c.sel[q0:q1], np.int64), axis=2)
        keep = (s >= 0) & (s < nblk)
        keep[..., 1:] &= s[..., 1:] != s[..., :-1]
        bl = s * c.bs
        bh = np.minimum(bl + c.bs, sk) - 1
        n = np.minimum(bh, hi[:, None, None]) - np.maximum(bl, lo[:, None, None]) + 1
        out[q0:q1] = np.where(keep, np.clip(n, 0, None), 0).sum(axis=2)
    return out


def kept_pairs(c):
    """Kept (query token, key) pairs summed over (token, kv head)."""
    return int(kept_per_token(c).sum())


def prefill_flops(c):
    """4*d flops per kept (query, key) pair per query head; the G query heads of a kv head share its
    selection, so each (token, kv head) pair count is taken G times."""
    return 4.0 * c.d * (c.Hq // c.Hkv) * kept_pairs(c)


def decode_bytes(c):
    """Algorithmic gathered bytes: K and V row (d bf16 each) per distinct valid (token, kv head)."""
    n = 0
    for b in range(c.B):
        L = int(c.cache_seqlens[b])
        for hk in range(c.Hkv):
            s = c.sel[b, hk]
            n += np.unique(s[(s >= 0) & (s < L)]).size
    return n * 2 * c.d * 2


# ---------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------------------------
REASONS = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    def __init__(self, gpu_index, path):
        self.path = path
        self.proc = None
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first(self, limit_s=3.0):
        """Block until nvidia-smi has written its first sample (it takes a few hundred ms to start), so a
        short timed region still falls between samples."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < limit_s and self.proc.poll() is None:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                return
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
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
                rows.append((float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return None
        mx = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * mx] or rows
        reasons = set()
        for _, _, rs in rows:
            for name, val in zip(REASONS[1:], rs[1:]):
                if val.lower() not in ("not active", "0", "0x0000000000000000"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


def physical_gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ---------------------------------------------------------------------------------------------
# Multi-rank reductions (independent replicas: the only collectives are these timing reductions)
# ---------------------------------------------------------------------------------------------
def max_over_ranks(vals, world, device):
    """Element-wise max of per-rank timings; every rank calls it the same number of times."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput in units/s: each of `world` ranks processes `units_per_rank`, and the
    job takes the slowest rank's `ms`."""
    return world * units_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------------------------
def cpu_oracle_rate(c, seconds, seed=0):
    """Time the fp64 oracle on random (token, head) rows of the prefill workload, sized to
    about `seconds` of CPU work; returns (TFLOP/s, rows, threads, seconds)."""
    import oracle

    rng = np.random.default_rng(seed)
    kept = kept_per_token(c)  # (total_q, Hkv)
    G = c.Hq // c.Hkv

    def run(n):
        rows = np.sort(rng.choice(c.total_q * c.Hq, size=n, replace=False)).astype(np.int64)
        flops = 4.0 * c.d * kept[rows // c.Hq, (rows % c.Hq) // G].sum()
        t0 = time.perf_counter()
        oracle.fwd(c, rows=rows)
        return flops, time.perf_counter() - t0, n

    threads = oracle.default_threads()
    cap = c.total_q * c.Hq
    n = min(cap, 64 * threads)
    while True:  # grow the sample until one run takes most of the requested time
        f, t, n = run(n)
        if t >= 0.6 * seconds or n >= cap:
            return f / t / 1e12, n, threads, t
        n = int(min(cap, max(n + 1, n * min(8.0, seconds / max(t, 1e-3)))))


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import sparse_flashattention_b200 as sfa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm, tf_burst, tf_sust, peak_kind = peaks()

    if args.part == "decode-small":
        pc = W.small_config(2)
    elif args.shrink > 1:
        pc = PREFILL_CONFIGS[args.prefill_config](shrink=args.shrink)
    else:
        pc = PREFILL_CONFIGS[args.prefill_config]()
    P = W.upload_prefill(pc, dev)
    flops = prefill_flops(pc)
    # Profiling aids: 'prefill' skips the 9.7 GB decode cache (a tiny decode case stands in);
    # 'decode-small' runs the decode shape with shorter caches (about 1.3 GB) for ncu captures.
    if args.part == "prefill":
        dc = W.make_decode(5, 2, 32, 8, 128, 256, 1024, 2048, 256, 16)
    elif args.part == "decode-small":
        dc = W.make_decode(5, 32, 32, 8, 128, 256, 4096, 16384, 2048, 128, parallel_values=True)
    else:
        dc = W.config5(parallel_values=True)
    D = W.upload_decode(dc, dev)
    gbytes = decode_bytes(dc)

    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    dout = torch.empty_like(D["q"])
    dlse = torch.empty((dc.B, dc.Hq), dtype=torch.float32, device=dev)
    dws = torch.empty(sfa.decode_workspace_size(dc.B, dc.Hq, dc.Hkv, dc.d, dc.topk, 0), dtype=torch.uint8,
                      device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    launches = [0]

    def prefill_call(c, T):
        """The public sfa_fwd call on one uploaded prefill case, with its own outputs and workspace."""
        o = torch.empty_like(T["q"])
        l = torch.empty((c.Hq, c.total_q), dtype=torch.float32, device=dev)
        w = torch.empty(max(1, sfa.fwd_workspace_size(c.batch, c.max_sq, c.max_sk, c.total_q, c.Hq, c.Hkv, c.d,
                                                      c.topk, c.bs)), dtype=torch.uint8, device=dev)

        def run():
            sfa.fwd(T["q"], T["k"], T["v"], T["cu_q"], T["sel"], c.bs, cu_seqlens_k=T["cu_k"], max_seqlen_q=c.max_sq,
                    max_seqlen_k=c.max_sk, causal=bool(c.causal), window=(c.wl, c.wr), out=o, lse=l, workspace=w,
                    status=status)
            launches[0] += sfa.last_launch_count()
        run.out, run.lse, run.ws = o, l, w
        return run

    prefill = prefill_call(pc, P)
    out, lse, ws = prefill.out, prefill.lse, prefill.ws
    prefill()
    prefill_launches = sfa.last_launch_count()

    def decode_call():
        sfa.decode(D["q"], D["k_cache"], D["v_cache"], D["block_table"], D["cache_seqlens"], D["sel"], out=dout,
                   lse=dlse, workspace=dws, status=status)
        launches[0] += sfa.last_launch_count()

    # one step: the whole public prefill call on the headline workload, then the whole decode call
    stages = [prefill, decode_call]
    if args.part == "prefill":
        stages = [prefill, lambda: None]
    K, Wm = args.steps, args.warmup
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(K)]

    def step(i=None):
        flush.fill_((i or 0) & 0xFF)
        if i is not None:
            ev[i][0].record(stream)
        for s, fn in enumerate(stages):
            fn()
            if i is not None:
                ev[i][s + 1].record(stream)

    # clocks: the sampler starts before the warm-up and has its first sample before the timed region
    import tempfile
    sampler = ClockSampler(physical_gpu_index(local_rank), os.path.join(tempfile.gettempdir(),
                                                                        f"sfa_bench_clocks_{os.getpid()}.csv")) \
        if rank == 0 else None
    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")
    launches[0] = 0
    if sampler:
        sampler.wait_first()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(K):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    n_launch = launches[0]

    stage_ms = np.array([[ev[i][s].elapsed_time(ev[i][s + 1]) for s in range(len(stages))] for i in range(K)])
    region_ms = t_start.elapsed_time(t_end)
    mean = stage_ms.mean(axis=0)
    region_ms, prefill_ms, decode_ms = max_over_ranks([region_ms, *mean.tolist()], world, dev)
    step_ms = prefill_ms + decode_ms
    value = job_rate(world, flops, prefill_ms) / 1e12
    attend_tflops = job_rate(1, flops, prefill_ms) / 1e12
    dec_gbs = job_rate(world, gbytes, decode_ms) / 1e9
    dec_attend_gbs = dec_gbs / world
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")

    # ---- the NSA branches beside the selected attention (not part of the step): the sliding-window
    # branch (window 512 as in the NSA module example, causal) and the three-branch gated mix, on the
    # prefill workload's tensors; L2 flushed before every repetition, CUDA events on the stream.
    extras = None
    want = (lambda name: True) if args.extras is None else (lambda name: name in args.extras.split(","))
    if not args.no_extras and (args.part != "decode-small" or args.extras is not None):
        def timed(fn, reps=10):
            for _ in range(3):
                fn()
            ts = []
            for _ in range(reps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            return float(np.mean(ts))

        # ---- the other prefill configurations, each its whole public call (parity cases beside the step)
        cfg_lines = {}
        for n in sorted(PREFILL_CONFIGS):
            if n == args.prefill_config or not want("prefill_configs"):
                continue
            xc = PREFILL_CONFIGS[n]()
            xT = W.upload_prefill(xc, dev)
            xrun = prefill_call(xc, xT)
            xrun()
            xl = sfa.last_launch_count()
            xf = prefill_flops(xc)
            x_ms = max_over_ranks([timed(xrun, reps=20)], world, dev)[0]
            tfl = xf / (x_ms * 1e-3) / 1e12
            cfg_lines[str(n)] = {"workload": PREFILL_NAMES[n], "ms": round(x_ms, 4),
                                 "effective_gflop": round(xf / 1e9, 3), "effective_tflops": round(tfl, 2),
                                 "frac": round(tfl / tf_burst, 4), "launches": xl,
                                 "peak_source": f"{peak_kind} bf16 burst"}
            del xT, xrun
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the prefill configuration runs")
        # the NSA branches and the backward run on the varlen NSA workload (configuration 2)
        bc = pc if args.prefill_config == 2 else W.config2()
        BP = P if args.prefill_config == 2 else W.upload_prefill(bc, dev)
        brun = prefill_call(bc, BP)
        brun()
        b_out, b_lse = brun.out, brun.lse
        b_flops = prefill_flops(bc)
        wl = 512
        seq = np.diff(bc.cu_q).tolist()
        wpairs = sum(int(np.minimum(np.arange(L) + 1, wl + 1).sum()) for L in seq)
        wflops = 4.0 * bc.d * bc.Hq * wpairs
        wws = torch.empty(256, dtype=torch.uint8, device=dev)
        wout = torch.empty_like(b_out)
        wlse = torch.empty_like(b_lse)
        gates = [torch.rand((bc.total_q, bc.Hq), dtype=torch.float32, device=dev) for _ in range(3)]
        mix = torch.empty_like(b_out)

        def run_window():
            sfa.window_fwd(BP["q"], BP["k"], BP["v"], BP["cu_q"], cu_seqlens_k=BP["cu_k"], max_seqlen_q=bc.max_sq,
                           max_seqlen_k=bc.max_sk, causal=True, window=(wl, 0), out=wout, lse=wlse, workspace=wws,
                           status=status)

        def run_mix():
            sfa.gated_combine([(b_out, gates[0]), (wout, gates[1]), (BP["q"], gates[2])], out=mix)

        # Backward of the selected attention on the same workload (d 128, bs 64): dq, dk, dv from the
        # forward's out / lse and a seeded dout; 2.5x the forward's effective flops (five products
        # of the kept pairs instead of two).
        bwd_line = None
        if bc.d == 128 and bc.bs == 64 and want("backward"):
            g_out = torch.randn(b_out.shape, generator=torch.Generator(device=dev).manual_seed(5), device=dev,
                                dtype=torch.float32).to(torch.bfloat16)
            bdq, bdk, bdv = torch.empty_like(BP["q"]), torch.empty_like(BP["k"]), torch.empty_like(BP["v"])
            bws = torch.empty(sfa.bwd_workspace_size(bc.batch, bc.max_sq, bc.max_sk, bc.total_q, bc.Hq, bc.Hkv, bc.d,
                                                     bc.topk, bc.bs), dtype=torch.uint8, device=dev)

            def run_bwd():
                sfa.bwd(BP["q"], BP["k"], BP["v"], b_out, g_out, b_lse, BP["cu_q"], BP["sel"], bc.bs, cu_seqlens_k=BP["cu_k"],
                        max_seqlen_q=bc.max_sq, max_seqlen_k=bc.max_sk, causal=bool(bc.causal),
                        window=(bc.wl, bc.wr), dq=bdq, dk=bdk, dv=bdv, workspace=bws, status=status)

            b_ms = max_over_ranks([timed(run_bwd)], world, dev)[0]
            bflops = 2.5 * b_flops
            bwd_line = {"workload": PREFILL_NAMES[2] + "; seeded dout; dq, dk, dv", "ms": round(b_ms, 4),
                        "effective_tflops": round(bflops / (b_ms * 1e-3) / 1e12, 2),
                        "frac": round(bflops / (b_ms * 1e-3) / 1e12 / tf_burst, 4),
                        "peak_source": f"{peak_kind} bf16 burst", "launches": 7,
                        "flops_note": "2.5x the forward's effective flops (S, dP, dQ, dK, dV over the kept pairs)"}
        # In-place KV-cache append on the decode workload's cache: one new token per sequence written at
        # position L - 1 (the decode query's own position); bytes = the new rows read + written.
        append_line = index_line = fp8_line = nsa_line = None
        if want("kv_append"):
            akn = torch.randn((dc.B, 1, dc.Hkv, dc.d), device=dev).to(torch.bfloat16)
            akv = torch.randn((dc.B, 1, dc.Hkv, dc.d), device=dev).to(torch.bfloat16)
            apos = (D["cache_seqlens"] - 1).to(torch.int32)

            def run_append():
                sfa.kv_append(akn, akv, D["k_cache"], D["v_cache"], D["block_table"], apos, status=status)

            a_ms = max_over_ranks([timed(run_append)], world, dev)[0]
            a_bytes = 2 * 2 * dc.B * dc.Hkv * dc.d * 2
            append_line = {"workload": f"B {dc.B}, 1 new token, Hkv {dc.Hkv}, d {dc.d}, page {dc.page}",
                           "us": round(a_ms * 1e3, 2), "gbs": round(a_bytes / (a_ms * 1e-3) / 1e9, 1), "launches": 1,
                           "note": "launch-latency bound (256 KB moved)"}
        # Decode index producer (exact FP8 scores over every cached key, top-k positions) on the decode
        # workload: topk = its selection size, the last 128 positions forced as in its recipe.  Bytes = the
        # K rows it scans.  Guarded so a failure here only marks this line.
        if want("index_topk"):
            try:
                itopk = int(dc.sel.shape[2])
                isel = torch.empty((dc.B, dc.Hkv, itopk), dtype=torch.int32, device=dev)
                istatus = torch.zeros(1, dtype=torch.int32, device=dev)
                iws = torch.empty(sfa.index_topk_workspace_size(dc.B, dc.Hkv, D["block_table"].shape[1], dc.page)
                                  if hasattr(sfa, "index_topk_workspace_size") else 1, dtype=torch.uint8, device=dev)

                def run_index():
                    sfa.index_topk(D["q"], D["k_cache"], D["block_table"], D["cache_seqlens"], itopk, n_local=128,
                                   out=isel, workspace=iws, status=istatus)

                i_ms = max_over_ranks([timed(run_index)], world, dev)[0]
                i_bytes = int(np.asarray(dc.cache_seqlens, np.int64).sum()) * dc.Hkv * dc.d * 2
                index_line = {"workload": f"decode workload, topk {itopk} (last 128 forced), every cached key scored",
                              "ms": round(i_ms, 4), "gbs": round(i_bytes / (i_ms * 1e-3) / 1e9, 1),
                              "frac": round(i_bytes / (i_ms * 1e-3) / 1e9 / hbm, 4), "peak_source": peak_kind,
                              "launches": 2, "status": int(istatus.item())}
            except Exception as exc:  # noqa: BLE001 - reported in the line, the rest of the bench goes on
                index_line = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        # FP8 E4M3 caches (the decode workload quantized per (sequence, kv head) on the device): the same
        # gathered rows at one byte per value.
        if want("decode_fp8"):
            try:
                fk, fv, fkd, fvd = W.quantize_cache_e4m3_device(dc, D)
                f_out = torch.empty_like(dout)
                f_lse = torch.empty_like(dlse)

                def run_fp8():
                    sfa.decode_fp8(D["q"], fk, fv, D["block_table"], D["cache_seqlens"], D["sel"], k_descale=fkd,
                                   v_descale=fvd, out=f_out, lse=f_lse, workspace=dws, status=status)

                f_ms = max_over_ranks([timed(run_fp8, reps=20)], world, dev)[0]
                f_bytes = gbytes // 2
                fp8_line = {"workload": DECODE_PART_NAMES[args.part] + ", caches E4M3 + per (sequence, kv head) descales",
                            "ms": round(f_ms, 4), "gathered_bytes": int(f_bytes),
                            "gbs": round(f_bytes / (f_ms * 1e-3) / 1e9, 1),
                            "frac": round(f_bytes / (f_ms * 1e-3) / 1e9 / hbm, 4), "peak_source": peak_kind,
                            "speedup_vs_bf16_cache": round(decode_ms / f_ms, 3), "launches": 1}
                del fk, fv
            except Exception as exc:  # noqa: BLE001 - reported in the line, the rest of the bench goes on
                fp8_line = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        if want("nsa_branches"):
            w_ms = max_over_ranks([timed(run_window)], world, dev)[0]
            m_ms = max_over_ranks([timed(run_mix)], world, dev)[0]
            mix_bytes = 4 * bc.total_q * bc.Hq * bc.d * 2 + 3 * bc.total_q * bc.Hq * 4
            nsa_line = {
                "window_branch": {"workload": "the prefill workload's q/k/v, causal, window (512, 0), no selection",
                                  "ms": round(w_ms, 4), "effective_tflops": round(wflops / (w_ms * 1e-3) / 1e12, 2),
                                  "frac": round(wflops / (w_ms * 1e-3) / 1e12 / tf_burst, 4),
                                  "peak_source": f"{peak_kind} bf16 burst", "launches": 1},
                "gated_combine": {"workload": "3 branches of (total_q, Hq, d) bf16 + fp32 gates -> bf16",
                                  "ms": round(m_ms, 4), "gbs": round(mix_bytes / (m_ms * 1e-3) / 1e9, 1),
                                  "frac": round(mix_bytes / (m_ms * 1e-3) / 1e9 / hbm, 4), "peak_source": peak_kind},
            }
        extras = {"nsa_branches": nsa_line, "backward": bwd_line, "kv_append": append_line,
                  "index_topk": index_line, "prefill_configs": cfg_lines, "decode_fp8": fp8_line}
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the NSA branch runs")

    # ---- end to end through the public API with host buffers (pinned), copies inside the timing
    e2e = None
    if not args.no_e2e:
        import torch as T
        hp = {k: T.from_numpy(np.ascontiguousarray(getattr(pc, k))).pin_memory() for k in ("q", "k", "v", "sel")}
        hcu = T.from_numpy(pc.cu_q).pin_memory()
        dq = {k: T.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in
              (("q", dc.q), ("bt", dc.block_table), ("lens", dc.cache_seqlens), ("sel", dc.sel))}
        h_out = T.empty(out.shape, dtype=T.bfloat16).pin_memory()
        h_lse = T.empty(lse.shape, dtype=T.float32).pin_memory()
        h_dout = T.empty(dout.shape, dtype=T.bfloat16).pin_memory()
        h_dlse = T.empty(dlse.shape, dtype=T.float32).pin_memory()
        dq_dev = {k: T.empty(v.shape, dtype=v.dtype, device=dev) for k, v in dq.items()}
        h2d = sum(t.numel() * t.element_size() for t in list(hp.values()) + [hcu] + [hcu])
        d2h = h_out.numel() * 2 + h_lse.numel() * 4
        dh2d = sum(t.numel() * t.element_size() for t in dq.values())
        dd2h = h_dout.numel() * 2 + h_dlse.numel() * 4
        Ke = max(4, min(K, 20))
        # Two device buffer sets, so step i+1's inputs go in (copy stream) while step i computes
        # (compute stream) and step i-1's results come out (copy-back stream): a serving loop's overlap.
        # Every step still copies its own inputs in and its results back inside the timed region.
        pin = [{"q": P["q"], "k": P["k"], "v": P["v"], "sel": P["sel"], "cu_q": P["cu_q"], "cu_k": P["cu_k"]},
               {"q": T.empty_like(P["q"]), "k": T.empty_like(P["k"]), "v": T.empty_like(P["v"]),
                "sel": T.empty_like(P["sel"]), "cu_q": T.empty_like(P["cu_q"]), "cu_k": T.empty_like(P["cu_k"])}]
        pout = [(out, lse), (T.empty_like(out), T.empty_like(lse))]
        din = [dq_dev, {k: T.empty_like(v) for k, v in dq_dev.items()}]
        dout2 = [(dout, dlse), (T.empty_like(dout), T.empty_like(dlse))]

        def pre_h2d(b):
            d = pin[b]
            d["q"].view(T.uint16).copy_(hp["q"], non_blocking=True)
            d["k"].view(T.uint16).copy_(hp["k"], non_blocking=True)
            d["v"].view(T.uint16).copy_(hp["v"], non_blocking=True)
            d["sel"].copy_(hp["sel"], non_blocking=True)
            d["cu_q"].copy_(hcu, non_blocking=True)
            d["cu_k"].copy_(hcu, non_blocking=True)

        def pre_compute(b):
            d = pin[b]
            sfa.fwd(d["q"], d["k"], d["v"], d["cu_q"], d["sel"], pc.bs, cu_seqlens_k=d["cu_k"], max_seqlen_q=pc.max_sq,
                    max_seqlen_k=pc.max_sk, out=pout[b][0], lse=pout[b][1], workspace=ws, status=status)

        def pre_d2h(b):
            h_out.view(T.uint16).copy_(pout[b][0].view(T.uint16), non_blocking=True)
            h_lse.copy_(pout[b][1], non_blocking=True)

        def dec_h2d(b):
            for k2 in dq:
                din[b][k2].copy_(dq[k2], non_blocking=True)

        def dec_compute(b):
            d = din[b]
            sfa.decode(d["q"].view(T.bfloat16), D["k_cache"], D["v_cache"], d["bt"], d["lens"], d["sel"],
                       out=dout2[b][0], lse=dout2[b][1], workspace=dws, status=status)

        def dec_d2h(b):
            h_dout.view(T.uint16).copy_(dout2[b][0].view(T.uint16), non_blocking=True)
            h_dlse.copy_(dout2[b][1], non_blocking=True)

        s_in, s_cmp, s_out = T.cuda.Stream(dev), T.cuda.Stream(dev), T.cuda.Stream(dev)

        def pipelined_ms(h2d_fn, compute_fn, d2h_fn, steps):
            ev_in = [T.cuda.Event() for _ in range(2)]
            ev_cmp = [T.cuda.Event() for _ in range(2)]
            ev_out = [T.cuda.Event() for _ in range(2)]
            t0, t1 = T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)
            T.cuda.synchronize()
            t0.record(s_in)
            for i in range(steps):
                b = i & 1
                with T.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_cmp[b])  # step i-2 has finished reading this input set
                    h2d_fn(b)
                    ev_in[b].record(s_in)
                with T.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[b])
                    if i >= 2:
                        s_cmp.wait_event(ev_out[b])  # step i-2's results have been copied out
                    compute_fn(b)
                    ev_cmp[b].record(s_cmp)
                with T.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[b])
                    d2h_fn(b)
                    ev_out[b].record(s_out)
            t1.record(s_out)
            T.cuda.synchronize()
            return t0.elapsed_time(t1) / steps

        pipelined_ms(pre_h2d, pre_compute, pre_d2h, 3)  # warm-up
        pipelined_ms(dec_h2d, dec_compute, dec_d2h, 3)
        if world > 1:
            dist.barrier()
        e_pre = pipelined_ms(pre_h2d, pre_compute, pre_d2h, Ke)
        e_dec = pipelined_ms(dec_h2d, dec_compute, dec_d2h, Ke)
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the end-to-end run")
        e_pre, e_dec = max_over_ranks([e_pre, e_dec], world, dev)
        e2e = {"value": round(job_rate(world, flops, e_pre) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d + dh2d), "d2h_bytes_per_step": int(d2h + dd2h),
               "decode": {"value": round(job_rate(world, gbytes, e_dec) / 1e9, 1), "unit": "GB/s"},
               "note": "pinned host inputs copied in and outputs (out, lse) copied back every step, with the "
                       "copies of neighbouring steps overlapping the compute on separate streams (two device "
                       "buffer sets); the decode KV cache is resident state, its per-step inputs are q, "
                       "block_table, cache_seqlens, sel_tok_idx"}
    return dict(value=value, prefill_launches=prefill_launches, prefill_ms=prefill_ms, decode_ms=decode_ms,
                step_ms=step_ms, region_ms=region_ms, attend_tflops=attend_tflops,
                dec_gbs=dec_gbs, dec_attend_gbs=dec_attend_gbs, flops=flops, gbytes=gbytes, clocks=clocks,
                launches=n_launch, e2e=e2e, extras=extras, hbm=hbm, tf_burst=tf_burst, tf_sust=tf_sust,
                peak_kind=peak_kind,
                pc=pc, dc=dc,
                traffic=args.traffic if args.traffic is not None else kernel_traffic(f"prefill_c{args.prefill_config}"),
                dec_traffic=kernel_traffic("decode_split_kernel"))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sfa", choices=["sfa", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the lines beside the step: NSA window branch, gated mix, backward, KV append, "
                         "index top-k")
    ap.add_argument("--extras", default=None,
                    help="profiling aid: comma list of the lines beside the step to run (prefill_configs, "
                         "nsa_branches, backward, kv_append, index_topk, decode_fp8); default all")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--part", default="all", choices=["all", "prefill", "decode-small"],
                    help="'prefill' times only the prefill stages (a small decode case stands in); for profiling")
    ap.add_argument("--prefill-config", type=int, default=4, choices=[1, 2, 3, 4],
                    help="headline prefill workload (default 4, the largest single-GPU configuration); the "
                         "others are timed beside it")
    ap.add_argument("--shrink", type=int, default=1,
                    help="profiling aid: divide the headline NSA prefill workload's lengths by this (configs 2 "
                         "and 4); the line then names the smaller workload")
    ap.add_argument("--traffic", type=int, default=None,
                    help="dram bytes (read+write) per attend launch from an ncu capture of this kernel version")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.shrink < 1 or (args.shrink > 1 and args.prefill_config not in (2, 4)):
        ap.error("--shrink takes a positive factor and applies to prefill configs 2 and 4")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, rank, world)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_gpu(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    pc = r["pc"]
    line = {
        "metric": METRIC,
        "value": round(r["value"], 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["step_ms"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, seeded NSA block selection; seeded paged decode inputs)",
        "config": {"workload": (PREFILL_NAMES[args.prefill_config] + (f", lengths / {args.shrink}" if args.shrink > 1
                                                                       else "")) if args.part != "decode-small"
                   else "small",
                   "decode_workload": DECODE_PART_NAMES[args.part], "parallelism": f"independent x{world}",
                   "l2": "flushed by a 256 MiB write before every step (outside the kernel events)",
                   "timing": "CUDA events per stage on the launch stream, mean over steps, max over ranks"},
        "prefill": {"ms": round(r["prefill_ms"], 4), "effective_gflop": round(r["flops"] / 1e9, 2),
                    "launches": r["prefill_launches"]},
        "decode": {"value": round(r["dec_gbs"], 1), "unit": "GB/s", "ms": round(r["decode_ms"], 4),
                   "gathered_bytes": int(r["gbytes"]),
                   "roofline": {"bound": "hbm", "achieved": round(r["dec_attend_gbs"], 1), "peak": r["hbm"],
                                "unit": "GB/s", "frac": round(r["dec_attend_gbs"] / r["hbm"], 4),
                                "traffic": r["dec_traffic"], "traffic_unit": "B per decode_split_kernel launch",
                                "kernel": "sfa_decode whole call = one decode_split_kernel launch (splits merged "
                                          "in the CTA)",
                                "peak_source": r["peak_kind"]}},
        "roofline": {"bound": "tensor", "achieved": round(r["attend_tflops"], 2), "peak": r["tf_burst"],
                     "unit": "TFLOP/s", "frac": round(r["attend_tflops"] / r["tf_burst"], 4),
                     "traffic": r["traffic"], "traffic_unit": "B (dram read + write) per sfa_fwd call",
                     "kernel": f"sfa_fwd whole call ({r['prefill_launches']} kernel launches; achieved = the "
                               f"call's effective flops / the call's duration)",
                     "peak_source": f"{r['peak_kind']} bf16 burst",
                     "frac_of_sustained": round(r["attend_tflops"] / r["tf_sust"], 4) if r["tf_sust"] else None},
        "gpu_launches": r["launches"],
        "region_ms": round(r["region_ms"], 3),
    }
    if r["clocks"]:
        line["clocks"] = r["clocks"]
    if r["e2e"]:
        line["e2e"] = r["e2e"]
    if r["extras"]:
        for key, val in r["extras"].items():  # nsa_branches, backward, kv_append: beside the timed step
            if val is not None:
                line[key] = val
    if world == 1 and not args.no_cpu_baseline:
        v, n, thr, secs = cpu_oracle_rate(pc, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": f"{n} random (token, head) rows of the prefill workload, {secs:.1f} s"}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main_reference(args, rank, world):
    """The CPU oracle, as it stands, on a bounded sample of the prefill workload per step."""
    if rank != 0:
        return
    pc = PREFILL_CONFIGS[args.prefill_config]()
    import oracle
    oracle.build()
    steps, warm = args.steps, args.warmup
    budget = 150.0  # seconds of CPU for the whole run
    per = min(10.0, max(0.2, budget / (steps + warm)))
    rates, total_t, rows_tot = [], 0.0, 0
    for i in range(warm + steps):
        v, n, thr, t = cpu_oracle_rate(pc, per, seed=i)
        if i >= warm:
            rates.append(v)
            total_t += t
            rows_tot += n
    value = float(np.mean(rates))
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": round(1e3 * total_t / steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL_NAMES[args.prefill_config], "decode_workload": DECODE_NAME},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                             "sample": f"{rows_tot} random (token, head) rows over {steps} steps"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
