#!/usr/bin/env python
"""Benchmark: FlashBlock cached vs uncached block-diffusion attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One timed *step* is one block of denoising steps of one attention layer, the
cached FlashBlock way: the prefix partial at the refresh step(s), the
in-block partial fused with the merge on every denoising step, and the block's
append to the KV cache.  The uncached baseline (full attention over
[prefix ; block] on every denoising step, plus the same append) is timed the
same way right after.  Inputs are resident in HBM before the timed region;
the KV cache (537 MB at 128K context) is larger than the 126 MB L2, so no
flush is needed between steps.  The append writes the block's rows after the
prefix without advancing the prefix length, so every timed block sees exactly
the configured prefix.

By default each block is recorded once as a CUDA graph and replayed (the
library's calls are capturable); ``--no-graph`` issues every call from the
host.  The eager cached block is always timed too.  CUDA events around the
prefix pass inside the timed blocks give the roofline figures of the dominant
kernel; the line also gives the pass timed 16 times back to back in a graph
(no event nodes next to it) and, where the KV cache fits in L2, after an L2
flush.

``value`` is cached attention tokens/s over all ranks (B * S tokens finalized
per block per rank).  Under torchrun each rank runs an independent replica
(weak scaling; the path has no collective).  Rank 0 prints one JSON line.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only) and prints the same kind of line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention µs/denoise-step and tokens/s, cached vs uncached; prefix-pass HBM GB/s"

# DRAM bytes read + written by one launch of the prefix-pass attention kernel,
# from one `ncu --clock-control none` capture of that launch on the workload
# (dram__bytes_read.sum + dram__bytes_write.sum), with the hash of the
# kernel sources it was captured on (see kernel_source_hash).  An entry whose
# hash differs from the built sources is not reported: the kernel changed
# since the counters were taken.
NCU_TRAFFIC = {
    # profiles/prefix_pass_long_ctx.md, capture b53_traffic_lc
    "long_ctx": {"bytes": 537209088 + 2964736, "sources": "8db3988978716104"},
}
KERNEL_SOURCES = ("fb_attn_tc.cu", "fb_attn_common.cuh", "fb_ptx.cuh", "fb_internal.h", "fb_api.cu")


def kernel_source_hash():
    """sha256 (first 16 hex digits) over the sources that decide the prefix
    pass's kernel code and launch plan."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "block_diffusion_attention_b200", "csrc", name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """Captured DRAM bytes per prefix-pass launch, or None when there is no
    capture of the current kernel sources."""
    e = NCU_TRAFFIC.get(workload)
    if e is None or e["sources"] != kernel_source_hash():
        return None
    return e["bytes"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_ctx")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--residual", action="store_true",
                    help="sparse workloads: residual reuse (cache the unselected chunks, recompute the selected ones)")
    ap.add_argument("--no-graph", action="store_true",
                    help="issue every call from the host instead of replaying one CUDA graph per block")
    ap.add_argument("--policy", choices=["headwise", "threshold"], default=None,
                    help="adaptive reuse: decide per step which units refresh (dense workloads)")
    ap.add_argument("--gamma", type=float, default=0.9, help="head-wise policy: similarity threshold")
    ap.add_argument("--tau", type=int, default=None, help="threshold policy: updated-token count (default S/4)")
    ap.add_argument("--eps", type=float, default=0.25, help="threshold policy: change that marks a token updated")
    ap.add_argument("--phases", default="cached,uncached,e2e",
                    help="comma list of timed phases (profiling runs may keep only 'cached')")
    return ap.parse_args()


L2_BYTES = 126e6  # B200 L2


def kv_cache_bytes(w):
    """Bytes of the workload's valid prefix K and V."""
    return 2 * w.batch * w.prefix_len * w.num_kv_heads * w.head_dim * (2 if w.dtype == "bf16" else 4)


def workload_config(w, extra=None):
    cfg = {
        "workload": (f"{w.name}: B{w.batch} Hq{w.num_q_heads}/Hkv{w.num_kv_heads} D{w.head_dim} "
                     f"block {w.block_len} prefix {w.prefix_len}"
                     + (f" (varlen from {w.prefix_min})" if w.prefix_min else "")
                     + f", {w.steps} denoising steps per block, refresh at {list(w.refresh)}"
                     + (f", top-{w.topk} of {w.chunk_size}-token chunks" if w.topk else "")),
        "global_batch": w.batch,
        "seq_len": w.prefix_len,
        "block_len": w.block_len,
        "denoise_steps": w.steps,
        "parallelism": "replicas",
        "l2": "KV cache larger than the 126 MB L2 at this workload; no flush" if kv_cache_bytes(w) > L2_BYTES else
              "KV cache fits in L2: the replayed blocks and prefix_gbs are L2-warm; prefix_pass_l2_cold_us times "
              "the pass after a 256 MB scratch read (L2 left holding clean lines), prefix_pass_l2_cold_dirty_us "
              "after a 256 MB scratch write (dirty lines written back during the pass)",
    }
    if extra:
        cfg.update(extra)
    return cfg


def prefix_bytes(w, lens, residual=False):
    """Algorithmic bytes of one prefix pass: K+V of the valid (or selected,
    or -- residual mode -- unselected) prefix rows, Q, and the written O_pre
    (f32) and LSE_pre (f32)."""
    if w.topk and residual:
        eff = sum(int(L) - min(int(L), w.topk * w.chunk_size) for L in lens)
    elif w.topk:
        eff = sum(min(int(L), w.topk * w.chunk_size) for L in lens)
    else:
        eff = sum(int(L) for L in lens)
    kv = 2 * eff * w.num_kv_heads * w.head_dim * 2
    rows = w.batch * w.block_len * w.num_q_heads
    return kv + rows * w.head_dim * 2 + rows * w.head_dim * 4 + rows * 4


def prefix_flops(w, lens, residual=False):
    if w.topk and residual:
        eff = sum(int(L) - min(int(L), w.topk * w.chunk_size) for L in lens)
    else:
        eff = sum(min(int(L), w.topk * w.chunk_size) if w.topk else int(L) for L in lens)
    return 4.0 * w.num_q_heads * w.block_len * eff * w.head_dim


def prefix_kernel_name(w):
    """The kernel that runs the workload's prefix pass, as the library picks
    it: fp32 on the CUDA cores; bf16 on the tensor cores with two 128-row
    query tiles per CTA where a (b, kv head) unit has at least two
    (S x G packed rows), else one."""
    if w.dtype != "bf16":
        return "prefix pass: attn_simt_kernel (fp32, CUDA cores)"
    tiles = -(-(w.block_len * w.group) // 128)
    kern = "attn_tc2_kernel<EPI_PARTIAL>" if tiles >= 2 else "attn_tc_kernel<EPI_PARTIAL>"
    return f"prefix pass: {kern} (+ combine_kernel when the keys are split)"


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return (j.get("hbm_gbs", 6650.0), j.get("bf16_tflops", 1590.0),
                j.get("bf16_tflops_sustained", 1400.0), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, read through NVML every
    10 ms on a background thread (read-only queries)."""

    # NVML clocks-event-reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.samples = []
        self._stop = None
        self._thread = None

    def _handle(self, pynvml):
        # map the CUDA device to its NVML handle through the PCI bus id
        import torch
        props = torch.cuda.get_device_properties(self.cuda_index)
        bus = getattr(props, "pci_bus_id", None)
        dom = getattr(props, "pci_domain_id", 0)
        dev = getattr(props, "pci_device_id", None)
        if bus is not None and dev is not None:
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0".encode())
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.error = str(e)
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((sm, rs))
                except Exception:
                    pass
                self._stop.wait(0.01)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        sm = [x[0] for x in self.samples]
        reasons = sorted({name for _, rs in self.samples for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": "NVML every 10 ms, first warm-up block to the last timed phase"}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------
# Oracle timing (CPU baseline and the reference arm)
# --------------------------------------------------------------------------

def oracle_block_sample(w, K, V, lens, heads=1):
    """Time the oracle's cached block on the first `heads` kv heads of the
    workload (one block: refresh + every denoising step's in-block partial and
    merge).  Returns the measured seconds of that sample; the sample does
    heads / Hkv of the block's attention work (the kv heads are independent
    and equal in size)."""
    import numpy as np
    from block_diffusion_attention_b200 import synth
    from oracle import flashblock_oracle as ora
    G = w.group
    hs = slice(0, heads)
    qs = slice(0, heads * G)
    Kc = synth.as_dtype(w, K[:, :, hs])[1]
    Vc = synth.as_dtype(w, V[:, :, hs])[1]
    base = synth.block_base(w, 0)
    steps = []
    for s in range(w.steps):
        Q, Kb, Vb = synth.step_inputs(w, 0, s, base)
        steps.append((synth.as_dtype(w, Q[:, :, qs])[1], synth.as_dtype(w, Kb[:, :, hs])[1],
                      synth.as_dtype(w, Vb[:, :, hs])[1]))
    lens64 = np.asarray(lens, dtype=np.int64)
    chunk_fn = None
    if w.topk:
        Km, valid = ora.chunk_means(Kc, lens64, w.chunk_size)
        chunk_fn = lambda Q: ora.select_chunks(Q, Km, valid, w.topk)  # noqa: E731
    t0 = time.perf_counter()
    ora.cached_block([x[0] for x in steps], [x[1] for x in steps], [x[2] for x in steps], Kc, Vc, lens64,
                     w.softmax_scale, w.refresh, chunk_fn, w.chunk_size)
    return time.perf_counter() - t0


def oracle_sample_record(w, seconds, heads=1, reps=1):
    """The oracle's measured sample as a rate: one sample finalizes
    heads / Hkv of the attention of the block's B * S tokens, so its
    throughput is B * S * heads / Hkv tokens over the measured seconds per
    sample (`seconds`, the mean of `reps` samples; no time is extrapolated)."""
    frac = heads / w.num_kv_heads
    return {"value": w.batch * w.block_len * frac / seconds, "unit": "tokens/s",
            "sample": f"the oracle's cached block (refresh + {w.steps} denoising steps) on {heads} of "
                      f"{w.num_kv_heads} kv heads, i.e. {frac:g} of the block's attention work"
                      + (f", timed {reps} times" if reps > 1 else "")
                      + "; the rate is that work over its measured time",
            "sample_seconds_measured": seconds, "sample_fraction_of_block": frac, "sample_repeats": reps}


def sample_heads(w, K, V, lens, target_s):
    """kv heads per oracle sample so that one sample takes about target_s
    (at least one head, at most all): a one-head sample is timed first.
    Returns (heads, seconds of the one-head sample)."""
    t1 = oracle_block_sample(w, K, V, lens, heads=1)
    return max(1, min(w.num_kv_heads, int(target_s / max(t1, 1e-9)))), t1


def run_reference(args):
    from block_diffusion_attention_b200 import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    K, V, lens = synth.prefix_kv(w)
    # each step one sample of about min(5 s, 120 s / (steps + warmup)) of
    # oracle work, so that the whole run stays within a few minutes
    heads, _ = sample_heads(w, K, V, lens, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    times = []
    for i in range(args.warmup + args.steps):
        t = oracle_block_sample(w, K, V, lens, heads=heads)
        if i >= args.warmup:
            times.append(t)
    per_step = sum(times) / len(times)  # measured seconds of one sample step
    rec = oracle_sample_record(w, per_step, heads=heads, reps=len(times))
    tok_s = rec["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "step": "one bounded sample of the workload's block (see cpu_baseline.sample); ms_per_step is its "
                "measured time",
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": rec["sample"], "sample_seconds_measured": per_step,
                         "sample_fraction_of_block": rec["sample_fraction_of_block"],
                         "sample_repeats": rec["sample_repeats"]},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    from block_diffusion_attention_b200 import flashblock as fbl
    from block_diffusion_attention_b200 import synth
    from block_diffusion_attention_b200.schedule import CachedBlockAttention

    from block_diffusion_attention_b200 import ranks
    rank, world, local = ranks.rank_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    fbl.load()
    phases = set(args.phases.split(","))

    w0 = synth.WORKLOADS[args.workload]
    # the append rows sit after the prefix; the prefix length stays fixed;
    # each rank runs its own replica (its own seeds)
    w = ranks.replica_workload(w0, rank).scaled(blocks=1)
    K, V, lens = synth.prefix_kv(w)
    Kt = synth.as_dtype(w, K)[0].cuda()
    Vt = synth.as_dtype(w, V)[0].cuda()
    del K, V
    base = synth.block_base(w, 0)
    if args.policy is not None and (w.topk or args.residual):
        raise SystemExit("--policy runs on the dense workloads")
    tau = args.tau if args.tau is not None else max(1, w.block_len // 4)
    if args.policy == "headwise":
        raw = synth.headwise_steps(w, 0, w.steps, base=base)
    elif args.policy == "threshold":
        raw = synth.threshold_steps(w, 0, w.steps, base=base)
    else:
        raw = [synth.step_inputs(w, 0, s, base) for s in range(w.steps)]
    step_in = [tuple(synth.as_dtype(w, x)[0] for x in t) for t in raw]
    del raw
    dev_in = [tuple(x.cuda() for x in t) for t in step_in]
    outs = [torch.empty_like(dev_in[0][0]) for _ in range(w.steps)]
    stream = torch.cuda.current_stream()

    def new_layer():
        layer = CachedBlockAttention(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_len, w.capacity,
                                     dtype=w.dtype, softmax_scale=w.softmax_scale,
                                     chunk_size=w.chunk_size if w.topk else 0, topk=w.topk,
                                     residual=args.residual, policy=policy, gamma=args.gamma, tau=tau,
                                     eps=args.eps)
        layer.load_prefix(Kt, Vt, lens)
        return layer

    policy = None

    def barrier():
        ranks.barrier()

    def max_over_ranks(x):
        return ranks.max_over_ranks(x, device="cuda")

    res = {}

    def timed(block_fn, layer):
        """W untimed blocks, then K blocks between CUDA events; max over ranks."""
        for _ in range(args.warmup):
            block_fn(None)
        layer.check()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        n0 = fbl.fb_launch_count()
        t0.record(stream)
        for k in range(args.steps):
            block_fn(k)
        t1.record(stream)
        n1 = fbl.fb_launch_count()
        torch.cuda.synchronize()
        layer.check()
        res.setdefault("launch_counts", []).append(n1 - n0)
        return max_over_ranks(t0.elapsed_time(t1))

    # ---- cached (FlashBlock) path
    policy = args.policy
    cached = new_layer()
    nref = 1 if policy else len(w.refresh)
    use_graph = not args.no_graph

    def issue_block(pre_events=None):
        """One block of calls; pre_events[i] = (select start, prefix start,
        prefix end) around refresh i."""
        pi = 0
        for s in range(w.steps):
            Q, Kb, Vb = dev_in[s]
            if policy:
                # every step decides which units refresh; step 0 refreshes all
                # of them (its mask + masked prefix pass is the timed pair)
                if s == 0 and pre_events is not None:
                    pre_events[0][0].record()
                    pre_events[0][1].record()  # no separate selection step
                    cached.adapt(Q, Kb, Vb, first=True)
                    pre_events[0][2].record()
                else:
                    cached.adapt(Q, Kb, Vb, first=(s == 0))
            elif s in w.refresh:
                # current stream: the capture stream while a graph is recorded
                if pre_events is not None:
                    pre_events[pi][0].record()
                cached.select(Q)
                if pre_events is not None:
                    pre_events[pi][1].record()
                cached.prefix(Q)
                if pre_events is not None:
                    pre_events[pi][2].record()
                pi += 1
            if s == w.steps - 1:
                # the block's last step carries the append (rows written
                # after the prefix, its length kept: a fixed workload)
                cached.step_append(Q, Kb, Vb, out=outs[s], advance=False)
            else:
                cached.step(Q, Kb, Vb, out=outs[s])

    res["lens0"] = [int(x) for x in cached.lens.cpu()]
    # clocks are sampled from the first warm-up block to the end of the last timed phase
    sampler = ClockSampler(local)
    sampler.start()
    # eager host launches (reported beside the graph numbers)
    res["ms_cached_eager"] = timed(lambda k: issue_block(), cached)
    res["launches_per_block"] = res["launch_counts"][0] / args.steps
    if use_graph:
        # the headline: one CUDA graph per block, replayed K times.  The
        # prefix-pass duration comes from a second timed run of the same K
        # blocks, each replaying its own copy of the graph with external event
        # nodes around the pass: an event node between two kernels ends the
        # early start (programmatic dependent launch) of the second one, so
        # those nodes cost a few microseconds per block and stay out of the
        # headline.
        def ev_pair():
            return tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(3))

        def capture(pre_events):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                issue_block(pre_events)
            return g

        torch.cuda.synchronize()
        warm = capture(None)
        ev_pre = [[ev_pair() for _ in range(nref)] for _ in range(args.steps)]
        graphs = [capture(ev_pre[k]) for k in range(args.steps)]

        def replay(k):
            (warm if k is None else graphs[k]).replay()

        res["ms_cached"] = timed(lambda k: warm.replay(), cached)
        res["ms_cached_evented"] = timed(replay, cached)
        res["pre_ms"] = [b.elapsed_time(c) for evs in ev_pre for a, b, c in evs]
        res["sel_ms"] = [a.elapsed_time(b) for evs in ev_pre for a, b, c in evs]
        del graphs, warm
    else:
        ev_pre = [[tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
                   for _ in range(nref)] for _ in range(args.steps)]
        res["ms_cached"] = timed(lambda k: issue_block(None if k is None else ev_pre[k]), cached)
        res["pre_ms"] = [b.elapsed_time(c) for evs in ev_pre for a, b, c in evs]
        res["sel_ms"] = [a.elapsed_time(b) for evs in ev_pre for a, b, c in evs]
    res["launches"] = int(res["launches_per_block"] * args.steps)
    res["lens1"] = [int(x) for x in cached.lens.cpu()]
    if policy:
        # share of the units the policy refreshes after the first step (one
        # eager block after the timed region, the masks read at each step)
        frac = []
        for s, (Q, Kb, Vb) in enumerate(dev_in):
            cached.cached_step(s, Q, Kb, Vb, out=outs[s])
            if s > 0:
                frac.append(float(cached.unit_mask.float().mean()))
        res["refresh_fraction"] = sum(frac) / len(frac) if frac else None
    # block-step latency on its own: 64 back-to-back denoising steps in one graph
    reps = 64
    Q, Kb, Vb = dev_in[1 % w.steps]
    for _ in range(4):
        cached.step(Q, Kb, Vb, out=outs[0])
    torch.cuda.synchronize()
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps):
        for _ in range(reps):
            cached.step(Q, Kb, Vb, out=outs[0])
    g_steps.replay()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g_steps.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    res["blk_ms"] = [e0.elapsed_time(e1) / reps]
    del g_steps
    if not policy:
        # the prefix pass on its own: 16 passes back to back in one graph,
        # CUDA events around the replay (each pass's start overlaps its
        # predecessor's end, as inside a block without event nodes)
        Q0 = dev_in[0][0]
        cached.select(Q0)
        for _ in range(3):
            cached.prefix(Q0)
        torch.cuda.synchronize()
        g_pre = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_pre):
            for _ in range(16):
                cached.prefix(Q0)
        g_pre.replay()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_pre.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        res["pre_b2b_ms"] = e0.elapsed_time(e1) / 16
        del g_pre
    if not policy and kv_cache_bytes(w) < L2_BYTES:
        # The KV cache fits in L2, so the replayed blocks time the prefix pass
        # L2-warm.  Cold figures, the pass timed alone after the cache has
        # been evicted from L2 by (a) a read of a 256 MB scratch buffer: the
        # L2 then holds clean lines, as after other layers' weight reads;
        # (b) a write of it: the L2 then holds 126 MB of dirty lines, whose
        # write-back to HBM runs during the pass and is charged to it.
        flush = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
        total = torch.zeros((), dtype=torch.int64, device="cuda")
        Q0 = dev_in[0][0]
        for key, evict in (("pre_cold_ms", lambda k: torch.sum(flush, 0, dtype=torch.int64, out=total)),
                           ("pre_cold_dirty_ms", lambda k: flush.fill_(k & 0xFF))):
            cold = []
            for k in range(args.warmup + args.steps):
                evict(k)
                a = torch.cuda.Event(enable_timing=True)
                c = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                cached.select(Q0)
                cached.prefix(Q0)
                c.record(stream)
                if k >= args.warmup:
                    cold.append((a, c))
            torch.cuda.synchronize()
            res[key] = [a.elapsed_time(c) for a, c in cold]
        del flush, total
    if not policy:
        # The method's reuse error on these synthetic inputs (outside every
        # timed region): per denoising step, the relative distance of the
        # cached output from the uncached one, both from this library.
        errs = []
        for s_ in range(w.steps):
            Q, Kb, Vb = dev_in[s_]
            if s_ in w.refresh:
                cached.select(Q)
                cached.prefix(Q)
            oc = cached.step(Q, Kb, Vb).float()
            of = cached.full(Q, Kb, Vb).float()
            errs.append(float((oc - of).norm() / of.norm()))
        res["reuse_err"] = errs
    cached.check()
    del cached

    # ---- uncached baseline: full attention at every denoising step
    if "uncached" in phases:
        unc = new_layer()
        if use_graph:
            g_unc = unc.capture_block(dev_in, outs, w.refresh, append_kv=(dev_in[-1][1], dev_in[-1][2]),
                                      cached=False, advance=False)
            res["ms_unc"] = timed(lambda k: g_unc.replay(), unc)
            del g_unc
        else:
            def uncached_block(k):
                unc.run_block(dev_in, outs, w.refresh, (dev_in[-1][1], dev_in[-1][2]), advance=False,
                              cached=False)
            res["ms_unc"] = timed(uncached_block, unc)
        del unc

    # ---- end to end through the public API: every block's inputs copied in
    # from pinned host memory and its outputs read back, inside the timed
    # region.  The copies run on a second stream and overlap the compute:
    # block k computes from device copy k % 2 while copy (k + 1) % 2 receives
    # block k + 1's inputs and gives back block k - 1's outputs (the first
    # block's inputs and the last block's outputs are copied before and after
    # the loop, still inside the timed region).
    if "e2e" in phases:
        e2e_layer = new_layer()
        host_in = torch.cat([x.reshape(-1) for t in step_in for x in t]).pin_memory()
        dev_flat = [torch.empty_like(host_in, device="cuda") for _ in range(2)]

        def views(buf):
            out, off = [], 0
            for t in step_in:
                v = []
                for x in t:
                    v.append(buf[off:off + x.numel()].view(x.shape))
                    off += x.numel()
                out.append(tuple(v))
            return out

        stages = [views(dev_flat[0]), views(dev_flat[1])]
        oshape = (w.steps,) + tuple(dev_in[0][0].shape)
        odt = dev_in[0][0].dtype
        outs_dev = [torch.empty(oshape, dtype=odt, device="cuda") for _ in range(2)]
        host_out = torch.empty(oshape, dtype=odt).pin_memory()
        # one stream per copy direction, so the two DMA directions overlap too
        h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_body(i):
            main = torch.cuda.current_stream()
            for cs in (h2d_stream, d2h_stream):
                cs.wait_stream(main)  # the other copies' last readers are done
            with torch.cuda.stream(h2d_stream):
                dev_flat[1 - i].copy_(host_in, non_blocking=True)
            with torch.cuda.stream(d2h_stream):
                host_out.copy_(outs_dev[1 - i], non_blocking=True)
            e2e_layer.run_block(stages[i], outs_dev[i], w.refresh, append_kv=(stages[i][-1][1], stages[i][-1][2]),
                                advance=False)
            main.wait_stream(h2d_stream)
            main.wait_stream(d2h_stream)

        if use_graph:
            e2e_body(0)
            e2e_body(1)
            torch.cuda.synchronize()
            graphs_e2e = []
            for i in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    e2e_body(i)
                graphs_e2e.append(g)
            run_block = lambda i: graphs_e2e[i].replay()  # noqa: E731
        else:
            run_block = e2e_body

        def e2e_blocks(n):
            dev_flat[0].copy_(host_in, non_blocking=True)
            for k in range(n):
                run_block(k % 2)
            host_out.copy_(outs_dev[(n - 1) % 2], non_blocking=True)

        e2e_blocks(args.warmup)
        torch.cuda.synchronize()
        e2e_layer.check()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        e2e_blocks(args.steps)
        t1.record(stream)
        torch.cuda.synchronize()
        e2e_layer.check()
        res["ms_e2e"] = max_over_ranks(t0.elapsed_time(t1))
        res["h2d"] = host_in.numel() * host_in.element_size()
        res["d2h"] = host_out.numel() * host_out.element_size()

        # each copy direction on its own (after the timed region), so the
        # copy share of the end-to-end figure can be read off the line
        def copy_ms(fn, cs):
            times = []
            for _ in range(5):
                a = torch.cuda.Event(enable_timing=True)
                c = torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(cs):
                    a.record(cs)
                    fn()
                    c.record(cs)
                cs.synchronize()
                times.append(a.elapsed_time(c))
            return statistics.median(times)

        res["h2d_ms"] = copy_ms(lambda: dev_flat[0].copy_(host_in, non_blocking=True), h2d_stream)
        res["d2h_ms"] = copy_ms(lambda: host_out.copy_(outs_dev[0], non_blocking=True), d2h_stream)
        if use_graph:
            del graphs_e2e
        del e2e_layer
    res["graph"] = use_graph

    res["clocks"] = sampler.stop()
    if world > 1:
        dist.barrier()
    if rank == 0:
        report(args, w0, w, world, res)
    if world > 1:
        dist.destroy_process_group()
    return 0


def e2e_bound(res, args):
    """The longest of the three things an end-to-end block overlaps: its
    compute (the device-timed cached block) and each copy direction timed
    alone."""
    parts = {"compute": res["ms_cached"] / args.steps, "host-to-device copies": res["h2d_ms"],
             "device-to-host copies": res["d2h_ms"]}
    return max(parts, key=parts.get)


def report(args, w0, w, world, res):
    policy = args.policy
    tau = args.tau if args.tau is not None else max(1, w.block_len // 4)
    from block_diffusion_attention_b200 import synth
    tokens = world * w.batch * w.block_len * args.steps

    def tps(ms):
        return tokens / (ms / 1e3) if ms and ms == ms else None

    pre_avg = sum(res["pre_ms"]) / len(res["pre_ms"])
    cold_us = (sum(res["pre_cold_ms"]) / len(res["pre_cold_ms"]) * 1e3) if res.get("pre_cold_ms") else None
    cold_dirty_us = ((sum(res["pre_cold_dirty_ms"]) / len(res["pre_cold_dirty_ms"]) * 1e3)
                     if res.get("pre_cold_dirty_ms") else None)
    blk_avg = sum(res["blk_ms"]) / len(res["blk_ms"])
    mid = [(a + b) / 2 for a, b in zip(res["lens0"], res["lens1"])]
    abytes = prefix_bytes(w, mid, args.residual)
    hbm_peak, tc_peak, tc_sustained, peak_kind = measured_peaks()
    achieved = abytes / (pre_avg / 1e3) / 1e9
    pflops = prefix_flops(w, mid, args.residual)
    tflops = pflops / (pre_avg / 1e3) / 1e12
    # the prefix pass is HBM-bound below the ridge point (measured bf16 peak /
    # measured copy bandwidth, ~258 flop/B) and tensor-bound above it
    intensity = pflops / abytes
    ridge = tc_peak * 1e12 / (hbm_peak * 1e9)
    if intensity > ridge:
        # the prefix pass runs inside a multi-millisecond block: sustained peak
        roof = {"bound": "tensor", "achieved": tflops, "peak": tc_sustained, "unit": "TFLOP/s",
                "frac": tflops / tc_sustained, "peak_source": f"{peak_kind} bf16_tflops_sustained",
                "hbm_gbs": achieved}
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "peak_source": f"{peak_kind} hbm_gbs",
                "tensor_tflops": tflops, "tensor_frac": tflops / tc_peak}
    traffic = None if args.residual else recorded_traffic(w.name)
    roof.update({"traffic": traffic,
                 "traffic_over_algorithmic": (traffic / abytes) if traffic else None,
                 "kernel": prefix_kernel_name(w),
                 "algorithmic_bytes_per_launch": abytes, "algorithmic_flops_per_launch": pflops,
                 "intensity_flop_per_byte": intensity})
    ms_c = res["ms_cached"]
    ms_u = res.get("ms_unc")
    line = {
        "metric": METRIC, "value": tps(ms_c), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_c / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) K/V, scaled Q, per-step drift)",
        "config": workload_config(w0, {"prefix_rows_during_timing": [min(res["lens0"]), max(res["lens1"])],
                                       **({"sparse_mode": "residual reuse (refresh caches the unselected "
                                                          "chunks; every step recomputes the selected ones)"}
                                          if args.residual else {}),
                                       **({"policy": ({"name": "headwise", "gamma": args.gamma,
                                                       "inputs": "per-unit query jumps (p = 0.35 per step)"}
                                                      if policy == "headwise" else
                                                      {"name": "threshold", "tau": tau, "eps": args.eps,
                                                       "inputs": "per-sequence token updates, uniform in [0, S/2]"})}
                                          if policy else {})}),
        "cached_us_per_denoise_step": ms_c * 1e3 / (args.steps * w.steps),
        "cached_eager_us_per_denoise_step": res["ms_cached_eager"] * 1e3 / (args.steps * w.steps),
        "cached_with_prefix_events_us_per_denoise_step": (res["ms_cached_evented"] * 1e3 / (args.steps * w.steps)
                                                           if "ms_cached_evented" in res else None),
        "launch_mode": "one CUDA graph per block" if res["graph"] else "eager host launches",
        "uncached_us_per_denoise_step": ms_u * 1e3 / (args.steps * w.steps) if ms_u else None,
        "uncached_tokens_per_s": tps(ms_u),
        "cached_over_uncached_speedup": (ms_u / ms_c) if ms_u else None,
        "prefix_pass_us": pre_avg * 1e3,
        "chunk_select_us": (sum(res["sel_ms"]) / len(res["sel_ms"]) * 1e3) if w.topk else None,
        "block_step_us": blk_avg * 1e3,
        "refresh_fraction": res.get("refresh_fraction"),
        "prefix_gbs": achieved,
        "prefix_pass_back_to_back_us": (res["pre_b2b_ms"] * 1e3) if res.get("pre_b2b_ms") else None,
        "prefix_gbs_back_to_back": (abytes / (res["pre_b2b_ms"] * 1e-3) / 1e9) if res.get("pre_b2b_ms") else None,
        "prefix_pass_l2_cold_us": cold_us,
        "prefix_gbs_l2_cold": (abytes / (cold_us * 1e-6) / 1e9) if cold_us else None,
        "prefix_hbm_frac_l2_cold": (abytes / (cold_us * 1e-6) / 1e9 / hbm_peak) if cold_us else None,
        "prefix_pass_l2_cold_dirty_us": cold_dirty_us,
        "roofline": roof,
        "clocks": res["clocks"],
        "reuse_error": ({"per_denoise_step": res["reuse_err"], "refresh_steps": list(w.refresh),
                         "definition": "||O_cached - O_uncached||_F / ||O_uncached||_F of one block, both outputs "
                                       "from this library; refresh steps show bf16 rounding (plus, for top-k "
                                       "workloads, the sparse selection's own error), reuse steps the method's "
                                       "approximation under the synthetic per-step drift"}
                        if "reuse_err" in res else None),
        "e2e": ({"value": tps(res["ms_e2e"]), "unit": "tokens/s", "h2d_bytes_per_step": res["h2d"],
                 "d2h_bytes_per_step": res["d2h"], "ms_per_step": res["ms_e2e"] / args.steps,
                 **({"h2d_ms_per_step_alone": res["h2d_ms"], "d2h_ms_per_step_alone": res["d2h_ms"],
                     "h2d_gbs": res["h2d"] / (res["h2d_ms"] * 1e-3) / 1e9,
                     "d2h_gbs": res["d2h"] / (res["d2h_ms"] * 1e-3) / 1e9,
                     "bound_by": e2e_bound(res, args)} if "h2d_ms" in res else {}),
                 "copies": "pinned host buffers; each block's inputs in and outputs out on one stream per "
                           "direction, overlapping the neighbouring blocks' compute"}
                if "ms_e2e" in res else None),
        "gpu_launches": res["launches"],
        "gpu_launches_per_step": res["launches"] / args.steps,
    }
    if not args.no_cpu_baseline and world == 1:
        # about 10-20 s of oracle work: samples of up to ~10 s each (as many
        # kv heads as fit), repeated until ~10 s have been timed
        K, V, lens_np = synth.prefix_kv(w0)
        heads, t1 = sample_heads(w0, K, V, lens_np, 10.0)
        times = [t1] if heads == 1 else []
        while sum(times) < 10.0 and len(times) < 50:
            times.append(oracle_block_sample(w0, K, V, lens_np, heads=heads))
        line["cpu_baseline"] = dict(oracle_sample_record(w0, sum(times) / len(times), heads=heads, reps=len(times)),
                                    cores=cpu_threads(), kind="oracle")
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
