"""Benchmark: MoE-layer tokens/s of the V3-shaped prefill layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3_prefill]
                    [--impl reference] [--no-cpu-baseline] [--graph] [--pow2] [--ep]
                    [--gemm | --backward]

One step = one forward pass of the whole layer (route, the permutation's
index tables, the 1x128 quantisation with the dispatch's row scatter fused in,
grouped GEMM 1 with fused SwiGLU + requantisation, grouped GEMM 2, combine,
bias update) over one batch of T tokens, with the FP8 weights already
resident (they are quantised once, before timing).  With N
GPUs (torchrun, one process per GPU) every rank runs its own batch of T
tokens over the full expert set and the per-expert load counts are summed
with an NCCL all-reduce before the bias update (weak scaling).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; between steps a 512 MB buffer is overwritten to
flush the 126 MB L2 (outside the events).  The reported time is the max over
ranks of the summed step times.  Clocks are polled through NVML every 2 ms
during the timed region.  The dominant GEMM's roofline counts each timed
step's own active experts (their routing is replayed untimed afterwards).
The end-to-end figure (e2e) runs the same steps through
MoELayer.forward_host_stream from pinned host buffers, the copies inside the
timed region.  The sequence-wise balance loss, fused into the router's
selection, is timed on its own (graph-replayed calls).

``--impl reference`` times the CPU oracle instead (rank 0 only) on a bounded
sample of the same workload and prints the same JSON line with
"impl": "reference".

Other modes (one GPU, their own JSON line): ``--pow2`` runs the layer with
power-of-two scales (the tensor core applies them); ``--graph`` times CUDA-graph
replays of the step; ``--gemm`` times the standalone 4096x7168x2048
block-scaled GEMM; ``--backward`` times the backward of the expert FFNs
(Dgrad and Wgrad) per phase; ``--ep`` shards the routed experts over the N
ranks (expert parallelism, FP8 dispatch as NCCL all-to-alls).
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

METRIC = "MoE-layer tokens/s on 1 B200; grouped FP8 GEMM TFLOPS as % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_name(cfg) -> str:
    lim = f"G={cfg.G} M={cfg.M}" if cfg.M < cfg.G else "no group limit"
    return (f"{cfg.name}: DeepSeekMoE layer forward, T={cfg.T} d={cfg.d} E={cfg.E} routed "
            f"({lim}) top-{cfg.K} +{cfg.n_shared} shared, SwiGLU I={cfg.I}, FP8 E4M3 1x128 "
            f"activations / 128x128 weights")


# --------------------------------------------------------------- clocks ---
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, polled every 2 ms
    through NVML from a thread while the timed region runs (a 3.5 ms step
    needs a period far below nvidia-smi's).  The device is matched by PCI
    bus id, so CUDA_VISIBLE_DEVICES remapping does not pick another GPU.
    Falls back to ``nvidia-smi -lms 200`` when NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.nvml = None
        self.thread = None
        self.samples = []
        self.stop_flag = False
        self.win = None
        self.max_mhz = None
        self.handle = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        bus = getattr(torch.cuda.get_device_properties(self.idx), "pci_bus_id", None)
        if bus is not None:
            dom = getattr(torch.cuda.get_device_properties(self.idx), "pci_domain_id", 0)
            dev = getattr(torch.cuda.get_device_properties(self.idx), "pci_device_id", 0)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def _poll(self, pynvml, h):
        try:
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self.max_mhz = None
        while not self.stop_flag:
            try:
                self.samples.append((time.perf_counter(),
                                     pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     pynvml.nvmlDeviceGetCurrentClocksEventReasons(h),
                                     pynvml.nvmlDeviceGetPowerUsage(h)))
            except Exception:  # noqa: BLE001 - a failed read drops one sample
                pass
            time.sleep(0.002)

    def sample_until(self, done) -> None:
        """Poll from the calling thread until done() is true (the GPU work of
        the timed region has drained): the region's samples do not depend on
        the polling thread being scheduled while the host enqueues."""
        if self.nvml is None or self.handle is None:
            return
        pynvml, h = self.nvml, self.handle
        while not done():
            try:
                self.samples.append((time.perf_counter(),
                                     pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     pynvml.nvmlDeviceGetCurrentClocksEventReasons(h),
                                     pynvml.nvmlDeviceGetPowerUsage(h)))
            except Exception:  # noqa: BLE001
                return
            time.sleep(0.001)

    def window(self, t0: float, t1: float):
        """Keep only samples taken between t0 and t1 (time.perf_counter)."""
        self.win = (t0, t1)

    def start(self):
        import threading
        try:
            pynvml, h = self._nvml_handle()
            self.nvml = pynvml
            self.handle = h
            self.thread = threading.Thread(target=self._poll, args=(pynvml, h), daemon=True)
            self.thread.start()
            return
        except Exception:  # noqa: BLE001 - no NVML: use nvidia-smi
            self.nvml = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join()
            smp = self.samples
            if self.win is not None:
                smp = [x for x in smp if self.win[0] <= x[0] <= self.win[1]]
            if not smp:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                        "reasons": ["no samples in the timed region"], "source": "nvml"}
            reasons, masks = set(), set()
            for _, _, bits, _ in smp:
                masks.add(int(bits))
                for b, n in self.REASONS.items():
                    if bits & b:
                        reasons.add(n)
            return {"sm_mhz": statistics.median(x[1] for x in smp), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(reasons), "samples": len(smp),
                    "power_w_median": round(statistics.median(x[3] for x in smp) / 1000.0, 1),
                    "reason_masks": sorted(hex(m) for m in masks),
                    "source": "nvml, polled every 2 ms, samples inside the timed region"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 200 ms"}


# ------------------------------------------------------- FP8 tensor peak ---
def measure_fp8_peak(dev, block_scaled: bool, launches: int = 8, iters: int = 8192,
                     sustain_s: float = 0.0) -> dict:
    """Dense FP8 rate of this GPU, measured live with the library's MMA loop
    (moe_fp8_mma_peak: one CTA per SM, 128x256x32 E4M3 tcgen05 MMAs from
    shared memory, no global traffic).  ``block_scaled`` times the
    kind::mxf8f6f4.block_scale instruction the power-of-two GEMM issues,
    otherwise the kind::f8f6f4 one of the promoting GEMM.  Burst = the best of
    ``launches`` separate launches (about 2 ms each at full clock, 30 ms
    apart); with
    sustain_s > 0 the launches also run back to back for that long and the
    median of the second half is the sustained rate."""
    import torch

    from fp8_block_scaled_sigmoid_b200 import _abi

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.empty(sms, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flops = 0
    for _ in range(2):
        flops = _abi.moe_fp8_mma_peak(block_scaled, iters, sms, sink, err)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(launches)]
    for a, b in ev:
        torch.cuda.synchronize()
        time.sleep(0.03)          # let the power controller settle between bursts
        a.record()
        _abi.moe_fp8_mma_peak(block_scaled, iters, sms, sink, err)
        b.record()
    torch.cuda.synchronize()
    burst = max(flops / (a.elapsed_time(b) / 1e3) / 1e12 for a, b in ev)
    out = {"tflops": round(burst, 1), "kind": "mxf8f6f4.block_scale" if block_scaled
           else "f8f6f4", "sms": sms, "iters": iters}
    if sustain_s > 0:
        rates = []
        t_end = time.perf_counter() + sustain_s
        while time.perf_counter() < t_end:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(10):
                _abi.moe_fp8_mma_peak(block_scaled, iters, sms, sink, err)
            b.record()
            b.synchronize()
            rates.append(10 * flops / (a.elapsed_time(b) / 1e3) / 1e12)
        tail = rates[len(rates) // 2:]
        out["sustained_tflops"] = round(statistics.median(tail), 1)
        out["sustained_s"] = sustain_s
    _abi.raise_dev_err(err)
    return out


def run_peak(args):
    """Measure the FP8 tensor peak (both MMA kinds, burst and sustained) with
    clocks sampled during each, one JSON line."""
    import torch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    res = {"metric": "dense FP8 tensor-core TFLOP/s (tcgen05 MMA loop, no global memory)",
           "unit": "TFLOP/s", "n_gpus": 1}
    for bs in (False, True):
        sampler = ClockSampler(0)
        sampler.start()
        if sampler.proc is not None:
            time.sleep(0.3)
        t0 = time.perf_counter()
        r = measure_fp8_peak(dev, bs, launches=10, sustain_s=4.0)
        sampler.window(t0, time.perf_counter())
        r["clocks"] = sampler.stop()
        res["block_scaled" if bs else "f8f6f4"] = r
        time.sleep(2.0)
    print(json.dumps(res), flush=True)


# ------------------------------------------------------- CPU oracle leg ---
def oracle_sample_rate(cfg, u_host, cent_host, bias_host, expert_weights, route_tokens,
                       ffn_tokens: int):
    """Time the single-threaded C++ oracle (oracle/moe_oracle_ref.cpp, fp64)
    on a bounded sample of the layer and return (seconds per token,
    description).  Router logits, selection, 1x128 quantisation, permutation
    and the bias update run over ``route_tokens`` tokens; the expert FFNs
    (grouped GEMM 1, SwiGLU + requantisation, grouped GEMM 2; routed and
    shared) and the combine over the first ``ffn_tokens`` of them, one expert
    at a time.  ``expert_weights(e)`` returns the quantised (w1q, w1s, w2q,
    w2s) of one expert as numpy arrays (weight preparation is not timed, as on
    the GPU)."""
    import numpy as np
    from oracle import cpp_oracle as C

    ur = u_host[:route_tokens]
    t0 = time.perf_counter()
    idx, gate, _ = C.route(ur, cent_host, bias_host, cfg.G, cfg.M, cfg.K)
    xq, xs = C.quant_1x128(ur)
    counts, offsets, src_row, dst_of = C.permute(idx, cfg.E)
    _ = xq[src_row], xs[src_row]
    C.bias_update(counts, route_tokens, cfg.K, cfg.gamma, bias_host)
    t_route = time.perf_counter() - t0
    # the sampled tokens' pairs, grouped by expert, plus the shared expert's rows
    S = ffn_tokens
    c_s, off_s, src_s, dst_s = C.permute(idx[:S], cfg.E)
    P = S * cfg.K
    xq_s = np.concatenate([xq[src_s], xq[:S]])
    xs_s = np.concatenate([xs[src_s], xs[:S]])
    offs = C.segment_offsets_with_shared(off_s, S)
    Y = np.zeros((P + S, cfg.d))
    t_ffn = 0.0
    n_exp = 0
    for e in range(cfg.E + 1):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r1 == r0:
            continue
        w1q, w1s, w2q, w2s = expert_weights(e)
        n_exp += 1
        seg = np.array([0, r1 - r0], np.int32)
        t1 = time.perf_counter()
        gu = C.grouped_gemm(xq_s[r0:r1], xs_s[r0:r1], w1q[None], w1s[None], seg)
        hq, hs = C.swiglu_quant(gu, cfg.I)
        Y[r0:r1] = C.grouped_gemm(hq, hs, w2q[None], w2s[None], seg)
        t_ffn += time.perf_counter() - t1
    t1 = time.perf_counter()
    C.combine(Y[:P], dst_s, gate[:S], Y[P:], ur[:S])
    t_ffn += time.perf_counter() - t1
    per_token = t_route / route_tokens + t_ffn / S
    desc = (f"C++ oracle, 1 thread: logits+select+quant+permute+bias-update over {route_tokens} "
            f"tokens ({t_route:.2f} s); expert FFNs ({cfg.K} routed + 1 shared per token: "
            f"{P} + {S} rows over {n_exp} experts) + combine for {S} tokens ({t_ffn:.2f} s); "
            f"rate = 1/(route time per token + FFN time per token)")
    return per_token, desc


# ------------------------------------------------------------- GPU arm ---
def run_gpu(args):
    import torch
    import torch.distributed as dist

    from fp8_block_scaled_sigmoid_b200 import _abi, configs, inputs
    from fp8_block_scaled_sigmoid_b200.layer import MoELayer, make_fp8_weights, max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist.group.WORLD

    cfg = configs.PRESETS[args.config]
    cfg_rank = cfg.with_(seed=cfg.seed + rank)       # each rank its own token batch
    if args.ep:
        return run_ep(args, cfg, cfg_rank, dev, pg, world, rank, local)
    w1q, w1s, w2q, w2s = make_fp8_weights(cfg, dev, pow2=args.pow2)  # same on every rank
    cent = inputs.draw_centroids(cfg, dev)
    bias = inputs.draw_bias(cfg, dev)
    u = inputs.draw_u(cfg_rank, dev)
    layer = MoELayer(cfg, cent, bias.clone(), w1q, w1s, w2q, w2s, process_group=pg,
                     pow2=args.pow2)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def barrier():
        if pg is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        layer.forward(u)
    barrier()
    layer.check()

    # permute = counts, offsets, row maps and tile table; quant = the 1x128
    # quantisation with the dispatch's row scatter fused in
    names = ["route", "permute", "quant", "gemm1", "gemm2", "combine", "bias"]
    use_graph = world == 1 and args.graph
    sampler = ClockSampler(local) if rank == 0 else None

    def start_sampler():
        if sampler:
            sampler.start()
            if sampler.proc is not None:
                time.sleep(0.3)  # nvidia-smi needs a moment before its first sample

    # headline: K eager steps with an event between every call (with --graph,
    # K CUDA-graph replays of the step are timed as the headline instead)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(args.steps)]
    # the bias the timed steps start from: their routing is replayed after the
    # timed region to count each step's active experts (the bias update moves
    # the routing from step to step)
    bias_t0 = layer.bias.clone()
    if not use_graph:
        start_sampler()
    barrier()
    t_lo = time.perf_counter()
    lc0 = _abi.launch_count
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e = ev[i]
        e[0].record(st)
        layer.step_route(u)
        e[1].record(st)
        layer.step_permute()
        e[2].record(st)
        layer.step_quant(u)
        e[3].record(st)
        layer.step_gemm1()
        e[4].record(st)
        layer.step_gemm2()
        e[5].record(st)
        layer.step_combine(u)
        e[6].record(st)
        layer.step_bias_update()
        e[7].record(st)
    if sampler:
        sampler.sample_until(ev[-1][-1].query)
    barrier()
    t_hi = time.perf_counter()
    launches = _abi.launch_count - lc0
    layer.check()
    step_ms = [ev[i][0].elapsed_time(ev[i][-1]) for i in range(args.steps)]
    j1, j2 = names.index("gemm1"), names.index("gemm2")
    gemm1_ms = [ev[i][j1].elapsed_time(ev[i][j1 + 1]) for i in range(args.steps)]
    gemm2_ms = [ev[i][j2].elapsed_time(ev[i][j2 + 1]) for i in range(args.steps)]
    # untimed replay of the timed steps' routing (same bias sequence, same
    # inputs, deterministic): the experts each step's GEMMs streamed
    bias_t1 = layer.bias.clone()
    layer.bias.copy_(bias_t0)
    step_counts = []
    for i in range(args.steps):
        layer.step_route(u)
        layer.step_permute()
        step_counts.append(layer.perm["counts"].clone())
        layer.step_bias_update()
    layer.bias.copy_(bias_t1)
    step_counts = [c.cpu() for c in step_counts]
    per_kernel = {n: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps
                  for j, n in enumerate(names)}
    eager_ms = max_over_ranks(sum(step_ms), dev, pg)
    total_ms = eager_ms
    if use_graph:
        # headline: the whole step replayed from a CUDA graph, one host call
        # per step (same kernels, same order; the L2 flush stays outside)
        graph, per_replay = layer.capture(u)
        for i in range(args.warmup):
            flush.fill_(i & 0xFF)
            graph.replay()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        start_sampler()
        barrier()
        t_lo = time.perf_counter()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            gev[i][0].record(st)
            graph.replay()
            gev[i][1].record(st)
        if sampler:
            sampler.sample_until(gev[-1][1].query)
        barrier()
        t_hi = time.perf_counter()
        layer.check()
        launches = per_replay * args.steps
        total_ms = sum(a.elapsed_time(b) for a, b in gev)
        del graph
    if sampler:
        sampler.window(t_lo, t_hi)
    clocks = sampler.stop() if sampler else None
    tokens = cfg.T * world * args.steps
    value = tokens / (total_ms / 1e3)

    # end to end through the public API with pinned host buffers: every step
    # copies its batch in (host -> device) and its output out (device -> host);
    # forward_host_stream overlaps step i's compute with step i+1's input copy
    # and step i-1's output copy.  No L2 flush here: the 11.3 GB of FP8 weights
    # that every step streams already exceed L2.
    u_host = u.cpu().pin_memory()
    out_hosts = [torch.empty(cfg.T, cfg.d, dtype=torch.float32).pin_memory() for _ in range(2)]
    layer.forward_host_stream([u_host] * 2, out_hosts)
    barrier()
    e2e0, e2e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e0.record(st)
    layer.forward_host_stream([u_host] * args.steps, [out_hosts[i & 1] for i in range(args.steps)])
    e2e1.record(st)
    barrier()
    e2e_ms = max_over_ranks(e2e0.elapsed_time(e2e1), dev, pg)
    e2e_value = tokens / (e2e_ms / 1e3)
    out_host = out_hosts[0]

    # the sequence-wise balance loss (eqs. 17-20) of this batch, one sequence
    # of T tokens: the router's selection pass computes it (integer sums per
    # sequence, the last block finishes the loss).  Its cost is the route
    # with the loss minus the route without it; the three-pass form from
    # kept logits is timed beside it.
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)
    bstate = _abi.BalanceLossState(cfg.T, cfg.E, cfg.T, 1e-4, with_fp=True, device=dev)
    rws = torch.empty(max(_abi.moe_route_workspace_size(cfg.T, cfg.d, cfg.E), 16),
                      dtype=torch.uint8, device=dev)
    bl_ws = torch.empty(max(_abi.moe_seq_balance_loss_ws(cfg.T, cfg.E, cfg.T), 16),
                        dtype=torch.uint8, device=dev)

    def timed(fn, n):
        # n calls recorded into one CUDA graph, so the device time is measured
        # and not the host's per-call overhead (these kernels run for a few us)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(st)
        g.replay()
        b_.record(st)
        b_.synchronize()
        del g
        return a_.elapsed_time(b_) * 1e3 / n

    reps = max(args.steps, 10)
    t_plain = timed(lambda: _abi.moe_route(u, layer.centroids, layer.bias, cfg.G, cfg.M, cfg.K,
                                           ws=rws), reps)
    t_aux = timed(lambda: _abi.moe_route(u, layer.centroids, layer.bias, cfg.G, cfg.M, cfg.K,
                                         ws=rws, aux=bstate), reps)
    _abi.moe_route(u, layer.centroids, layer.bias, cfg.G, cfg.M, cfg.K, logits_out=logits, ws=rws)
    t_3p = timed(lambda: _abi.moe_seq_balance_loss(logits, cfg.K, cfg.T, ws=bl_ws), reps)
    barrier()
    balance_loss = {"extra_us": round(t_aux - t_plain, 2),
                    "route_us": round(t_plain, 2), "route_with_loss_us": round(t_aux, 2),
                    "three_pass_from_logits_us": round(t_3p, 2), "seq_len": cfg.T,
                    "how": "device time per call, 10+ calls replayed from one CUDA graph"}
    del logits, bstate, rws, bl_ws

    # roofline of the dominant kernel (grouped GEMM 1 with the SwiGLU epilogue):
    # algorithmic bytes of each timed step (its own active experts) over the
    # GEMM's total time in those steps
    counts = step_counts[-1]
    active = sum(int((c > 0).sum()) + cfg.n_shared for c in step_counts) / len(step_counts)
    rows = cfg.pairs + cfg.T
    w1_bytes = active * 2 * cfg.I * cfg.d * (1 + 4.0 / (128 * 128))
    a_bytes = rows * cfg.d * (1 + 4.0 / 128)
    h_bytes = rows * cfg.I * (1 + 4.0 / 128)
    g1_bytes = w1_bytes + a_bytes + h_bytes
    w2_bytes = active * cfg.I * cfg.d * (1 + 4.0 / (128 * 128))
    g2_bytes = w2_bytes + rows * cfg.I * (1 + 4.0 / 128) + rows * cfg.d * 4
    g1_flops = 2.0 * rows * cfg.d * 2 * cfg.I
    g2_flops = 2.0 * rows * cfg.I * cfg.d
    t1 = sum(gemm1_ms) / len(gemm1_ms) / 1e3
    t2 = sum(gemm2_ms) / len(gemm2_ms) / 1e3
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp8 = measure_fp8_peak(dev, args.pow2)
    fp8_peak = fp8["tflops"]
    achieved = g1_bytes / t1 / 1e9
    gemm_name = "grouped_gemm_fp8_pow2" if args.pow2 else "grouped_gemm_fp8"
    traffic = read_traffic(gemm_name, cfg.name)
    # the dominant kernel's bound: weight streaming below the ridge point
    # (FP8 peak / HBM bandwidth, in FLOP per byte), the tensor pipe above it
    ridge = fp8_peak * 1e12 / (hbm * 1e9)
    src_note = (f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback")
    if g1_flops / g1_bytes < ridge:
        roofline = {"kernel": f"{gemm_name} (GEMM 1, SwiGLU+quant epilogue)", "bound": "hbm",
                    "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4), "traffic": traffic,
                    "peak_source": f"hbm_gbs, {src_note}", "algorithmic_bytes": int(g1_bytes)}
    else:
        tf1 = g1_flops / t1 / 1e12
        roofline = {"kernel": f"{gemm_name} (GEMM 1, SwiGLU+quant epilogue)",
                    "bound": "tensor", "achieved": round(tf1, 1), "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": round(tf1 / fp8_peak, 4), "traffic": traffic,
                    "peak_source": f"measured in this run: tcgen05 kind::{fp8['kind']} MMA loop, "
                                   "best of 8 launches (moe_fp8_mma_peak)",
                    "algorithmic_flops": int(g1_flops), "algorithmic_bytes": int(g1_bytes)}
    # the memory-bound kernels against the measured copy bandwidth, with
    # their algorithmic bytes: quant reads u (2 B/elem) and writes every FP8
    # row once per destination (the token copy and K routed rows, 1 B/elem +
    # 4 B per 128); combine reads K+1 fp32 rows and u, writes fp32
    Tn, dn = cfg.T, cfg.d
    q_bytes = Tn * dn * 2 + (cfg.pairs + Tn) * dn * (1 + 4.0 / 128)
    c_bytes = Tn * ((cfg.K + 1) * 4 * dn + 2 * dn + 4 * dn)
    r_bytes = Tn * dn * 2 + cfg.E * dn * 2 + Tn * cfg.K * 8
    tq, tc = per_kernel["quant"] / 1e3, per_kernel["combine"] / 1e3
    tr = per_kernel["route"] / 1e3
    memory_kernels = {
        "quant_scatter": {"bytes": int(q_bytes), "gbs": round(q_bytes / tq / 1e9, 1),
                          "frac": round(q_bytes / tq / 1e9 / hbm, 4)},
        "combine": {"bytes": int(c_bytes), "gbs": round(c_bytes / tc / 1e9, 1),
                    "frac": round(c_bytes / tc / 1e9 / hbm, 4)},
        "permute_index_us": round(per_kernel["permute"] * 1e3, 1),
        # the router: u and the centroids read once, the indices and gates
        # written; its logits GEMM is a bf16 tensor-core product (2·T·E·d)
        "route": {"bytes": int(r_bytes), "gbs": round(r_bytes / tr / 1e9, 1),
                  "frac": round(r_bytes / tr / 1e9 / hbm, 4),
                  "bf16_tflops": round(2.0 * Tn * cfg.E * dn / tr / 1e12, 1),
                  "note": "logits GEMM (bf16 tensor cores, split over K) + one warp per token "
                          "selection; bound by the selection's instruction issue, not HBM"},
        "peak": hbm, "unit": "GB/s"}
    gemm = {"gemm1_tflops": round(g1_flops / t1 / 1e12, 1),
            "gemm2_tflops": round(g2_flops / t2 / 1e12, 1),
            "gemm1_gbs": round(achieved, 1), "gemm2_gbs": round(g2_bytes / t2 / 1e9, 1),
            "layer_gemm_tflops": round((g1_flops + g2_flops) / (t1 + t2) / 1e12, 1),
            "fp8_peak_tflops": fp8_peak,
            "frac_fp8_peak": round((g1_flops + g2_flops) / (t1 + t2) / 1e12 / fp8_peak, 4),
            "fp8_peak_note": f"measured in this run: tcgen05 kind::{fp8['kind']} MMA loop on all "
                             f"{fp8['sms']} SMs, best of 8 launches (moe_fp8_mma_peak)"}
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "synthetic (seeded; random-init weights of the V3-shaped layer)",
        "config": {"workload": workload_name(cfg), "tokens_per_gpu": cfg.T,
                   "parallelism": f"dp{world} (full expert set per GPU, load counts all-reduced)"
                   if world > 1 else "single GPU",
                   "l2": "512 MB buffer written between timed steps; FP8 weights (11.3 GB) > L2",
                   "scales": "powers of two; the tensor core applies them (UE8M0 block scaling)"
                   if args.pow2 else "fp32 amax/448; promoted per 128-wide K block"},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(u_host.numel() * u_host.element_size()),
                "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
                "how": "MoELayer.forward_host_stream over the timed steps: per step a pinned "
                       "host->device copy of u and a device->host copy of the output, "
                       "overlapped with the neighbouring steps' compute on copy streams"},
        "gpu_launches": launches,
        "step_launch": "one CUDA-graph replay per step" if use_graph else "eager calls",
        "roofline": roofline,
        "gemm": gemm,
        "kernel_ms": {k: round(v, 4) for k, v in per_kernel.items()},
        "memory_kernels": memory_kernels,
        "seq_balance_loss": balance_loss,
        "loads": {"max": int(counts.max()), "mean": float(counts.float().mean()),
                  "active_experts": round(active - cfg.n_shared, 1),
                  "how": "routing of the timed steps, replayed untimed from their starting "
                         "bias; max and mean of the last step, active experts averaged over "
                         "the steps"},
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, layer, u, bias)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if pg is not None:
        dist.barrier()
        dist.destroy_process_group()


def read_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}/{workload}")
    if not ent:
        return None
    src = os.path.join(ROOT, "fp8_block_scaled_sigmoid_b200", "csrc", ent.get("source", ""))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return ent["bytes_per_launch"] if h == ent.get("source_sha256_16") else None


def cpu_baseline(cfg, layer, u, bias):
    """The C++ oracle on the host, one thread, on a bounded sample of the
    same workload (the layer's own inputs and FP8 weights, copied to the
    host one expert at a time)."""
    u_h = u.float().cpu().numpy()
    cent_h = layer.centroids.float().cpu().numpy()
    b_h = bias.cpu().numpy()

    def weights(e):
        return (layer.w1q[e].cpu().numpy(), layer.w1s[e].cpu().numpy(),
                layer.w2q[e].cpu().numpy(), layer.w2s[e].cpu().numpy())

    per_token, desc = oracle_sample_rate(cfg, u_h, cent_h, b_h, weights, min(cfg.T, 256),
                                         min(cfg.T, 32))
    return {"value": round(1.0 / per_token, 3), "unit": "tokens/s", "cores": 1,
            "host_cpus": os.cpu_count(), "kind": "oracle", "sample": desc}


# ------------------------------------------------------- reference arm ---
def run_reference(args):
    """The reference arm: the C++ oracle (one thread, fp64) on the host cores,
    each step a bounded sample of the workload -- the route over 64 tokens,
    the FFNs and the combine of the first 2.  The FP8 weights of the experts
    those tokens use are prepared once, before timing (numpy oracle
    quantiser, as the GPU arm quantises its weights outside the step)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from fp8_block_scaled_sigmoid_b200 import configs, inputs
    from oracle import cpp_oracle as C
    from oracle import moe_oracle as O

    cfg = configs.PRESETS[args.config]
    route_tokens, ffn_tokens = min(cfg.T, 64), min(cfg.T, 2)
    u = inputs.draw_u(cfg).float().numpy()[:route_tokens]
    cent = inputs.draw_centroids(cfg).float().numpy()
    bias = inputs.draw_bias(cfg).numpy()
    cache = {}

    def weights(e):
        if e not in cache:       # weight preparation (not timed)
            w1 = inputs.draw_w1(cfg, e).float().numpy()
            w2 = inputs.draw_w2(cfg, e).float().numpy()
            cache[e] = O.quant_128x128(w1) + O.quant_128x128(w2)
        return cache[e]

    # prepare the sampled tokens' experts before timing
    idx0, _, _ = C.route(u[:ffn_tokens], cent, bias, cfg.G, cfg.M, cfg.K)
    for e in sorted(set(idx0.reshape(-1).tolist()) | {cfg.E}):
        weights(int(e))
    times, desc = [], ""
    for i in range(args.warmup + args.steps):
        per_token, desc = oracle_sample_rate(cfg, u, cent, bias, weights, route_tokens,
                                             ffn_tokens)
        if i >= args.warmup:
            times.append(per_token)
    per_token = sum(times) / len(times)
    value = 1.0 / per_token
    cb = {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "host_cpus": os.cpu_count(),
          "kind": "oracle", "sample": desc}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_token * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": workload_name(cfg), "tokens_per_gpu": cfg.T,
                   "parallelism": "CPU oracle (C++, one thread), rank 0 only"},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_gemm(args):
    """Standalone block-scaled GEMM: A 4096x7168 (1x128 tiles, 1% outliers
    x50) times B^T, B 7168x2048 (128x128 blocks), fp32 out."""
    import torch

    from fp8_block_scaled_sigmoid_b200 import _abi, configs, inputs

    dev = torch.device("cuda", 0)
    cfg = configs.STANDALONE_GEMM
    a, bt = inputs.draw_gemm(cfg, dev)
    aq, sa = _abi.fp8_quant_1x128(a, pow2=args.pow2)
    bq, sb = _abi.fp8_quant_128x128(bt.unsqueeze(0), pow2=args.pow2)
    offs = torch.tensor([0, cfg.M], dtype=torch.int32, device=dev)
    mt = cfg.M // 128
    tg, ts, nt = _abi.moe_tile_table(offs, mt)
    D = torch.empty(cfg.M, cfg.N, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, mt, D=D, pow2=args.pow2)
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    sampler.start()
    if sampler.proc is not None:
        time.sleep(0.3)
    times = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        _abi.grouped_gemm_fp8_blockscaled(aq, sa, bq, sb, offs, tg, ts, nt, mt, D=D, pow2=args.pow2)
        e1.record()
        sampler.sample_until(e1.query)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    clocks = sampler.stop()
    fp8 = measure_fp8_peak(dev, args.pow2)
    fp8_peak = fp8["tflops"]
    ms = statistics.median(times)
    tf = cfg.flops / (ms / 1e3) / 1e12
    print(json.dumps({
        "metric": "standalone block-scaled FP8 GEMM TFLOP/s", "value": round(tf, 1),
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "dtype": "fp8_e4m3",
        "config": {"workload": f"{cfg.name}: A {cfg.M}x{cfg.K} (1x128 scales, 1% outliers x50) "
                               f"x B^T {cfg.N}x{cfg.K} (128x128 scales), fp32 out"
                               + (", power-of-two scales applied by the tensor core"
                                  if args.pow2 else ""),
                   "l2": "512 MB buffer written between timed launches"},
        "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": round(tf / fp8_peak, 4),
                     "peak_source": f"measured in this run: tcgen05 kind::{fp8['kind']} MMA "
                                    "loop, best of 8 launches (moe_fp8_mma_peak)"},
        "clocks": clocks}), flush=True)


def run_ep(args, cfg, cfg_rank, dev, pg, world, rank, local):
    """Expert parallelism: each rank holds E/world routed experts (plus the
    shared one) and its own batch of T tokens; the routed rows travel to
    their experts' ranks and back as NCCL all-to-alls (ep.MoELayerEP).  Weak
    scaling: T tokens per rank.  Timed per step with CUDA events, max over
    ranks; clocks sampled as in the main mode."""
    import torch
    import torch.distributed as dist

    from fp8_block_scaled_sigmoid_b200 import _abi, ep, inputs
    from fp8_block_scaled_sigmoid_b200.layer import make_fp8_weights, max_over_ranks

    shard = ep.ExpertShard(cfg.E, world, rank)
    experts = [cfg.E] + list(range(shard.e0, shard.e1))      # the shared expert first
    w = make_fp8_weights(cfg, dev, experts=experts)
    layer = ep.MoELayerEP(cfg, inputs.draw_centroids(cfg, dev), inputs.draw_bias(cfg, dev), *w,
                          shard, process_group=pg)
    u = inputs.draw_u(cfg_rank, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def barrier():
        if pg is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        layer.forward(u)
    barrier()
    layer.check()
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
        if sampler.proc is not None:
            time.sleep(0.3)
    barrier()
    t_lo = time.perf_counter()
    total = 0.0
    lc0 = _abi.launch_count
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        layer.forward(u)
        e1.record(st)
        if sampler:
            sampler.sample_until(e1.query)
        e1.synchronize()   # the next step's dispatch plan reads its split sizes on the host
        total += e0.elapsed_time(e1)
    barrier()
    t_hi = time.perf_counter()
    launches = _abi.launch_count - lc0
    layer.check()
    if sampler:
        sampler.window(t_lo, t_hi)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(total, dev, pg)
    result = {
        "metric": METRIC + " (expert parallel)", "value": round(cfg.T * world * args.steps / (ms / 1e3), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3", "data": "synthetic (seeded)",
        "config": {"workload": workload_name(cfg), "tokens_per_gpu": cfg.T,
                   "parallelism": f"ep{world} ({shard.per_rank} routed experts per GPU + shared; "
                                  "FP8 dispatch and output return as NCCL all-to-alls)",
                   "l2": "512 MB buffer written between timed steps"},
        "gpu_launches": launches, "roofline": None,
        "roofline_note": "per-kernel times are not separated in this mode",
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if pg is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_backward(args):
    """Backward of the expert FFNs at the configured layer size (one GPU):
    forward_train once per step (untimed), then the timed backward with the
    weight gradients.  Tokens/s = T / backward time."""
    import torch

    from fp8_block_scaled_sigmoid_b200 import _abi, configs, inputs
    from fp8_block_scaled_sigmoid_b200.layer import MoELayer, make_fp8_weights

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = configs.PRESETS[args.config]
    w1q, w1s, w2q, w2s = make_fp8_weights(cfg, dev, pow2=args.pow2)
    layer = MoELayer(cfg, inputs.draw_centroids(cfg, dev), inputs.draw_bias(cfg, dev), w1q, w1s,
                     w2q, w2s, pow2=args.pow2)
    u = inputs.draw_u(cfg, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed + 77)
    dout = torch.randn(cfg.T, cfg.d, generator=g, device=dev) * 0.01
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    layer.forward_train(u, update_bias=False)
    layer.transposed_weights()
    for _ in range(args.warmup):
        layer.backward(dout)
    torch.cuda.synchronize()
    layer.check()
    names = ["combine_backward", "dgrad2", "swiglu_backward", "dgrad1", "unpermute", "quant_128x1",
             "wgrad2", "wgrad1"]
    per = {n: 0.0 for n in names}
    total = 0.0
    sampler = ClockSampler(0)
    sampler.start()
    if sampler.proc is not None:
        time.sleep(0.3)
    launches = 0
    t_lo = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev = [torch.cuda.Event(enable_timing=True)]
        ev[0].record(st)

        def mark(name, ev=ev):
            e = torch.cuda.Event(enable_timing=True)
            e.record(st)
            ev.append(e)
        lc0 = _abi.launch_count
        layer.backward(dout, mark=mark)
        launches += _abi.launch_count - lc0
        sampler.sample_until(ev[-1].query)
        torch.cuda.synchronize()
        for j, n in enumerate(names):
            per[n] += ev[j].elapsed_time(ev[j + 1])
        total += ev[0].elapsed_time(ev[-1])
    t_hi = time.perf_counter()
    layer.check()
    sampler.window(t_lo, t_hi)
    clocks = sampler.stop()
    per = {n: round(v / args.steps, 4) for n, v in per.items()}
    ms = total / args.steps
    rows = cfg.pairs + cfg.T
    counts = layer.perm["counts"].cpu()
    G = cfg.E + cfg.n_shared
    ldt = _abi.wgrad_ld(layer.max_tiles)
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp8_peak = measure_fp8_peak(dev, True)["tflops"]   # Wgrad is block-scaled
    # Wgrad of W1: both token-major operands once, the fp32 gradient of every expert written
    ktot = 128 * int(layer.perm["n_tiles"].item())
    w1_bytes = (2 * cfg.I + cfg.d) * ktot * (1 + 1.0 / 128) + G * 2 * cfg.I * cfg.d * 4
    w1_flops = 2.0 * rows * 2 * cfg.I * cfg.d
    t_w1 = per["wgrad1"] / 1e3
    dg_flops = 2.0 * rows * cfg.I * cfg.d
    result = {
        "metric": "MoE expert-FFN backward tokens/s on 1 B200 (Dgrad + Wgrad, FP8)",
        "value": round(cfg.T / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "dtype": "fp8_e4m3", "data": "synthetic (seeded)",
        "config": {"workload": workload_name(cfg) + "; backward of the expert FFNs for a seeded "
                   "fp32 output gradient, weight gradients fp32 [G][N][K]",
                   "scales": "powers of two" if args.pow2 else "fp32 weights/activations, "
                   "power-of-two gradients", "l2": "512 MB buffer written between steps"},
        "gpu_launches": launches // args.steps,
        "kernel_ms": per,
        "roofline": {"kernel": "grouped_gemm_fp8_wgrad (dW1)", "bound": "hbm",
                     "achieved": round(w1_bytes / t_w1 / 1e9, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(w1_bytes / t_w1 / 1e9 / hbm, 4),
                     "algorithmic_bytes": int(w1_bytes), "traffic": None,
                     "peak_source": f"hbm_gbs, {src}"},
        "gemm_tflops": {"dgrad2": round(dg_flops / (per["dgrad2"] / 1e3) / 1e12, 1),
                        "dgrad1": round(dg_flops * 2 / (per["dgrad1"] / 1e3) / 1e12, 1),
                        "wgrad2": round(dg_flops / (per["wgrad2"] / 1e3) / 1e12, 1),
                        "wgrad1": round(w1_flops / t_w1 / 1e12, 1), "fp8_peak": fp8_peak},
        "loads": {"max": int(counts.max()), "active_experts": int((counts > 0).sum())},
        "clocks": clocks,
    }
    print(json.dumps(result), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="v3_prefill")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time CUDA-graph replays of the step instead of eager calls (one GPU)")
    ap.add_argument("--pow2", action="store_true",
                    help="power-of-two scale variant (tensor-core UE8M0 block scaling)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: routed experts sharded over the N ranks")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward of the expert FFNs (Dgrad + Wgrad) instead")
    ap.add_argument("--gemm", action="store_true",
                    help="time the standalone 4096x7168x2048 block-scaled GEMM instead")
    ap.add_argument("--peak", action="store_true",
                    help="measure the dense FP8 tensor-core peak (MMA loop) instead")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.peak:
        run_peak(args)
    elif args.gemm:
        run_gemm(args)
    elif args.backward:
        run_backward(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
