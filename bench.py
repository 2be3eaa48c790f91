"""Benchmark of the W4A8 routed-expert MoE layer on B200.

One step = one ``w4a8_moe_forward`` (activation quantisation, routing +
permutation, gate/up grouped GEMM + SwiGLU, intermediate requantisation, down
grouped GEMM, combine) over one batch of synthetic tokens.  Prints one JSON
line.  ``--impl reference`` times the CPU oracle instead (the only other
place this script runs ``oracle/``).

Multi-GPU: one process per GPU (torchrun); each rank runs its own batch
through its own copy of the experts (data parallel, no collective on the data
path): weak scaling, value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import hashlib
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200 + % of HBM (decode) / FP8-peak (prefill) roofline"
DEFAULT_CONFIG = workloads.CONFIGS[1].name
KERNELS_PER_STEP = 8   # act_quant, route topk/scan/scatter, gemm1, inter_quant, gemm2, combine
SHARED_KERNELS_PER_STEP = 5   # tables, input group quant, gate/up GEMM, h group quant, down GEMM


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sus=d.get("bf16_tflops_sustained", d["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    NVML is polled from a thread every ~2 ms (the timed region of a short run is
    only tens of milliseconds); the device is found by its PCI bus id, so the
    sample is of the GPU this process runs on whatever CUDA_VISIBLE_DEVICES is.
    """

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device: torch.device, period_s: float = 0.002):
        self.device, self.period_s = device, period_s
        self.samples, self.max_mhz, self.reasons, self.err = [], None, set(), None
        self._stop = None

    def _handle(self, nv):
        try:
            p = torch.cuda.get_device_properties(self.device)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report no samples rather than guess
            self.err = f"{type(e).__name__}: {e}"
            return self
        self._stop = threading.Event()

        def run():
            while True:
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.reasons.update(n for n, b in self.REASONS.items() if r & b)
                except Exception as e:
                    self.err = f"{type(e).__name__}: {e}"
                    return
                if self._stop.wait(self.period_s):
                    return

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
               "samples": len(self.samples), "source": "nvml"}
        if self.err:
            out["error"] = self.err
        return out


def build_layer(cfg, device, w4, variant: str = "w4a8"):
    """Pack every expert's seeded bf16 weights on the device and lay them out for the GEMMs (not timed)."""
    E, H, I = cfg.E, cfg.H, cfg.I
    if variant == "channel-int8":
        p13 = torch.empty(E, 2 * I, H // 8, dtype=torch.int32, device=device)
        s13 = torch.empty(E, 2 * I, dtype=torch.bfloat16, device=device)
        p2 = torch.empty(E, H, I // 8, dtype=torch.int32, device=device)
        s2 = torch.empty(E, H, dtype=torch.bfloat16, device=device)
        for e in range(E):
            w13, w2 = workloads.gen_expert_weights(cfg, e, device=device)
            w4.w4a8_pack_int4_channel(w13, packed=p13[e], scales=s13[e])
            w4.w4a8_pack_int4_channel(w2, packed=p2[e], scales=s2[e])
        p13, n13 = w4.w4a8_prepare_experts_channel_b200(p13, packed_out=p13)
        p2, n2 = w4.w4a8_prepare_experts_channel_b200(p2, packed_out=p2)
        torch.cuda.synchronize(device)
        return w4.W4A8ChannelInt8Layer(p13, s13, n13, p2, s2, n2, cfg.k)
    p13 = torch.empty(E, 2 * I, H // 8, dtype=torch.int32, device=device)
    s13 = torch.empty(E, 2 * I, H // 128, dtype=torch.bfloat16, device=device)
    p2 = torch.empty(E, H, I // 8, dtype=torch.int32, device=device)
    s2 = torch.empty(E, H, I // 128, dtype=torch.bfloat16, device=device)
    for e in range(E):
        w13, w2 = workloads.gen_expert_weights(cfg, e, device=device)
        w4.w4a8_pack_int4(w13, packed=p13[e], scales=s13[e])
        w4.w4a8_pack_int4(w2, packed=p2[e], scales=s2[e])
    p13, s13g = w4.w4a8_prepare_experts_b200(p13, s13, packed_out=p13)
    p2, s2g = w4.w4a8_prepare_experts_b200(p2, s2, packed_out=p2)
    torch.cuda.synchronize(device)
    del s13, s2
    if variant == "w4a8+shared":   # plus the FP8 128x128-block shared expert
        ws13, ws2 = workloads.gen_shared_weights(cfg, device=device)
        shared = w4.SharedExpertFP8.from_bf16(ws13, ws2)
        torch.cuda.synchronize(device)
        return w4.W4A8MoELayerShared(p13, s13g, p2, s2g, cfg.k, shared)
    return w4.W4A8MoELayer(p13, s13g, p2, s2g, cfg.k)


def max_over_ranks(dist, values, device):
    """Element-wise max over all ranks of a list of timings (every rank calls it,
    at the same point): the job is as slow as its slowest rank."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def whole_job_throughput(tokens_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Tokens of all ranks over all timed steps per second of the (max-over-ranks) time."""
    return tokens_per_rank * world * steps / (ms / 1e3)


def kernel_source_id() -> str:
    """Git blob id of the grouped GEMM source, which keys the DRAM traffic records."""
    path = os.path.join(ROOT, "w4a8_quantized_moe_b200", "csrc", "grouped_gemm.cu")
    data = open(path, "rb").read()
    return hashlib.sha1(b"blob %d\0" % len(data) + data).hexdigest()


def recorded_traffic(workload: str, kernel: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch from the ncu record in
    profiles/dram_traffic.txt, or None when there is none for this workload and
    kernel or the kernel source has changed since it was taken.  The workload is
    the config name, with ":<variant>" appended for variants other than w4a8."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sid = kernel_source_id()
    for ln in open(path):
        f = ln.split()
        if len(f) == 4 and not ln.startswith("#") and f[0] == workload and f[1] == kernel:
            return float(f[2]) if f[3] == sid else None
    return None


def algorithmic_work(cfg, counts, variant: str = "w4a8"):
    """Algorithmic bytes and FLOPs of each grouped GEMM for the given expert counts."""
    T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
    A = T * k
    active = int(np.count_nonzero(counts))
    if variant == "channel-int8":   # one bf16 scale and one int32 nibble sum per row
        w13_bytes = 2 * I * H // 2 + 2 * I * (2 + 4)
        w2_bytes = H * I // 2 + H * (2 + 4)
    else:                           # one bf16 scale per 128-wide group
        w13_bytes = 2 * I * H // 2 + 2 * I * (H // 128) * 2
        w2_bytes = H * I // 2 + H * (I // 128) * 2
    g1 = dict(bytes=active * w13_bytes + T * H + T * 4 + A * I * 4 + A * 4 + A * 8,
              flops=2 * A * 2 * I * H)
    g2 = dict(bytes=active * w2_bytes + A * I + A * 4 + A * H * 4, flops=2 * A * H * I)
    return g1, g2, active


def shared_work(cfg):
    """Algorithmic bytes and FLOPs of the shared expert's two GEMMs (E4M3 weights,
    one float32 scale per 128 x 128 block, per-token-group activation scales)."""
    T, H, I = cfg.T, cfg.H, cfg.I
    s1 = dict(bytes=2 * I * H + (2 * I // 128) * (H // 128) * 4 + T * H + T * (H // 128) * 4
              + T * I * 4, flops=2 * T * 2 * I * H)
    s2 = dict(bytes=H * I + (H // 128) * (I // 128) * 4 + T * I + T * (I // 128) * 4 + T * H * 4,
              flops=2 * T * H * I)
    return s1, s2


class OracleSample:
    """The CPU oracle on a seeded sample of tokens, experts quantised up front."""

    def __init__(self, cfg, n_tokens: int, seed_tokens: int = 7, variant: str = "w4a8"):
        import oracle
        self.oracle, self.cfg = oracle, cfg
        self.act_format = "int8" if variant == "channel-int8" else "fp8"
        self.shared = None
        try:
            from threadpoolctl import threadpool_info
            self.cores = max((p.get("num_threads", 1) for p in threadpool_info()), default=None)
        except Exception:
            self.cores = None
        self.cores = self.cores or os.cpu_count()
        f = lambda t: oracle.bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy()
                                              .view(np.uint16))
        self.hidden = f(workloads.gen_hidden(cfg))
        self.logits = workloads.gen_logits(cfg).numpy()
        rng = np.random.default_rng(seed_tokens)
        self.tokens = np.sort(rng.choice(cfg.T, size=min(n_tokens, cfg.T), replace=False))
        ids, _ = oracle.route_topk(self.logits, cfg.k)

        def weights(e):
            a, b = workloads.gen_expert_weights(cfg, e)
            return f(a), f(b)

        self.store = oracle.ExpertStore(
            cfg.E, weights,
            quantize=oracle.rtn_quantize_int4_channel if self.act_format == "int8" else None)
        for e in sorted(set(ids[self.tokens].reshape(-1).tolist())):
            self.store[e]                          # quantise outside the timed region
        if variant == "w4a8+shared":
            a, b = workloads.gen_shared_weights(cfg)
            self.shared = (*oracle.quant_fp8_block(f(a)), *oracle.quant_fp8_block(f(b)))

    def run(self) -> float:
        t0 = time.perf_counter()
        self.oracle.moe_forward(self.hidden, self.logits, self.store, self.cfg.k,
                                tokens=self.tokens, act_format=self.act_format,
                                shared=self.shared)
        return time.perf_counter() - t0

    def describe(self, dt: float) -> str:
        return (f"{len(self.tokens)} of {self.cfg.T} tokens of {self.cfg.name} per step "
                f"(their {self.cfg.k} experts each, RTN-quantised before timing), float64 "
                f"numpy, {dt:.2f} s per step")


def cpu_baseline(cfg, n_tokens: int, variant: str = "w4a8"):
    s = OracleSample(cfg, n_tokens, variant=variant)
    dt = s.run()
    return dict(value=len(s.tokens) / dt, unit="tokens/s", cores=s.cores, kind="oracle",
                sample=s.describe(dt))


def bench_reference(args, cfg, rank):
    if rank != 0:
        return 0
    s = OracleSample(cfg, max(1, args.ref_tokens), variant=args.variant)
    for _ in range(args.warmup):
        s.run()
    times = [s.run() for _ in range(args.steps)]
    tot = sum(times)
    value = len(s.tokens) * args.steps / tot
    line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * tot / args.steps, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=cfg.name, T=cfg.T, H=cfg.H, I=cfg.I, E=cfg.E, k=cfg.k,
                            variant=args.variant, sample_tokens_per_step=len(s.tokens)),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=s.cores, kind="oracle",
                                  sample=s.describe(tot / args.steps)),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG,
                    choices=[c.name for c in workloads.CONFIGS])
    ap.add_argument("--cpu-tokens", type=int, default=2,
                    help="tokens in the oracle sample of cpu_baseline (0: skip)")
    ap.add_argument("--ref-tokens", type=int, default=1,
                    help="tokens per step of the --impl reference arm")
    ap.add_argument("--experts", type=int, default=0,
                    help="run the workload with this many experts instead (a smaller case for "
                         "profiler captures; recorded in config)")
    ap.add_argument("--variant", default="w4a8", choices=["w4a8", "channel-int8", "w4a8+shared"],
                    help="w4a8: group-128 INT4 experts x FP8 E4M3 activations (default); "
                         "channel-int8: per-channel INT4 experts x per-token INT8 activations; "
                         "w4a8+shared: w4a8 plus the FP8 128x128-block shared expert")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with this many tokens instead (a smaller case for "
                         "profiler captures; recorded in config)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    cfg = workloads.config_by_name(args.config)
    if args.experts:
        cfg = cfg.with_(name=f"{cfg.name}_E{args.experts}", E=args.experts,
                        forced_empty=min(cfg.forced_empty, args.experts // 16))
    if args.tokens:
        cfg = cfg.with_(name=f"{cfg.name}_T{args.tokens}", T=args.tokens)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return bench_reference(args, cfg, rank)

    import w4a8_quantized_moe_b200 as w4
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    layer = build_layer(cfg, device, w4, args.variant)
    rank_cfg = cfg.with_(seed=cfg.seed + 7919 * rank)      # each rank its own batch
    hidden = workloads.gen_hidden(rank_cfg, device=device)
    logits = workloads.gen_logits(rank_cfg, device=device)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=device)
    ws = layer.workspace(cfg.T)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)

    shared = args.variant == "w4a8+shared"
    n_ev = 2 * w4.NUM_STAGES + (8 if shared else 0)

    def step(events=None):
        if events:
            # torch only reports elapsed time for events it recorded itself; the
            # library re-records each one at its stage boundary later in the stream
            for e in events:
                e.record(stream)
        kw = {}
        if shared:
            kw["shared_stage_events"] = events[2 * w4.NUM_STAGES:] if events else None
            events = events[:2 * w4.NUM_STAGES] if events else None
        layer(hidden, logits, out=out, aux={"expert_offsets": offsets}, stage_events=events, **kw)

    for _ in range(args.warmup):
        step()
    w4.w4a8_check_device_error(device)
    counts = np.diff(offsets.cpu().numpy().astype(np.int64))

    # ---------------- device-resident timing (kernel path)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
          for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(ev[i])
        t_end.record(stream)
        torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    w4.w4a8_check_device_error(device)
    ms = t_start.elapsed_time(t_end)
    stage_ms = [statistics.mean(ev[i][2 * s].elapsed_time(ev[i][2 * s + 1])
                                for i in range(args.steps)) for s in range(n_ev // 2)]

    # ---------------- end to end through the public API, host buffers
    h_host = hidden.cpu().pin_memory()
    l_host = logits.cpu().pin_memory()
    o_host = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    h_dev = torch.empty_like(hidden)
    l_dev = torch.empty_like(logits)

    def e2e_step():
        h_dev.copy_(h_host, non_blocking=True)
        l_dev.copy_(l_host, non_blocking=True)
        layer(h_dev, l_dev, out=out)
        o_host.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e_start.elapsed_time(e_end)

    if dist:
        ms, e2e_ms, *stage_ms = max_over_ranks(dist, [ms, e2e_ms] + stage_ms, device)

    value = whole_job_throughput(cfg.T, world, args.steps, ms)
    e2e_value = whole_job_throughput(cfg.T, world, args.steps, e2e_ms)

    pk = peaks()
    g1, g2, active = algorithmic_work(cfg, counts, args.variant)
    prefill = cfg.T >= 4096
    gi = 2 if stage_ms[2] >= stage_ms[4] else 4          # dominant kernel: the slower GEMM
    work = g1 if gi == 2 else g2
    kname = "grouped_gemm_gate_up" if gi == 2 else "grouped_gemm_down"
    traffic_key = cfg.name if args.variant == "w4a8" else f"{cfg.name}:{args.variant}"
    if prefill:
        achieved = work["flops"] / (stage_ms[gi] / 1e3) / 1e12
        peak = 2.0 * pk["bf16_sus"]                     # FP8 = 2 x bf16 (nominal ratio)
        roof = dict(bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s",
                    frac=achieved / peak, traffic=recorded_traffic(traffic_key, kname), kernel=kname,
                    peak_source=f"{pk['src']} sustained bf16 x 2")
    else:
        achieved = work["bytes"] / (stage_ms[gi] / 1e3) / 1e9
        peak = pk["hbm"]
        roof = dict(bound="hbm", achieved=achieved, peak=peak, unit="GB/s", frac=achieved / peak,
                    traffic=recorded_traffic(traffic_key, kname), kernel=kname,
                    peak_source=f"{pk['src']} HBM copy")

    line = dict(
        metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms / args.steps, higher_is_better=True, scaling="weak",
        vs_baseline=None,
        dtype="s8xint4-s32acc" if args.variant == "channel-int8" else "e4m3xint4-f32acc",
        data="synthetic",
        config=dict(workload=cfg.name, T=cfg.T, H=cfg.H, I=cfg.I, E=cfg.E, k=cfg.k,
                    variant=args.variant, active_experts=active,
                    parallelism=f"dp{world}" if world > 1 else "single",
                    l2=("inputs larger than L2: %.2f GB of packed experts streamed per step"
                        % ((g1["bytes"] + g2["bytes"]) / 1e9))),
        stage_ms={n: round(x, 5) for n, x in
                  zip(w4.STAGE_NAMES + (w4.SHARED_STAGE_NAMES if shared else []), stage_ms)},
        roofline=roof,
        e2e=dict(value=e2e_value, unit="tokens/s",
                 h2d_bytes_per_step=cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4,
                 d2h_bytes_per_step=cfg.T * cfg.H * 2),
        gpu_launches=(KERNELS_PER_STEP + (SHARED_KERNELS_PER_STEP if shared else 0)) * args.steps,
        clocks=clk.summary(),
    )
    if shared:   # the shared expert's slower GEMM against the same peak
        s1, s2 = shared_work(cfg)
        # stages 6..9: shared input quantisation, gate/up GEMM, requantisation, down GEMM
        si = 1 if stage_ms[7] >= stage_ms[9] else 3
        sw_, st_ = (s1, stage_ms[7]) if si == 1 else (s2, stage_ms[9])
        sname = "shared_gemm_gate_up" if si == 1 else "shared_gemm_down"
        if prefill:
            a_ = sw_["flops"] / (st_ / 1e3) / 1e12
            line["shared_roofline"] = dict(bound="tensor", achieved=a_, peak=roof["peak"],
                                           unit="TFLOP/s", frac=a_ / roof["peak"], kernel=sname)
        else:
            a_ = sw_["bytes"] / (st_ / 1e3) / 1e9
            line["shared_roofline"] = dict(bound="hbm", achieved=a_, peak=roof["peak"],
                                           unit="GB/s", frac=a_ / roof["peak"], kernel=sname)
    if rank == 0 and world == 1 and args.cpu_tokens > 0:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_tokens, args.variant)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
