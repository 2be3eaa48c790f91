"""Benchmark of the W4A8 routed-expert MoE layer on B200.

One step = one ``w4a8_moe_forward`` (activation quantisation, routing +
permutation, gate/up grouped GEMM + SwiGLU, intermediate requantisation, down
grouped GEMM, combine) over one batch of synthetic tokens.  Prints one JSON
line: the headline workload (decode, 64 tokens, by default) and, on one GPU,
a ``per_config`` entry for every workload.  ``--impl reference`` times the
CPU oracle instead (the only other place this script runs ``oracle/``).

Multi-GPU: one process per GPU (torchrun).  ``--parallel ep`` (the default
for more than one GPU): expert parallelism -- each rank holds E / N of the
experts and its own batch of tokens; the step all-gathers the quantised
tokens, runs each rank's experts on them and reduce-scatters the partial
sums (NCCL).  ``--parallel replicas``: every rank holds all experts and runs
its own batch with no collective on the data path.  Both are weak scaling:
value = all ranks' tokens / max-over-ranks time.
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
# expert-parallel step: act quant, top-k, then local hist/scan/scatter, gather,
# gemm1, inter_quant, gemm2, partial combine, and the final bf16 cast (each
# GEMM twice under split tiling)
EP_KERNELS_PER_STEP = 11
# the all-to-all(v) dispatch adds the plan and the send-row gather; its
# combine of the returned rows takes the place of the bf16 cast
EP_A2A_EXTRA_KERNELS = 2
L2_BYTES = 126 * 10**6
SEGMENT_BINS = [(0, 0), (1, 8), (9, 32), (33, 128), (129, 512), (513, 2048), (2049, 1 << 31)]


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


def build_layer(cfg, device, w4, variant: str = "w4a8", experts=None):
    """Pack the seeded bf16 weights of every expert (or of the range ``experts`` =
    (begin, count), for one expert-parallel rank) on the device and lay them out
    for the GEMMs (not timed)."""
    H, I = cfg.H, cfg.I
    e0, E = experts if experts is not None else (0, cfg.E)
    if variant == "channel-int8":
        p13 = torch.empty(E, 2 * I, H // 8, dtype=torch.int32, device=device)
        s13 = torch.empty(E, 2 * I, dtype=torch.bfloat16, device=device)
        p2 = torch.empty(E, H, I // 8, dtype=torch.int32, device=device)
        s2 = torch.empty(E, H, dtype=torch.bfloat16, device=device)
        for e in range(E):
            w13, w2 = workloads.gen_expert_weights(cfg, e0 + e, device=device)
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
        w13, w2 = workloads.gen_expert_weights(cfg, e0 + e, device=device)
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


def shared_fused(w4, cfg, variant: str) -> bool:
    """Whether the library runs the shared expert's GEMMs inside the routed GEMM
    launches for this workload: decode-sized batches (at most 32 tokens per
    expert on average) without split tiling, the default decode shapes, and
    W4A8_SHARED_FUSED not 0."""
    if variant != "w4a8+shared" or os.environ.get("W4A8_SHARED_FUSED", "1") == "0":
        return False
    if int(os.environ.get("W4A8_GEMM_DECODE_SHAPE", "0") or 0) != 0:
        return False
    no_split = w4.w4a8_moe_forward_launches(cfg.T, cfg.E, cfg.k) == KERNELS_PER_STEP
    return cfg.T * cfg.k <= 32 * cfg.E and no_split


def layer_work(cfg, counts, variant: str = "w4a8"):
    """Algorithmic bytes and FLOPs of the whole layer (one step): the HBM bytes
    of every active expert's weights and scales, the hidden states and logits
    read, the output written, and the intermediates that cross HBM between the
    kernels (h written and read as float32, its codes, the float32 Y rows
    written and read); FLOPs 6 A H I."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    A = T * k
    active = int(np.count_nonzero(counts))
    if variant == "channel-int8":
        per_expert = 2 * I * H // 2 + 2 * I * 6 + H * I // 2 + H * 6
    else:
        per_expert = 2 * I * H // 2 + 2 * I * (H // 128) * 2 + H * I // 2 + H * (I // 128) * 2
    nbytes = (active * per_expert + T * H * 2 + T * E * 4 + T * H * 2 + A * I * (4 + 4 + 1)
              + A * H * 4 * 2)
    return dict(bytes=nbytes, flops=6 * A * H * I)


def segment_histogram(counts):
    """Segment sizes (tokens per expert) in bins, with the active count and the maximum."""
    c = np.asarray(counts, dtype=np.int64)
    bins = {(f"{lo}" if lo == hi else f"{lo}-{hi}" if hi < (1 << 31) else f">={lo}"):
            int(np.count_nonzero((c >= lo) & (c <= hi))) for lo, hi in SEGMENT_BINS}
    return dict(bins=bins, active=int(np.count_nonzero(c)), max=int(c.max(initial=0)),
                experts=int(c.size))


def input_digest(hidden: torch.Tensor, logits: torch.Tensor) -> str:
    """sha256 of the generated hidden-state and logit bytes, as the oracle sees them."""
    h = hashlib.sha256()
    for t in (hidden, logits):
        h.update(t.contiguous().view(torch.uint8).cpu().numpy().tobytes())
    return h.hexdigest()


def roofline(work, ms, prefill: bool, pk, kernel=None, traffic=None):
    """Achieved / peak for ``work`` (dict with bytes and flops) done in ``ms``:
    HBM bytes against the measured copy bandwidth for decode-shaped batches,
    FLOPs against the FP8 dense rate (2 x the measured bf16 GEMM rate, the
    nominal FP8 / bf16 ratio) for prefill-shaped ones."""
    if prefill:
        achieved = work["flops"] / (ms / 1e3) / 1e12
        peak, peak_sus = 2.0 * pk["bf16"], 2.0 * pk["bf16_sus"]
        out = dict(bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s",
                   frac=achieved / peak, frac_of_sustained=achieved / peak_sus,
                   peak_source=f"{pk['src']} bf16 GEMM burst x 2 (FP8 dense); sustained x 2 = "
                               f"{peak_sus:.1f}")
    else:
        achieved = work["bytes"] / (ms / 1e3) / 1e9
        out = dict(bound="hbm", achieved=achieved, peak=pk["hbm"], unit="GB/s",
                   frac=achieved / pk["hbm"], peak_source=f"{pk['src']} HBM copy")
    if kernel is not None:
        out["kernel"] = kernel
        out["traffic"] = traffic
    return out


class OracleSample:
    """The CPU oracle on a seeded sample of tokens, experts quantised up front."""

    MAX_ROWS = 256

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
        # the tokens are drawn from the first rows of the workload's generator
        # (same recipe; generating all T rows on the host would dominate)
        self.rows = min(cfg.T, self.MAX_ROWS)
        self.hidden = f(workloads.gen_hidden(cfg, T=self.rows))
        self.logits = workloads.gen_logits(cfg, T=self.rows).numpy()
        rng = np.random.default_rng(seed_tokens)
        self.tokens = np.sort(rng.choice(self.rows, size=min(n_tokens, self.rows),
                                         replace=False))
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
                f"(drawn from the generator's first {self.rows} rows; their {self.cfg.k} "
                f"experts each, RTN-quantised before timing), float64 numpy, {dt:.2f} s per step")


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


def run_single(cfg, args, device, w4, cpu_tokens: int):
    """One workload on one GPU: device-timed steps with per-stage events and
    clock samples, then the end-to-end loop through host buffers.  Returns the
    fields of the JSON line for this workload."""
    layer = build_layer(cfg, device, w4, args.variant)
    hidden = workloads.gen_hidden(cfg, device=device)
    logits = workloads.gen_logits(cfg, device=device)
    digest = input_digest(hidden, logits) if args.digest else None
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=device)
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

    # per-stage CUDA events (the stage breakdown and the dominant kernel's time)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
          for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    t_start.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize(device)
    w4.w4a8_check_device_error(device)
    ms_eager = t_start.elapsed_time(t_end)
    stage_ms = [statistics.mean(ev[i][2 * s_].elapsed_time(ev[i][2 * s_ + 1])
                                for i in range(args.steps)) for s_ in range(n_ev // 2)]

    # the timed steps: the same forward captured once as a CUDA graph and
    # replayed (the library's kernels without the per-call host work)
    graph = w4.capture_graph(lambda: layer(hidden, logits, out=out))
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            graph.replay()
        t_end.record(stream)
        torch.cuda.synchronize(device)
    w4.w4a8_check_device_error(device)
    ms = t_start.elapsed_time(t_end)

    # end to end: inputs copied in from pinned host memory and the output read
    # back every step, each step waiting for its output on the host before the
    # next one starts (the graph reads the buffers the copies fill)
    h_host = hidden.cpu().pin_memory()
    l_host = logits.cpu().pin_memory()
    o_host = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    done = torch.cuda.Event()

    def e2e_step():
        hidden.copy_(h_host, non_blocking=True)
        logits.copy_(l_host, non_blocking=True)
        graph.replay()
        o_host.copy_(out, non_blocking=True)
        done.record(stream)
        done.synchronize()

    for _ in range(args.warmup):
        e2e_step()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e_start.elapsed_time(e_end)

    pk = peaks()
    g1, g2, active = algorithmic_work(cfg, counts, args.variant)
    prefill = cfg.T >= 4096
    gi = 2 if stage_ms[2] >= stage_ms[4] else 4          # dominant kernel: the slower GEMM
    kname = "grouped_gemm_gate_up" if gi == 2 else "grouped_gemm_down"
    traffic_key = cfg.name if args.variant == "w4a8" else f"{cfg.name}:{args.variant}"
    del graph
    res = dict(
        cfg=cfg, ms=ms, ms_eager=ms_eager, e2e_ms=e2e_ms, stage_ms=stage_ms, counts=counts,
        active=active,
        roofline=roofline(g1 if gi == 2 else g2, stage_ms[gi], prefill, pk, kname,
                          recorded_traffic(traffic_key, kname)),
        roofline_layer=roofline(layer_work(cfg, counts, args.variant), ms / args.steps, prefill,
                                pk),
        clocks=clk.summary(), digest=digest, l2_bytes=g1["bytes"] + g2["bytes"])
    if shared and shared_fused(w4, cfg, args.variant):
        # one launch per projection carries both experts' tiles: the dominant
        # launch's work is the routed projection's plus the shared expert's
        s1, s2 = shared_work(cfg)
        fw = {k_: (g1 if gi == 2 else g2)[k_] + (s1 if gi == 2 else s2)[k_]
              for k_ in ("bytes", "flops")}
        res["roofline"] = roofline(fw, stage_ms[gi], prefill, pk,
                                   kname + " (with the shared expert)")
        res["shared_fused"] = True
    elif shared:   # the shared expert's slower GEMM against the same peak
        s1, s2 = shared_work(cfg)
        # stages 6..9: shared input quantisation, gate/up GEMM, requantisation, down GEMM
        si = 1 if stage_ms[7] >= stage_ms[9] else 3
        sw_, st_ = (s1, stage_ms[7]) if si == 1 else (s2, stage_ms[9])
        res["shared_roofline"] = roofline(sw_, st_, prefill, pk,
                                          "shared_gemm_gate_up" if si == 1 else "shared_gemm_down")
    if cpu_tokens > 0:
        res["cpu_baseline"] = cpu_baseline(cfg, cpu_tokens, args.variant)
    del layer
    return res


def step_launches(w4, cfg, variant: str) -> int:
    """This library's kernel launches in one step of the variant."""
    if variant == "channel-int8":
        return KERNELS_PER_STEP
    n = w4.w4a8_moe_forward_launches(cfg.T, cfg.E, cfg.k)
    if variant != "w4a8+shared":
        return n
    # the shared GEMMs inside the routed launches: tables and the two quantisers
    return n + (SHARED_KERNELS_PER_STEP - 2 if shared_fused(w4, cfg, variant)
                else SHARED_KERNELS_PER_STEP)


def config_fields(cfg, res, args, world=1, parallelism="single"):
    streamed = res["l2_bytes"]
    c = dict(workload=cfg.name, T=cfg.T, H=cfg.H, I=cfg.I, E=cfg.E, k=cfg.k,
             variant=args.variant, active_experts=res["active"], parallelism=parallelism,
             segments=segment_histogram(res["counts"]),
             l2=(("inputs larger than L2: %.2f GB of packed experts streamed per step"
                  % (streamed / 1e9)) if streamed > L2_BYTES else
                 ("L2-resident: %.1f MB of packed experts fit in the %d MB L2, so the HBM "
                  "roofline fraction means nothing here" % (streamed / 1e6, L2_BYTES // 10**6))),
             timed_as="CUDA graph replay of the forward (stage_ms from a separate eager pass "
                      "with per-stage events, %.4f ms per step)" % (res["ms_eager"] / args.steps))
    if res.get("digest"):
        c["inputs_sha256"] = res["digest"]
    if args.variant == "w4a8+shared":
        c["shared_gemms"] = ("second phase of the routed GEMM launches" if res.get("shared_fused")
                             else "launches of their own")
    return c


def stage_names(w4, shared):
    return w4.STAGE_NAMES + (w4.SHARED_STAGE_NAMES if shared else [])


def run_expert_parallel(cfg, args, device, w4, dist, rank, world):
    """Expert parallelism over the ranks: rank g holds experts
    expert_partition(E, world)[g] and its own batch of cfg.T tokens."""
    from w4a8_quantized_moe_b200.ep import ExpertParallelMoE, expert_partition
    b, n = expert_partition(cfg.E, world)[rank]
    local = build_layer(cfg, device, w4, experts=(b, n)) if n else None
    weights = ((local.w13_packed, local.w13_scales, local.w2_packed, local.w2_scales)
               if local is not None else None)
    ep = ExpertParallelMoE(weights, cfg.E, cfg.k, b, n, cfg.H, cfg.I, tokens_per_rank=cfg.T,
                           dispatch=args.ep_dispatch)
    rank_cfg = cfg.with_(seed=cfg.seed + 7919 * rank)      # each rank its own batch
    hidden = workloads.gen_hidden(rank_cfg, device=device)
    logits = workloads.gen_logits(rank_cfg, device=device)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        ep(hidden, logits, out=out)
    w4.w4a8_check_device_error(device)
    # the rows this rank's experts serve: every rank's routed ids (each rank's
    # batch comes from its own seed, so they are routed again here, untimed)
    all_ids = [w4.w4a8_moe_route_topk(workloads.gen_logits(cfg.with_(seed=cfg.seed + 7919 * g),
                                                           device=device), cfg.k)[0]
               for g in range(world)]
    gat_ids = torch.cat(all_ids).cpu().numpy()
    local_counts = np.array([np.count_nonzero(gat_ids == e) for e in range(b, b + n)])
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        t_start.record(stream)
        for _ in range(args.steps):
            ep(hidden, logits, out=out)
        t_end.record(stream)
        torch.cuda.synchronize(device)
    dist.barrier()
    w4.w4a8_check_device_error(device)
    ms = t_start.elapsed_time(t_end)

    h_host = hidden.cpu().pin_memory()
    l_host = logits.cpu().pin_memory()
    o_host = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    h_dev, l_dev = torch.empty_like(hidden), torch.empty_like(logits)
    done = torch.cuda.Event()

    def e2e_step():
        h_dev.copy_(h_host, non_blocking=True)
        l_dev.copy_(l_host, non_blocking=True)
        ep(h_dev, l_dev, out=out)
        o_host.copy_(out, non_blocking=True)
        done.record(stream)
        done.synchronize()

    for _ in range(args.warmup):
        e2e_step()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(device)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e_start.elapsed_time(e_end)
    dist.barrier()
    return dict(ms=ms, e2e_ms=e2e_ms, local_counts=local_counts, experts=(b, n),
                clocks=clk.summary())


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
    ap.add_argument("--per-config", type=int, default=1,
                    help="on one GPU, also time every other workload into per_config (0: no)")
    ap.add_argument("--parallel", default="ep", choices=["ep", "replicas"],
                    help="more than one GPU: expert parallelism (default) or full replicas")
    ap.add_argument("--ep-dispatch", default="all_gather", choices=["all_gather", "all_to_all"],
                    help="expert parallelism: all-gather every token to every rank (default) or "
                         "all-to-all(v) each token to the ranks of its experts")
    ap.add_argument("--digest", type=int, default=1,
                    help="log the sha256 of each workload's generated inputs (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    cfg = workloads.config_by_name(args.config)
    custom = bool(args.experts or args.tokens)
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
    dtype = "s8xint4-s32acc" if args.variant == "channel-int8" else "e4m3xint4-f32acc"
    shared = args.variant == "w4a8+shared"

    if world == 1:
        head = run_single(cfg, args, device, w4, args.cpu_tokens)
        line = dict(
            metric=METRIC, value=whole_job_throughput(cfg.T, 1, args.steps, head["ms"]),
            unit="tokens/s", n_gpus=1, steps=args.steps, warmup=args.warmup,
            ms_per_step=head["ms"] / args.steps, higher_is_better=True, scaling="weak",
            vs_baseline=None, dtype=dtype, data="synthetic",
            config=config_fields(cfg, head, args),
            stage_ms={n_: round(x, 5) for n_, x in zip(stage_names(w4, shared), head["stage_ms"])},
            roofline=head["roofline"], roofline_layer=head["roofline_layer"],
            e2e=dict(value=whole_job_throughput(cfg.T, 1, args.steps, head["e2e_ms"]),
                     unit="tokens/s", h2d_bytes_per_step=cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4,
                     d2h_bytes_per_step=cfg.T * cfg.H * 2, host_round_trip_per_step=True),
            gpu_launches=step_launches(w4, cfg, args.variant) * args.steps,
            clocks=head["clocks"])
        if "shared_roofline" in head:
            line["shared_roofline"] = head["shared_roofline"]
        if "cpu_baseline" in head:
            line["cpu_baseline"] = head["cpu_baseline"]
        if args.per_config and not custom:
            per = {}
            for c in workloads.CONFIGS:
                r = head if c.name == cfg.name else run_single(c, args, device, w4, 1)
                torch.cuda.empty_cache()
                per[c.name] = dict(
                    ms_per_step=r["ms"] / args.steps,
                    tokens_per_s=whole_job_throughput(c.T, 1, args.steps, r["ms"]),
                    e2e_tokens_per_s=whole_job_throughput(c.T, 1, args.steps, r["e2e_ms"]),
                    stage_ms={n_: round(x, 5) for n_, x in
                              zip(stage_names(w4, shared), r["stage_ms"])},
                    roofline=r["roofline"], roofline_layer=r["roofline_layer"],
                    config=config_fields(c, r, args), clocks=r["clocks"],
                    gpu_launches=step_launches(w4, c, args.variant) * args.steps)
                if "cpu_baseline" in r:
                    per[c.name]["cpu_baseline"] = r["cpu_baseline"]
                if "shared_roofline" in r:
                    per[c.name]["shared_roofline"] = r["shared_roofline"]
            line["per_config"] = per
        print(json.dumps(line), flush=True)
        return 0

    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        if args.parallel == "ep":
            from w4a8_quantized_moe_b200.ep import expert_partition
            if args.variant != "w4a8":
                raise SystemExit("--parallel ep runs the w4a8 variant only")
            r = run_expert_parallel(cfg, args, device, w4, dist, rank, world)
            ms, e2e_ms = max_over_ranks(dist, [r["ms"], r["e2e_ms"]], device)
            b, n = r["experts"]
            pk = peaks()
            T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
            Tg = T * world
            per_expert = 2 * I * H // 2 + 2 * I * (H // 128) * 2 + H * I // 2 + H * (I // 128) * 2
            A_loc = int(r["local_counts"].sum())
            work = dict(bytes=int(np.count_nonzero(r["local_counts"])) * per_expert
                        + Tg * H + Tg * 4 + A_loc * I * 9 + A_loc * H * 8 + Tg * H * 4,
                        flops=6 * A_loc * H * I)
            line = dict(
                metric=METRIC, value=whole_job_throughput(T, world, args.steps, ms),
                unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms / args.steps, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype=dtype, data="synthetic",
                config=dict(workload=cfg.name, T=T, H=H, I=I, E=cfg.E, k=k, variant=args.variant,
                            parallelism=f"ep{world}", tokens_per_rank=T,
                            experts_per_rank=[n_ for _, n_ in expert_partition(cfg.E, world)],
                            rank0_experts_served=int(np.count_nonzero(r["local_counts"])),
                            dispatch=("all-gather of E4M3 codes, scales, ids, weights (NCCL)"
                                      if args.ep_dispatch == "all_gather" else
                                      "all-to-all(v) of each token's E4M3 codes, scale, ids, "
                                      "weights to the ranks of its experts (NCCL)"),
                            combine=("reduce-scatter of float32 partial sums (NCCL)"
                                     if args.ep_dispatch == "all_gather" else
                                     "all-to-all(v) of float32 partial sums back, summed in "
                                     "rank order")),
                roofline=roofline(work, ms / args.steps, T * world >= 4096, pk,
                                  "ep_step (rank 0: dispatch + local experts + combine)"),
                e2e=dict(value=whole_job_throughput(T, world, args.steps, e2e_ms),
                         unit="tokens/s", h2d_bytes_per_step=world * (T * H * 2 + T * cfg.E * 4),
                         d2h_bytes_per_step=world * T * H * 2, host_round_trip_per_step=True),
                gpu_launches=(EP_KERNELS_PER_STEP + w4.w4a8_moe_forward_launches(
                    T * world, cfg.E, k) - KERNELS_PER_STEP
                    + (EP_A2A_EXTRA_KERNELS if args.ep_dispatch == "all_to_all" else 0))
                * args.steps,
                clocks=r["clocks"])
        else:
            layer = build_layer(cfg, device, w4, args.variant)
            rank_cfg = cfg.with_(seed=cfg.seed + 7919 * rank)
            hidden = workloads.gen_hidden(rank_cfg, device=device)
            logits = workloads.gen_logits(rank_cfg, device=device)
            out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=device)
            stream = torch.cuda.current_stream(device)
            for _ in range(args.warmup):
                layer(hidden, logits, out=out)
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            dist.barrier()
            torch.cuda.synchronize(device)
            with ClockSampler(device) as clk:
                t0.record(stream)
                for _ in range(args.steps):
                    layer(hidden, logits, out=out)
                t1.record(stream)
                torch.cuda.synchronize(device)
            dist.barrier()
            w4.w4a8_check_device_error(device)
            (ms,) = max_over_ranks(dist, [t0.elapsed_time(t1)], device)
            line = dict(
                metric=METRIC, value=whole_job_throughput(cfg.T, world, args.steps, ms),
                unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms / args.steps, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype=dtype, data="synthetic",
                config=dict(workload=cfg.name, T=cfg.T, H=cfg.H, I=cfg.I, E=cfg.E, k=cfg.k,
                            variant=args.variant, parallelism=f"replicas{world}"),
                gpu_launches=KERNELS_PER_STEP * args.steps, clocks=clk.summary())
        dist.barrier()
    finally:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
