"""Benchmark of the GDN layer on B200: prefill tokens/s and decode GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workloads (synthetic, seeded; see linear_attention_12_b200/inputs.py):
  * prefill: B=1, L=32768, 16 QK / 48 V heads, d=128, bf16 q/k/v, fp32 gates,
    S0 = 0, chunk 64 -- the headline ``value`` (tokens/s, whole job); the same
    prefill with its output state pass on mma.sync instead of tcgen05 -- the
    ``prefill_mma_sync`` object;
  * decode: 256 sequences x 48 V heads (16 QK heads), fp32 states updated in
    place (805 MB) -- reported in the ``decode`` object (GB/s);
  * multi-token decode: 4 tokens per sequence for the same 256 x 48 heads, a
    state checkpoint after each (4.0 GB moved) -- the ``decode_multi`` object;
  * gradients of the same prefill (dq, dk, dv and the gate gradients) -- the
    ``backward`` object (tokens/s and the tensor roofline);
  * prefill of one 8-way tensor-parallel shard (2 QK / 6 V heads, L=32768),
    with and without the library's sequence split -- the ``prefill_shard`` object;
  * front end: the short convolution, q/k normalisation and gate activations
    over the raw inputs of the L=32768 prefill (1.37 GB moved) -- reported in
    the ``frontend`` object (GB/s).
Each rank runs its own replica (the layer shards by sequence and head with no
exchange step; nothing is communicated), so scaling is weak.  Timing: W
untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize(); CUDA events on the launching stream; the max over
ranks is reported.  Inputs (1.09 GB per prefill step, 1.6 GB per decode step)
are larger than L2, so no flush is needed between iterations.

``--impl reference`` times the fp64 CPU oracle (the only reference
implementation there is) on rank 0, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (L=32K, 48 V heads) and decode GB/s vs roofline, 1 B200"
L = 32768  # the benchmarked sequence length (--seq-len overrides it for profiling captures)
H_QK, H_V, D = 16, 48, 128
DEC_B = 256
# Algorithmic bytes: q, k (H_qk*d bf16 each), v and o (H_v*d bf16 each), two fp32 gates
# per V head; plus the final state (H_v * d * d fp32) once per sequence.
BYTES_PER_TOKEN = 2 * H_QK * D * 2 + 2 * H_V * D * 2 + 2 * H_V * 4          # 33,152
STATE_BYTES = H_V * D * D * 4                                                 # 3,145,728
# Algorithmic FLOPs per token per V head: 6 d^2 (W S, Q S, K^T Delta) + 3 C d
# (three triangular C x C x d products at half) + 2 C d / 3 (grams at half,
# shared by the 3 V heads of a QK head), C = 64.
FLOP_PER_TOKEN = H_V * (6 * D * D + 3 * 64 * D + (2 * 64 * D) // 3)
# B200 HBM3e bandwidth as specified (HGX), beside the measured copy peak
HBM_SPEC_GBS = 7700.0


def dec_bytes(B):
    """One decode step: the fp32 states read and written, plus the tokens."""
    return 2 * B * H_V * D * D * 4 + B * (2 * H_QK * D * 2 + 2 * H_V * D * 2 + 2 * H_V * 4)


DEC_BYTES = dec_bytes(DEC_B)
# multi-token decode (speculative verification, M = 4 tokens: 3 drafted + 1):
# the state read once and written after each token, plus the tokens' inputs/outputs
DM_M = 4
def dm_bytes(B):
    return ((1 + DM_M) * B * H_V * D * D * 4
            + B * DM_M * (2 * H_QK * D * 2 + 2 * H_V * D * 2 + 2 * H_V * 4))
# gradients of the prefill, per token: q, k, v, dO and the gates read, dq, dk, dv and
# the gate gradients written; FLOPs of the chunk form per (chunk, value head):
# forward re-run 4 C d^2 + 2 C^2 d, reverse chain 6 C d^2 + 4 C^2 d, per-chunk
# gradients 12 C d^2 + 20 C^2 d + 4 C^3  (C = 64)
BW_BYTES_PER_TOKEN = (2 * H_QK * D * 2 + 2 * H_V * D * 2 + 2 * H_V * 4) + \
                     (2 * H_QK * D * 2 + H_V * D * 2 + 2 * H_V * 4)                  # 53,504
BW_FLOP_PER_TOKEN = H_V * (22 * D * D + 26 * 64 * D + 4 * 64 * 64)                  # 28.3 M
# front end, per token: raw q, k, v read and normalised q, k, v written (bf16),
# a, b read and log_alpha, beta written (fp32); plus the conv weight once
FE_BYTES_PER_TOKEN = 2 * (2 * H_QK + H_V) * D * 2 + 4 * H_V * 4                # 41,728
FE_WEIGHT_BYTES = (2 * H_QK + H_V) * D * 4 * 4                                  # 163,840


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region.

    Reads NVML every ~2 ms from a thread (nvidia-smi's 200 ms loop would see
    at most one sample of a region that lasts tens of milliseconds); only
    samples taken between __enter__ and __exit__ count.  Falls back to
    ``nvidia-smi -lms 200`` when NVML cannot be opened.  Only reads settings.
    """

    # NVML clock-event reason bits -> names used in the output
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []       # (time, sm_mhz, reason bits)
        self.max_mhz = None
        self.source = None
        self.proc = None
        self.smi_lines = []
        self._stop = threading.Event()
        self.t_start = self.t_stop = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.gpu)
        try:
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, nv, h):
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.monotonic(), float(mhz), int(bits)))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            t_wait = time.monotonic() + 2.0
            while not self.samples and time.monotonic() < t_wait:
                time.sleep(0.001)
        except Exception:
            self.source = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
                self.thread = threading.Thread(target=self._read_smi, daemon=True)
                self.thread.start()
                time.sleep(0.5)  # let nvidia-smi start before the region
            except (OSError, FileNotFoundError):
                self.proc = None
        self.t_start = time.monotonic()
        return self

    def _read_smi(self):
        for line in self.proc.stdout:
            self.smi_lines.append(line.strip())

    def __exit__(self, *a):
        self.t_stop = time.monotonic()
        self._stop.set()
        if self.proc is not None:
            time.sleep(0.3)  # one more nvidia-smi sample
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        elif self.source == "nvml":
            self.thread.join(timeout=1.0)

    def summary(self):
        if self.source == "nvml":
            inside = [(m, b) for t, m, b in self.samples if self.t_start <= t <= self.t_stop]
            if not inside:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["not recorded"],
                        "source": "nvml"}
            reasons = sorted({nm for _, b in inside for bit, nm in self.REASONS.items() if b & bit})
            return {"sm_mhz": statistics.median(m for m, _ in inside), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(inside), "source": "nvml"}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.smi_lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["not recorded"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_decode(args, dev, stream, world):
    """Time decode steps on the 256-sequence workload; returns (ms per step, GB/s)."""
    import torch
    from linear_attention_12_b200 import gdn, inputs
    B = args.decode_batch
    dc = inputs.make_decode(B, H_QK, H_V, D, seed=4)
    S = dc.S0.to(dev)
    dq, dk_, dv_, dla, dbe = (x.to(dev) for x in dc.step(0))
    do = torch.empty((B, H_V, D), dtype=torch.bfloat16, device=dev)
    dec_steps = max(args.steps, 20)
    for _ in range(max(args.warmup, 3)):
        gdn.decode_step(dq, dk_, dv_, dla, dbe, S, o=do)
    torch.cuda.synchronize()
    barrier(world)
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(dec_steps):
        gdn.decode_step(dq, dk_, dv_, dla, dbe, S, o=do)
    d1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    dec_ms = max_over_ranks(d0.elapsed_time(d1), world) / dec_steps
    assert gdn.last_device_error() == gdn.GDN_OK
    return dec_ms, dec_bytes(B) / (dec_ms / 1e3) / 1e9


def run_decode_multi(args, dev, stream, world):
    """Time M = 4 token verification steps on the 256-sequence workload;
    returns (ms per call, GB/s)."""
    import torch
    from linear_attention_12_b200 import gdn, inputs
    B = args.decode_batch
    dc = inputs.make_decode(B, H_QK, H_V, D, seed=4)
    S_in = dc.S0.to(dev)
    win = [x.to(dev) for x in dc.window(0, DM_M)]
    o = torch.empty((B, DM_M, H_V, D), dtype=torch.bfloat16, device=dev)
    S_steps = torch.empty((B, DM_M, H_V, D, D), dtype=torch.float32, device=dev)
    n = max(args.steps, 10)
    for _ in range(max(args.warmup, 3)):
        gdn.decode_multi(*win, S_in, o=o, S_steps=S_steps)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        gdn.decode_multi(*win, S_in, o=o, S_steps=S_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / n
    assert gdn.last_device_error() == gdn.GDN_OK
    return ms, dm_bytes(B) / (ms / 1e3) / 1e9


def run_prefill_shard(args, dev, stream, world, L):
    """The prefill of one tensor-parallel shard (1/8 of the heads: 2 QK, 6 V),
    with the library's automatic sequence split and without it; returns
    (segments, ms with the split, ms without)."""
    import torch
    from linear_attention_12_b200 import gdn, inputs
    hq, hv = H_QK // 8, H_V // 8
    case = inputs.make_prefill(f"prefill_shard_L{L}", [L], hq, hv, seed=6)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    la, be, cu = case.log_alpha.to(dev), case.beta.to(dev), case.cu_seqlens.to(dev)
    o = torch.empty((L, hv, D), dtype=torch.bfloat16, device=dev)
    Sf = torch.empty((1, hv, D, D), dtype=torch.float32, device=dev)
    seg = gdn.auto_segments(1, L, hq, hv)
    out = []
    for s in (0, 1):
        ws = torch.empty(max(gdn.workspace_size(1, L, hq, hv, segments=s), 256),
                         dtype=torch.uint8, device=dev)
        for _ in range(max(args.warmup, 3)):
            gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws, segments=s)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n = max(args.steps, 10)
        e0.record(stream)
        for _ in range(n):
            gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws, segments=s)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        out.append(max_over_ranks(e0.elapsed_time(e1), world) / n)
        assert gdn.last_device_error() == gdn.GDN_OK
    return seg, out[0], out[1]


def run_backward(args, case, dev, stream, world, L):
    """Time the gradients of the L-token prefill (the same inputs): the recomputing
    backward, and the training pair (saving forward, backward from the saved
    states).  Returns (ms per backward, calls, ms per training forward, ms per
    saved backward)."""
    import torch
    from linear_attention_12_b200 import gdn
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    la, be, cu = case.log_alpha.to(dev), case.beta.to(dev), case.cu_seqlens.to(dev)
    gen = torch.Generator().manual_seed(7)
    dO = torch.randn((L, H_V, D), generator=gen).to(torch.bfloat16).to(dev)
    ws = torch.empty(int(gdn.lib().gdn_prefill_backward_workspace_size(1, L, H_QK, H_V, D, D,
                                                                      gdn.GDN_BF16)),
                     dtype=torch.uint8, device=dev)
    n = max(3, min(args.steps, 10))
    for _ in range(max(args.warmup, 3)):
        gdn.prefill_backward(q, k, v, la, be, dO, cu_seqlens=cu, workspace=ws)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        gdn.prefill_backward(q, k, v, la, be, dO, cu_seqlens=cu, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    assert gdn.last_device_error() == gdn.GDN_OK
    bw_ms = max_over_ranks(e0.elapsed_time(e1), world) / n

    # a training step: the saving forward, then the gradients from its saved states
    o, Sf = torch.empty_like(v), torch.empty((1, H_V, D, D), dtype=torch.float32, device=dev)

    def train_fwd():
        gdn.prefill_train(q, k, v, la, be, cu_seqlens=cu, o=o, S_final=Sf, workspace=ws)

    def train_bwd():
        gdn.prefill_backward(q, k, v, la, be, dO, cu_seqlens=cu, workspace=ws, saved=True)

    for _ in range(max(args.warmup, 3)):
        train_fwd()
        train_bwd()
    torch.cuda.synchronize()
    barrier(world)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    fwd_ms = bwd_ms = 0.0
    for _ in range(n):
        ev[0].record(stream)
        train_fwd()
        ev[1].record(stream)
        train_bwd()
        ev[2].record(stream)
        torch.cuda.synchronize()
        fwd_ms += ev[0].elapsed_time(ev[1])
        bwd_ms += ev[1].elapsed_time(ev[2])
    barrier(world)
    assert gdn.last_device_error() == gdn.GDN_OK
    return (bw_ms, n, max_over_ranks(fwd_ms / n, world), max_over_ranks(bwd_ms / n, world))


def run_frontend(args, dev, stream, world, L):
    """Time the front end on raw inputs of the prefill's shape; returns
    (ms per call, GB/s)."""
    import torch
    from linear_attention_12_b200 import gdn, inputs
    fc = inputs.make_frontend(f"frontend_L{L}", [L], H_QK, H_V, d=D, seed=5)
    qr, kr, vr, a, b, w = (x.to(dev) for x in (fc.q_raw, fc.k_raw, fc.v_raw, fc.a, fc.b,
                                                fc.conv_w))
    del fc
    cu = torch.tensor([0, L], dtype=torch.int32, device=dev)
    out = (torch.empty_like(qr), torch.empty_like(kr), torch.empty_like(vr),
           torch.empty_like(a), torch.empty_like(b))
    fe_steps = max(args.steps, 20)
    for _ in range(max(args.warmup, 3)):
        gdn.frontend(qr, kr, vr, w, a, b, cu, out=out)
    torch.cuda.synchronize()
    barrier(world)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(fe_steps):
        gdn.frontend(qr, kr, vr, w, a, b, cu, out=out)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    fe_ms = max_over_ranks(f0.elapsed_time(f1), world) / fe_steps
    assert gdn.last_device_error() == gdn.GDN_OK
    return fe_ms, (FE_BYTES_PER_TOKEN * L + FE_WEIGHT_BYTES) / (fe_ms / 1e3) / 1e9


def run_e2e(args, case, cu, ws, stream, world, L):
    """Prefill through the public API with the inputs in pinned host memory:
    each step copies q, k, v and the gates in and o and S_final out.  Steps
    are pipelined as a serving loop would run them: the uploads, the prefill
    and the downloads go on three streams over two sets of device buffers, so
    that step i + 1's upload and step i - 1's download overlap step i (PCIe
    copies run both ways at once).  Timed from the first upload to the last
    download."""
    import torch
    from linear_attention_12_b200 import gdn
    dev = cu.device
    hin = [x.pin_memory() for x in (case.q, case.k, case.v, case.log_alpha, case.beta)]
    ho = torch.empty((L, H_V, D), dtype=torch.bfloat16).pin_memory()
    hS = torch.empty((1, H_V, D, D), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = ho.numel() * ho.element_size() + hS.numel() * hS.element_size()
    din = [[torch.empty_like(x, device=dev) for x in hin] for _ in range(2)]
    dout = [(torch.empty((L, H_V, D), dtype=torch.bfloat16, device=dev),
             torch.empty((1, H_V, D, D), dtype=torch.float32, device=dev)) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    read_done = [None, None]    # the prefill that last read input set b
    drained = [None, None]      # the download that last read output set b

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if read_done[b] is not None:
                s_in.wait_event(read_done[b])
            for d, h in zip(din[b], hin):
                d.copy_(h, non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_in)
        stream.wait_event(up)
        if drained[b] is not None:
            stream.wait_event(drained[b])
        q, k, v, la, be = din[b]
        o, Sf = dout[b]
        gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws, stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
        read_done[b] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            ho.copy_(o, non_blocking=True)
            hS.copy_(Sf, non_blocking=True)
            dr = torch.cuda.Event()
            dr.record(s_out)
        drained[b] = dr

    e2e_steps = max(4, min(args.steps, 10))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    assert gdn.last_device_error() == gdn.GDN_OK
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    return world * L / (e2e_ms / 1e3), e2e_ms, h2d, d2h


def run_prefill_workload(args, case, dev, stream, world):
    """Time gdn_prefill on one workload (inputs resident in HBM, workspace
    allocated outside the timing); returns ms per call (max over ranks)."""
    import torch
    from linear_attention_12_b200 import gdn
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    la, be = case.log_alpha.to(dev), case.beta.to(dev)
    S0 = None if case.S0 is None else case.S0.to(dev)
    cu = case.cu_seqlens.to(dev)
    o = torch.empty((case.T, H_V, D), dtype=torch.bfloat16, device=dev)
    Sf = torch.empty((case.N, H_V, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.workspace_size(case.N, case.T, H_QK, H_V, D, gdn.GDN_BF16),
                     dtype=torch.uint8, device=dev)

    def step():
        gdn.prefill(q, k, v, la, be, S0, cu, o=o, S_final=Sf, workspace=ws)

    n = max(3, min(args.steps, 10))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    assert gdn.last_device_error() == gdn.GDN_OK
    ms = max_over_ranks(a.elapsed_time(b), world) / n
    del q, k, v, la, be, S0, o, Sf, ws
    torch.cuda.empty_cache()
    return ms, n


def run_prefill_tiny(args, dev, stream, world):
    """The tiny fp32 prefill (B=1, L=256, 1 QK / 1 V head): launch-bound, so timed
    for the record only; returns a line with its CPU baseline (the oracle on the
    whole workload, rank 0 at N=1)."""
    import torch
    from linear_attention_12_b200 import gdn, inputs
    case = inputs.tiny_fp32()
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    la, be, cu = case.log_alpha.to(dev), case.beta.to(dev), case.cu_seqlens.to(dev)
    o = torch.empty((case.T, case.H_v, D), dtype=torch.float32, device=dev)
    Sf = torch.empty((case.N, case.H_v, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, gdn.workspace_size(case.N, case.T, case.H_qk, case.H_v, D,
                                               gdn.GDN_F32)), dtype=torch.uint8, device=dev)

    def step():
        gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws)

    n = 50
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    assert gdn.last_device_error() == gdn.GDN_OK
    us = max_over_ranks(a.elapsed_time(b), world) / n * 1e3
    line = {"value": case.T / (us / 1e6), "unit": "tokens/s", "us_per_call": us,
            "tokens": case.T, "steps": n,
            "workload": "tiny prefill B=1 L=256 H_qk=1 H_v=1 d=128, all fp32, S0=0 "
                        "(launch-bound: three launches, one fp32 -> bf16 copy of q, k, v and the two passes)"}
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        t0 = time.perf_counter()
        oracle.prefill(case.q, case.k, case.v, case.log_alpha, case.beta, None, case.cu_seqlens,
                       n_threads=1)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": case.T / dt, "unit": "tokens/s", "cores": 1,
                                "kind": "oracle", "sample": f"the whole workload, fp64, {dt:.3f} s"}
    del q, k, v, la, be, cu, o, Sf, ws
    return line


def prefill_workload_line(case, ms, steps, hbm_peak, tf_peak, workload, cpu):
    """Throughput and roofline of one prefill workload (bf16 q/k/v, o; fp32 gates,
    states): bytes = the tokens' algorithmic bytes + S0 (if given) + S_final."""
    T, N = case.T, case.N
    nbytes = BYTES_PER_TOKEN * T + (2 if case.S0 is not None else 1) * N * STATE_BYTES
    flops = FLOP_PER_TOKEN * T
    t_hbm = nbytes / (hbm_peak * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    gbs = nbytes / (ms / 1e3) / 1e9
    line = {
        "value": T / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms, "tokens": T,
        "sequences": N, "workload": workload, "steps": steps,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak, "bytes_per_call": nbytes,
                     "roofline_us": max(t_hbm, t_tc) * 1e6, "hbm_term_us": t_hbm * 1e6,
                     "tensor_term_us": t_tc * 1e6},
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def traffic_from_profile(L):
    """DRAM bytes per prefill launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "prefill_traffic.json")
    src = os.path.join(ROOT, "linear_attention_12_b200", "csrc", "gdn_prefill.cu")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if d.get("kernel_source_sha256") != sha:
        return None
    return d["dram_bytes_per_token"] * L + d.get("dram_bytes_fixed", 0)


def run_ours(args):
    import torch
    from linear_attention_12_b200 import gdn, inputs

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, tf_peak, tf_sust, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    # ---------------- prefill workload, inputs resident in HBM
    case = inputs.qwen_prefill_32k(args.seq_len)
    L = args.seq_len
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    la, be = case.log_alpha.to(dev), case.beta.to(dev)
    cu = case.cu_seqlens.to(dev)
    o = torch.empty((L, H_V, D), dtype=torch.bfloat16, device=dev)
    Sf = torch.empty((1, H_V, D, D), dtype=torch.float32, device=dev)

    # the path's workspace (chunk-operator records), allocated once, outside the timing
    ws = torch.empty(gdn.workspace_size(1, L, H_QK, H_V, D, gdn.GDN_BF16), dtype=torch.uint8,
                     device=dev)

    def prefill_step():
        gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws)

    for _ in range(args.warmup):
        prefill_step()
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            prefill_step()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    kern_avg_ms = statistics.mean(kern_ms)
    assert gdn.last_device_error() == gdn.GDN_OK
    ms_per_step = total_ms / args.steps
    value = world * L * args.steps / (total_ms / 1e3)

    bytes_per_launch = BYTES_PER_TOKEN * L + STATE_BYTES
    flops_per_launch = FLOP_PER_TOKEN * L
    achieved_gbs = bytes_per_launch / (kern_avg_ms / 1e3) / 1e9
    t_hbm = bytes_per_launch / (hbm_peak * 1e9)
    t_tc = flops_per_launch / (tf_peak * 1e12)

    # ---------------- the same prefill with its output state pass on mma.sync
    tc_ms = None
    if not args.no_tc:
        def alt_step():
            gdn.prefill(q, k, v, la, be, None, cu, o=o, S_final=Sf, workspace=ws,
                        state_pass="mma_sync")
        for _ in range(args.warmup):
            alt_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            alt_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        assert gdn.last_device_error() == gdn.GDN_OK
        tc_ms = max_over_ranks(a.elapsed_time(b), world) / args.steps

    # ---------------- decode workload (states in place)
    dec_ms = dec_gbs = None
    if not args.no_decode:
        dec_ms, dec_gbs = run_decode(args, dev, stream, world)

    # ---------------- multi-token decode (verification of 3 drafted tokens)
    dm_ms = dm_gbs = None
    if not args.no_decode:
        dm_ms, dm_gbs = run_decode_multi(args, dev, stream, world)

    # ---------------- gradients of the same prefill
    bw = None
    if not args.no_backward:
        bw = run_backward(args, case, dev, stream, world, L)

    # ---------------- prefill of a tensor-parallel shard (few heads: sequence split)
    shard = None
    if not args.no_shard:
        shard = run_prefill_shard(args, dev, stream, world, L)

    # ---------------- the other prefill workloads: packed varlen batch with S0, and
    # the long-context prefill (each timed alone; inputs resident)
    varlen = long_ctx = tiny = None
    if not args.no_workloads:
        tiny = run_prefill_tiny(args, dev, stream, world)
        vcase = inputs.varlen_8seq()
        ms, n = run_prefill_workload(args, vcase, dev, stream, world)
        vcpu = None
        if world == 1 and not args.no_cpu_baseline:
            vcpu = cpu_baseline(vcase, args.cpu_tokens)
        varlen = prefill_workload_line(
            vcase, ms, n, hbm_peak, tf_peak,
            f"packed varlen prefill: {vcase.N} sequences, lengths uniform in [1024, 8192] "
            f"(T={vcase.T}), H_qk={H_QK} H_v={H_V} d={D} bf16, S0 ~ N(0, 0.02^2)", vcpu)
        del vcase
        lcase = inputs.long_256k(args.long_len)
        ms, n = run_prefill_workload(args, lcase, dev, stream, world)
        lcpu = None
        if world == 1 and not args.no_cpu_baseline:
            lcpu = cpu_baseline(lcase, args.cpu_tokens)
        long_ctx = prefill_workload_line(
            lcase, ms, n, hbm_peak, tf_peak,
            f"long-context prefill B=1 L={lcase.T} H_qk={H_QK} H_v={H_V} d={D} bf16, "
            "long-memory gates log_alpha = -softplus(N(-2, 1)), S0 = 0", lcpu)
        del lcase

    # ---------------- front end on raw inputs of the same shape
    fe_ms = fe_gbs = None
    if not args.no_frontend:
        fe_ms, fe_gbs = run_frontend(args, dev, stream, world, L)

    # ---------------- end to end through the public API, host buffers
    e2e_value = e2e_ms = None
    h2d = d2h = 0
    if not args.no_e2e:
        e2e_value, e2e_ms, h2d, d2h = run_e2e(args, case, cu, ws, stream, world, L)

    # ---------------- CPU baseline (the oracle as it stands), rank 0 at N=1 only
    cpu = dec_cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, args.cpu_baseline_tokens)
        if not args.no_decode:
            dec_cpu = decode_cpu_baseline(args.decode_batch, args.cpu_decode_seqs)
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                "workload": f"prefill B=1 L={L} H_qk={H_QK} H_v={H_V} d={D} bf16 q/k/v, "
                            "fp32 gates/state, chunk 64, S0=0",
                "global_batch": world,
                "seq_len": L,
                "parallelism": f"replicas x{world}",
                "l2": "inputs larger than L2 (1.09 GB per step); no flush",
            },
            "roofline": {
                "bound": "hbm",
                "achieved": achieved_gbs,
                "peak": hbm_peak,
                "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak,
                "frac_of_spec": achieved_gbs / HBM_SPEC_GBS,
                "traffic": traffic_from_profile(L),
                "peak_source": peak_src,
                "kernel": "prefill path: chunk_ops_kernel + state_tc_kernel (tcgen05)",
                "kernel_us": kern_avg_ms * 1e3,
                "roofline_us": max(t_hbm, t_tc) * 1e6,
                "hbm_term_us": t_hbm * 1e6,
                "tensor_term_us": t_tc * 1e6,
                "frac_of_roofline_time": max(t_hbm, t_tc) / (kern_avg_ms / 1e3),
                "tflops": flops_per_launch / (kern_avg_ms / 1e3) / 1e12,
            },
            "prefill_mma_sync": None if tc_ms is None else {
                "value": L / (tc_ms / 1e3),
                "unit": "tokens/s",
                "ms_per_call": tc_ms,
                "ms_per_call_default": ms_per_step,
                "ratio_to_default": ms_per_step / tc_ms,
                "workload": "the headline prefill with its output state pass on warp-level "
                            "mma.sync (gdn_prefill_mma) instead of the tcgen05 pass the "
                            "library picks at this shape",
                "steps": args.steps,
            },
            "decode": None if dec_gbs is None else {
                "value": dec_gbs,
                "unit": "GB/s",
                "us_per_step": dec_ms * 1e3,
                "bytes_per_step": dec_bytes(args.decode_batch),
                "peak": hbm_peak,
                "frac": dec_gbs / hbm_peak,
                "frac_of_copy_peak": dec_gbs / hbm_peak,
                "frac_of_spec": dec_gbs / HBM_SPEC_GBS,
                "spec_gbs": HBM_SPEC_GBS,
                "workload": f"decode B={args.decode_batch} H_qk={H_QK} H_v={H_V} d={D}, "
                            "fp32 state in place",
                "steps": max(args.steps, 20),
                **({"cpu_baseline": dec_cpu} if dec_cpu is not None else {}),
            },
            "prefill_tiny": tiny,
            "prefill_varlen": varlen,
            "prefill_long": long_ctx,
            "decode_multi": None if dm_gbs is None else {
                "value": dm_gbs,
                "unit": "GB/s",
                "us_per_call": dm_ms * 1e3,
                "tokens_per_s": args.decode_batch * DM_M / (dm_ms / 1e3),
                "bytes_per_call": dm_bytes(args.decode_batch),
                "peak": hbm_peak,
                "frac": dm_gbs / hbm_peak,
                "workload": f"decode of M={DM_M} tokens per sequence, B={args.decode_batch} H_qk={H_QK} "
                            f"H_v={H_V} d={D}, fp32 state read once, a checkpoint per token",
                "steps": max(args.steps, 10),
            },
            "backward": None if bw is None else {
                "value": L / (bw[0] / 1e3),
                "unit": "tokens/s",
                "ms_per_call": bw[0],
                "roofline": {
                    "bound": "tensor",
                    "achieved": BW_FLOP_PER_TOKEN * L / (bw[0] / 1e3) / 1e12,
                    "peak": tf_peak,
                    "unit": "TFLOP/s",
                    "frac": BW_FLOP_PER_TOKEN * L / (bw[0] / 1e3) / 1e12 / tf_peak,
                    "flop_per_call": BW_FLOP_PER_TOKEN * L,
                    "hbm_bytes_per_call": BW_BYTES_PER_TOKEN * L,
                    "hbm_term_us": BW_BYTES_PER_TOKEN * L / (hbm_peak * 1e9) * 1e6,
                    "tensor_term_us": BW_FLOP_PER_TOKEN * L / (tf_peak * 1e12) * 1e6,
                },
                "workload": f"gradients of the prefill B=1 L={L} H_qk={H_QK} H_v={H_V} d={D} bf16 "
                            "(dq, dk, dv, dlog_alpha, dbeta; S0 = 0, no state gradient)",
                "steps": bw[1],
                "train_step": {
                    "ms_forward": bw[2],
                    "ms_backward": bw[3],
                    "ms_per_step": bw[2] + bw[3],
                    "tokens_per_s": L / ((bw[2] + bw[3]) / 1e3),
                    "ms_per_step_recomputing": ms_per_step + bw[0],
                    "what": "gdn_prefill_train (outputs + saved states) then "
                            "gdn_prefill_backward_saved, against gdn_prefill then "
                            "gdn_prefill_backward (which re-runs the forward)",
                },
            },
            "prefill_shard": None if shard is None else {
                "value": L / (shard[1] / 1e3),
                "unit": "tokens/s",
                "ms_per_call": shard[1],
                "segments": shard[0],
                "ms_per_call_unsplit": shard[2],
                "speedup_from_split": shard[2] / shard[1],
                "workload": f"prefill B=1 L={L} H_qk={H_QK // 8} H_v={H_V // 8} d={D} bf16 "
                            "(one shard of 8-way tensor parallelism)",
                "steps": max(args.steps, 10),
            },
            "frontend": None if fe_gbs is None else {
                "value": fe_gbs,
                "unit": "GB/s",
                "us_per_call": fe_ms * 1e3,
                "bytes_per_call": FE_BYTES_PER_TOKEN * L + FE_WEIGHT_BYTES,
                "peak": hbm_peak,
                "frac": fe_gbs / hbm_peak,
                "workload": f"front end L={L} H_qk={H_QK} H_v={H_V} d={D} bf16, width-4 conv, "
                            "no activation, eps 1e-6",
                "steps": max(args.steps, 20),
            },
            "e2e": None if e2e_value is None else {
                "value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "uploads, prefill and downloads on three streams, two buffer sets"},
            # per step: chunk_ops_kernel + state_tc_kernel
            "gpu_launches": 2 * args.steps,
            "clocks": clocks.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline(case, tokens):
    """The fp64 oracle on all 48 V heads of the first ``tokens`` tokens of the
    first sequence (from its S0 when the workload has one)."""
    import oracle
    T = min(tokens, int(case.cu_seqlens[1]))
    n_threads = oracle.default_threads()
    args = (case.q[:T], case.k[:T], case.v[:T], case.log_alpha[:T], case.beta[:T])
    S0 = None if case.S0 is None else case.S0[:1]
    t0 = time.perf_counter()
    oracle.prefill(*args, S0=S0, want_o=True, n_threads=n_threads)
    dt = time.perf_counter() - t0
    return {"value": T / dt, "unit": "tokens/s", "cores": min(n_threads, H_V),
            "kind": "oracle",
            "sample": f"first {T} tokens of sequence 0 (of {case.T} tokens in {case.N} "
                      f"sequences), all {H_V} V heads, fp64, {dt:.1f} s"}


def decode_cpu_baseline(B, seqs):
    """The fp64 oracle's decode step on the first ``seqs`` sequences of the decode
    batch (all 48 V heads), scaled to GB/s by the same algorithmic bytes."""
    import oracle
    from linear_attention_12_b200 import inputs
    dc = inputs.make_decode(B, H_QK, H_V, D, seed=4)
    n = min(seqs, B)
    q, k, v, la, be = (x[:n] for x in dc.step(0))
    n_threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.decode_step(q, k, v, la, be, dc.S0[:n], n_threads=n_threads)
    dt = time.perf_counter() - t0
    return {"value": dec_bytes(n) / dt / 1e9, "unit": "GB/s", "cores": n_threads,
            "kind": "oracle", "us_per_step_sample": dt * 1e6,
            "sample": f"one step of the first {n} of {B} sequences, all {H_V} V heads, fp64, "
                      f"{dt:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from linear_attention_12_b200 import inputs
    case = inputs.qwen_prefill_32k(L)
    import oracle
    oracle.build()
    T = min(args.cpu_tokens, L)
    for _ in range(args.warmup):
        cpu_baseline(case, min(T, 256))
    times = []
    for _ in range(args.steps):
        r = cpu_baseline(case, T)
        times.append(T / r["value"])
    value = args.steps * T / sum(times)
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {
            "workload": f"prefill B=1 L={L} H_qk={H_QK} H_v={H_V} d={D} (oracle on a "
                        f"{T}-token sample per step)",
            "global_batch": 1, "seq_len": L, "parallelism": "cpu threads",
        },
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"],
                         "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-tokens", type=int, default=2048,
                    help="tokens per step of the reference arm's oracle sample (all 48 heads)")
    ap.add_argument("--cpu-baseline-tokens", type=int, default=L,
                    help="tokens of the cpu_baseline oracle sample (all 48 heads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=L,
                    help="prefill length (the benchmark is L=32768; smaller only for profiling)")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--decode-batch", type=int, default=DEC_B,
                    help="sequences of the decode workloads (256; smaller only for profiling)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer measurement")
    ap.add_argument("--no-frontend", action="store_true", help="skip the front-end measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the gradient measurement")
    ap.add_argument("--no-alt", "--no-tc", dest="no_tc", action="store_true",
                    help="skip the comparison leg: the prefill through the state pass the "
                         "library does not pick at this shape (mma.sync)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the packed-varlen and long-context prefill workloads")
    ap.add_argument("--long-len", type=int, default=262144,
                    help="length of the long-context prefill workload (262144)")
    ap.add_argument("--cpu-decode-seqs", type=int, default=16,
                    help="sequences of the decode batch in the decode cpu_baseline sample")
    ap.add_argument("--no-shard", action="store_true",
                    help="skip the tensor-parallel-shard prefill measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
