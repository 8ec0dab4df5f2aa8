"""Benchmark of the MoE layer hot path on B200.

One step = one pass of the whole layer over one batch of synthetic tokens:
router logits -> top-K -> dispatch (histogram, scan, positions, scatter into
the expert-sorted and the rank-packed buffers) -> gate/up grouped GEMM -> down
grouped GEMM -> combine; for a stack of layers, every layer in turn with
x_(l+1) = bf16(x_l + MoE_l(x_l)). Default workload: the stack of four MoE layers
(N=32768 tokens, d=4096, f=1536, E=64, K=6, W=8 virtual ranks, capacity factor
1.25), the largest single-GPU configuration, with every point of its capacity
factor {1.0, 1.25, 2.0} x Zipf skew {0, 1.2} grid timed as well.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Multi-GPU (torchrun, one process per GPU): the layer does not shard on one GPU's
path, so every rank runs an independent replica on its own batch (no
collective on the data path); the reported time is the max over ranks and the
value counts the tokens of all ranks ("scaling": "weak").

The headline value times K replays of the step captured once as a CUDA graph; the
same K steps launched eagerly, with events between the stages, give the per-stage
times ("eager", "stages_ms"). Prints one JSON line on rank 0.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "moe_layer_tokens_per_s"
UNIT = "tokens/s"


# --------------------------------------------------------------------------- distributed harness

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str):
    import datetime

    import torch.distributed as dist
    world, rank, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when single-process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(tokens_per_rank: float, elapsed_s: float, device=None) -> dict:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    t_max = max_over_ranks(elapsed_s, device)
    total = sum_over_ranks(tokens_per_rank, device)
    return dict(elapsed_max_s=t_max, tokens_total=total, value=total / t_max if t_max > 0 else 0.0)


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks, power and throttle reasons while running: through NVML every
    10 ms in a thread (read-only queries), else with nvidia-smi every 100 ms."""

    # NVML clock-event reason bits
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                   ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:  # the CUDA device by its PCI address (CUDA and NVML may number GPUs differently)
            p = torch.cuda.get_device_properties(self.gpu_index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu_index)

    def _poll(self, nv, h):
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append(dict(sm=float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                      smax=float(smax),
                                      power=nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                      reasons={n for n, bit in self.REASON_BITS if reasons & bit}))
            except Exception:
                pass
            self.stop.wait(0.01)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            return self
        except Exception:
            self.thread = None
        self.path = os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 100 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
            self._read_smi()

    def _read_smi(self):
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    flags = {name for name, v in (("hw_slowdown", parts[5]),
                                                  ("hw_thermal_slowdown", parts[6]),
                                                  ("sw_thermal_slowdown", parts[7]),
                                                  ("sw_power_cap", parts[8]))
                             if v.lower() == "active"}
                    self.rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                          power=float(parts[3]) if parts[3] not in ("[N/A]", "")
                                          else 0.0, reasons=flags))
                except ValueError:
                    continue
        try:
            os.remove(self.path)
        except OSError:
            pass

    def summary(self) -> dict:
        rows = self.rows
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "source": self.source}
        # every sample falls inside the timed region (the sampler runs only there); NVML's
        # power reading is averaged, so it does not tell busy samples from idle ones
        reasons = sorted(set().union(*(r["reasons"] for r in rows)))
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": reasons,
                "samples": len(rows), "source": self.source}


# --------------------------------------------------------------------------- GPU arm

# DRAM bytes per launch of the gate/up grouped GEMM at full size, from one-pass ncu captures
# (the Mixtral shape from its half-size case, scaled x2: weights, rows and h all double),
# summarised in profiles/.
# A figure holds only for the kernel code it was measured on (kernel_source_hash of
# grouped_gemm.cuh: comments and whitespace do not count).
_UP_SHA = "5d9c986bcab4eb5e75d5a505601235db5f1094189b4665fedb8a52bf68bf5ea7"
MEASURED_UP_TRAFFIC = {
    # workload: (kernel source sha256, bytes per launch)
    "mixtral_prefill": (_UP_SHA, 2 * (995.3e6 + 112.5e6)),      # half-size capture x 2
    "mixtral_prefill_fp8": (_UP_SHA, 2 * (487.8e6 + 104.3e6)),  # half-size capture x 2
    "e128_skew": (_UP_SHA, 894.8e6 + 34.7e6),
    "e128_skew_fp8": (_UP_SHA, 444.1e6 + 32.6e6),
    # the return payload changes the down GEMM and the combine, not the gate/up GEMM
    "mixtral_prefill_fp8_return": (_UP_SHA, 2 * (487.8e6 + 104.3e6)),
    "e128_skew_fp8_return": (_UP_SHA, 444.1e6 + 32.6e6),
    "decode": (_UP_SHA, 6080.8e6 + 3.8e6),
    "decode_fp8": (_UP_SHA, 3042.2e6 + 3.8e6),
    "stack4": (_UP_SHA, 4041.5e6 + 597.3e6),                    # one layer's launch
}


def kernel_source_hash(path: str) -> str:
    """sha256 of a source file with its comments and whitespace removed: the code the
    traffic figures were measured on, unaffected by edits to comments."""
    import re
    with open(path, "r", encoding="utf-8") as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()


def up_traffic(workload: str):
    sha_ref, nbytes = MEASURED_UP_TRAFFIC.get(workload, (None, None))
    if sha_ref is None:
        return None
    path = os.path.join(ROOT, "combine_grouped_gemm_router_b200", "csrc", "grouped_gemm.cuh")
    try:
        sha = kernel_source_hash(path)
    except OSError:
        return None
    return nbytes if sha == sha_ref else None


PEER_COPY_GBS = 770.0  # measured NVLink peer copy per direction per GPU on this GPU type


def exchange_report(m, D, row_bytes: int) -> dict:
    """The exchange of layer 0's packed rows as W ranks would run it (host planning only; nothing
    crosses a link here): the contention-free order from moe_exchange_schedule, its length in
    rows (equal to tau_min), and, for contrast, the plain rotation order in which, in round s,
    rank i sends to rank (i + s) mod W and a round lasts as long as its largest block."""
    W = D.shape[0]
    dst, ln, span = m.moe_exchange_schedule(D)
    rotation = sum(int(max(D[i, (i + s) % W] for i in range(W))) for s in range(1, W))
    return {"phases": int(len(ln)), "makespan_rows": span, "rotation_rows": rotation,
            "makespan_us_at_peer_copy": span * row_bytes / (PEER_COPY_GBS * 1e3),
            "rotation_us_at_peer_copy": rotation * row_bytes / (PEER_COPY_GBS * 1e3)}


def placement_report(m, counts, L: int, E: int, P: int) -> dict:
    """Expert placement over P GPUs from the affinity counts the timed steps accumulated:
    the fraction of inter-layer token hops that cross GPUs with contiguous placement and with
    moe_place_experts' placement, and the host time the placement took."""
    t0 = time.perf_counter()
    _, cost, base = m.moe_place_experts(counts, L, E, P, starts=16)
    host_s = time.perf_counter() - t0
    hops = int(counts.sum())
    return {"gpus": P, "hops": hops,
            "cross_fraction_contiguous": base / hops if hops else 0.0,
            "cross_fraction_placed": cost / hops if hops else 0.0,
            "host_s": host_s}


def kernel_launches(w) -> int:
    """Kernels the library launches for one layer of workload w, by the same rules as its
    host code: routing 2 (the router weights' transposition, then the fused projection + top-K
    kernel, E > 32 and N >= 2048), 1 (the fused kernel alone, E = 32) or 2 (projection, then
    selection); per dispatch pass the histogram / look-back kernel and the
    placement kernel (the pass's control words are cleared by a memset, not a kernel); with
    re-routing a positions-only pass, the ranking kernel, then the full pass; each grouped GEMM
    once, or twice (CTA-pair tiles, then single-CTA tiles) when the experts average at least
    768 rows and the K extent allows pair stages, and for fp16 h one more gate/up launch (the
    range pass, which does nothing while h is in fp16's range); the quantisation of h on the
    FP8 path; the shared MLP's offsets and GEMMs; the combine."""
    N, d, f, E, K, W = w.N, w.d, w.f, w.E, w.K, w.W
    NK = N * K
    C = NK if not w.cf > 0 else min(NK, math.ceil(w.cf * N * K / E))
    pair = min(NK // E, C) >= 768
    n = (2 if E > 32 else 1) if (E >= 32 and N >= 2048) else 2
    n += (2 + 1 + 2) if w.reroute else 2
    atom = 128 if w.fp8 else 64
    n += 2 if pair and (d // atom) % 2 == 0 else 1                     # gate/up
    n += 0 if w.fp8 else 1                      # the fp16 range pass (does nothing in range)
    n += 1 if w.fp8 else 0                                              # h -> e4m3
    n += (2 if pair and (f // atom) % 2 == 0 else 1) if d % 256 == 0 else 1   # down
    if w.shared_f > 0:
        sp = N >= 768
        n += 1 + (2 if sp else 1) + 1 + ((2 if sp else 1) if d % 256 == 0 else 1)
    n += 1  # combine
    return n


def algorithmic_work(w, R: int, E_act: int) -> dict:
    """Algorithmic flops and bytes per launch of each stage (see the design notes);
    E_act = experts with at least one kept row (only their weights are read)."""
    N, d, f, E, K = w.N, w.d, w.f, w.E, w.K
    eb = 1 if w.fp8 else 2  # bytes per GEMM operand element
    return dict(
        up_flops=4.0 * d * f * R,
        down_flops=2.0 * d * f * R,
        # gate/up: W1 and W3 of the active experts, the x_sorted rows, h written (bf16)
        up_bytes=2.0 * E_act * f * d * eb + R * d * eb + R * f * 2,
        logits_bytes=N * d * 2 + E * d * 4 + N * E * 4,
        # scatter: read each token row once, write every kept row twice (sorted + packed)
        # (the FP8 payload writes one byte per element and a 4-byte scale per row)
        scatter_bytes=(N * d * 2 + 2 * R * (d + 4) + N * K * 4 * 3 if w.fp8
                       else N * d * 2 + 2 * R * d * 2 + N * K * 4 * 3),
        # combine: read every kept expert row (fp32, or a block payload: e4m3 or fp16 codes and
        # one exponent byte per 32 columns), the routing, write the bf16 out
        combine_bytes=(R * (d + d // 32) if w.fp8_return else
                       R * (2 * d + d // 32) if w.y_f16 else R * d * 4) + N * K * 8 + N * d * 2,
    )


def gemm_peak_choice(peaks: dict, timed_s: float, clocks: dict) -> tuple:
    """The bf16 peak the GEMM roofline divides by: the burst cuBLAS figure (a GEMM timed
    alone), unless the timed region lasted at least a second and the clock record shows the
    power cap holding the SM clock below its maximum, the condition the sustained figure (a
    seconds-long GEMM loop under the power cap) was measured in."""
    capped = ("sw_power_cap" in (clocks.get("reasons") or []) and clocks.get("sm_mhz")
              and clocks.get("sm_max_mhz") and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
    if timed_s >= 1.0 and capped:
        return peaks["bf16_tflops_sustained"], "bf16 sustained (timed region >= 1 s, power-capped)"
    return peaks["bf16_tflops"], "bf16 burst"


def run_gpu(args, w) -> dict:
    import torch

    import combine_grouped_gemm_router_b200 as m
    from moe_workloads import STACK_GRID_CF, STACK_GRID_S, make_layer_inputs, make_shared_inputs
    from moe_workloads import zipf_bias

    world, rank = init_dist("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # one step = the whole stack of w.layers layers (one layer unless the workload is a stack)
    L = w.layers
    shared = w.shared_f > 0
    if w.fp8 and (w.reroute or shared):
        raise ValueError("the FP8 path is benchmarked without re-routing or a shared MLP")
    layers = [make_layer_inputs(w, seed=args.seed + rank, device=str(dev), layer=l, with_x=(l == 0))
              for l in range(L)]
    inp = layers[0]

    def make(wl):
        # the layer's output is bf16, as the hidden states it replaces (a stack's next input)
        return m.make_shape(wl.N, wl.d, wl.f, wl.E, wl.K, wl.W, wl.cf, out_bf16=True,
                            slot_major=wl.slot_major, reroute=wl.reroute,
                            fp8_return=wl.fp8_return, y_f16=wl.y_f16)

    shape = make(w)
    # a stack also times every point of its capacity-factor x Zipf-skew grid (same weights)
    grid = [w.with_(cf=cf, s=s) for cf in STACK_GRID_CF for s in STACK_GRID_S] \
        if (L > 1 and not args.no_grid and w.affinity == 0.0) else []
    shapes = [shape] + [make(g) for g in grid]
    RA = max(m.moe_rows_alloc(s_) for s_ in shapes)
    ws = torch.empty(max(m.moe_workspace_size(s_) for s_ in shapes), dtype=torch.uint8,
                     device=dev)
    x = inp["x"]
    N, K, E, W, d, f = w.N, w.K, w.E, w.W, w.d, w.f
    topk_idx = [torch.empty(N, K, dtype=torch.int32, device=dev) for _ in range(L)]
    topk_w = torch.empty(N, K, dtype=torch.float32, device=dev)
    # the logits rank the candidates of re-routed assignments
    logits = torch.empty(N, E, dtype=torch.float32, device=dev) if w.reroute else None
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = [torch.empty(E + 1, dtype=torch.int32, device=dev) for _ in range(L)]
    row_of = torch.empty(N * K, dtype=torch.int32, device=dev)
    assign = torch.empty(RA, dtype=torch.int32, device=dev)
    pay_dt = torch.uint8 if w.fp8 else torch.bfloat16  # e4m3 codes or bf16 rows
    x_sorted = torch.empty(RA, d, dtype=pay_dt, device=dev)
    x_packed = torch.empty(RA, d, dtype=pay_dt, device=dev)
    if w.fp8:
        # the FP8 payload's row scales; the experts' W1, W3 quantised once (weights are static)
        sorted_scale = torch.empty(RA, dtype=torch.float32, device=dev)
        packed_scale = torch.empty(RA, dtype=torch.float32, device=dev)
        for lw in layers:
            for k in ("w1", "w3", "w2"):
                q = torch.empty(lw[k].shape, dtype=torch.uint8, device=dev)
                sc = torch.empty(lw[k].shape[:-1], dtype=torch.float32, device=dev)
                m.moe_quantize_rows_e4m3(lw[k], q, sc)
                lw[k + "q"], lw[k + "s"] = q, sc
        h_q = torch.empty(RA, f, dtype=torch.uint8, device=dev)
        h_scale = torch.empty(RA, dtype=torch.float32, device=dev)
    else:
        # the down projection reads fp16 h and an fp16 copy of W2, made once (static weights)
        for lw in layers:
            lw["w2h"] = m.w2_for(shape, lw["w2"])
    torch.cuda.synchronize(dev)
    D = torch.empty(W * W, dtype=torch.int64, device=dev)
    pk_off = torch.empty(W * W + 1, dtype=torch.int64, device=dev)
    h = torch.empty(RA, f, dtype=torch.bfloat16 if w.fp8 else torch.float16, device=dev)
    # fp32 expert outputs, or the FP8 return payload (e4m3 codes + block exponents)
    y = torch.empty(max(m.moe_y_bytes(s_) for s_ in shapes), dtype=torch.uint8, device=dev)
    if L > 1:  # x_{l+1} = bf16(x_l + MoE_l(x_l)), ping-pong buffers
        xbuf = [torch.empty(N, d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        affinity = torch.zeros(L - 1, E, E, dtype=torch.int64, device=dev)
        out = xbuf[(L - 1) % 2]
    else:
        out = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
    if shared:  # Residual-MoE: the shared dense MLP on every token
        sh = make_shared_inputs(w, seed=args.seed + rank, device=str(dev))
        sh["ws2h"] = m.w2_for(shape, sh["ws2"])
        h_s = torch.empty(N, w.shared_f, dtype=torch.float16, device=dev)
        y_s = torch.empty(N, d, dtype=torch.float32, device=dev)
        ws_s = torch.empty(256, dtype=torch.uint8, device=dev)

    stage_names = ["route", "dispatch", "expert_up", "expert_down"] + (
        ["shared_expert"] if shared else []) + ["combine"]
    n_ev = len(stage_names) + 1

    def step(ev=None, shp=shape, biases=None):
        """One step; ev (optional) is [layer][n_ev] events around the stages; biases
        (optional) replaces each layer's router bias (the grid's Zipf skew)."""
        st = torch.cuda.current_stream(dev)
        for l in range(L):
            lw = layers[l]
            bias = lw["bias"] if biases is None else biases
            xin = x if l == 0 else xbuf[(l - 1) % 2]
            dst = xbuf[l % 2] if L > 1 else out
            e = ev[l] if ev is not None else None
            if e is not None:
                e[0].record(st)
            m.moe_route(shp, xin, lw["w_router"], bias, topk_idx[l], topk_w, logits, ws, st)
            if e is not None:
                e[1].record(st)
            if w.fp8:
                m.moe_dispatch_fp8(shp, xin, topk_idx[l], counts, kept, offsets[l], row_of,
                                   assign, x_sorted, sorted_scale, x_packed=x_packed,
                                   packed_scale=packed_scale, rank_matrix=D,
                                   packed_offsets=pk_off, ws=ws, stream=st)
            elif w.reroute:
                m.moe_dispatch_reroute(shp, xin, logits, topk_idx[l], counts, kept, offsets[l],
                                       row_of, assign, x_sorted, x_packed=x_packed, rank_matrix=D,
                                       packed_offsets=pk_off, ws=ws, stream=st)
            else:
                m.moe_dispatch(shp, xin, topk_idx[l], counts, kept, offsets[l], row_of, assign,
                               x_sorted, x_packed, D, pk_off, None, ws, st)
            if e is not None:
                e[2].record(st)
            if w.fp8:
                m.moe_expert_up_fp8(shp, x_sorted, sorted_scale, offsets[l], lw["w1q"],
                                    lw["w1s"], lw["w3q"], lw["w3s"], h, st)
            else:
                m.moe_expert_up(shp, x_sorted, offsets[l], lw["w1"], lw["w3"], h, st)
            if e is not None:
                e[3].record(st)
            if w.fp8:  # the kept rows of h to e4m3, then the e4m3 down GEMM
                m.moe_quantize_rows_e4m3(h, h_q, h_scale, rows_dev=offsets[l][E:], stream=st)
                m.moe_expert_down_fp8(shp, h_q, h_scale, offsets[l], lw["w2q"], lw["w2s"], y,
                                      st)
            else:
                m.moe_expert_down(shp, h, offsets[l], lw["w2h"], y, st)
            j = 4
            if e is not None:
                e[j].record(st)
            if shared:
                m.moe_shared_expert(shp, w.shared_f, xin, sh["ws1"], sh["ws3"], sh["ws2h"], h_s,
                                    y_s, ws_s, st)
                j += 1
                if e is not None:
                    e[j].record(st)
            m.moe_combine(shp, y, row_of, topk_w, dst, residual=xin if L > 1 else None,
                          shared_y=y_s if shared else None, stream=st)
            if e is not None:
                e[j + 1].record(st)
            if l > 0:
                m.moe_affinity_accumulate(N, E, K, topk_idx[l - 1], topk_idx[l], affinity[l - 1],
                                          st)

    def timed(n_steps, shp=shape, biases=None, with_clocks=False):
        """n_steps eager steps between a barrier and a synchronize on each side, CUDA events
        around the whole run and between the stages of every step (on the stream the kernels
        run on). Returns (elapsed s, per-stage ms: mean over steps of the sum over the
        stack's layers, clock summary or None)."""
        events = [[[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(L)]
                  for _ in range(n_steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        sampler = ClockSampler(local) if with_clocks else None
        if sampler is not None:
            sampler.__enter__()
        t0.record(stream)
        for i in range(n_steps):
            step(events[i], shp, biases)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if sampler is not None:
            sampler.__exit__(None, None, None)
        barrier()
        stage = {name: statistics.mean(sum(ev[l][j].elapsed_time(ev[l][j + 1]) for l in range(L))
                                       for ev in events)
                 for j, name in enumerate(stage_names)}
        return t0.elapsed_time(t1) / 1e3, stage, (sampler.summary() if sampler else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if m.moe_get_device_error(True) != 0:
        raise RuntimeError("device error during warm-up")

    # eager launches with CUDA events between the stages: the per-stage times and the
    # dominant kernel's mean launch duration
    elapsed_eager_s, stage_ms, clock_summary = timed(args.steps, with_clocks=args.no_graph)
    R_layers = [int(o[E].item()) for o in offsets]
    act_layers = [int(((o[1:] - o[:-1]) > 0).sum().item()) for o in offsets]
    R = R_layers[0]
    agg_eager = aggregate(float(N * args.steps), elapsed_eager_s, dev)

    # the headline: the same step captured once in a CUDA graph (how a serving loop runs it)
    # and replayed K times between a barrier and a synchronize, the clocks sampled meanwhile;
    # the host launch overhead disappears, which matters for small (decode) steps
    eager_res = {"value": agg_eager["value"], "unit": UNIT,
                 "ms_per_step": agg_eager["elapsed_max_s"] / args.steps * 1e3}
    if args.no_graph:
        agg, elapsed_s, timing = agg_eager, elapsed_eager_s, "eager launches"
    else:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(dev)
        barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(local)
        sampler.__enter__()
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        sampler.__exit__(None, None, None)
        barrier()
        clock_summary = sampler.summary()
        elapsed_s = g0.elapsed_time(g1) / 1e3
        agg = aggregate(float(N * args.steps), elapsed_s, dev)
        timing = "CUDA graph of one step, replayed"
        if m.moe_get_device_error(True) != 0:
            raise RuntimeError("device error during the graph replays")
        del graph

    peaks = load_peaks()
    up_peak_bf16, up_peak_name = gemm_peak_choice(peaks, elapsed_s, clock_summary or {})

    def work_of(R_list, A_list, wl):
        tot = {}
        for Rl, Al in zip(R_list, A_list):
            for k, v in algorithmic_work(wl, Rl, Al).items():
                tot[k] = tot.get(k, 0.0) + v
        return tot

    # the grid of a stack: every (capacity factor, Zipf skew) point, timed the same way on the
    # same weights (the bias carries the skew; the capacity factor is in the shape)
    grid_res = []
    for gw, gshape in zip(grid, shapes[1:]):
        gb = zipf_bias(E, gw.s)
        gb = None if gb is None else gb.to(dev)
        for _ in range(3):
            step(None, gshape, gb)
        torch.cuda.synchronize(dev)
        gs, gstage, _ = timed(args.grid_steps, gshape, gb)
        gR = [int(o[E].item()) for o in offsets]
        gA = [int(((o[1:] - o[:-1]) > 0).sum().item()) for o in offsets]
        gwk = work_of(gR, gA, gw)
        up_s, down_s = gstage["expert_up"] / 1e3, gstage["expert_down"] / 1e3
        g_agg = aggregate(float(N * args.grid_steps), gs, dev)
        gemm_tf = (gwk["up_flops"] + gwk["down_flops"]) / (up_s + down_s) / 1e12
        grid_res.append({
            "capacity_factor": gw.cf, "zipf_s": gw.s, "tokens_per_s": g_agg["value"],
            "ms_per_step": g_agg["elapsed_max_s"] / args.grid_steps * 1e3,
            "layer_tokens_per_s": g_agg["value"] * L, "rows_kept": gR,
            "drop_rate": 1.0 - sum(gR) / float(L * N * K),
            "stages_ms": {k: round(v, 4) for k, v in gstage.items()},
            "gate_up_tflops": gwk["up_flops"] / up_s / 1e12,
            "gemm_tflops": gemm_tf, "gemm_frac_of_bf16_burst": gemm_tf / peaks["bf16_tflops"]})
    if m.moe_get_device_error(True) != 0:
        raise RuntimeError("device error during the timed runs")

    # the routing report of layer 0 (untimed): one more route + dispatch with the counters on,
    # then the derived figures (drop rate, per-rank send/receive balance, cross-rank fraction,
    # expert-load spread, effective capacity factor, the exchange-time bound tau_min)
    stats_buf = m.stats_buffer(dev)
    l0 = layers[0]
    m.moe_route(shape, x, l0["w_router"], l0["bias"], topk_idx[0], topk_w, logits, ws, stream)
    if w.reroute:
        m.moe_dispatch_reroute(shape, x, logits, topk_idx[0], counts, kept, offsets[0], row_of,
                               assign, x_sorted, x_packed=x_packed, rank_matrix=D,
                               packed_offsets=pk_off, stats=stats_buf, ws=ws, stream=stream)
    elif w.fp8:
        m.moe_dispatch_fp8(shape, x, topk_idx[0], counts, kept, offsets[0], row_of, assign,
                           x_sorted, sorted_scale, x_packed=x_packed, packed_scale=packed_scale,
                           rank_matrix=D, packed_offsets=pk_off, stats=stats_buf, ws=ws,
                           stream=stream)
    else:
        m.moe_dispatch(shape, x, topk_idx[0], counts, kept, offsets[0], row_of, assign, x_sorted,
                       x_packed, D, pk_off, stats_buf, ws, stream)
    st0 = m.read_stats(stats_buf, stream)
    rep0 = m.report_dict(m.moe_derive_report(shape, st0, D.cpu().numpy(), kept.cpu().numpy()))
    routing = {"rows_kept": st0.rows, "dropped": st0.dropped, "active_experts": st0.active_experts,
               "dedup_pairs": st0.dedup_pairs, "rerouted": st0.rerouted,
               **{k: rep0[k] for k in ("drop_rate", "send_max_over_min", "recv_max_over_min",
                                       "cross_rank_fraction", "load_std_over_mean",
                                       "capacity_factor_effective", "tau_min_tokens")}}
    routing["exchange"] = exchange_report(m, D.cpu().numpy().reshape(W, W),
                                          row_bytes=(d + 4) if w.fp8 else 2 * d)
    if L > 1:
        routing["placement"] = placement_report(m, affinity.cpu().numpy(), L, E, W)
    err = m.moe_get_device_error(True)

    # end to end through the public API: every step copies its input from pinned host memory,
    # runs moe_layer (each layer of a stack in turn) and copies the bf16 result back; the copies
    # of one step overlap the layers of the previous one (two buffers, one copy stream each way)
    e2e = None
    if not args.no_e2e:
        lws_bytes = (m.moe_layer_shared_workspace_size(shape, w.shared_f) if shared
                     else m.moe_layer_workspace_size(shape))
        lws = torch.empty(lws_bytes, dtype=torch.uint8, device=dev)
        x_host = x.cpu().pin_memory()
        out_host = [torch.empty(N, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        out_dev = [torch.empty(N, d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        mid = [torch.empty_like(x) for _ in range(2)] if L > 1 else None
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev_comp[b])  # buffer b's previous layer has read its input
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # buffer b's previous result has left the device
            xin = x_dev[b]
            for l in range(L):
                lw = layers[l]
                dst = out_dev[b] if l == L - 1 else mid[l % 2]
                res = xin if L > 1 else None
                if shared:
                    m.moe_layer_shared(shape, w.shared_f, xin, lw["w_router"], lw["bias"],
                                       lw["w1"], lw["w3"], lw["w2h"], sh["ws1"], sh["ws3"],
                                       sh["ws2h"], dst, residual=res, ws=lws, stream=stream)
                elif w.fp8:
                    m.moe_layer_fp8(shape, xin, lw["w_router"], lw["bias"], lw["w1q"], lw["w1s"],
                                    lw["w3q"], lw["w3s"], lw["w2q"], lw["w2s"], dst, residual=res,
                                    ws=lws, stream=stream)
                else:
                    m.moe_layer(shape, xin, lw["w_router"], lw["bias"], lw["w1"], lw["w3"],
                                lw["w2h"], dst, residual=res, ws=lws, stream=stream)
                xin = dst
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(args.steps):
            e2e_step(i)
        for b in range(2):
            stream.wait_event(ev_out[b])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_agg = aggregate(float(N * args.steps), e0.elapsed_time(e1) / 1e3, dev)
        e2e = {"value": e2e_agg["value"], "unit": UNIT, "h2d_bytes_per_step": N * d * 2,
               "d2h_bytes_per_step": N * d * 2,
               "note": "pinned host input and output; copies overlap the previous step's layers"}
        del lws

    # algorithmic work of one step (all layers of a stack)
    work = work_of(R_layers, act_layers, w)
    up_ratio = 2.0 if w.fp8 else 1.0  # e4m3 tensor throughput is twice bf16's (nominal)
    up_peak = up_peak_bf16 * up_ratio
    up_s = stage_ms["expert_up"] / 1e3
    down_s = stage_ms["expert_down"] / 1e3
    up_tflops = work["up_flops"] / up_s / 1e12
    down_tflops = work["down_flops"] / down_s / 1e12
    gemm_tflops = (work["up_flops"] + work["down_flops"]) / (up_s + down_s) / 1e12
    stages = {k: round(v, 4) for k, v in stage_ms.items()}
    hbm = peaks["hbm_gbs"]
    comb_gbs = work["combine_bytes"] / (stage_ms["combine"] / 1e3) / 1e9
    # the dominant kernel's roofline: tensor-bound when its flops per algorithmic byte exceed
    # the machine balance (peak flops / copy bandwidth), else HBM-bound (decode, and layers
    # with few rows per expert, stream weights)
    up_gbs = work["up_bytes"] / up_s / 1e9
    intensity = work["up_flops"] / work["up_bytes"]
    balance = up_peak * 1e12 / (hbm * 1e9)
    kernel_name = ("grouped GEMM gate/up on e4m3 (moe_expert_up_fp8, tcgen05 kind::f8f6f4)"
                   if w.fp8 else "grouped GEMM gate/up (moe_expert_up, tcgen05)")
    tensor_line = {"achieved": up_tflops, "peak": up_peak, "unit": "TFLOP/s",
                   "frac": up_tflops / up_peak,
                   "peak_source": (peaks["source"] + " " + up_peak_name +
                                   (" x 2 (the nominal e4m3/bf16 dense ratio)" if w.fp8 else "")),
                   "frac_of_burst": up_tflops / (peaks["bf16_tflops"] * up_ratio),
                   "frac_of_sustained": up_tflops / (peaks["bf16_tflops_sustained"] * up_ratio)}
    hbm_line = {"achieved": up_gbs, "peak": hbm, "unit": "GB/s", "frac": up_gbs / hbm,
                "peak_source": peaks["source"] + " copy bandwidth"}
    roofline = {"kernel": kernel_name, "bound": "tensor" if intensity >= balance else "hbm"}
    roofline.update(tensor_line if intensity >= balance else hbm_line)
    roofline.update({"traffic": up_traffic(w.name),
                     "launches_per_step": L,
                     "algorithmic_flops_per_launch": work["up_flops"] / L,
                     "algorithmic_bytes_per_launch": work["up_bytes"] / L,
                     "mean_launch_ms": stage_ms["expert_up"] / L,
                     "flops_per_byte": intensity, "machine_balance": balance,
                     "other_bound": ({"unit": "GB/s", "achieved": up_gbs, "frac": up_gbs / hbm}
                                     if intensity >= balance else
                                     {"unit": "TFLOP/s", "achieved": up_tflops,
                                      "frac": up_tflops / up_peak})})
    ms_step = agg["elapsed_max_s"] / args.steps * 1e3
    res = {
        "metric": METRIC,
        "value": agg["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": (("e4m3 (dispatch payload, both expert GEMMs' operands and the return "
                   "payload), fp32 accumulate" if w.fp8_return else
                   "e4m3 (dispatch payload and both expert GEMMs' operands), fp32 accumulate")
                  if w.fp8 else "bf16 (x, W1, W3), fp16 (h, W2), fp32 accumulate" + (
                      "; y as fp16 codes + block exponents" if w.y_f16 else "")),
        "data": "synthetic (seeded: x N(0,1), router per the workload, experts N(0,0.02^2); "
                "random-init weights)",
        "config": {"workload": w.name, "N": N, "d": d, "f": f, "E": E, "K": K, "W": W,
                   "shared_f": w.shared_f,
                   "capacity_factor": w.cf if w.cf > 0 else "dropless", "zipf_s": w.s,
                   "rows_kept": R_layers if L > 1 else R, "layers": L,
                   "step": (f"the {L}-layer stack, x_(l+1) = bf16(x_l + MoE_l(x_l))" if L > 1
                            else "one layer"),
                   "output": "bf16 [N][d], the fp32 sum rounded once",
                   "y_payload": ("e4m3 codes + exponent per 32 columns" if w.fp8_return else
                                 "fp16 codes + exponent per 32 columns" if w.y_f16 else "fp32"),
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {L * 3 * E * d * f * 2 / 1e9:.2f} GB of expert "
                         "weights streamed per step, no flush"},
        "per_layer": {"layer_tokens_per_s": agg["value"] * L, "ms_per_layer": ms_step / L},
        "roofline": roofline,
        "stages_ms": stages,
        "grouped_gemm": {"tflops": gemm_tflops, "gate_up_tflops": up_tflops,
                         "down_tflops": down_tflops,
                         "frac_of_bf16_burst": gemm_tflops / peaks["bf16_tflops"],
                         "frac_of_bf16_sustained": gemm_tflops / peaks["bf16_tflops_sustained"]},
        "combine": {"gbs": comb_gbs, "frac_of_hbm": comb_gbs / hbm, "frac_of_8tbs": comb_gbs / 8000.0},
        "shared_expert": ({"ms": stage_ms["shared_expert"],
                           "tflops": 6.0 * d * w.shared_f * N / (stage_ms["shared_expert"] / 1e3) / 1e12}
                          if shared else None),
        "dispatch": {"ms": stage_ms["dispatch"],
                     "scatter_bytes": work["scatter_bytes"],
                     # the whole dispatch stage (histogram, scans, positions, scatter) against
                     # the scatter's bytes alone: a lower bound on the scatter kernel's rate
                     "gbs": work["scatter_bytes"] / (stage_ms["dispatch"] / 1e3) / 1e9,
                     "frac_of_hbm": work["scatter_bytes"] / (stage_ms["dispatch"] / 1e3) / 1e9
                     / hbm},
        "route": {"ms": stage_ms["route"],
                  "tflops_fp32": 2.0 * N * d * E * L / (stage_ms["route"] / 1e3) / 1e12},
        "grid": grid_res or None,
        "routing": routing,
        "clocks": clock_summary,
        "gpu_launches": (L * kernel_launches(w) + (L - 1)) * args.steps,
        "timing": timing,
        "eager": eager_res,
        "device_error": err,
        "e2e": e2e,
    }
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, layers, args.cpu_sample_tokens,
                                           sh if shared else None)
    return res if rank == 0 else None


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "of measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "of fallback"}


# --------------------------------------------------------------------------- CPU oracle legs

def sample_size(w, seconds: float, cores: int) -> int:
    """Tokens of a sample the oracle finishes in about `seconds` on `cores` host cores, from
    its work per token (the router's 2*d*E fp32 multiply-adds at about 0.7 GFLOP/s and the
    experts' K*6*d*f fp64 flops at about 2 GFLOP/s per core, measured on this oracle), every
    layer of a stack; a multiple of W, at least W, at most N."""
    per_core_s = w.layers * (2.0 * w.d * w.E / 0.7e9 + w.K * 6.0 * w.d * (w.f + w.shared_f)
                             / 2.0e9)
    S = int(seconds * max(cores, 1) / per_core_s)
    return max(w.W, min(w.N, (S // w.W) * w.W))


def slice_inputs(w, layers_cpu: list, S: int) -> tuple:
    """The first S tokens of the workload's batch (S a multiple of W) and its weights: the
    bounded sample the oracle is timed on. The capacity is the same factor of the smaller
    batch (C = ceil(cf * S * K / E))."""
    S = max(w.W, (min(S, w.N) // w.W) * w.W)
    return w.with_(N=S), layers_cpu[0]["x"][:S].contiguous()


def oracle_step(ws, layers_cpu: list, x, shared_cpu=None):
    """One step of the oracle on the sample: the whole layer (route, dispatch, the experts,
    combine) for every token of the sample, every layer of a stack in turn with
    x_(l+1) = bf16(x_l + out_l). The FP8 workloads run on the operands quantised once outside
    the timing (static weights), the token rows quantised inside it."""
    import numpy as np
    import torch

    import oracle
    for l, lw in enumerate(layers_cpu):
        inp = dict(lw, x=x)
        if ws.fp8:
            xq, sx = oracle.quantize_rows_e4m3(x)
            as_bf16 = lambda u: torch.from_numpy(u.view(np.int16)).view(torch.bfloat16)
            inp = dict(lw["deq"], x=as_bf16(oracle.dequantize_rows_bf16(xq, sx)),
                       w_router=lw["w_router"], bias=lw["bias"])
        r = oracle.layer(inp, ws.K, ws.W, ws.cf, order=int(ws.slot_major), reroute=ws.reroute)
        out = r["out"]
        if shared_cpu is not None:
            out = out + oracle.shared_expert(x, shared_cpu["ws1"], shared_cpu["ws3"],
                                             shared_cpu["ws2"])
        if len(layers_cpu) > 1:
            xf = oracle.bf16_bits_to_f64(oracle.as_u16(x))
            x = torch.from_numpy(oracle.round_bf16(xf + out).view(np.int16)).view(torch.bfloat16)
    return x


def prepare_oracle_layers(w, layers: list) -> list:
    """Host copies of every layer's inputs for the oracle; for the FP8 workloads also the
    dequantised e4m3 weights (made once: the weights are static)."""
    import numpy as np
    import torch

    import oracle
    oracle.build()
    out = []
    for lw in layers:
        c = {k: (None if v is None else v.cpu()) for k, v in lw.items()
             if k in ("x", "w_router", "bias", "w1", "w3", "w2")}
        if w.fp8:
            as_bf16 = lambda u: torch.from_numpy(u.view(np.int16)).view(torch.bfloat16)
            c["deq"] = {k: as_bf16(oracle.dequantize_rows_bf16(*oracle.quantize_rows_e4m3(c[k])))
                        for k in ("w1", "w3", "w2")}
        out.append(c)
    return out


def cpu_threads() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def cpu_baseline(w, layers, sample_tokens: int, shared=None) -> dict:
    """The oracle as it stands, timed on the host cores on a bounded sample of the workload:
    the first `sample_tokens` tokens through the whole layer (or stack); measured, not
    extrapolated."""
    lc = prepare_oracle_layers(w, layers)
    sh = None if shared is None else {k: v.cpu() for k, v in shared.items()}
    ws, x = slice_inputs(w, lc, sample_tokens or sample_size(w, 15.0, cpu_threads()))
    t0 = time.perf_counter()
    oracle_step(ws, lc, x, sh)
    t = time.perf_counter() - t0
    return {"value": ws.N / t, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "seconds": t,
            "sample": f"the first {ws.N} of the {w.N} tokens through the whole "
                      + (f"{w.layers}-layer stack" if w.layers > 1 else "layer")
                      + " (route, dispatch, experts, combine; capacity ceil(cf*S*K/E)), "
                        "measured"}


def run_reference(args, w) -> dict:
    from moe_workloads import make_layer_inputs
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    layers = [make_layer_inputs(w, seed=args.seed, device="cpu", layer=l, with_x=(l == 0))
              for l in range(w.layers)]
    sh = None
    if w.shared_f > 0:
        from moe_workloads import make_shared_inputs
        sh = make_shared_inputs(w, seed=args.seed, device="cpu")
    lc = prepare_oracle_layers(w, layers)
    ws, x = slice_inputs(w, lc, args.ref_sample_tokens or sample_size(w, 1.0, cpu_threads()))
    times = []
    wall0 = time.perf_counter()
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_step(ws, lc, x, sh)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = ws.N * len(times) / total
    sample = (f"each step: the first {ws.N} of the {w.N} tokens through the whole "
              + (f"{w.layers}-layer stack" if w.layers > 1 else "layer")
              + " (route, dispatch, experts, combine; capacity ceil(cf*S*K/E)), measured")
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "impl": "reference",
        "config": {"workload": w.name, "N": w.N, "d": w.d, "f": w.f, "E": w.E, "K": w.K,
                   "W": w.W, "capacity_factor": w.cf if w.cf > 0 else "dropless",
                   "zipf_s": w.s, "layers": w.layers, "tokens_per_step": ws.N},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - wall0,
    }
    return res


# --------------------------------------------------------------------------- main

def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="stack4")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample-tokens", type=int, default=0,
                    help="tokens of the cpu_baseline sample (0: about 15 s of oracle work)")
    ap.add_argument("--ref-sample-tokens", type=int, default=0,
                    help="tokens per step of the reference arm (0: about 1 s of oracle work)")
    ap.add_argument("--grid-steps", type=int, default=10,
                    help="timed steps per point of a stack's capacity-factor x skew grid")
    ap.add_argument("--no-grid", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches instead of replaying the step's CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--y-f32", action="store_true",
                    help="the expert outputs travel to the combine as fp32 rows instead of the "
                         "default fp16 codes with one power-of-two exponent per 32 columns "
                         "(bf16-path workloads; the FP8 workloads keep their own payloads)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with this many tokens instead of its own N (a reduced "
                         "case for profiler captures; not a benchmark configuration)")
    return ap.parse_args(argv)


def select_workload(args):
    """The workload the arguments name: its token count replaced by --tokens, and on the bf16
    path the fp16 return payload unless --y-f32 (the FP8 workloads keep their own payloads)."""
    from moe_workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.tokens > 0:
        w = w.with_(N=args.tokens)
    if not w.fp8 and not args.y_f32:
        w = w.with_(y_f16=True)
    return w


def main(argv=None):
    args = parse(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = select_workload(args)
    if args.impl == "reference":
        res = run_reference(args, w)
    else:
        res = run_gpu(args, w)
    if res is not None:
        print(json.dumps(res), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
