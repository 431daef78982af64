#!/usr/bin/env python
"""Benchmark of the TIDE hot path on B200: RS reduce + AG placement, HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama70b]
    python bench.py --impl reference ...          # the CPU oracle, timed on host cores
    python bench.py --suite                       # every workload, one JSON line each

A step is one pass of the hot path over one synthetic parameter group:
tide_ag_place (SM engine) places the rank-major bf16 all-gather buffer into
padded per-parameter storage, then tide_rs_reduce (rank order, x fl32(1/W))
reduces the W simulated ranks' bf16 gradients into fp32 rank-major shards.
The metric is algorithmic HBM bytes moved per second (bytes each element must
cross HBM once: RS 2W B read per valid element + 4 B written per shard
element; AG 2 B read per valid element + 2 B written per padded element).

Timing: W untimed steps, then K steps between a barrier + synchronize on each
side, CUDA events on the launching stream, max over ranks.  Inputs are
generated on the device by the seeded generator and exceed L2.

With N > 1 processes (torchrun, one per GPU) the default is the exchange: the
group's W ranks are spread over the N GPUs (W/N each); every process holds only
its ranks' gradients and all-gather shards, maps the other processes' buffers
through CUDA IPC, places every rank's shard into its own parameters
(tide_ag_gather_place, peer loads over NVLink) and reduces the shards of the
ranks it holds (tide_rs_reduce with one-rank plans, peer loads).  The value is
all processes' algorithmic bytes over the slowest process's step time
(--mode replicas runs N independent single-GPU copies instead).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "RS/AG-place achieved HBM GB/s and % of B200 peak (70B layer, W=8)"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--mode", choices=["exchange", "replicas"], default=None,
                    help="with N > 1 processes the default is exchange: spread the group's ranks "
                         "over the GPUs and exchange over NVLink; replicas runs N independent "
                         "copies.  --mode exchange with one process runs the exchange path in a "
                         "one-process group (all ranks on this GPU)")
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama70b")
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--max-ctas", type=int, default=0)
    ap.add_argument("--rs-order", choices=["rank", "tree"], default="rank",
                    help="summation order of the step's reduce-scatter (tree: pairs by levels)")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-m1", action="store_true",
                    help="skip the one-rank training-step record (layout-conversion share)")
    ap.add_argument("--interference", action="store_true",
                    help="run the full concurrent-GEMM interference sweep (3 trials, both RS kernels) "
                         "instead of the quick one")
    ap.add_argument("--no-interference", action="store_true",
                    help="skip the concurrent-GEMM interference record")
    ap.add_argument("--suite", action="store_true", help="one JSON line per workload")
    ap.add_argument("--jsonl", default=None,
                    help="also append one flat row per (workload, op, mode, ctas) to this file")
    ap.add_argument("--profile-small", action="store_true",
                    help="a short run of the sweep_w8 workload, sized for an ncu capture")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(*rel):
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


RS_SOURCES = ("fsdp2_layout_aware_b200/csrc/rs_reduce.cu", "fsdp2_layout_aware_b200/csrc/reduce_ranks.cuh",
              "fsdp2_layout_aware_b200/csrc/device_common.cuh")
AG_SOURCES = ("fsdp2_layout_aware_b200/csrc/ag_place.cu", "fsdp2_layout_aware_b200/csrc/device_common.cuh")


TRAFFIC_WORKLOAD = "sweep_w8"


def ncu_traffic(kernel: str, sources, alg_read: int, alg_write: int):
    """Per-launch DRAM traffic of `kernel` on a full launch, scaled from a small-case capture.

    profiles/ncu_traffic.txt holds, per kernel, one ncu capture on the sweep_w8 group (inputs
    larger than L2, under 1 GB on the device): dram__bytes_read.sum, dram__bytes_write.sum,
    the bytes its SMs wrote into L2 ((lts__t_sectors_op_write.sum - the ltcfabric share) x
    32 B), and that launch's algorithmic read and write bytes.
    Reads scale by read/alg_read.  The small case ends with part of its output still dirty in
    L2 (not yet in dram__bytes_write), so writes scale by the bytes the kernel wrote into L2,
    all of which reach DRAM.  Returns (traffic bytes or None, source note).  None when the
    kernel's sources changed since the capture.
    """
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None, "no capture"
    digest = source_digest(*sources)
    for line in open(path):
        parts = line.split()
        if line.startswith("#") or len(parts) < 8 or parts[0] != kernel:
            continue
        if parts[2] != digest:
            return None, "sources changed since the capture"
        rd, wr, l2w, ard, awr = (float(x) for x in parts[3:8])
        traffic = rd / ard * alg_read + max(wr, l2w) / awr * alg_write
        return traffic, (f"scaled from the {parts[1]} capture: read x{rd / ard:.4f}, "
                         f"write x{max(wr, l2w) / awr:.4f} of the algorithmic bytes")
    return None, "no capture"


class ClockSampler:
    """Polls NVML for SM clock and clock-event reasons while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML absent: report it rather than guess
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=_reduce_device(device))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def _reduce_device(device):
    """Where a small all-reduce tensor lives: the GPU under NCCL, the host under gloo."""
    import torch.distributed as dist
    return "cpu" if dist.get_backend() == "gloo" else device


def replica_throughput(n_ranks: int, bytes_per_rank_step: int, max_step_ms: float) -> float:
    """Whole-job GB/s of independent replicas: all ranks' bytes over the slowest rank's time."""
    return n_ranks * bytes_per_rank_step / (max_step_ms * 1e-3) / 1e9


def alg_bytes(group, L):
    W = group.world
    N = sum(group.numel(i) for i in range(group.n_params))
    Npad = W * L.Ns
    return {"rs": 2 * W * N + 4 * Npad, "ag": 2 * N + 2 * Npad, "stage": 4 * W * N,
            "slot_rs": 2 * W * N + 4 * Npad, "N": N, "Npad": Npad,
            "rs_read": 2 * W * N, "rs_write": 4 * Npad, "ag_read": 2 * N, "ag_write": 2 * Npad}


# --------------------------------------------------------------------------- our arm


class Workload:
    """Device buffers of one parameter group, plus the plan."""

    def __init__(self, group, seed, device):
        import torch
        import synth
        from fsdp2_layout_aware_b200 import tide as T
        self.group = group
        self.plan = T.Plan(group.shapes, group.world, device=device)
        self.Ns = self.plan.shard_numel
        W = group.world
        self.grads = synth.dev_grads(group, seed, device=device)
        self.ag = synth.dev_ag(group, self.Ns, seed, device=device)
        self.out = torch.empty(W * self.Ns, dtype=torch.float32, device=device)
        self.params = [torch.empty(self.plan.query(i)["padded_numel"], dtype=torch.bfloat16,
                                   device=device) for i in range(group.n_params)]
        # pointer tables marshalled once, as a training loop would per bucket
        self.grads_t = T.TensorTable([g for row in self.grads for g in row])
        self.params_t = T.TensorTable(self.params)
        self.slots = None

    def ensure_slots(self):
        import torch
        if self.slots is None:
            n = self.group.world * self.Ns
            self.slots = [torch.empty(n, dtype=torch.bfloat16, device=self.out.device)
                          for _ in range(self.group.world)]
        return self.slots

    def drop_slots(self):
        self.slots = None

    def params_poison(self):
        """Fill the parameter storage (pads included) with a bit pattern no call writes."""
        import torch
        for p in self.params:
            p.view(torch.int16).fill_(-1)


def timed_calls(fn, K, stream, flush=None, warmup=2):
    """Mean device time of fn() over K calls, each bracketed by events on `stream`,
    after `warmup` untimed calls (first-call costs: streams and events a plan
    creates on first use, allocator growth in torch's own kernels)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def make_flush(device, nbytes):
    """Evict the workload from L2 by reading a buffer twice the size of L2.

    A read leaves only clean lines behind, so the timed kernel does not pay for
    writing the flush buffer back (the previous step's dirty outputs are written
    back during the flush itself).
    """
    import torch
    buf = torch.ones(nbytes // 4, dtype=torch.float32, device=device)
    return lambda: buf.sum()


def same_run_copy(device, nbytes=4 * 2 ** 30, K=5):
    """This GPU's copy bandwidth in this run: one device-to-device cudaMemcpyAsync of
    `nbytes` (torch's copy_ between two contiguous buffers), timed with CUDA events over K
    copies after two untimed ones.  Each copy reads and writes `nbytes`, both far larger
    than L2, so the figure is HBM's; the kernels' fractions against it sit beside the
    roofline's fraction of the recorded peak."""
    import torch
    src = torch.ones(nbytes // 2, dtype=torch.bfloat16, device=device)
    dst = torch.empty_like(src)
    ms = timed_calls(lambda: dst.copy_(src), K, torch.cuda.current_stream(device))
    del src, dst
    torch.cuda.empty_cache()
    return ms, 2 * nbytes


def run_variants(wl, K, stream, peak, flush):
    """The other hot-path modes on the same workload, each timed on its own.

    Every mode meant to give the plain call's bits is compared, on the device,
    with the plain tide_rs_reduce / tide_ag_place output of the same inputs
    ("same_bits_as_plain"); the plain calls are pinned to the CPU oracle by the
    test suite.  Tree order has its own bits and is not compared."""
    import torch
    from fsdp2_layout_aware_b200 import tide as T
    B = alg_bytes(wl.group, oracle_free_layout(wl))
    out = {}
    wl.plan.rs_reduce(wl.grads_t, wl.out)
    wl.plan.ag_place(wl.ag, wl.params_t)
    torch.cuda.synchronize()
    ref_out = wl.out.view(torch.int32).clone()
    ref_params = [p.view(torch.int16).clone() for p in wl.params]

    def same_rs():
        torch.cuda.synchronize()
        return bool(torch.equal(wl.out.view(torch.int32), ref_out))

    def same_ag():
        torch.cuda.synchronize()
        return all(bool(torch.equal(p.view(torch.int16), q)) for p, q in zip(wl.params, ref_params))

    def rec(name, ms, nbytes, launches, plan=None, same=None):
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                     "alg_bytes": nbytes, "kernel_launches": launches}
        if plan is not None:
            k, n = plan.last_launch()
            out[name]["kernel"] = T.KERNEL_NAMES[k] if k >= 0 else "copy engines"
            out[name]["ctas"] = n if k >= 0 else 0
        if same is not None:
            out[name]["same_bits_as_plain"] = same()

    wl.params_poison()
    rec("ag_place_ce", timed_calls(lambda: wl.plan.ag_place(wl.ag, wl.params_t, engine=T.TIDE_ENGINE_CE),
                                   K, stream, flush), B["ag"], 0, wl.plan, same_ag)
    rec("rs_reduce_tree", timed_calls(lambda: wl.plan.rs_reduce(wl.grads_t, wl.out, order=T.TIDE_ORDER_TREE),
                                      K, stream, flush), B["rs"], 1, wl.plan)
    tma_plan = T.Plan(wl.group.shapes, wl.group.world, device=wl.out.device, tma=True)
    wl.out.fill_(float("nan"))
    rec("rs_reduce_tma", timed_calls(lambda: tma_plan.rs_reduce(wl.grads_t, wl.out), K, stream, flush),
        B["rs"], 1, tma_plan, same_rs)
    tma_plan.close()
    # the exchange as one rank runs it: rank 0 reduces its own shard ...
    rank0 = T.Plan(wl.group.shapes, wl.group.world, device=wl.out.device, rank=0)
    n0 = sum(min(rank0.query(i)["chunk_numel"], wl.group.numel(i)) for i in range(wl.group.n_params))
    shard0 = torch.full((wl.Ns,), float("nan"), device=wl.out.device)
    rec("rs_reduce_one_rank", timed_calls(lambda: rank0.rs_reduce(wl.grads_t, shard0), K, stream, flush),
        2 * wl.group.world * n0 + 4 * wl.Ns, 1, rank0,
        lambda: bool(torch.equal(shard0.view(torch.int32), ref_out[: wl.Ns])))
    rank0.close()
    del shard0
    # ... and places every rank's shard, each from its own buffer (here: row r of the input)
    flat_ag = wl.ag.reshape(-1)
    shards = T.TensorTable([flat_ag[r * wl.Ns: (r + 1) * wl.Ns] for r in range(wl.group.world)])
    for eng, name in ((T.TIDE_ENGINE_SM, "sm"), (T.TIDE_ENGINE_CE, "ce")):
        wl.params_poison()
        rec(f"ag_gather_place_{name}",
            timed_calls(lambda: wl.plan.ag_gather_place(shards, wl.params_t, engine=eng), K, stream, flush),
            B["ag"], 1 if eng == 0 else 0, wl.plan, same_ag)
    del shards, flat_ag
    slots = wl.ensure_slots()
    for eng, name in ((T.TIDE_ENGINE_SM, "sm"), (T.TIDE_ENGINE_CE, "ce")):
        rec(f"slot_stage_{name}", timed_calls(lambda: wl.plan.rs_stage(wl.grads_t, slots, engine=eng),
                                              K, stream, flush), B["stage"], 1 if eng == 0 else 0, wl.plan)
    wl.out.fill_(float("nan"))
    rec("slot_reduce", timed_calls(lambda: wl.plan.rs_reduce_slots(slots, wl.out), K, stream, flush),
        B["slot_rs"], 1, wl.plan, same_rs)
    # both phases: one after the other (CE staging, then the reduce kernel) ...
    wl.out.fill_(float("nan"))
    rec("slot_reuse_serial_ce",
        timed_calls(lambda: wl.plan.rs_reduce(wl.grads_t, wl.out, slots=slots, engine=T.TIDE_ENGINE_CE),
                    K, stream, flush), B["stage"] + B["slot_rs"], 1, wl.plan, same_rs)
    # ... and overlapped: the copy engines stage run s+1 while the SMs reduce run s
    cs = torch.cuda.Stream(wl.out.device)
    W = wl.group.world
    # (a full-grid reduction keeps the copy engines from progressing beside it, so the
    # overlapped runs cap the reduction at one CTA per SM; one segment is the serial order)
    sms = torch.cuda.get_device_properties(wl.out.device).multi_processor_count
    for nseg in sorted({1, min(4, W), W}):
        cap = 0 if nseg == 1 else sms
        wl.out.fill_(float("nan"))
        rec(f"slot_reuse_pipelined_seg{nseg}",
            timed_calls(lambda: wl.plan.rs_reduce_pipelined(wl.grads_t, wl.out, slots, nseg, cs,
                                                            max_ctas=cap),
                        K, stream, flush), B["stage"] + B["slot_rs"], nseg, wl.plan, same_rs)
        out[f"slot_reuse_pipelined_seg{nseg}"]["max_ctas"] = cap
    wl.drop_slots()
    del slots
    # Context: the stock FSDP2 layout conversion with torch's own kernels on the same GPU
    # (gradients packed by torch._chunk_cat into a fp32 rank-major buffer per rank, summed in
    # rank order, scaled; all-gather copy-out by torch.split_with_sizes_copy).  Same bits as
    # ours; rated against the same algorithmic bytes so the GB/s compare directly.
    Ns = wl.Ns
    chunks = [wl.plan.query(i)["chunk_numel"] for i in range(wl.group.n_params)]
    pack = torch.empty(W, Ns, dtype=torch.float32, device=wl.out.device)
    stock = torch.empty(W, Ns, dtype=torch.float32, device=wl.out.device)
    stock_params = [torch.empty(W * c, dtype=torch.bfloat16, device=wl.out.device) for c in chunks]

    def stock_rs():
        for k in range(W):
            torch._chunk_cat(wl.grads[k], dim=0, num_chunks=W, out=stock if k == 0 else pack)
            if k:
                stock.add_(pack)
        stock.mul_(1.0 / W)

    def stock_ag():
        torch.split_with_sizes_copy(wl.ag.view(W, Ns), chunks, dim=1,
                                    out=[p.view(W, c) for p, c in zip(stock_params, chunks)])

    rec("stock_torch_pack_reduce", timed_calls(stock_rs, K, stream, flush), B["rs"], 2 * W)
    rec("stock_torch_copyout", timed_calls(stock_ag, K, stream, flush), B["ag"], 1)
    wl.plan.rs_reduce(wl.grads_t, wl.out)
    wl.plan.ag_place(wl.ag, wl.params_t)
    torch.cuda.synchronize()
    out["stock_torch_pack_reduce"]["same_bits_as_tide"] = bool(
        torch.equal(stock.view(-1).view(torch.int32), wl.out.view(torch.int32)))
    # stock copy-out also copies the all-gather buffer's pad slots; compare valid rows only
    same = True
    for i, (p, q) in enumerate(zip(stock_params, wl.params)):
        n = wl.group.numel(i)
        same &= bool(torch.equal(p[:n].view(torch.int16), q[:n].view(torch.int16)))
    out["stock_torch_copyout"]["same_valid_bits_as_tide"] = same
    del pack, stock, stock_params
    # fp32 gradients (FSDP2's, accumulated with gradient sync off) through fp32 slots: each
    # rank's gradients widened to fp32 (exactly) and staged into its own slot, then the slots
    # reduced in rank order, which must give the plain reduction's bits
    f32_bytes = 4 * W * W * Ns
    if f32_bytes <= 32 * 2 ** 30:
        N = B["N"]
        slots32 = [torch.empty(W * Ns, dtype=torch.float32, device=wl.out.device) for _ in range(W)]
        for k in range(W):
            g32 = T.TensorTable([t.float() for t in wl.grads[k]])
            if k == 0:
                rec("stage_one_f32_ce",
                    timed_calls(lambda: wl.plan.rs_stage_one_f32(g32, slots32[0], engine=T.TIDE_ENGINE_CE),
                                K, stream, flush), 8 * N, 0, wl.plan)
                rec("stage_one_f32", timed_calls(lambda: wl.plan.rs_stage_one_f32(g32, slots32[0]),
                                                 K, stream, flush), 8 * N, 1, wl.plan)
            else:
                wl.plan.rs_stage_one_f32(g32, slots32[k])
            del g32
        wl.out.fill_(float("nan"))
        rec("slot_reduce_f32", timed_calls(lambda: wl.plan.rs_reduce_slots_f32(slots32, wl.out),
                                           K, stream, flush), 4 * W * N + 4 * W * Ns, 1, wl.plan, same_rs)
        del slots32
        # ... and read in place, every rank's fp32 gradients at once (TIDE-RS itself)
        g32_all = T.TensorTable([t.float() for row in wl.grads for t in row])
        wl.out.fill_(float("nan"))
        rec("rs_reduce_f32", timed_calls(lambda: wl.plan.rs_reduce_f32(g32_all, wl.out), K, stream, flush),
            4 * W * N + 4 * W * Ns, 1, wl.plan, same_rs)
        del g32_all
    else:
        out["slot_reduce_f32"] = {"skipped": f"fp32 slots of {f32_bytes / 2 ** 30:.0f} GiB"}
    del ref_out, ref_params
    wl.drop_slots()
    return out


# (op, mode) of each timed entry of a bench line, for the flat JSONL log
ROW_KINDS = {
    "rs_reduce_kernel": ("rs_reduce", "SM, rank order"),
    "ag_place_kernel": ("ag_place", "SM"),
    "ag_place_ce": ("ag_place", "copy engines"),
    "rs_reduce_tree": ("rs_reduce", "SM, tree order"),
    "rs_reduce_tma": ("rs_reduce", "SM bulk-copy kernel, rank order"),
    "slot_stage_sm": ("slot_stage", "SM"),
    "slot_stage_ce": ("slot_stage", "copy engines"),
    "slot_reduce": ("slot_reduce", "SM, rank order"),
    "slot_reuse_serial_ce": ("slot_reuse", "copy-engine staging, then reduce"),
    "rs_reduce_one_rank": ("rs_reduce", "one rank's shard (one-rank plan), rank order"),
    "ag_gather_place_sm": ("ag_gather_place", "SM, from per-rank shards"),
    "ag_gather_place_ce": ("ag_gather_place", "copy engines, from per-rank shards"),
    "stage_one_f32": ("slot_stage", "fp32 gradients of one rank, SM"),
    "stage_one_f32_ce": ("slot_stage", "fp32 gradients of one rank, copy engines"),
    "slot_reduce_f32": ("slot_reduce", "fp32 slots, SM, rank order"),
    "rs_reduce_f32": ("rs_reduce", "fp32 gradients read in place, SM, rank order"),
    "stock_torch_pack_reduce": ("stock_rs", "torch _chunk_cat pack + add"),
    "stock_torch_copyout": ("stock_ag", "torch split_with_sizes_copy"),
}


def rs_sm_time(rs_ms: float, rs_ctas: int, variants: dict, sms: int) -> dict:
    """SM time of the reduce-scatter's layout work, stock against TIDE: SMs held x duration,
    the one-GPU analogue of the pages' lower RS SM time (weekinpapers.com, Abstract).  A
    TIDE kernel holds min(CTAs, SMs) SMs for its launch, copy-engine staging holds none, and
    torch's pack and add kernels are counted at the whole GPU."""
    stock = sms * variants["stock_torch_pack_reduce"]["ms"]
    tide = min(rs_ctas, sms) * rs_ms
    slot = variants["slot_reduce"]
    reuse = min(slot.get("ctas", sms), sms) * slot["ms"]
    return {"unit": "SM-ms", "stock_pack_reduce": round(stock, 2), "tide_rs_reduce": round(tide, 2),
            "tide_slot_reuse_ce": round(reuse, 2),
            "note": "Slot-Reuse with copy-engine staging: the staging holds no SM, the reduction "
                    "of the slots does",
            "stock_over_tide": round(stock / tide, 2), "stock_over_slot_reuse_ce": round(stock / reuse, 2)}


def jsonl_rows(res, group_name, world):
    """One flat row per (config, op, mode, ctas) of a bench line."""
    rows = []
    cpu = res.get("cpu_baseline") or {}
    entries = list(res.get("kernels", {}).items()) + list(res.get("variants", {}).items())
    for name, e in entries:
        if "skipped" in e:
            continue
        op, mode = ROW_KINDS.get(name, (name, ""))
        if name.startswith("slot_reuse_pipelined_seg"):
            op, mode = "slot_reuse", f"pipelined, {name.rsplit('seg', 1)[1]} segments"
        same = e.get("same_bits_as_plain", e.get("same_bits_as_tide", e.get("same_valid_bits_as_tide")))
        rows.append({
            "config": group_name, "world": world, "op": op, "mode": mode, "entry": name,
            "kernel": e.get("kernel"), "ctas": e.get("ctas"), "alg_bytes": e["alg_bytes"],
            "ms": e["ms"], "GB/s": e["GB/s"], "frac_of_measured_peak": e["frac_of_peak"],
            "dram_bytes_per_launch": e.get("traffic"),
            "same_bits_as_plain": same,
            "oracle_GB/s": cpu.get("value"), "oracle_cores": cpu.get("cores"),
            "host_cores": len(os.sched_getaffinity(0)),
            "sm_mhz": (res.get("clocks") or {}).get("sm_mhz"),
        })
    return rows


def oracle_free_layout(wl):
    """Layout sizes from the plan (the product side never calls the oracle)."""
    class L:
        pass
    L.Ns = wl.Ns
    return L


def run_e2e(wl, K, stream):
    """The step through the C-ABI with host buffers: H2D inputs, AG + RS, D2H results.

    Every step copies all its inputs from pinned host memory and reads all its
    outputs (fp32 shards and placed parameters) back.  Three streams pipeline
    consecutive steps: step i+1's H2D starts once step i's kernels have
    consumed the inputs, while step i's D2H runs on the other copy direction;
    step i+1's kernels wait for step i's D2H before overwriting the outputs.
    Returns (pipelined ms/step, serial ms/step, h2d bytes, d2h bytes, pinned?).
    """
    import torch
    dev = wl.out.device
    need = (sum(t.numel() * t.element_size() for row in wl.grads for t in row) + wl.ag.numel() * 2 +
            wl.out.numel() * 4 + sum(p.numel() * 2 for p in wl.params))
    # every rank on this node pins its own copy; fall back to pageable host memory
    # rather than pin more than about half of what the host has free
    local = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    try:
        import psutil
        pin = need * local < 0.5 * psutil.virtual_memory().available
    except Exception:
        pin = True
    host = (lambda t: t.pin_memory()) if pin else (lambda t: t)
    g_host = [[host(t.cpu()) for t in row] for row in wl.grads]
    ag_host = host(wl.ag.cpu())
    out_host = host(torch.empty(wl.out.shape, dtype=wl.out.dtype))
    par_host = [host(torch.empty(p.shape, dtype=p.dtype)) for p in wl.params]
    h2d = sum(t.numel() * t.element_size() for row in g_host for t in row) + ag_host.numel() * 2
    d2h = out_host.numel() * 4 + sum(p.numel() * 2 for p in par_host)
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def h2d_copies(st):
        for row_d, row_h in zip(wl.grads, g_host):
            for d, h in zip(row_d, row_h):
                d.copy_(h, non_blocking=True)
        wl.ag.copy_(ag_host, non_blocking=True)

    def kernels(st):
        wl.plan.ag_place(wl.ag, wl.params_t, stream=st)
        wl.plan.rs_reduce(wl.grads_t, wl.out, stream=st)

    def d2h_copies(st):
        out_host.copy_(wl.out, non_blocking=True)
        for d, h in zip(wl.params, par_host):
            h.copy_(d, non_blocking=True)

    def serial_step():
        with torch.cuda.stream(stream):
            h2d_copies(stream); kernels(stream); d2h_copies(stream)

    def pipelined(n):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(s_in)
        done_cmp, done_out = None, None
        for _ in range(n):
            with torch.cuda.stream(s_in):
                if done_cmp is not None:
                    s_in.wait_event(done_cmp)      # inputs consumed by the previous step
                h2d_copies(s_in)
                done_in = ev(); done_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(done_in)
                if done_out is not None:
                    s_cmp.wait_event(done_out)     # previous outputs read back
                kernels(s_cmp)
                done_cmp = ev(); done_cmp.record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_cmp)
                d2h_copies(s_out)
                done_out = ev(); done_out.record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n

    serial_step()
    serial_ms = timed_calls(serial_step, max(1, min(K, 3)), stream)
    pipelined(1)
    ms = pipelined(K)
    del g_host, ag_host, out_host, par_host
    return ms, serial_ms, h2d, d2h, pin


# --------------------------------------------------------------------------- the oracle on host cores


def oracle_items(group, max_elems=16 * 2 ** 20):
    """The work items of an oracle sample: row blocks (i, a, b, inner) of the group's params.

    Each block (rows a..b-1 of param i, at most max_elems elements) is run as a
    one-param group over the same W: per element the same work as in the whole
    group (W bf16 reads, W-1 fp32 adds, the scale, one fp32 write; the copy-out).
    """
    items = []
    for i, shape in enumerate(group.shapes):
        d0 = shape[0]
        inner = 1
        for x in shape[1:]:
            inner *= x
        if d0 * inner == 0:
            continue
        rows = max(1, min(d0, max_elems // inner))
        for a in range(0, d0, rows):
            items.append((i, a, min(d0, a + rows), inner))
    return items


def oracle_item_bytes(W, item):
    """(RS, AG) algorithmic bytes of one item as a one-param group over W ranks."""
    _, a, b, inner = item
    n = (b - a) * inner
    npad = W * (-(-(b - a) // W)) * inner
    return 2 * W * n + 4 * npad, 2 * n + 2 * npad


def oracle_item_inputs(group, seed, item):
    """Host inputs of one item: each rank's gradient rows a..b-1 of param i, and an all-gather
    buffer of the item's layout (values drawn by the seeded generator)."""
    import numpy as np
    import synth
    i, a, b, inner = item
    W = group.world
    n = (b - a) * inner
    shape = (b - a, inner) if len(group.shapes[i]) > 1 else (b - a,)
    grads = []
    for k in range(W):
        if i in synth.zero_grad_params(group, seed, k):
            grads.append([np.zeros(n, dtype=np.uint16)])
        else:
            grads.append([synth.fill_bf16(n, seed, synth.STREAM_GRAD, k, i, group.grad_sigma,
                                          idx0=a * inner)])
    npad = W * (-(-(b - a) // W)) * inner
    ag = synth.fill_bf16(npad, seed, synth.STREAM_AG, 0, i, group.param_sigma, idx0=W * a * inner)
    return shape, grads, ag


def oracle_item_run(W, inputs):
    """One item through the oracle as it stands: RS x fl32(1/W), then the AG copy-out.
    Returns (RS seconds, AG seconds)."""
    import oracle
    shape, grads, ag = inputs
    t0 = time.perf_counter()
    oracle.rs_reduce(W, (shape,), grads, 1)
    t1 = time.perf_counter()
    oracle.ag_copyout(W, (shape,), ag)
    return t1 - t0, time.perf_counter() - t1


def _oracle_worker(root, group_name, seed, items, n_passes, barrier, queue):
    """One host process of the all-cores oracle: generate its items, then run n_passes passes
    over them, each started together with the other workers at a barrier."""
    if root not in sys.path:
        sys.path.insert(0, root)
    from synth import configs
    group = configs.by_name(group_name)
    inputs = [oracle_item_inputs(group, seed, it) for it in items]
    times = []
    for _ in range(n_passes):
        barrier.wait()
        t0 = time.perf_counter()
        for inp in inputs:
            oracle_item_run(group.world, inp)
        times.append(time.perf_counter() - t0)
    queue.put(times)


def oracle_pool_passes(group, seed, items, n_workers, n_passes):
    """Per pass, the wall time of the all-cores oracle over `items`: n_workers spawned processes
    (each item goes whole to one worker, balanced by bytes), started together at a barrier;
    a pass ends when the slowest worker ends.  Input generation is outside the passes."""
    import multiprocessing as mp
    W = group.world
    n_workers = max(1, min(n_workers, len(items)))
    bins = [[] for _ in range(n_workers)]
    load = [0] * n_workers
    for it in sorted(items, key=lambda it: -sum(oracle_item_bytes(W, it))):
        j = load.index(min(load))
        bins[j].append(it)
        load[j] += sum(oracle_item_bytes(W, it))
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(n_workers)
    queue = ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(ROOT, group.name, seed, b, n_passes, barrier, queue))
             for b in bins]
    for p in procs:
        p.start()
    try:
        results = [queue.get(timeout=1800) for _ in procs]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    return [max(r[j] for r in results) for j in range(n_passes)], n_workers


def oracle_sample(group, budget_bytes):
    """The items of the group, in group order, up to `budget_bytes` algorithmic bytes (at least
    one item), and that byte count."""
    W = group.world
    items, total = [], 0
    for it in oracle_items(group):
        rb, ab = oracle_item_bytes(W, it)
        if items and total + rb + ab > budget_bytes:
            break
        items.append(it)
        total += rb + ab
    return items, total


def sample_budget_bytes(group, cap_bytes=None):
    """The oracle sample's byte budget: the whole group, unless its inputs would take more than
    a third of the host's available memory (every worker holds its items' inputs at once)."""
    W = group.world
    whole = sum(sum(oracle_item_bytes(W, it)) for it in oracle_items(group))
    budget = whole if cap_bytes is None else min(whole, cap_bytes)
    try:
        import psutil
        avail = psutil.virtual_memory().available
        # inputs are about (2W + 2) / (2W + 4 + 4) of the algorithmic bytes; allow for outputs too
        budget = min(budget, int(avail / 3))
    except Exception:
        pass
    return budget


def describe_sample(group, items, nbytes):
    idx = sorted({i for i, _, _, _ in items})
    names = [group.names[i] if group.names else str(i) for i in idx]
    if len(names) > 12:
        names = names[:6] + ["..."] + names[-3:]
    return (f"{group.name}: {len(items)} row blocks of params {names} (each block of at most "
            f"16M elements run as a one-param group over W={group.world}), RS x fl32(1/W) + AG "
            f"copy-out, {nbytes / 1e9:.2f} GB algorithmic; input generation excluded")


def cpu_baseline(group, seed, budget_s, cap_bytes=None):
    """The oracle as it stands on the host cores, on one sample of the workload, timed twice:
    single-threaded in this process (until `budget_s` of oracle time), and on every available
    core with one process per core over the same blocks (the blocks are independent, so the
    oracle code and its bits are unchanged).  The all-cores figure is the headline."""
    W = group.world
    items, nbytes = oracle_sample(group, sample_budget_bytes(group, cap_bytes))
    rs_s = ag_s = 0.0
    rs_b = ag_b = 0
    single_items = []
    for it in items:
        r, a = oracle_item_run(W, oracle_item_inputs(group, seed, it))
        rs_s += r
        ag_s += a
        rb, ab = oracle_item_bytes(W, it)
        rs_b += rb
        ag_b += ab
        single_items.append(it)
        if rs_s + ag_s >= budget_s:
            break
    single_bytes = rs_b + ag_b
    cores = len(os.sched_getaffinity(0))
    passes, workers = oracle_pool_passes(group, seed, items, cores, 2)
    wall = min(passes)
    value = nbytes / wall / 1e9
    return {"value": round(value, 3), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": describe_sample(group, items, nbytes) +
                      f"; {workers} processes, best of 2 passes",
            "seconds": round(wall, 3),
            "single_thread": {
                "value": round(single_bytes / (rs_s + ag_s) / 1e9, 3), "unit": "GB/s", "cores": 1,
                "sample": f"the first {len(single_items)} of those blocks, "
                          f"{single_bytes / 1e9:.2f} GB algorithmic",
                "seconds": round(rs_s + ag_s, 2),
                # the two oracle steps timed apart: pack + reduce, and the all-gather copy-out
                "rs_pack_reduce": {"GB/s": round(rs_b / rs_s / 1e9, 3), "seconds": round(rs_s, 2)},
                "ag_copyout": {"GB/s": round(ag_b / ag_s / 1e9, 3) if ag_s > 0 else None,
                               "seconds": round(ag_s, 3)}},
            "host": host_cpu()}


def host_cpu():
    """CPU model and the cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "cores_available": len(os.sched_getaffinity(0))}


def gemm_kernel_launch(a, b, c):
    """Name and grid (CTAs) of the kernel torch.matmul(a, b, out=c) launches, read from a
    torch profiler trace (no ncu)."""
    import tempfile
    import torch
    from torch.profiler import ProfilerActivity, profile
    torch.matmul(a, b, out=c)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        torch.matmul(a, b, out=c)
        torch.cuda.synchronize()
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "trace.json")
        prof.export_chrome_trace(path)
        with open(path) as f:
            trace = json.load(f)
    kernels = [e for e in trace.get("traceEvents", []) if e.get("cat") == "kernel"]
    if not kernels:
        return {"kernel": None, "grid": None, "ctas": None}
    k = max(kernels, key=lambda e: e.get("dur", 0))
    grid = k.get("args", {}).get("grid")
    ctas = grid[0] * grid[1] * grid[2] if grid else None
    return {"kernel": k.get("name"), "grid": grid, "ctas": ctas,
            "cluster": k.get("args", {}).get("cluster")}


def run_interference(device, seed, quick=False):
    """Slowdown of a concurrent bf16 GEMM vs the RS kernel's CTA count (sweep_w8 group).

    GEMMs: the configured 8192x8192x8192 (cuBLAS picks a 1024-CTA kernel on
    B200, i.e. not single-wave) and 3072x3072x16384, whose kernel fits in one
    wave; each GEMM's kernel and grid come from a torch profiler trace.  Per
    point: the GEMM batch alone, then concurrently with back-to-back RS launches
    on a second stream (started first, enough of them to outlast the GEMMs twice
    over); slowdown = median(concurrent) / median(alone) - 1.  Done for the
    load/store RS kernel at 8, 16, 32 and all CTAs, and for the Slot-Reuse
    staging on the copy engines (no SM; its bytes are the staging's).  The full
    sweep (quick=False) takes three trials per point and adds the bulk-copy (TMA)
    kernel; quick=True takes one trial and shorter GEMM batches (about 10 s in
    all, for the default bench line).
    """
    import torch
    from synth import configs
    from fsdp2_layout_aware_b200 import tide as T
    t_start = time.perf_counter()
    group = configs.sweep(8)
    wl = Workload(group, seed, device)
    plans = {"lsu": wl.plan, "tma": T.Plan(group.shapes, group.world, device=device, tma=True)}
    trials = 1 if quick else 3
    B = alg_bytes(group, oracle_free_layout(wl))
    short = T.Plan(group.shapes, group.world, device=device, short_ctas=True)
    s_gemm = torch.cuda.Stream(device)
    s_gemm_hi = torch.cuda.Stream(device, priority=-5)    # the device's highest priority
    s_rs = torch.cuda.Stream(device)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    res = {"rs_workload": "sweep_w8 (16 x 512x4096 params, W=8), rank order, x fl32(1/W)",
           "trials": trials, "sm_count": sms, "gemms": []}
    for (m, n, k, n_gemm) in ((8192, 8192, 8192, 40), (3072, 3072, 16384, 120)):
        if quick:
            n_gemm //= 2
        a = torch.randn(m, k, dtype=torch.bfloat16, device=device)
        b = torch.randn(k, n, dtype=torch.bfloat16, device=device)
        c = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        launch = gemm_kernel_launch(a, b, c)

        def gemm_batch():
            for _ in range(n_gemm):
                torch.matmul(a, b, out=c)

        def gemm_alone(sg=s_gemm):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            with torch.cuda.stream(sg):
                e0.record(sg); gemm_batch(); e1.record(sg)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n_gemm

        # warm both GEMM streams: cuBLAS sets up a stream's workspace on its first GEMM, and a
        # cold high-priority stream would inflate that point's time alone
        for _ in range(3 if quick else 5):
            gemm_alone()
            gemm_alone(s_gemm_hi)
        g = {"gemm": f"bf16 {m}x{n}x{k} torch.matmul (cuBLAS), {n_gemm} per batch",
             "kernel": launch["kernel"], "grid": launch["grid"], "ctas": launch["ctas"],
             "single_wave": (launch["ctas"] <= sms) if launch["ctas"] else None, "points": []}
        # CTA caps: the single-wave GEMM leaves sm_count - 144 = 4 SMs idle on B200, so caps of
        # 2 and 4 fit beside it and 8 and more do not
        caps = {"lsu": (2, 4, 8, 16, 32, 0), "tma": (4,) if quick else (2, 4, 8, 16, 32, 0)}
        points = [(kind, plans[kind], ctas, B["rs"],
                   lambda plan=plans[kind], ctas=ctas: plan.rs_reduce(wl.grads_t, wl.out, max_ctas=ctas,
                                                                      stream=s_rs),
                   s_gemm)
                  for kind in ("lsu", "tma") for ctas in caps[kind]]
        slots = T.TensorTable(wl.ensure_slots())
        points.append(("ce_stage", wl.plan, 0, B["stage"],
                       lambda: wl.plan.rs_stage(wl.grads_t, slots, engine=T.TIDE_ENGINE_CE, stream=s_rs),
                       s_gemm))
        # short-lived CTAs (one per tile), with the GEMM's stream at the default priority and
        # at the highest; the persistent full grid with the high-priority GEMM for contrast
        points.append(("lsu_short_gemm_high_priority", short, 0, B["rs"],
                       lambda: short.rs_reduce(wl.grads_t, wl.out, stream=s_rs), s_gemm_hi))
        if not quick:
            points.append(("lsu_short", short, 0, B["rs"],
                           lambda: short.rs_reduce(wl.grads_t, wl.out, stream=s_rs), s_gemm))
            points.append(("lsu_gemm_high_priority", wl.plan, 0, B["rs"],
                           lambda: wl.plan.rs_reduce(wl.grads_t, wl.out, stream=s_rs), s_gemm_hi))
        for kind, plan, ctas, nbytes, call, sg in points:
            rs_ms = timed_calls(call, 3 if quick else 5, s_rs)
            n_ctas = max(0, plan.last_launch()[1]) if kind != "ce_stage" else 0
            alone, conc, rs_conc = [], [], []
            for _ in range(trials):
                alone.append(gemm_alone(sg))
                reps = int((alone[-1] * n_gemm * 2.0) / max(rs_ms, 1e-3)) + 2
                torch.cuda.synchronize()
                r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(s_rs):
                    r0.record(s_rs)
                    for _ in range(reps):
                        call()
                    r1.record(s_rs)
                with torch.cuda.stream(sg):
                    e0.record(sg); gemm_batch(); e1.record(sg)
                torch.cuda.synchronize()
                conc.append(e0.elapsed_time(e1) / n_gemm)
                rs_conc.append(r0.elapsed_time(r1) / reps)
            ga, gc = statistics.median(alone), statistics.median(conc)
            g["points"].append({
                "rs_kernel": kind, "max_ctas": ctas, "ctas": n_ctas, "rs_ms_alone": round(rs_ms, 4),
                "rs_GBps_alone": round(nbytes / (rs_ms * 1e-3) / 1e9, 1),
                "rs_ms_concurrent": round(statistics.median(rs_conc), 4),
                "gemm_ms_alone": round(ga, 4), "gemm_ms_concurrent": round(gc, 4),
                "gemm_slowdown": round(gc / ga - 1.0, 4),
                "rs_cta_ms_per_call": round(n_ctas * rs_ms, 2)})
        res["gemms"].append(g)
        del a, b, c, slots
        wl.drop_slots()
    plans["tma"].close()
    short.close()
    del wl
    torch.cuda.empty_cache()
    res["seconds"] = round(time.perf_counter() - t_start, 1)
    return res


def run_m1_step(wl, steps, tokens=8192):
    """One data-parallel rank's step on one layer group, with the stock FSDP2 layout
    conversion and with TIDE's calls: the single-GPU analogue of the pages' measurement that
    layout conversion takes 6.4 % of step time on Llama-3.1 70B at 8K tokens per GPU
    (weekinpapers.com, Abstract; kongchang.com, "The Root of FSDP2 Communication Overhead").

    Compute: every 2-D parameter is a linear layer; forward Y = X W^T, backward dX = dY W
    and dW = dY^T X for `tokens` tokens (bf16 torch.matmul, cuBLAS), with W the placed
    parameter and dW written into this rank's (rank 0's) gradient, so the step reads what
    the all-gather placed and the reduce-scatter reads what the backward wrote.  The
    attention core, norms and activations are left out (linear layers only).
      stock: copy-out (torch.split_with_sizes_copy, all-gather buffer -> parameters),
             compute, pack of this rank's gradients into a fp32 rank-major buffer
             (torch._chunk_cat), then this rank's shard reduced in rank order from the W
             ranks' packed buffers (the other W-1 were packed beforehand, as their own
             ranks would have) and scaled -- the reduction NCCL would do;
      tide:  tide_ag_place, compute, tide_rs_reduce with this rank's one-rank plan
             (bf16 gradients read where they lie, no pack).
    The network transfers are absent on one GPU in both.  Layout conversion in the stock
    step = copy-out + pack; its share is over the stock step.  Both give the same shard bits.
    """
    import torch
    from fsdp2_layout_aware_b200 import tide as T
    g = wl.group
    W, Ns = g.world, wl.Ns
    dev = wl.out.device
    stream = torch.cuda.current_stream(dev)
    lin = [i for i, sh in enumerate(g.shapes) if len(sh) == 2]
    dims_in = sorted({g.shapes[i][1] for i in lin})
    dims_out = sorted({g.shapes[i][0] for i in lin})
    gen = torch.Generator(device=dev).manual_seed(7)
    X = {d: torch.randn(tokens, d, device=dev, dtype=torch.bfloat16, generator=gen) for d in dims_in}
    dY = {d: torch.randn(tokens, d, device=dev, dtype=torch.bfloat16, generator=gen) for d in dims_out}
    Y = {d: torch.empty(tokens, d, device=dev, dtype=torch.bfloat16) for d in dims_out}
    dX = {d: torch.empty(tokens, d, device=dev, dtype=torch.bfloat16) for d in dims_in}
    flops = sum(6 * tokens * g.shapes[i][0] * g.shapes[i][1] for i in lin)
    chunks = [wl.plan.query(i)["chunk_numel"] for i in range(g.n_params)]
    stock_params = [torch.empty(W * c, dtype=torch.bfloat16, device=dev) for c in chunks]
    my_grads = wl.grads[0]

    def compute(params):
        for i in lin:
            d_out, d_in = g.shapes[i]
            w = params[i][: d_out * d_in].view(d_out, d_in)
            torch.matmul(X[d_in], w.t(), out=Y[d_out])
            torch.matmul(dY[d_out], w, out=dX[d_in])
            torch.matmul(dY[d_out].t(), X[d_in], out=my_grads[i])

    # chunk 0 of the other ranks' packed fp32 buffers, as their own ranks would have packed
    # and sent them; this rank packs its whole gradient set into `own` every step
    own = torch.empty(W, Ns, dtype=torch.float32, device=dev)
    recv = torch.empty(W, Ns, dtype=torch.float32, device=dev)
    for k in range(1, W):
        torch._chunk_cat(wl.grads[k], dim=0, num_chunks=W, out=own)
        recv[k].copy_(own[0])
    stock_shard = torch.empty(Ns, dtype=torch.float32, device=dev)
    rank0 = T.Plan(g.shapes, W, device=dev, rank=0)
    tide_shard = torch.empty(Ns, dtype=torch.float32, device=dev)
    params_t = wl.params_t

    def phases_stock():
        return [lambda: torch.split_with_sizes_copy(wl.ag.view(W, Ns), chunks, dim=1,
                                                    out=[p.view(W, c) for p, c in zip(stock_params, chunks)]),
                lambda: compute(stock_params),
                lambda: torch._chunk_cat(my_grads, dim=0, num_chunks=W, out=own),
                lambda: _rank_order_shard(own[0], recv, stock_shard, W)]

    def phases_tide():
        return [lambda: wl.plan.ag_place(wl.ag, params_t),
                lambda: compute(wl.params),
                lambda: rank0.rs_reduce(wl.grads_t, tide_shard)]

    def record(phases, evs):
        evs[0].record(stream)
        for j, f in enumerate(phases):
            f()
            evs[j + 1].record(stream)

    # the two steps alternate, so that clock and power-cap drift hits both alike
    n = max(3, min(steps, 10))
    ps, pt = phases_stock(), phases_tide()
    for _ in range(2):
        for f in ps + pt:
            f()
    torch.cuda.synchronize()
    ev_s = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ps) + 1)] for _ in range(n)]
    ev_t = [[torch.cuda.Event(enable_timing=True) for _ in range(len(pt) + 1)] for _ in range(n)]
    for es, et in zip(ev_s, ev_t):
        record(ps, es)
        record(pt, et)
    torch.cuda.synchronize()
    ts = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev_s) for j in range(len(ps))]
    tt = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev_t) for j in range(len(pt))]
    same = bool(torch.equal(stock_shard.view(torch.int32), tide_shard.view(torch.int32)))
    rank0.close()
    stock_ms, tide_ms = sum(ts), sum(tt)
    conv = ts[0] + ts[2]
    del own, recv, stock_params, X, dY, Y, dX
    torch.cuda.empty_cache()
    return {
        "what": f"one rank's step on the {g.name} group: linear-layer forward + backward at "
                f"{tokens} tokens (bf16 cuBLAS), AG placement and reduce-scatter of its shard; "
                "network transfers absent",
        "tokens": tokens, "gemm_tflop": round(flops / 1e12, 2),
        "stock_ms": {"copyout": round(ts[0], 4), "compute": round(ts[1], 4), "pack": round(ts[2], 4),
                     "reduce_own_shard": round(ts[3], 4), "step": round(stock_ms, 4)},
        "tide_ms": {"ag_place": round(tt[0], 4), "compute": round(tt[1], 4),
                    "rs_reduce_own_shard": round(tt[2], 4), "step": round(tide_ms, 4)},
        "layout_conversion_share_stock": round(conv / stock_ms, 4),
        "pages_share": 0.064,
        "compute_TFLOPs": round(flops / (ts[1] * 1e-3) / 1e12, 1),
        "step_time_reduction": round(1.0 - tide_ms / stock_ms, 4),
        "same_shard_bits": same,
    }


def _rank_order_shard(own_chunk, recv, out, W):
    """Rank 0's shard summed in rank order 0..W-1 (its own packed chunk, then the chunks
    received from ranks 1..W-1), scaled by fl32(1/W): the stock reduce-scatter's arithmetic
    on one rank, with torch's kernels."""
    out.copy_(own_chunk)
    for k in range(1, W):
        out.add_(recv[k])
    out.mul_(1.0 / W)


def bench_workload(args, group, rank, world, device, dist_on):
    import torch
    from fsdp2_layout_aware_b200 import tide as T
    peak, peak_src = load_peaks()
    wl = Workload(group, args.seed, device)
    B = alg_bytes(group, oracle_free_layout(wl))
    stream = torch.cuda.current_stream(device)
    in_bytes = 2 * B["N"] * group.world
    flush = None if in_bytes > 4 * L2_BYTES else make_flush(device, 2 * L2_BYTES)

    order = T.TIDE_ORDER_TREE if args.rs_order == "tree" else T.TIDE_ORDER_RANK

    def step():
        wl.plan.ag_place(wl.ag, wl.params_t, max_ctas=args.max_ctas)
        wl.plan.rs_reduce(wl.grads_t, wl.out, max_ctas=args.max_ctas, order=order)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    wl.plan.check()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        start.record(stream)
        for e in evs:
            if flush is not None:
                flush()
            e[0].record(stream)
            wl.plan.ag_place(wl.ag, wl.params_t, max_ctas=args.max_ctas)
            e[1].record(stream)
            wl.plan.rs_reduce(wl.grads_t, wl.out, max_ctas=args.max_ctas, order=order)
            e[2].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    wl.plan.check()
    rs_kernel, rs_ctas = wl.plan.last_launch()
    total_ms = start.elapsed_time(end)
    ag_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    rs_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    step_ms = ag_ms + rs_ms if flush is not None else total_ms / K
    step_ms, ag_ms, rs_ms = max_over_ranks([step_ms, ag_ms, rs_ms], device)

    step_bytes = B["ag"] + B["rs"]
    value = replica_throughput(world, step_bytes, step_ms)
    rs_gbs = B["rs"] / (rs_ms * 1e-3) / 1e9
    ag_gbs = B["ag"] / (ag_ms * 1e-3) / 1e9
    rs_name = T.KERNEL_NAMES[rs_kernel]
    rs_traffic, rs_traffic_src = ncu_traffic(rs_name, RS_SOURCES, B["rs_read"], B["rs_write"])
    ag_traffic, ag_traffic_src = ncu_traffic("ag", AG_SOURCES, B["ag_read"], B["ag_write"])
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32", "data": "synthetic",
        "config": {
            "workload": f"{group.name} layer group, W={group.world} simulated ranks, "
                        f"{group.n_params} params, {B['N']} elements",
            "step": f"tide_ag_place(SM) + tide_rs_reduce({args.rs_order} order, x fl32(1/W))",
            "alg_bytes_per_step": step_bytes, "max_ctas": args.max_ctas,
            "l2": ("inputs larger than L2, no flush" if flush is None else
                   "L2 flushed (256 MB read) before every timed step"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(rs_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(rs_gbs / peak, 4), "peak_source": f"{peak_src} hbm_gbs",
                     "kernel": f"rs_reduce_kernel ({rs_name})", "alg_bytes_per_launch": B["rs"],
                     "avg_launch_ms": round(rs_ms, 4),
                     "traffic": None if rs_traffic is None else round(rs_traffic),
                     "traffic_source": rs_traffic_src},
        "kernels": {
            "rs_reduce_kernel": {"ms": round(rs_ms, 4), "GB/s": round(rs_gbs, 1),
                                 "frac_of_peak": round(rs_gbs / peak, 4), "alg_bytes": B["rs"],
                                 "ctas": rs_ctas, "kernel": rs_name,
                                 "traffic": None if rs_traffic is None else round(rs_traffic)},
            "ag_place_kernel": {"ms": round(ag_ms, 4), "GB/s": round(ag_gbs, 1),
                                "frac_of_peak": round(ag_gbs / peak, 4), "alg_bytes": B["ag"],
                                "ctas": wl.plan.launch_ctas(T.K_AG, args.max_ctas),
                                "traffic": None if ag_traffic is None else round(ag_traffic),
                                "traffic_source": ag_traffic_src}},
        "gpu_launches": 2 * K,
        "clocks": clk.summary(),
        "workspace_bytes": wl.plan.workspace_bytes,
        # what the stock path would hold instead: one full-group fp32 rank-major buffer per rank
        "stock_fp32_buffer_bytes": 4 * group.world * wl.Ns,
    }
    if not args.profile_small:   # a capture run keeps a few hundred MB on the device
        copy_ms, copy_bytes = same_run_copy(device)
        copy_ms = max_over_ranks([copy_ms], device)[0]
        copy_gbs = copy_bytes / (copy_ms * 1e-3) / 1e9
        res["copy_same_run"] = {"what": "device-to-device cudaMemcpyAsync of 4 GiB (reads and writes "
                                        "4 GiB), after the timed steps, 5 copies",
                                "ms": round(copy_ms, 4), "GB/s": round(copy_gbs, 1),
                                "rs_frac": round(rs_gbs / copy_gbs, 4),
                                "ag_frac": round(ag_gbs / copy_gbs, 4),
                                "step_frac": round(value / world / copy_gbs, 4)}
    if not args.no_variants:
        # the step's figures above stand even if a variant fails: record the error instead
        try:
            res["variants"] = run_variants(wl, max(3, min(K, 20)), stream, peak, flush)
            res["rs_sm_time"] = rs_sm_time(rs_ms, rs_ctas, res["variants"],
                                           torch.cuda.get_device_properties(device).multi_processor_count)
        except Exception as e:  # noqa: BLE001
            res["variants_error"] = f"{type(e).__name__}: {e}"
            wl.drop_slots()
    if group.name == "llama70b" and not args.no_m1 and world == 1:
        try:
            res["m1_step"] = run_m1_step(wl, K)
        except Exception as e:  # noqa: BLE001
            res["m1_step_error"] = f"{type(e).__name__}: {e}"
    if not args.no_e2e:
        e2e_ms, serial_ms, h2d, d2h, pinned = run_e2e(wl, max(1, args.e2e_steps), stream)
        e2e_ms, serial_ms = max_over_ranks([e2e_ms, serial_ms], device)
        res["e2e"] = {"value": round(replica_throughput(world, step_bytes, e2e_ms), 2), "unit": "GB/s",
                      "serial_value": round(replica_throughput(world, step_bytes, serial_ms), 2),
                      "pipelining": "3 streams: H2D of step i+1 and D2H of step i overlap",
                      "host_memory": "pinned" if pinned else "pageable (not enough free RAM to pin)",
                      "ms_per_step": round(e2e_ms, 3), "steps": max(1, args.e2e_steps),
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del wl
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    from synth import configs
    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    # one process per GPU; if a node runs more processes than it has GPUs (a one-GPU check of
    # the multi-process path), processes share GPUs and meet over gloo, since NCCL needs
    # distinct GPUs
    n_dev = torch.cuda.device_count()
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    shared_device = local_world > n_dev
    torch.cuda.set_device(local % n_dev)
    device = torch.device("cuda", local % n_dev)
    exchange = args.mode == "exchange" or (args.mode is None and world > 1)
    dist_on = world > 1 or exchange
    if dist_on:
        import datetime
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                import socket
                with socket.socket() as sk:
                    sk.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        if shared_device:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=device)
    try:
        if exchange:
            res = run_exchange(args, configs.by_name(args.workload), rank, world, device, shared_device)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.suite:
            names = configs.ALL
        elif args.profile_small:
            names = ("sweep_w8",)
        else:
            names = (args.workload,)
        for name in names:
            res = bench_workload(args, configs.by_name(name), rank, world, device, dist_on)
            if rank == 0 and world == 1 and not args.no_cpu and not args.profile_small:
                res["cpu_baseline"] = cpu_baseline(configs.by_name(name), args.seed, args.cpu_budget_s)
            if name == names[0] and world == 1 and not args.no_interference and not args.profile_small:
                try:
                    res["interference"] = run_interference(device, args.seed, quick=not args.interference)
                except Exception as e:  # noqa: BLE001  (the step's figures above stand)
                    res["interference_error"] = f"{type(e).__name__}: {e}"
            if rank == 0:
                print(json.dumps(res), flush=True)
                if args.jsonl:
                    with open(args.jsonl, "a") as f:
                        for row in jsonl_rows(res, name, configs.by_name(name).world):
                            f.write(json.dumps(row) + "\n")
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


# --------------------------------------------------------------------------- the exchange across GPUs


NVLINK_PEER_GBS = 770.0   # measured peer copy per direction per GPU on this machine's B200s


def exchange_bytes(group, L_c, Ns, mine, n_procs):
    """Algorithmic bytes of one process's step in the exchange, and the part that crosses
    NVLink into this GPU.  RS: chunk k of all W ranks' gradients read for each held rank k
    (2 B per valid element per rank), its fp32 [Ns] shard written; AG: every rank's shard read
    (2 B per valid element), this GPU's padded parameters written (2 B per element)."""
    W = group.world
    per = W // n_procs
    valid = [[max(0, min(L_c[i], group.numel(i) - r * L_c[i])) for i in range(group.n_params)]
             for r in range(W)]
    vr = [sum(v) for v in valid]
    mine = list(mine)
    rs_read = sum(2 * W * vr[k] for k in mine)
    rs_write = 4 * Ns * len(mine)
    ag_read = 2 * sum(vr)
    ag_write = 2 * W * sum(L_c)
    rs_nvlink = sum(2 * (W - per) * vr[k] for k in mine)
    ag_nvlink = sum(2 * vr[r] for r in range(W) if r not in mine)
    return {"rs": rs_read + rs_write, "ag": ag_read + ag_write, "rs_read": rs_read,
            "rs_write": rs_write, "ag_read": ag_read, "ag_write": ag_write,
            "rs_nvlink": rs_nvlink, "ag_nvlink": ag_nvlink}


def run_exchange(args, group, proc, n_procs, device, shared_device):
    """The data-parallel exchange across GPUs: the group's W ranks spread over n processes
    (one per GPU, W/n ranks each).  Each process holds only its ranks' gradients and
    all-gather shards; peers' arenas are mapped through CUDA IPC into the pointer tables.
    A step: tide_ag_gather_place of all W shards into this GPU's parameters (peer loads on
    the SMs), then, per held rank k, tide_rs_reduce of rank k's shard with its one-rank plan
    (chunk k of every rank's gradients, peer loads).  Ranks meet only at host barriers: the
    arenas are written once before the timed region and only read inside it."""
    import torch
    import torch.distributed as dist
    import synth
    from fsdp2_layout_aware_b200 import exchange as X
    from fsdp2_layout_aware_b200 import tide as T
    W, P = group.world, group.n_params
    peak, peak_src = load_peaks()
    full = T.Plan(group.shapes, W, device=device)
    Ns = full.shard_numel
    L_c = [full.query(i)["chunk_numel"] for i in range(P)]
    lay = X.arena_layout(group.shapes, W, n_procs, Ns)
    mine = list(X.ranks_of(proc, W, n_procs))
    grads = torch.zeros(lay.grad_elems, dtype=torch.bfloat16, device=device)
    shards = torch.zeros(lay.shard_elems, dtype=torch.bfloat16, device=device)
    for j, k in enumerate(mine):
        zero = synth.zero_grad_params(group, args.seed, k)
        for i in range(P):
            o = j * lay.grad_stride + lay.grad_off[i]
            v = grads[o: o + lay.numel[i]]
            if i not in zero and v.numel():
                synth.dev_fill_bf16(v, args.seed, synth.STREAM_GRAD, k, i, group.grad_sigma)
        o = j * lay.shard_stride
        if Ns:
            synth.dev_fill_bf16(shards[o: o + Ns], args.seed, synth.STREAM_AG, k, 0, group.param_sigma)
    torch.cuda.synchronize()
    dist.barrier()                                   # every process's arenas are filled
    exports = X.all_exports(X.export({"grads": grads, "shards": shards}))
    peers = X.PeerMaps(exports, proc, device.index,
                       {"grads": grads.data_ptr(), "shards": shards.data_ptr()})
    try:
        gp, gn = X.grad_table(lay, W, n_procs, peers.bases("grads", n_procs))
        gtab = T.PointerTable(gp, gn, keep=[grads])
        stab = T.PointerTable(X.shard_table(lay, W, n_procs, peers.bases("shards", n_procs)),
                              [Ns] * W, keep=[shards])
        plans = {k: T.Plan(group.shapes, W, device=device, rank=k) for k in mine}
        outs = {k: torch.empty(Ns, dtype=torch.float32, device=device) for k in mine}
        params = [torch.empty(W * c, dtype=torch.bfloat16, device=device) for c in L_c]
        ptab = T.TensorTable(params)
        stream = torch.cuda.current_stream(device)
        B = exchange_bytes(group, L_c, Ns, mine, n_procs)

        def ag(engine=T.TIDE_ENGINE_SM):
            full.ag_gather_place(stab, ptab, engine=engine)

        def rs():
            for k in mine:
                plans[k].rs_reduce(gtab, outs[k])

        for _ in range(args.warmup):
            ag()
            rs()
        torch.cuda.synchronize()
        full.check()
        for p in plans.values():
            p.check()
        K = args.steps
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(device.index) as clk:
            for e in evs:
                e[0].record(stream)
                ag()
                e[1].record(stream)
                rs()
                e[2].record(stream)
            torch.cuda.synchronize()
        dist.barrier()
        ag_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        rs_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        step_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
        step_ms, ag_ms, rs_ms = max_over_ranks([step_ms, ag_ms, rs_ms], device)
        # the copy-engine placement from peers' shards, timed on its own
        ce_ms = timed_calls(lambda: ag(T.TIDE_ENGINE_CE), max(3, min(K, 10)), stream)
        dist.barrier()
        ce_ms = max_over_ranks([ce_ms], device)[0]
        # the reduction as the pages' two-phase pipeline: the copy engines pull this GPU's rows of
        # every rank's gradients (peers' over NVLink) into local slots, the SMs reduce them
        # segment by segment; compared on the device with the plain call's shards
        pipe = {"segments": min(4, W)}
        try:
            rows = {k: [torch.empty(Ns, dtype=torch.bfloat16, device=device) for _ in range(W)]
                    for k in mine}
            cs = torch.cuda.Stream(device)
            plain = {k: outs[k].clone() for k in mine}

            def rs_pipe():
                for k in mine:
                    plans[k].rs_reduce_pipelined(gtab, outs[k], rows[k], pipe["segments"], cs)

            pipe_ms = timed_calls(rs_pipe, max(3, min(K, 10)), stream)
            torch.cuda.synchronize()
            pipe["same_bits_as_plain"] = all(
                bool(torch.equal(outs[k].view(torch.int32), plain[k].view(torch.int32))) for k in mine)
            del rows, plain
        except Exception as e:  # noqa: BLE001  (the step's figures stand)
            pipe_ms, pipe["error"] = -1.0, f"{type(e).__name__}: {e}"
        dist.barrier()
        pipe_ms = max_over_ranks([pipe_ms], device)[0]
        k_rs, ctas_rs = plans[mine[0]].last_launch()
        nccl = None
        if not shared_device and not args.no_interference:
            short_plans = {k: T.Plan(group.shapes, W, device=device, rank=k, short_ctas=True)
                           for k in mine}

            def rs_on(st, pl, cap=0):
                for k in mine:
                    pl[k].rs_reduce(gtab, outs[k], stream=st, max_ctas=cap)

            try:
                nccl = run_nccl_compare(group, lay, mine, n_procs, device, grads,
                                        lambda st, cap=0: rs_on(st, plans, cap),
                                        lambda st: rs_on(st, short_plans))
            except Exception as e:  # noqa: BLE001  (the step's figures stand)
                nccl = {"error": f"{type(e).__name__}: {e}"}
            for pl in short_plans.values():
                pl.close()
        step_bytes = B["ag"] + B["rs"]
        total_bytes = _sum_over_ranks(step_bytes, device)
        value = total_bytes / (step_ms * 1e-3) / 1e9
        nv_bytes = B["rs_nvlink"] + B["ag_nvlink"]
        if shared_device:
            # the processes share this GPU: a "peer" read is a read of this GPU's own HBM
            roofline = {"bound": "hbm", "achieved": round(total_bytes / (step_ms * 1e-3) / 1e9, 1),
                        "peak": peak, "unit": "GB/s",
                        "frac": round(total_bytes / (step_ms * 1e-3) / 1e9 / peak, 4),
                        "peak_source": f"{peak_src} hbm_gbs",
                        "kernel": "step of all processes (gather placement + one-rank reductions)",
                        "traffic": None}
        else:
            nv_gbs = nv_bytes / (step_ms * 1e-3) / 1e9
            roofline = {"bound": "nvlink", "achieved": round(nv_gbs, 1), "peak": NVLINK_PEER_GBS,
                        "unit": "GB/s", "frac": round(nv_gbs / NVLINK_PEER_GBS, 4),
                        "peak_source": "measured peer copy per direction on this pool",
                        "kernel": "step (gather placement + one-rank reductions)",
                        "nvlink_bytes_in_per_gpu": nv_bytes, "traffic": None,
                        "hbm": {"achieved": round(step_bytes / (step_ms * 1e-3) / 1e9, 1),
                                "peak": peak, "peak_source": f"{peak_src} hbm_gbs"}}
        e2e = run_exchange_e2e(args, grads, shards, outs, params, ag, rs, stream, device)
        e2e = {"value": round(total_bytes / (e2e["ms_per_step"] * 1e-3) / 1e9, 2), "unit": "GB/s", **e2e}
        res = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": n_procs,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16/f32", "data": "synthetic",
            "config": {
                "workload": f"{group.name} layer group, W={W} ranks over {n_procs} GPUs "
                            f"({len(mine)} per GPU), {P} params",
                "step": "tide_ag_gather_place(SM, peer loads) + tide_rs_reduce per held rank "
                        "(one-rank plan, peer loads, rank order, x fl32(1/W))",
                "alg_bytes_per_step_all_gpus": total_bytes,
                "l2": "inputs larger than L2, no flush",
                "parallelism": f"dp{W} over {n_procs} GPUs, exchange over NVLink through CUDA IPC"
                               + (" (processes sharing one GPU)" if shared_device else "")},
            "roofline": roofline,
            "kernels": {
                "rs_reduce_one_rank": {"ms": round(rs_ms, 4), "alg_bytes": B["rs"],
                                       "nvlink_bytes": B["rs_nvlink"], "launches": len(mine),
                                       "kernel": T.KERNEL_NAMES[k_rs] if k_rs >= 0 else None,
                                       "ctas": ctas_rs},
                "ag_gather_place": {"ms": round(ag_ms, 4), "alg_bytes": B["ag"],
                                    "nvlink_bytes": B["ag_nvlink"]},
                "ag_gather_place_ce": {"ms": round(ce_ms, 4), "alg_bytes": B["ag"],
                                       "nvlink_bytes": B["ag_nvlink"], "kernel": "copy engines"},
                "rs_reduce_pipelined_ce": {"ms": round(pipe_ms, 4), "alg_bytes": B["rs"],
                                           "nvlink_bytes": B["rs_nvlink"],
                                           "kernel": "copy engines pull the rows, SMs reduce them",
                                           **pipe}},
            "gpu_launches": K * (1 + len(mine)),
            "clocks": clk.summary(),
            "e2e": e2e,
        }
        if nccl is not None:
            res["nccl_compare"] = nccl
        torch.cuda.synchronize()
        full.check()
        for p in plans.values():
            p.check()
    finally:
        torch.cuda.synchronize()
        dist.barrier()                               # no process still reads a peer's arena
        peers.close()
        dist.barrier()                               # every mapping is gone before any free
    return res


def run_nccl_compare(group, lay, mine, n_procs, device, grads, rs_tide, short_rs, seed=0):
    """Stock FSDP2 reduce-scatter across the GPUs against TIDE-RS, and the slowdown each gives
    a concurrent single-wave bf16 GEMM (3072x3072x16384) on the same GPU: the pages' point that
    the default NCCL reduce-scatter slows such a GEMM by 69 % (weekinpapers.com, Abstract;
    kongchang.com, "The Root of FSDP2 Communication Overhead").

    Stock, per process: each held rank's gradients packed into a fp32 rank-major buffer
    (torch._chunk_cat), summed over the held ranks, then torch.distributed.reduce_scatter_tensor
    (NCCL) over the processes, then x 1/W; rank-major order means each process receives its
    held ranks' shards.  TIDE: the step's one-rank reductions (rs_tide), and the same with
    short-lived CTAs (short_rs).  Interference: the GEMM batch alone, then with back-to-back
    reduce-scatters on a second stream; the NCCL loop length is agreed over the processes so
    every process issues the same collectives.  Every process takes every step in the same
    order."""
    import torch
    import torch.distributed as dist
    W, P = group.world, group.n_params
    per = len(mine)
    Ns = lay.shard_numel
    views = [[grads[j * lay.grad_stride + lay.grad_off[i]:
                    j * lay.grad_stride + lay.grad_off[i] + lay.numel[i]].view(group.shapes[i])
              for i in range(P)] for j in range(per)]
    pack = torch.empty(W, Ns, dtype=torch.float32, device=device)
    acc = torch.empty(W, Ns, dtype=torch.float32, device=device)
    out = torch.empty(per * Ns, dtype=torch.float32, device=device)
    s_comm = torch.cuda.Stream(device)
    s_gemm = torch.cuda.Stream(device)
    s_gemm_hi = torch.cuda.Stream(device, priority=-5)

    def stock_pack():
        for j in range(per):
            torch._chunk_cat(views[j], dim=0, num_chunks=W, out=acc if j == 0 else pack)
            if j:
                acc.add_(pack)

    def stock_rs():
        dist.reduce_scatter_tensor(out, acc.view(-1), op=dist.ReduceOp.SUM)
        out.mul_(1.0 / W)

    def ev_ms(fn, st, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            e0.record(st)
            for _ in range(n):
                fn()
            e1.record(st)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    for _ in range(2):
        with torch.cuda.stream(s_comm):
            stock_pack()
            stock_rs()
            rs_tide(s_comm)
    torch.cuda.synchronize()
    dist.barrier()
    t_pack = ev_ms(stock_pack, s_comm, 3)
    dist.barrier()
    t_nccl = ev_ms(stock_rs, s_comm, 5)
    dist.barrier()
    t_tide = ev_ms(lambda: rs_tide(s_comm), s_comm, 5)
    t_short = ev_ms(lambda: short_rs(s_comm), s_comm, 5)
    t_pack, t_nccl, t_tide, t_short = max_over_ranks([t_pack, t_nccl, t_tide, t_short], device)

    a = torch.randn(3072, 16384, dtype=torch.bfloat16, device=device)
    b = torch.randn(16384, 3072, dtype=torch.bfloat16, device=device)
    c = torch.empty(3072, 3072, dtype=torch.bfloat16, device=device)
    n_gemm = 60

    def gemm_batch():
        for _ in range(n_gemm):
            torch.matmul(a, b, out=c)

    def concurrent(sg, fn, reps):
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s_comm):
            for _ in range(reps):
                fn()
        with torch.cuda.stream(sg):
            e0.record(sg)
            gemm_batch()
            e1.record(sg)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n_gemm

    # the first batch on each stream warms it (cuBLAS sets up a stream's workspace on its
    # first GEMM); the second is timed
    alone = ev_ms(gemm_batch, s_gemm, 1) / n_gemm
    alone = ev_ms(gemm_batch, s_gemm, 1) / n_gemm
    alone_hi = ev_ms(gemm_batch, s_gemm_hi, 1) / n_gemm
    alone_hi = ev_ms(gemm_batch, s_gemm_hi, 1) / n_gemm
    cover = alone * n_gemm * 2.0

    def reps_for(t):
        r = int(cover / max(t, 1e-3)) + 2
        return int(max_over_ranks([r], device)[0])      # the same count on every process

    t_cap = ev_ms(lambda: rs_tide(s_comm, 4), s_comm, 2)
    t_cap = max_over_ranks([t_cap], device)[0]
    r_nccl, r_tide, r_short, r_cap = reps_for(t_nccl), reps_for(t_tide), reps_for(t_short), reps_for(t_cap)
    with_nccl = concurrent(s_gemm, stock_rs, r_nccl)
    with_tide = concurrent(s_gemm, lambda: rs_tide(s_comm), r_tide)
    with_short = concurrent(s_gemm_hi, lambda: short_rs(s_comm), r_short)
    with_cap = concurrent(s_gemm, lambda: rs_tide(s_comm, 4), r_cap)
    dist.barrier()
    alone, alone_hi, with_nccl, with_tide, with_short, with_cap = max_over_ranks(
        [alone, alone_hi, with_nccl, with_tide, with_short, with_cap], device)
    del pack, acc, out, a, b, c
    torch.cuda.empty_cache()
    return {
        "stock": "torch._chunk_cat pack of each held rank + sum, then NCCL reduce_scatter_tensor "
                 "over the processes, x 1/W",
        "stock_ms": {"pack": round(t_pack, 4), "nccl_reduce_scatter": round(t_nccl, 4)},
        "tide_rs_ms": round(t_tide, 4), "tide_rs_short_ctas_ms": round(t_short, 4),
        "tide_rs_4_ctas_ms": round(t_cap, 4),
        "gemm": "bf16 3072x3072x16384 torch.matmul, single wave",
        "gemm_ms_alone": round(alone, 4),
        "gemm_slowdown": {"nccl_reduce_scatter": round(with_nccl / alone - 1, 4),
                          "tide_rs": round(with_tide / alone - 1, 4),
                          "tide_rs_short_ctas_gemm_high_priority": round(with_short / alone_hi - 1, 4),
                          "tide_rs_4_ctas": round(with_cap / alone - 1, 4)},
        "reps": {"nccl": r_nccl, "tide": r_tide, "tide_short": r_short, "tide_4_ctas": r_cap},
    }


def _sum_over_ranks(x, device):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device(device))
    dist.all_reduce(t)
    return int(t.item())


def run_exchange_e2e(args, grads, shards, outs, params, ag, rs, stream, device):
    """The exchange step end to end: every step copies this process's arenas in from pinned
    host memory, meets the other processes at a barrier (their inputs are in place), runs the
    step, and reads its shards and parameters back.  Timed with events on the stream from the
    first copy in to the last copy out; max over processes."""
    import torch
    import torch.distributed as dist
    g_host = grads.cpu().pin_memory()
    s_host = shards.cpu().pin_memory()
    o_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in outs.items()}
    p_host = [torch.empty(p.shape, dtype=p.dtype).pin_memory() for p in params]
    h2d = g_host.numel() * 2 + s_host.numel() * 2
    d2h = sum(v.numel() * 4 for v in o_host.values()) + sum(p.numel() * 2 for p in p_host)
    n = max(1, min(args.e2e_steps, 5))
    times = []
    for j in range(n + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        dist.barrier()                               # nobody reads this arena while it is rewritten
        e0.record(stream)
        grads.copy_(g_host, non_blocking=True)
        shards.copy_(s_host, non_blocking=True)
        torch.cuda.synchronize()
        dist.barrier()                               # every process's inputs are in place
        ag()
        rs()
        for k, v in outs.items():
            o_host[k].copy_(v, non_blocking=True)
        for d, h in zip(params, p_host):
            h.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if j:
            times.append(e0.elapsed_time(e1))
    dist.barrier()
    ms = max_over_ranks([statistics.mean(times)], device)[0]
    total = _sum_over_ranks(h2d + 0, device)
    return {"ms_per_step": round(ms, 3), "steps": n, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "host_memory": "pinned",
            "all_gpus_h2d_bytes_per_step": total,
            "note": "serial per step; value is the whole job's algorithmic step bytes over the "
                    "slowest process's end-to-end step time"}


# --------------------------------------------------------------------------- reference arm


def run_reference(args):
    """The CPU oracle as it stands, on every host core, on the same sample as cpu_baseline.

    One process per core (the sample's row blocks are independent); every step is one pass
    over the sample, started together at a barrier; warm-up passes are untimed.  Under
    torchrun only rank 0 runs it."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from synth import configs
    group = configs.by_name(args.workload)
    items, nbytes = oracle_sample(group, sample_budget_bytes(group))
    cores = len(os.sched_getaffinity(0))
    passes, workers = oracle_pool_passes(group, args.seed, items, cores, args.warmup + args.steps)
    timed = passes[args.warmup:]
    dt = statistics.mean(timed)
    value = nbytes / dt / 1e9
    total = sum(group.numel(i) for i in range(group.n_params))
    sample = describe_sample(group, items, nbytes) + f"; {workers} processes, one pass per step"
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
           "scaling": "strong" if args.gpus > 1 else "weak",
           "vs_baseline": None, "dtype": "bf16/f32", "data": "synthetic",
           "config": {"workload": f"{group.name} layer group, W={group.world} simulated ranks, "
                                  f"{group.n_params} params, {total} elements",
                      "sample": sample},
           "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": workers, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
