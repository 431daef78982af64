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
side, CUDA events on the launching stream; multi-GPU runs are independent
replicas (no collective on the data path) and report the max over ranks.
Inputs are generated on the device by the seeded generator and exceed L2.
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
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama70b")
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--max-ctas", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--interference", action="store_true",
                    help="also run the concurrent-GEMM interference sweep")
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


def ncu_traffic(kernel: str, workload: str, sources):
    """Per-launch DRAM bytes from profiles/ncu_traffic.txt, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(*sources)
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
            return float(parts[3]) if parts[2] == digest else None
    return None


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
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def replica_throughput(n_ranks: int, bytes_per_rank_step: int, max_step_ms: float) -> float:
    """Whole-job GB/s of independent replicas: all ranks' bytes over the slowest rank's time."""
    return n_ranks * bytes_per_rank_step / (max_step_ms * 1e-3) / 1e9


def alg_bytes(group, L):
    W = group.world
    N = sum(group.numel(i) for i in range(group.n_params))
    Npad = W * L.Ns
    return {"rs": 2 * W * N + 4 * Npad, "ag": 2 * N + 2 * Npad, "stage": 4 * W * N,
            "slot_rs": 2 * W * N + 4 * Npad, "N": N, "Npad": Npad}


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
    for nseg in sorted({1, min(4, W), W}):
        wl.out.fill_(float("nan"))
        rec(f"slot_reuse_pipelined_seg{nseg}",
            timed_calls(lambda: wl.plan.rs_reduce_pipelined(wl.grads_t, wl.out, slots, nseg, cs),
                        K, stream, flush), B["stage"] + B["slot_rs"], nseg, wl.plan, same_rs)
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
    del pack, stock, stock_params, ref_out, ref_params
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
    "stock_torch_pack_reduce": ("stock_rs", "torch _chunk_cat pack + add"),
    "stock_torch_copyout": ("stock_ag", "torch split_with_sizes_copy"),
}


def jsonl_rows(res, group_name, world):
    """One flat row per (config, op, mode, ctas) of a bench line."""
    rows = []
    cpu = res.get("cpu_baseline") or {}
    entries = list(res.get("kernels", {}).items()) + list(res.get("variants", {}).items())
    for name, e in entries:
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


def cpu_baseline(group, seed, budget_s):
    """The oracle as it stands (single thread) on a bounded prefix of the group's params.

    Each sampled param is run as a one-param group over the same W (same
    per-element work: W bf16 reads, W-1 fp32 adds, scale, one fp32 write; and
    the copy-out), in group order until `budget_s` of oracle time is spent.
    """
    import numpy as np
    import oracle
    import synth
    from synth import configs
    W = group.world
    rs_s = ag_s = 0.0
    rs_b = ag_b = 0
    names = []
    for i in range(group.n_params):
        sub = configs.Group("sample", W, (group.shapes[i],))
        grads = [[synth.grad_host(group, seed, k, i)] for k in range(W)]
        L = oracle.layout(W, sub.shapes)
        ag = synth.fill_bf16(W * L.Ns, seed, synth.STREAM_AG, 0, i, group.param_sigma)
        t0 = time.perf_counter()
        oracle.rs_reduce(W, sub.shapes, grads, 1)
        t1 = time.perf_counter()
        oracle.ag_copyout(W, sub.shapes, ag)
        t2 = time.perf_counter()
        rs_s += t1 - t0
        ag_s += t2 - t1
        n = sub.numel(0)
        rs_b += 2 * W * n + 4 * W * L.Ns
        ag_b += 2 * n + 2 * W * L.Ns
        names.append(group.names[i] if group.names else str(i))
        del grads, ag
        if rs_s + ag_s >= budget_s:
            break
    spent, nbytes = rs_s + ag_s, rs_b + ag_b
    cores = 1
    return {"value": round(nbytes / spent / 1e9, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{group.name}: params {names} (each as a one-param group, W={W}), "
                      f"RS x fl32(1/W) + AG copy-out, {nbytes / 1e9:.2f} GB algorithmic, "
                      f"{spent:.1f} s single-thread C oracle, generation excluded",
            "seconds": round(spent, 2),
            # the two oracle steps timed apart: pack + reduce, and the all-gather copy-out
            "rs_pack_reduce": {"GB/s": round(rs_b / rs_s / 1e9, 3), "seconds": round(rs_s, 2)},
            "ag_copyout": {"GB/s": round(ag_b / ag_s / 1e9, 3) if ag_s > 0 else None,
                           "seconds": round(ag_s, 3)},
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


def run_interference(device, seed):
    """Slowdown of a concurrent bf16 GEMM vs the RS kernel's CTA count (sweep_w8 group).

    GEMMs: the configured 8192x8192x8192 (cuBLAS picks a 1024-CTA kernel on
    B200, i.e. not single-wave) and 3072x3072x16384, whose kernel fits in one
    wave.  Per point, three trials of: the GEMM batch alone, then concurrently
    with back-to-back RS launches on a second stream (started first, enough of
    them to outlast the GEMMs twice over); slowdown = median(concurrent) / median(alone)
    - 1.  Done for the load/store RS kernel and for the bulk-copy (TMA) one,
    and for the Slot-Reuse staging on the copy engines (no SM; its bytes are
    the staging's).
    """
    import torch
    from synth import configs
    from fsdp2_layout_aware_b200 import tide as T
    group = configs.sweep(8)
    wl = Workload(group, seed, device)
    plans = {"lsu": wl.plan, "tma": T.Plan(group.shapes, group.world, device=device, tma=True)}
    B = alg_bytes(group, oracle_free_layout(wl))
    s_gemm = torch.cuda.Stream(device)
    s_rs = torch.cuda.Stream(device)
    res = {"rs_workload": "sweep_w8 (16 x 512x4096 params, W=8), rank order, x fl32(1/W)",
           "trials": 3, "gemms": []}
    for (m, n, k, n_gemm) in ((8192, 8192, 8192, 40), (3072, 3072, 16384, 120)):
        a = torch.randn(m, k, dtype=torch.bfloat16, device=device)
        b = torch.randn(k, n, dtype=torch.bfloat16, device=device)
        c = torch.empty(m, n, dtype=torch.bfloat16, device=device)

        def gemm_batch():
            for _ in range(n_gemm):
                torch.matmul(a, b, out=c)

        def gemm_alone():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            with torch.cuda.stream(s_gemm):
                e0.record(s_gemm); gemm_batch(); e1.record(s_gemm)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n_gemm

        for _ in range(5):
            gemm_alone()
        g = {"gemm": f"bf16 {m}x{n}x{k} torch.matmul (cuBLAS), {n_gemm} per batch", "points": []}
        points = [(kind, plan, ctas, B["rs"],
                   lambda plan=plan, ctas=ctas: plan.rs_reduce(wl.grads_t, wl.out, max_ctas=ctas, stream=s_rs))
                  for kind, plan in plans.items() for ctas in (8, 16, 32, 0)]
        slots = T.TensorTable(wl.ensure_slots())
        points.append(("ce_stage", wl.plan, 0, B["stage"],
                       lambda: wl.plan.rs_stage(wl.grads_t, slots, engine=T.TIDE_ENGINE_CE, stream=s_rs)))
        for kind, plan, ctas, nbytes, call in points:
            rs_ms = timed_calls(call, 5, s_rs)
            n_ctas = max(0, plan.last_launch()[1]) if kind != "ce_stage" else 0
            alone, conc, rs_conc = [], [], []
            for _ in range(3):
                alone.append(gemm_alone())
                reps = int((alone[-1] * n_gemm * 2.0) / max(rs_ms, 1e-3)) + 2
                torch.cuda.synchronize()
                r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(s_rs):
                    r0.record(s_rs)
                    for _ in range(reps):
                        call()
                    r1.record(s_rs)
                with torch.cuda.stream(s_gemm):
                    e0.record(s_gemm); gemm_batch(); e1.record(s_gemm)
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
    del wl
    torch.cuda.empty_cache()
    return res


def bench_workload(args, group, rank, world, device, dist_on):
    import torch
    from fsdp2_layout_aware_b200 import tide as T
    peak, peak_src = load_peaks()
    wl = Workload(group, args.seed, device)
    B = alg_bytes(group, oracle_free_layout(wl))
    stream = torch.cuda.current_stream(device)
    in_bytes = 2 * B["N"] * group.world
    flush = None if in_bytes > 4 * L2_BYTES else make_flush(device, 2 * L2_BYTES)

    def step():
        wl.plan.ag_place(wl.ag, wl.params_t, max_ctas=args.max_ctas)
        wl.plan.rs_reduce(wl.grads_t, wl.out, max_ctas=args.max_ctas)

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
            wl.plan.rs_reduce(wl.grads_t, wl.out, max_ctas=args.max_ctas)
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
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32", "data": "synthetic",
        "config": {
            "workload": f"{group.name} layer group, W={group.world} simulated ranks, "
                        f"{group.n_params} params, {B['N']} elements",
            "step": "tide_ag_place(SM) + tide_rs_reduce(rank order, x fl32(1/W))",
            "alg_bytes_per_step": step_bytes, "max_ctas": args.max_ctas,
            "l2": ("inputs larger than L2, no flush" if flush is None else
                   "L2 flushed (256 MB read) before every timed step"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(rs_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(rs_gbs / peak, 4), "peak_source": f"{peak_src} hbm_gbs",
                     "kernel": "rs_reduce_kernel", "alg_bytes_per_launch": B["rs"],
                     "avg_launch_ms": round(rs_ms, 4),
                     "traffic": ncu_traffic("rs_reduce_kernel", group.name, RS_SOURCES)},
        "kernels": {
            "rs_reduce_kernel": {"ms": round(rs_ms, 4), "GB/s": round(rs_gbs, 1),
                                 "frac_of_peak": round(rs_gbs / peak, 4), "alg_bytes": B["rs"],
                                 "ctas": rs_ctas, "kernel": T.KERNEL_NAMES[rs_kernel]},
            "ag_place_kernel": {"ms": round(ag_ms, 4), "GB/s": round(ag_gbs, 1),
                                "frac_of_peak": round(ag_gbs / peak, 4), "alg_bytes": B["ag"],
                                "ctas": wl.plan.launch_ctas(T.K_AG, args.max_ctas),
                                "traffic": ncu_traffic("ag_place_kernel", group.name, AG_SOURCES)}},
        "gpu_launches": 2 * K,
        "clocks": clk.summary(),
        "workspace_bytes": wl.plan.workspace_bytes,
        # what the stock path would hold instead: one full-group fp32 rank-major buffer per rank
        "stock_fp32_buffer_bytes": 4 * group.world * wl.Ns,
    }
    if not args.no_variants:
        # the step's figures above stand even if a variant fails: record the error instead
        try:
            res["variants"] = run_variants(wl, max(3, min(K, 20)), stream, peak, flush)
        except Exception as e:  # noqa: BLE001
            res["variants_error"] = f"{type(e).__name__}: {e}"
            wl.drop_slots()
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
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
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
            if args.interference and name == names[0]:
                res["interference"] = run_interference(device, args.seed)
            if rank == 0:
                print(json.dumps(res), flush=True)
                if args.jsonl:
                    with open(args.jsonl, "a") as f:
                        for row in jsonl_rows(res, name, configs.by_name(name).world):
                            f.write(json.dumps(row) + "\n")
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


# --------------------------------------------------------------------------- reference arm


def run_reference(args):
    """The CPU oracle as it stands, on host cores, on a bounded sample of the workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    import synth
    from synth import configs
    group = configs.by_name(args.workload)
    W = group.world
    # per step: the largest param of the group that is at most 1/8 of the group, as a one-param group
    total = sum(group.numel(i) for i in range(group.n_params))
    cand = [i for i in range(group.n_params) if group.numel(i) <= total / 8] or [0]
    i = max(cand, key=group.numel)
    sub = configs.Group("sample", W, (group.shapes[i],))
    grads = [[synth.grad_host(group, args.seed, k, i)] for k in range(W)]
    L = oracle.layout(W, sub.shapes)
    ag = synth.fill_bf16(W * L.Ns, args.seed, synth.STREAM_AG, 0, i, group.param_sigma)
    n = sub.numel(0)
    step_bytes = (2 * W * n + 4 * W * L.Ns) + (2 * n + 2 * W * L.Ns)

    def step():
        oracle.ag_copyout(W, sub.shapes, ag)
        oracle.rs_reduce(W, sub.shapes, grads, 1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = step_bytes / dt / 1e9
    name = group.names[i] if group.names else str(i)
    sample = (f"{group.name}: param {name} {group.shapes[i]} as a one-param group over W={W}; "
              f"AG copy-out + RS x fl32(1/W), {step_bytes / 1e9:.3f} GB algorithmic per step")
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16/f32", "data": "synthetic",
           "config": {"workload": f"{group.name} layer group, W={W} simulated ranks, "
                                  f"{group.n_params} params, {total} elements",
                      "sample": sample},
           "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
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
