#!/usr/bin/env python
"""Benchmark of the MoLE lookup path on B200.

Workload (default): the 1B-activated-shaped MoLE model -- 16 layers, each with
its own table LUT[50304, 16, 2048] bf16 (3.3 GB) and router Wr[2048, 16] --
over a prefill batch of T = 16384 tokens with Zipf(1.1) ids.  One step is one
pass of the lookup path of a forward pass: the batch's token grouping
(mole_token_groups_build, once: every layer indexes its table with the same
token ids) and a combine for each of the 16 layers (router GEMV + softmax +
direct-addressed gather + gate-weighted sum), every layer with its own hidden
states.  Tables are seeded N(0, 0.02) fills (the combine's time does not
depend on the values); ids and hidden states rotate over a pool of 4 batches.
A step touches 16 distinct tables of 3.3 GB, so inputs are far larger than
the 126 MB L2.  --path plain runs mole_lookup_combine per layer instead.

Also measured in the same run (own keys in the JSON line): the one-off table
build (410M-shaped layer, tensor cores), the NF3-compressed table combine, the
other prefill cases of the 1B-shaped layer, and the offloaded table (a layer
table in pinned host memory, distinct rows staged over the host link).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch on its own GPU (weak scaling, no
data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mixture_lookup_experts_b200 import inputs  # noqa: E402

METRIC = "MoLE lookup-combine tokens/s & HBM GB/s vs 8 TB/s; LUT build TFLOP/s"
UNIT = "tokens/s"
KERNEL_SOURCES = ["mixture_lookup_experts_b200/csrc/combine.cu", "mixture_lookup_experts_b200/csrc/grouped.cu",
                  "mixture_lookup_experts_b200/csrc/router_tc.cu", "mixture_lookup_experts_b200/csrc/combine_common.cuh",
                  "mixture_lookup_experts_b200/csrc/common.cuh", "mixture_lookup_experts_b200/csrc/nf3.cuh",
                  "mixture_lookup_experts_b200/csrc/groups.cuh"]
PROFILE_SUMMARY = {"grouped": "profiles/combine_grouped_bf16_1b_T16384_zipf.md",
                   "plain": "profiles/combine_bf16_1b_T16384_zipf.md"}
KERNELS = {
    "grouped": "grouped_stream_kernel (mole_lookup_combine_groups, one launch per layer call)",
    "plain": "router_gates_kernel + gather_kernel (mole_lookup_combine, per layer call)",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--ids", choices=["zipf", "uniform"], default="zipf")
    ap.add_argument("--path", choices=["grouped", "plain"], default="grouped",
                    help="grouped: mole_lookup_combine_grouped (default); plain: mole_lookup_combine")
    ap.add_argument("--layers", type=int, default=None,
                    help="layer tables to allocate (default: the model's 16); fewer only for profiling runs")
    ap.add_argument("--no-extras", action="store_true", help="skip the build / NF3 / other-case legs")
    ap.add_argument("--no-offload", action="store_true", help="skip the host-resident (offloaded) table leg")
    ap.add_argument("--no-decode", action="store_true", help="skip the small-batch (decode) sweeps")
    ap.add_argument("--no-ffn", action="store_true", help="skip the FFN-block leg")
    ap.add_argument("--no-train", action="store_true", help="skip the training-step leg")
    ap.add_argument("--train-only", action="store_true", help="run only the training-step leg")
    ap.add_argument("--ffn-only", action="store_true", help="run only the FFN-block leg")
    ap.add_argument("--decode-only", action="store_true", help="run only the small-batch (decode) sweeps")
    ap.add_argument("--nf3-only", action="store_true",
                    help="run only the NF3-table leg on the main workload's batches (for profiling its kernels)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--build-only", action="store_true",
                    help="run only the table-build leg (for profiling the tensor-core kernels)")
    ap.add_argument("--build-experts", type=int, default=None,
                    help="experts in the build leg (default: the model's 16); fewer only for profiling runs")
    return ap.parse_args()


class Combiner:
    """The combine call of the chosen path.  grouped: the batch's token
    grouping is built once per step (prepare) and serves every layer's
    mole_lookup_combine_groups; plain: mole_lookup_combine per layer."""

    def __init__(self, mole, path: str, T: int, V: int, N: int, dev):
        import torch
        self.mole, self.path, self.V, self.N = mole, path, V, N
        self.groups = None
        if path == "grouped":
            self.groups = torch.empty(mole.mole_token_groups_workspace(T, N), dtype=torch.uint8, device=dev)

    def prepare(self, ids, stream):
        if self.path == "grouped":
            self.mole.mole_token_groups_build(ids, self.V, self.N, groups=self.groups, stream=stream)

    def __call__(self, ids, h, Wr, lut, out, stream):
        if self.path == "grouped":
            self.mole.mole_lookup_combine_groups(ids, self.groups, h, Wr, lut, out=out, stream=stream)
        else:
            self.mole.mole_lookup_combine(ids, h, Wr, lut, out=out, stream=stream)


def workload_config(T: int, kind: str, layers: int | None = None, path: str = "grouped") -> dict:
    s = inputs.SHAPES["1b"]
    layers = s.layers if layers is None else layers
    call = "mole_lookup_combine_groups" if path == "grouped" else "mole_lookup_combine"
    return {
        "workload": f"1B-shaped MoLE lookup path: {layers} layers x {call}"
                    f"{' (one grouping per step)' if path == 'grouped' else ''}, prefill T={T}, "
                    f"{'Zipf(1.1)' if kind == 'zipf' else 'uniform'} ids",
        "V": s.V, "D": s.D, "N": s.N, "layers": layers, "tokens_per_step": T, "ids": kind,
        "table_dtype": "bf16", "out_dtype": "f32",
        "l2": "inputs larger than L2 (each step reads its layers' distinct 3.3 GB tables)",
        "data": "seeded N(0,0.02) tables; ids and per-layer h rotate over a pool of 4 batches",
    }


def compact(x, digits: int = 6):
    """Floats rounded to `digits` significant digits, recursively (keeps the
    headline line short)."""
    if isinstance(x, float):
        return float(f"{x:.{digits}g}")
    if isinstance(x, dict):
        return {k: compact(v, digits) for k, v in x.items()}
    if isinstance(x, list):
        return [compact(v, digits) for v in x]
    return x


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, polled from a thread)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.ok = False
        self.samples, self.reasons = [], 0
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            # NVML may see more GPUs than CUDA does: find ours by PCI address
            pr = torch.cuda.get_device_properties(device_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _poll(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def launches_per_step(T: int, N: int, layers: int, path: str, n_sm: int | None = None) -> int:
    """This library's kernel launches in one timed step (bf16 table).  Grouped
    path: the grouping (plan kernel, plus the per-SM share kernel when a CTA's
    share fits, 16 + T/SMs < 256 tokens), then per layer one kernel (the
    interleaved or the CTA-local kernel, N <= 16) where the shares exist, else
    router + gather; plain path: router + gather per layer.  Below 1024 tokens
    one combine kernel per layer.  n_sm: the device's SM count (queried when
    not given)."""
    if n_sm is None:
        import torch
        n_sm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    if T < 1024:
        return layers
    if path != "grouped":
        return 2 * layers
    shares = (16 + -(-T // n_sm) + 15) // 16 * 16 < 256
    per_layer = 1 if (shares and N <= 16) else 2
    return (2 if shares else 1) + per_layer * layers


def profiled_traffic(path: str):
    """(bytes per launch, note) from the committed ncu summary if it was taken
    on the current kernel source; else (None, reason)."""
    p = os.path.join(ROOT, PROFILE_SUMMARY[path])
    if not os.path.exists(p):
        return None, "no ncu summary committed"
    fields = {}
    for line in open(p):
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "kernel_source_sha256")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != kernel_source_hash():
        return None, "kernel changed since the ncu capture"
    try:
        return float(fields["traffic_bytes_per_launch"]), "ncu dram__bytes_read.sum + dram__bytes_write.sum"
    except (KeyError, ValueError):
        return None, "summary lacks traffic"


def rank_seeds(base: int, rank: int):
    """(device generator seed, host rng seed) of a rank: each rank draws its own
    tables and batches (weak scaling: per-rank work is fixed as ranks grow)."""
    return base + 7919 * rank, base + 104729 * rank


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (the job takes as long as its
    slowest rank); a no-op on a single process."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tokens_per_s(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Tokens processed by all ranks divided by the slowest rank's time."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def combine_bytes(U: float, T: int, D: int, N: int) -> float:
    """Algorithmic bytes of one combine launch: unique table rows + h in +
    out (fp32) + router weights + ids."""
    return U * N * D * 2 + T * D * 2 + T * D * 4 + D * N * 2 + 4 * T


def nf3_bytes(U: float, T: int, D: int, N: int) -> float:
    return U * N * D * (3 / 8 + 2 / 64) + T * D * 2 + T * D * 4 + D * N * 2 + 4 * T


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    shape = inputs.SHAPES["1b"]
    V, D, N, L = shape.V, shape.D, shape.N, shape.layers
    sample_T = 256  # tokens per layer per step (bounded sample of the T-token batch)
    rng = np.random.default_rng(shape.seed)
    cores = oracle.max_threads()

    def one_step(seed):
        r = np.random.default_rng(seed)
        done = 0
        ids = inputs.draw_ids(r, sample_T, V, args.ids)  # the batch's ids, shared by the layers
        uniq, inv = np.unique(ids, return_inverse=True)
        for layer in range(L):
            rows = inputs.normal(r, (uniq.size, N, D), 0.02, "bf16")  # the rows this sample reads
            Wr = inputs.normal(r, (D, N), 0.02, "bf16")
            h = inputs.normal(r, (sample_T, D), 1.0, "bf16")
            gen = time.perf_counter()
            oracle.combine(inv.astype(np.int32), h, Wr, rows)
            done += time.perf_counter() - gen
        return done

    for i in range(args.warmup):
        one_step(1000 + i)
    times = [one_step(2000 + i) for i in range(args.steps)]
    total = sum(times)
    value = sample_T * args.steps / total  # tokens through all 16 layers per second
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.tokens, args.ids),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{sample_T} tokens per layer x {L} layers per step (input generation "
                                   f"excluded), fp64 C oracle with OpenMP over tokens"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    from mixture_lookup_experts_b200 import mole

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    if args.decode_only:
        res = decode_leg(mole, dev, stream)
        if rank == 0:
            print(json.dumps({"decode": res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    if args.train_only:
        _, bf16_peak, bf16_sust, _ = measured_peaks()
        g = torch.Generator(device=dev)
        g.manual_seed(inputs.SHAPES["1b"].seed)
        res = train_leg(mole, np.random.default_rng(7), g, dev, stream, max(3, args.warmup), (bf16_peak, bf16_sust))
        if rank == 0:
            print(json.dumps({"train": res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    if args.ffn_only:
        shape = inputs.SHAPES["1b"]
        g = torch.Generator(device=dev)
        g.manual_seed(shape.seed)
        luts = [(torch.randn((shape.V, shape.N, shape.D), generator=g, device=dev) * 0.02).to(torch.bfloat16)
                for _ in range(2)]
        routers = [(torch.randn((shape.D, shape.N), generator=g, device=dev) * 0.02).to(torch.bfloat16)]
        _, bf16_peak, bf16_sust, _ = measured_peaks()
        res = ffn_leg(mole, luts, routers, np.random.default_rng(shape.seed), g, dev, stream, max(3, args.warmup),
                      (bf16_peak, bf16_sust))
        if rank == 0:
            print(json.dumps({"ffn_block": res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    if args.build_only:
        hbm_peak, bf16_peak, bf16_sust, peak_kind = measured_peaks()
        res = build_leg(mole, dev, stream, bf16_peak, bf16_sust, peak_kind, reps=max(1, args.steps),
                        warmup=max(1, args.warmup), experts=args.build_experts)
        if rank == 0:
            print(json.dumps({"build": res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    shape = inputs.SHAPES["1b"]
    V, D, N = shape.V, shape.D, shape.N
    L = shape.layers if args.layers is None else max(1, args.layers)
    T = args.tokens
    W, K = args.warmup, args.steps

    # ---- layer tables and routers (seeded per rank) ----
    g = torch.Generator(device=dev)
    dev_seed, host_seed = rank_seeds(shape.seed, rank)
    g.manual_seed(dev_seed)
    luts = [(torch.randn((V, N, D), generator=g, device=dev) * 0.02).to(torch.bfloat16) for _ in range(L)]
    routers = [(torch.randn((D, N), generator=g, device=dev) * 0.02).to(torch.bfloat16) for _ in range(L)]
    # per-step batches: a pool of P distinct (ids, h) per layer slot, rotated
    P = 4
    rng = np.random.default_rng(host_seed)
    # every layer of a step indexes its table with the same token ids (the
    # batch's), with its own hidden states
    id_pool = [[torch.from_numpy(inputs.draw_ids(rng, T, V, args.ids)).to(dev)] * L for _ in range(P)]
    h_pool = [[(torch.randn((T, D), generator=g, device=dev)).to(torch.bfloat16) for _ in range(L)]
              for _ in range(P)]
    uniq_counts = [[int(torch.unique(x).numel()) for x in pool] for pool in id_pool]
    if args.nf3_only:
        res = nf3_leg(mole, luts, routers, id_pool, h_pool, uniq_counts, dev, stream, max(1, W), K, T, P, L)
        if rank == 0:
            print(json.dumps({"nf3": res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    out = torch.empty((T, D), dtype=torch.float32, device=dev)
    combine = Combiner(mole, args.path, T, V, N, dev)

    def step(i, events=None):
        """One step; with `events` (start, grouped, end) recorded around the
        grouping and the layer calls -- none between layers, so consecutive
        layer kernels overlap their launches (programmatic dependent launch)."""
        p = i % P
        if events is not None:
            events[0].record(stream)
        combine.prepare(id_pool[p][0], stream)
        if events is not None:
            events[1].record(stream)
        for layer in range(L):
            combine(id_pool[p][layer], h_pool[p][layer], routers[layer], luts[layer], out, stream)
        if events is not None:
            events[2].record(stream)

    # ---- warm-up ----
    for i in range(W):
        step(i)
    st = mole.mole_check(stream, timeout_ms=60000)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---- timed region: K steps, barrier + synchronize on both sides ----
    kern_events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        t_start.record(stream)
        for i in range(K):
            step(W + i, kern_events[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    st = mole.mole_check(stream, timeout_ms=60000)
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    # per layer call: the step's layer span / L (mean over the timed steps)
    layers_ms = [kern_events[i][1].elapsed_time(kern_events[i][2]) for i in range(K)]
    avg_kern_ms = sum(layers_ms) / (K * L)
    U_avg = sum(uniq_counts[(W + i) % P][l] for i in range(K) for l in range(L)) / (K * L)

    prep_ms = [kern_events[i][0].elapsed_time(kern_events[i][1]) for i in range(K)]
    avg_prep_ms = sum(prep_ms) / len(prep_ms)
    max_ms, max_kern_ms, max_prep_ms = max_over_ranks([elapsed_ms, avg_kern_ms, avg_prep_ms], dev)
    value = whole_job_tokens_per_s(world, T, K, max_ms)

    # ---- end to end through the C ABI with host buffers ----
    e2e = None if args.no_e2e else e2e_leg(combine, id_pool, h_pool, routers, luts, out, dev, stream, world, W, K,
                                           T, L)

    # ---- roofline of the combine kernel ----
    hbm_peak, bf16_peak, bf16_sust, peak_kind = measured_peaks()
    alg_bytes = combine_bytes(U_avg, T, D, N)
    achieved_gbs = alg_bytes / (max_kern_ms / 1e3) / 1e9
    traffic, traffic_note = profiled_traffic(args.path)
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": traffic, "kernel": KERNELS[args.path],
                "bytes_per_launch": alg_bytes, "unique_rows": U_avg, "avg_launch_us": max_kern_ms * 1e3,
                "peak_source": f"{peak_kind} hbm_gbs", "frac_of_8TBs": achieved_gbs / 8000.0,
                "traffic_source": traffic_note}

    line = headline(value=value, world=world, K=K, W=W, max_ms=max_ms,
                    cfg=workload_config(T, args.ids, L, args.path), roofline=roofline, e2e=e2e,
                    launches=K * launches_per_step(T, N, L, args.path),
                    prep_us=max_prep_ms * 1e3 if args.path == "grouped" else None, clocks=clocks.summary())

    # ---- extras, each printed as its own JSON line before the headline ----
    def leg(name, fn):
        res = fn()
        if rank == 0:
            print(json.dumps({"leg": name, name: res}), flush=True)

    if not args.no_extras:
        leg("cases", lambda: other_cases(mole, luts, routers, rng, g, dev, stream, W, T, args.ids, args.path, L))
        leg("nf3", lambda: nf3_leg(mole, luts, routers, id_pool, h_pool, uniq_counts, dev, stream, W, K, T, P, L))
        if not args.no_offload:
            leg("offload", lambda: offload_leg(mole, luts, routers, rng, g, dev, stream, W, L))
        if not args.no_ffn:
            leg("ffn_block", lambda: ffn_leg(mole, luts, routers, rng, g, dev, stream, W, (bf16_peak, bf16_sust)))
        del luts
        torch.cuda.empty_cache()
        if not args.no_decode:
            leg("decode", lambda: decode_leg(mole, dev, stream))
        if not args.no_train:
            leg("train", lambda: train_leg(mole, rng, g, dev, stream, W, (bf16_peak, bf16_sust)))
        leg("build", lambda: build_leg(mole, dev, stream, bf16_peak, bf16_sust, peak_kind))

    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = compact(cpu_baseline(args))
    if rank == 0:
        # the headline: one short line, printed last
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


HEADLINE_MAX_BYTES = 2048


def headline(*, value, world, K, W, max_ms, cfg, roofline, e2e, launches, prep_us, clocks, cpu=None) -> dict:
    """The headline JSON line (floats to 6 significant digits).  Printed
    last and kept under HEADLINE_MAX_BYTES so that a reader keeping only
    the tail of the output still holds all of it; the extra legs go on
    lines of their own before it."""
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline, "e2e": e2e,
        "gpu_launches": launches, "token_groups_build_us_per_step": prep_us, "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return compact(line)


def e2e_leg(combine, id_pool, h_pool, routers, luts, out, dev, stream, world, W, K, T, L):
    """The same metric through the C ABI with host buffers: per step the ids
    and the L hidden-state batches are copied host -> device from pinned
    memory, the L combine calls run, and the L outputs are copied back.  The
    copies run on their own streams, double-buffered on the device: layer
    l+1's h goes in while layer l combines and layer l-1's output comes back
    (the host link carries both directions at once), every copy and call
    ordered by events."""
    import torch
    import torch.distributed as dist
    D = out.shape[1]
    h_host = [torch.empty((T, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ids_host = torch.empty((T,), dtype=torch.int32).pin_memory()
    out_host = torch.empty((T, D), dtype=torch.float32).pin_memory()
    for s in range(min(2, L)):
        h_host[s].copy_(h_pool[0][s])
    ids_host.copy_(id_pool[0][0].cpu())
    h_stage = [torch.empty((T, D), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    o_stage = [out, torch.empty_like(out)]
    ids_stage = torch.empty((T,), dtype=torch.int32, device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n_ev = 4
    ev_h = [torch.cuda.Event() for _ in range(n_ev)]   # h of call g is on the device
    ev_c = [torch.cuda.Event() for _ in range(n_ev)]   # call g is done (its h buffer is free)
    ev_o = [torch.cuda.Event() for _ in range(n_ev)]   # call g's output is back (its buffer is free)
    ev_ids = torch.cuda.Event()
    g = [0]  # calls issued so far (events of call g at g % n_ev)

    def e2e_step():
        s_in.wait_stream(stream)  # the previous step's grouping has read ids_stage
        with torch.cuda.stream(s_in):
            ids_stage.copy_(ids_host, non_blocking=True)
            ev_ids.record(s_in)
        stream.wait_event(ev_ids)
        combine.prepare(ids_stage, stream)
        for layer in range(L):
            c = g[0]
            b = c % 2
            with torch.cuda.stream(s_in):
                if c >= 2:
                    s_in.wait_event(ev_c[(c - 2) % n_ev])
                h_stage[b].copy_(h_host[layer % 2], non_blocking=True)
                ev_h[c % n_ev].record(s_in)
            stream.wait_event(ev_h[c % n_ev])
            if c >= 2:
                stream.wait_event(ev_o[(c - 2) % n_ev])
            combine(ids_stage, h_stage[b], routers[layer], luts[layer], o_stage[b], stream)
            ev_c[c % n_ev].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[c % n_ev])
                out_host.copy_(o_stage[b], non_blocking=True)
                ev_o[c % n_ev].record(s_out)
            g[0] += 1
        stream.wait_event(ev_o[(g[0] - 1) % n_ev])  # the step ends when its last output is back

    for _ in range(min(W, 3)):
        e2e_step()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    K_e2e = max(1, min(K, 20))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for _ in range(K_e2e):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    (e_ms,) = max_over_ranks([e_start.elapsed_time(e_end)], dev)
    return {"value": whole_job_tokens_per_s(world, T, K_e2e, e_ms), "unit": UNIT,
            "h2d_bytes_per_step": L * T * D * 2 + T * 4, "d2h_bytes_per_step": L * T * D * 4,
            "steps": K_e2e, "note": f"per step: ids + {L} h H2D (pinned), {L} C-ABI calls, {L} outputs D2H; "
                                    f"copies overlapped with the calls on two copy streams"}


def time_block(fn, n, stream):
    """ms for n back-to-back calls between two CUDA events."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(n):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def time_launches(fn, n, stream):
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        ev[i][0].record(stream)
        fn(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def other_cases(mole, luts, routers, rng, g, dev, stream, W, T_main, kind_main, path_main, L):
    """The other prefill cases of the 1B-shaped layer, on both combine paths:
    one id batch shared by the L layers, the grouping built once (its time
    reported apart), per-layer combine calls timed."""
    import torch
    shape = inputs.SHAPES["1b"]
    V, D, N = shape.V, shape.D, shape.N
    hbm_peak = measured_peaks()[0]
    res = {}
    for T in (4096, 16384):
        for kind in ("zipf", "uniform"):
            ids = torch.from_numpy(inputs.draw_ids(rng, T, V, kind)).to(dev)
            hs = [torch.randn((T, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(L)]
            U = int(torch.unique(ids).numel())
            out = torch.empty((T, D), dtype=torch.float32, device=dev)
            for path in ("grouped", "plain"):
                if T == T_main and kind == kind_main and path == path_main:
                    continue
                combine = Combiner(mole, path, T, V, N, dev)
                combine.prepare(ids, stream)

                def fn(i):
                    lay = i % L
                    combine(ids, hs[lay], routers[lay], luts[lay], out, stream)

                for i in range(max(W, 3) * L):
                    fn(i)
                avg = time_block(fn, 4 * L, stream) / (4 * L)  # no events between calls
                prep = time_launches(lambda i: combine.prepare(ids, stream), 5, stream)
                b = combine_bytes(U, T, D, N)
                res[f"T{T}_{kind}_{path}"] = {"tokens_per_s_per_layer": T / (avg / 1e3), "avg_launch_us": avg * 1e3,
                                              "unique_rows": U, "achieved_gbs": b / (avg / 1e3) / 1e9,
                                              "frac_of_measured_hbm": b / (avg / 1e3) / 1e9 / hbm_peak,
                                              "token_groups_build_us": (sum(prep) / len(prep) * 1e3
                                                                        if path == "grouped" else None)}
                del combine
            del ids, hs, out
    return res


def nf3_leg(mole, luts, routers, id_pool, h_pool, uniq_counts, dev, stream, W, K, T, P, L):
    import torch
    shape = inputs.SHAPES["1b_nf3"]
    D, N = shape.D, shape.N
    hbm_peak = measured_peaks()[0]
    V = shape.V
    tables = [(torch.empty((V, N, D // 64, 24), dtype=torch.uint8, device=dev),
               torch.empty((V, N, D // 64), dtype=torch.float16, device=dev)) for _ in range(L)]
    mole.mole_quantize_lut_nf3(luts[0], *tables[0], stream=stream)  # warm-up
    q_ms = []
    for lay in range(L):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        mole.mole_quantize_lut_nf3(luts[lay], *tables[lay], stream=stream)
        e1.record(stream)
        q_ms.append((e0, e1))
    torch.cuda.synchronize()
    q_avg = sum(a.elapsed_time(b) for a, b in q_ms) / L
    out = torch.empty((T, D), dtype=torch.float32, device=dev)

    # one id batch per step (as the main metric); its grouping built once
    groups = [mole.mole_token_groups_build(id_pool[pp][0], shape.V, N, stream=stream) for pp in range(P)]

    def fn(i):
        p, lay = (i // L) % P, i % L
        c, s = tables[lay]
        mole.mole_lookup_combine_nf3_groups(id_pool[p][lay], groups[p], h_pool[p][lay], routers[lay], c, s, out=out,
                                            stream=stream)

    for i in range(W * L):
        fn(i)
    n = max(1, min(K, 20)) * L
    avg = time_block(fn, n, stream) / n  # per layer call, no events between calls
    U = sum(uniq_counts[(i // L) % P][i % L] for i in range(n)) / n
    b = nf3_bytes(U, T, D, N)
    assert mole.mole_check(stream) == 0
    q_bytes = V * N * D * 2 + V * N * D * 3 / 8 + V * N * (D // 64) * 2
    del tables, groups
    # ALU roofline (plain lane arithmetic): a gate-weighted FMA per (token,
    # expert, element) plus ~4 integer / conversion operations to decode each
    # element of each distinct row block (bit extract, two byte-permute
    # lookups, fp16 -> fp32), against 148 SMs x 128 lanes x the max SM clock
    lane_ops = T * N * D + 4.0 * U * N * D
    alu_peak = 148 * 128 * 1.965e9
    alu_us = lane_ops / alu_peak * 1e6
    return {"tokens_per_s": T / (avg / 1e3) / L, "tokens_per_s_per_layer": T / (avg / 1e3),
            "avg_launch_us": avg * 1e3, "achieved_gbs": b / (avg / 1e3) / 1e9,
            "frac_of_measured_hbm": b / (avg / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes_per_launch": b,
            "alu": {"bound": "alu", "lane_ops_per_launch": lane_ops, "peak_lane_ops_per_s": alu_peak,
                    "roofline_us": alu_us, "frac": alu_us / (avg * 1e3),
                    "model": "T*N*D FMAs + 4*U*N*D decode ops; 148 SMs x 128 lanes x 1.965 GHz"},
            "quantize_ms_per_layer": q_avg, "quantize_gbs": q_bytes / (q_avg / 1e3) / 1e9,
            "workload": f"1B-shaped NF3 table (codes + fp16 scale per 64), T={T}, same ids/h as the main case, "
                        f"mole_lookup_combine_nf3_groups (grouping built once per id batch, not timed here)"}


def offload_leg(mole, luts, routers, rng, g, dev, stream, W, L):
    """The page's deployment scenario: the 1B-shaped layer table (3.3 GB bf16;
    also its NF3 form) in pinned host memory.  Per batch each distinct id's
    row block crosses the host link once (mole_offload_stage) and the combine
    reads the staging buffer (mole_lookup_combine_offload).  Reported per
    batch size: link bytes per token, staging time and link GB/s (against a
    copy-engine copy of a contiguous pinned block), the combine, and a
    decode step over L layers with the next layer's rows staged on a second
    stream while this layer combines (two staging buffers)."""
    import torch
    shape = inputs.SHAPES["1b"]
    V, D, N, Dr = shape.V, shape.D, shape.N, shape.Dr
    row = N * D * 2
    host = torch.empty((V, N, D), dtype=torch.bfloat16, pin_memory=True)
    host.copy_(luts[0])
    codes = torch.empty((V, N, D // 64, 24), dtype=torch.uint8, device=dev)
    scales = torch.empty((V, N, D // 64), dtype=torch.float16, device=dev)
    mole.mole_quantize_lut_nf3(luts[0], codes, scales, stream=stream)
    hc = torch.empty(codes.shape, dtype=torch.uint8, pin_memory=True)
    hs = torch.empty(scales.shape, dtype=torch.float16, pin_memory=True)
    hc.copy_(codes)
    hs.copy_(scales)
    del codes, scales
    torch.cuda.synchronize()
    # the link's copy-engine rate: one contiguous 256 MiB pinned block to the device
    blk = 256 << 20
    src = host.view(-1).view(torch.uint8)[:blk]
    dst = torch.empty(blk, dtype=torch.uint8, device=dev)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    ce_ms = min(time_launches(lambda i: dst.copy_(src, non_blocking=True), 5, stream))
    ce_gbs = blk / (ce_ms / 1e3) / 1e9
    del dst
    moe_expert_bytes = 2 * D * Dr * 2  # one D x Dr and one Dr x D bf16 matrix
    res = {"workload": "1B-shaped layer table [50304, 16, 2048] bf16 (3.3 GB) and its NF3 form (0.68 GB) in pinned "
                       "host memory; Zipf(1.1) ids; grouping built once per batch (timed apart)",
           "h2d_copy_engine_gbs": ce_gbs,
           "moe_byte_model": {"expert_bytes": moe_expert_bytes,
                              "note": "an offloaded MoE moves the weights of each expert a batch activates "
                                      "(2 x D x Dr bf16 each; the routed experts of this layer before the table "
                                      "replaced them); MoLE moves only the batch's distinct N x D row blocks"},
           "cases": {}}
    for nf3 in (False, True):
        for T in ((1, 8, 64, 256, 4096, 16384) if not nf3 else (1, 64, 16384)):
            ids_np = inputs.draw_ids(rng, T, V, "zipf")
            U = int(np.unique(ids_np).size)
            ids = torch.from_numpy(ids_np).to(dev)
            groups = mole.mole_token_groups_build(ids, V, N, stream=stream)
            staging = torch.empty(mole.mole_offload_staging_bytes(T, V, N, D, nf3=nf3), dtype=torch.uint8,
                                  device=dev)
            h = torch.randn((T, D), generator=g, device=dev).to(torch.bfloat16)
            out = torch.empty((T, D), dtype=torch.float32, device=dev)
            tab, sc = (hc, hs) if nf3 else (host, None)

            def stage(i):
                mole.mole_offload_stage(T, groups, tab, sc, staging=staging, stream=stream)

            def comb(i):
                mole.mole_lookup_combine_offload(groups, h, routers[0], staging, V, nf3=nf3, out=out, stream=stream)

            def both(i):
                stage(i)
                comb(i)

            n = 20 if T <= 4096 else 6
            for i in range(max(W, 3)):
                both(i)
            st_ms = time_block(stage, n, stream) / n
            cb_ms = time_block(comb, n, stream) / n
            lay_ms = time_block(both, n, stream) / n
            grp_ms = time_block(lambda i: mole.mole_token_groups_build(ids, V, N, groups=groups, stream=stream), n,
                                stream) / n
            assert mole.mole_check(stream) == 0
            link = U * (N * (D // 64) * 26 if nf3 else row)
            res["cases"][f"T{T}{'_nf3' if nf3 else ''}"] = {
                "unique_rows": U, "link_bytes_per_layer": link, "link_bytes_per_token": link / T,
                "stage_us": st_ms * 1e3, "stage_link_gbs": link / (st_ms / 1e3) / 1e9,
                "stage_frac_of_copy_engine": link / (st_ms / 1e3) / 1e9 / ce_gbs,
                "combine_us": cb_ms * 1e3, "layer_us": lay_ms * 1e3, "token_groups_build_us": grp_ms * 1e3,
                "tokens_per_s_per_layer": T / (lay_ms / 1e3),
                "moe_bytes_per_layer_all_experts": N * moe_expert_bytes,
                "moe_over_mole_bytes_top1_per_token": moe_expert_bytes / (link / T)}
            del groups, staging, h, out, ids
    # decode step over L layers (one host table serves as every layer's: the link
    # traffic per layer is the same), sequential vs the next layer's staging
    # overlapped with this layer's combine
    side = torch.cuda.Stream(device=dev)
    for T in (1, 64):
        ids = torch.from_numpy(inputs.draw_ids(rng, T, V, "zipf")).to(dev)
        groups = torch.empty(mole.mole_token_groups_workspace(T, N), dtype=torch.uint8, device=dev)
        nbytes = mole.mole_offload_staging_bytes(T, V, N, D)
        stg = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        hs_l = [torch.randn((T, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(L)]
        out = torch.empty((T, D), dtype=torch.float32, device=dev)
        e_st = [torch.cuda.Event() for _ in range(L)]
        e_used = [torch.cuda.Event() for _ in range(2)]

        def seq_step(i):
            mole.mole_token_groups_build(ids, V, N, groups=groups, stream=stream)
            for lay in range(L):
                mole.mole_offload_stage(T, groups, host, staging=stg[0], stream=stream)
                mole.mole_lookup_combine_offload(groups, hs_l[lay], routers[lay], stg[0], V, out=out, stream=stream)

        def pipe_step(i):
            mole.mole_token_groups_build(ids, V, N, groups=groups, stream=stream)
            side.wait_stream(stream)
            mole.mole_offload_stage(T, groups, host, staging=stg[0], stream=side)
            e_st[0].record(side)
            for lay in range(L):
                if lay + 1 < L:
                    b = (lay + 1) % 2
                    if lay + 1 >= 2:
                        side.wait_event(e_used[b])
                    mole.mole_offload_stage(T, groups, host, staging=stg[b], stream=side)
                    e_st[lay + 1].record(side)
                stream.wait_event(e_st[lay])
                mole.mole_lookup_combine_offload(groups, hs_l[lay], routers[lay], stg[lay % 2], V, out=out,
                                                 stream=stream)
                e_used[lay % 2].record(stream)

        for i in range(3):
            seq_step(i)
            pipe_step(i)
        n = 20
        seq_ms = time_block(seq_step, n, stream) / n
        pipe_ms = time_block(pipe_step, n, stream) / n
        assert mole.mole_check(stream) == 0
        res["cases"][f"decode_T{T}_{L}layers"] = {
            "sequential_us_per_step": seq_ms * 1e3, "overlapped_us_per_step": pipe_ms * 1e3,
            "tokens_per_s": T / (pipe_ms / 1e3),
            "note": "per step: the grouping, then per layer the staging of its rows from host memory and its "
                    "combine; overlapped = the next layer staged on a second stream into the other staging buffer"}
        del ids, groups, stg, hs_l, out
    del host, hc, hs
    return res


def ffn_leg(mole, luts, routers, rng, g, dev, stream, W, peaks):
    """The MoLE FFN block of a 1B-shaped layer (§8(f) rank 1): one shared expert
    (D x 8192 GELU FFN, as wide as a routed expert), the routed mixture from the
    table, and the residual, for T = 16384 Zipf tokens.  mole_ffn_block = the
    grouped combine into a workspace, then the shared expert's two tcgen05
    GEMMs, the second adding the mixture and the residual in its epilogue."""
    import torch
    shape = inputs.SHAPES["1b"]
    V, D, N, Ds, T = shape.V, shape.D, shape.N, shape.Dr, 16384
    bf16_peak, bf16_sust = peaks
    W1s = (torch.randn((D, Ds), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W2s = (torch.randn((Ds, D), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    ids = torch.from_numpy(inputs.draw_ids(rng, T, V, "zipf")).to(dev)
    h = torch.randn((T, D), generator=g, device=dev).to(torch.bfloat16)
    res = torch.randn((T, D), generator=g, device=dev)
    out = torch.empty((T, D), dtype=torch.float32, device=dev)
    mix = torch.empty((T, D), dtype=torch.float32, device=dev)
    groups = mole.mole_token_groups_build(ids, V, N, stream=stream)
    ws = torch.empty(mole.mole_ffn_block_workspace(T, D, Ds), dtype=torch.uint8, device=dev)
    flops = 4.0 * T * D * Ds

    def block(i):
        mole.mole_ffn_block(ids, groups, h, routers[0], luts[i % len(luts)], W1s, W2s, "gelu", residual=res, out=out,
                            workspace=ws, stream=stream)

    def shared(i):
        mole.mole_shared_ffn(h, W1s, W2s, "gelu", out=out, workspace=ws, stream=stream)

    def unfused(i):  # the three terms apart: combine, shared expert, then two element-wise adds
        mole.mole_lookup_combine_groups(ids, groups, h, routers[0], luts[i % len(luts)], out=mix, stream=stream)
        mole.mole_shared_ffn(h, W1s, W2s, "gelu", out=out, workspace=ws, stream=stream)
        out.add_(mix).add_(res)

    res_line = {}
    for name, fn in (("ffn_block", block), ("shared_expert", shared), ("unfused", unfused)):
        for i in range(max(W, 3)):
            fn(i)
        n = 10
        ms = time_block(fn, n, stream) / n
        res_line[f"{name}_us"] = ms * 1e3
    assert mole.mole_check(stream) == 0
    sh = res_line["shared_expert_us"] / 1e6
    res_line.update({
        "workload": f"1B-shaped FFN block: T={T} Zipf tokens, shared expert {D}x{Ds} GELU FFN (bf16, fp32 "
                    f"accumulate), table [{V}, {N}, {D}] bf16, residual fp32",
        "tokens_per_s": T / (res_line["ffn_block_us"] / 1e6),
        "shared_expert_tflops": flops / sh / 1e12,
        "shared_expert_frac_of_bf16_peak": flops / sh / 1e12 / bf16_peak,
        "shared_expert_frac_of_sustained": (flops / sh / 1e12 / bf16_sust) if bf16_sust else None,
        "combine_share_us": res_line["ffn_block_us"] - res_line["shared_expert_us"],
    })
    del W1s, W2s, h, res, out, mix, ws, groups
    return res_line


def train_leg(mole, rng, g, dev, stream, W, peaks):
    """One MoLE layer's training step at the 1B shape, T = 4096 Zipf tokens
    (§8(f) rank 4): the forward evaluates the routed experts on the batch's
    distinct ids only (tcgen05 build GEMMs), then the combine; the backward
    (gate / router gradients, per-id dL/dY, the four expert GEMMs on the same
    tcgen05 kernels with transposed operand forms)."""
    import torch
    shape = inputs.SHAPES["1b"]
    V, D, N, Dr, T = shape.V, shape.D, shape.N, shape.Dr, 4096
    bf16_peak, _ = peaks
    rnd = lambda *sz, sd=0.02: (torch.randn(sz, generator=g, device=dev) * sd).to(torch.bfloat16)
    E, W1, W2, Wr, h = rnd(V, D), rnd(N, D, Dr), rnd(N, Dr, D), rnd(D, N), rnd(T, D, sd=1.0)
    ids = torch.from_numpy(inputs.draw_ids(rng, T, V, "zipf")).to(dev)
    groups = mole.mole_token_groups_build(ids, V, N, stream=stream)
    out = torch.empty((T, D), dtype=torch.float32, device=dev)
    cache = torch.empty(mole.mole_train_cache_bytes(T, V, N, D, Dr), dtype=torch.uint8, device=dev)
    dout = torch.randn((T, D), generator=g, device=dev)
    z = lambda *sz: torch.zeros(sz, dtype=torch.float32, device=dev)
    grads = dict(dh=z(T, D), dWr=z(D, N), dE=z(V, D), dW1=z(N, D, Dr), dW2=z(N, Dr, D))
    U = [0]

    def fwd(i):
        _, _, U[0] = mole.mole_train_forward(ids, groups, h, Wr, E, W1, W2, out=out, cache=cache, stream=stream)

    def bwd(i):
        mole.mole_train_backward(ids, groups, h, Wr, E, W1, W2, dout, cache, U[0], stream=stream, **grads)

    for i in range(max(W, 3)):
        fwd(i)
        bwd(i)
    n = 5
    f_ms = time_block(fwd, n, stream) / n
    b_ms = time_block(bwd, n, stream) / n
    assert mole.mole_check(stream) == 0
    flops_f = 4.0 * U[0] * D * Dr * N
    flops_b = 8.0 * U[0] * D * Dr * N
    res = {"workload": f"1B-shaped MoLE layer training step: T={T} Zipf tokens, {U[0]} distinct ids, N={N} experts "
                       f"{D}x{Dr} GELU FFN, bf16 weights, fp32 gradients",
           "distinct_ids": U[0], "forward_ms": f_ms, "backward_ms": b_ms,
           "tokens_per_s": T / ((f_ms + b_ms) / 1e3),
           "forward_expert_tflops": flops_f / (f_ms / 1e3) / 1e12,
           "backward_expert_tflops": flops_b / (b_ms / 1e3) / 1e12,
           "forward_frac_of_bf16_peak": flops_f / (f_ms / 1e3) / 1e12 / bf16_peak,
           "expert_flops_saved_vs_per_token": T / max(U[0], 1),
           "note": "forward: the table build restricted to the batch's distinct embedding rows (tcgen05) + the "
                   "grouped combine; the forward reads the distinct-id count back to the host (one sync); "
                   "backward expert GEMMs (dpre, dW2, dW1, dE) on tcgen05"}
    del E, W1, W2, cache, grads
    return res


def graph_pass_us(passes, stream, dev, replays=60, flush=None):
    """Median device time (us) of one replay of a CUDA graph captured from
    each of `passes` (one graph per pooled batch, replayed in rotation), and
    the same passes run eagerly (host-launched) for comparison.  With
    `flush` (a device buffer larger than L2) the buffer is rewritten before
    every timed pass, outside its events, so each pass starts with a cold L2.
    Returns (graph_us or None, eager_us, note)."""
    import torch
    P = len(passes)

    def timed(run, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            if flush is not None:
                flush.fill_(i & 0xff)
            ev[i][0].record(stream)
            run(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3

    for p in range(P):
        passes[p]()
    eager = timed(lambda i: passes[i % P](), 4 * P)
    try:
        graphs = []
        side = torch.cuda.Stream(device=dev)
        for p in range(P):
            gr = torch.cuda.CUDAGraph()
            side.wait_stream(stream)
            with torch.cuda.graph(gr, stream=side, capture_error_mode="thread_local"):
                passes[p]()
            stream.wait_stream(side)
            graphs.append(gr)
    except Exception as e:  # capture not possible: report the eager time only
        torch.cuda.synchronize()
        return None, eager, f"graph capture failed: {type(e).__name__}: {str(e)[:120]}"
    for i in range(3 * P):
        graphs[i % P].replay()
    us = timed(lambda i: graphs[i % P].replay(), replays)
    del graphs
    return us, eager, ("median of CUDA-graph replays (one graph per pooled batch, rotated)"
                       + ("; L2 flushed before each pass" if flush is not None else ""))


def decode_leg(mole, dev, stream):
    """Small batches on the 160M- and 410M-shaped models (decode, T <= 256,
    bf16 tables) and the NF3 1B-shaped sweep (T = 1 .. 16384).  One pass =
    the combine of every layer (own table, router, hidden states; the batch's
    ids shared), captured as a CUDA graph per pooled batch (4 batches,
    rotated, so consecutive replays read other ids), timed as the median of
    60 replays, the L2 flushed before every pass (a 256 MB write outside the
    pass's events: each pass starts cold, as after a step's other work); the
    eager (host-launched) pass is reported beside it, and the same passes
    preceded by mole_prefetch_rows of every layer's rows."""
    import torch
    hbm_peak = measured_peaks()[0]
    res = {}
    P = 4
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2x the L2: every pass starts cold
    sweeps = [("160m", (1, 8, 64), False), ("410m", (1, 2, 4, 8, 16, 32, 64, 128, 256), False),
              ("1b_nf3", (1, 8, 64, 256, 1024, 4096, 16384), True)]
    for name, Ts, nf3 in sweeps:
        shape = inputs.SHAPES[name]
        V, D, N, L = shape.V, shape.D, shape.N, shape.layers
        g = torch.Generator(device=dev)
        g.manual_seed(shape.seed)
        tables = []
        for _ in range(L):
            lut = (torch.randn((V, N, D), generator=g, device=dev) * 0.02).to(torch.bfloat16)
            if nf3:
                tables.append(mole.mole_quantize_lut_nf3(lut, stream=stream))
                del lut
            else:
                tables.append(lut)
        routers = [(torch.randn((D, N), generator=g, device=dev) * 0.02).to(torch.bfloat16) for _ in range(L)]
        zero_id = torch.zeros(1, dtype=torch.int32, device=dev)
        rng = np.random.default_rng(shape.seed)
        for T in Ts:
            ids = [torch.from_numpy(inputs.draw_ids(rng, T, V, "zipf")).to(dev) for _ in range(P)]
            U = sum(int(torch.unique(x).numel()) for x in ids) / P
            hs = [[torch.randn((T, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(L)] for _ in range(P)]
            outs = [torch.empty((T, D), dtype=torch.float32, device=dev) for _ in range(L)]
            groups = [mole.mole_token_groups_build(x, V, N, stream=stream) for x in ids] if T >= 1024 else None

            def prefetch_layers(p, lays):
                mole.mole_prefetch_rows(zero_id, [routers[x].view(1, -1) for x in lays])
                if nf3:
                    mole.mole_prefetch_rows(ids[p], [tables[x][0] for x in lays])
                    mole.mole_prefetch_rows(ids[p], [tables[x][1] for x in lays])
                else:
                    mole.mole_prefetch_rows(ids[p], [tables[x] for x in lays])

            def make_pass(p, prefetch=None):
                def run():
                    if prefetch == "all":  # every layer's rows and router for this step, asked of L2 up front
                        prefetch_layers(p, range(L))
                    elif prefetch == "ahead":
                        prefetch_layers(p, [0])
                    for lay in range(L):
                        if prefetch == "ahead" and lay + 1 < L:  # the next layer's, while this one runs
                            prefetch_layers(p, [lay + 1])
                        if nf3 and groups is not None:
                            mole.mole_lookup_combine_nf3_groups(ids[p], groups[p], hs[p][lay], routers[lay],
                                                                *tables[lay], out=outs[lay])
                        elif nf3:
                            mole.mole_lookup_combine_nf3(ids[p], hs[p][lay], routers[lay], *tables[lay],
                                                         out=outs[lay])
                        else:
                            mole.mole_lookup_combine(ids[p], hs[p][lay], routers[lay], tables[lay], out=outs[lay])
                return run

            graph_us, eager_us, note = graph_pass_us([make_pass(p) for p in range(P)], stream, dev, flush=flush)
            pf_us, pf_eager_us, _ = graph_pass_us([make_pass(p, "all") for p in range(P)], stream, dev, flush=flush)
            pa_us, pa_eager_us, _ = graph_pass_us([make_pass(p, "ahead") for p in range(P)], stream, dev,
                                                  flush=flush)
            st = mole.mole_check(stream)
            if st != 0:
                raise RuntimeError(f"device status {st} in the {name} T={T} sweep")
            pass_us = graph_us if graph_us is not None else eager_us
            b = (nf3_bytes if nf3 else combine_bytes)(U, T, D, N)
            res[f"{name}_T{T}"] = {
                "us_per_layer_call": pass_us / L, "us_per_pass": pass_us, "eager_us_per_pass": eager_us,
                "tokens_per_s": T / (pass_us / 1e6), "layer_tokens_per_s": T * L / (pass_us / 1e6),
                "unique_rows": U, "achieved_gbs": b / (pass_us / L / 1e6) / 1e9,
                "frac_of_measured_hbm": b / (pass_us / L / 1e6) / 1e9 / hbm_peak, "layers": L,
                "prefetch_all_us_per_layer_call": (pf_us if pf_us is not None else pf_eager_us) / L,
                "prefetch_ahead_us_per_layer_call": (pa_us if pa_us is not None else pa_eager_us) / L,
                "prefetch_note": "mole_prefetch_rows of the rows (and router) of every layer at the pass start "
                                 "(all), or of layer l+1 before layer l's combine (ahead)",
                "call": ("mole_lookup_combine_nf3_groups (grouping built once per batch, outside the pass)"
                         if nf3 and groups is not None else
                         "mole_lookup_combine_nf3" if nf3 else "mole_lookup_combine"),
                "timing": note}
            del ids, hs, outs, groups
        del tables, routers
        torch.cuda.empty_cache()
    return res


def build_leg(mole, dev, stream, bf16_peak, bf16_sust, peak_kind, reps=3, warmup=1, experts=None):
    import torch
    shape = inputs.SHAPES["410m"]
    V, D, N, Dr = shape.V, shape.D, shape.N if experts is None else max(1, experts), shape.Dr
    g = torch.Generator(device=dev)
    g.manual_seed(shape.seed)
    E = (torch.randn((V, D), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W1 = (torch.randn((N, D, Dr), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((N, Dr, D), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    lut = torch.empty((V, N, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(mole.mole_build_lut_workspace(V, D, N, Dr, torch.bfloat16, 0), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        mole.mole_build_lut(E, W1, W2, lut=lut, workspace=ws, stream=stream)
    ms = time_launches(lambda i: mole.mole_build_lut(E, W1, W2, lut=lut, workspace=ws, stream=stream), reps, stream)
    assert mole.mole_check(stream) == 0
    best = min(ms)
    flops = 4.0 * V * D * Dr * N
    tf = flops / (best / 1e3) / 1e12
    # the NF3 table straight from the build (quantising epilogue) vs build + quantiser
    codes = torch.empty((V, N, D // 64, 24), dtype=torch.uint8, device=dev)
    scales = torch.empty((V, N, D // 64), dtype=torch.float16, device=dev)
    mole.mole_build_lut_nf3(E, W1, W2, codes=codes, scales=scales, workspace=ws, stream=stream)
    nf3_ms = min(time_launches(lambda i: mole.mole_build_lut_nf3(E, W1, W2, codes=codes, scales=scales, workspace=ws,
                                                                 stream=stream), reps, stream))
    mole.mole_quantize_lut_nf3(lut, codes, scales, stream=stream)  # (its first launch loads the kernel)
    q_ms = min(time_launches(lambda i: mole.mole_quantize_lut_nf3(lut, codes, scales, stream=stream), reps, stream))
    assert mole.mole_check(stream) == 0
    del codes, scales
    return {"workload": f"410M-shaped table build V={V} D={D} N={N} Dr={Dr} GELU (2 tcgen05 GEMMs per expert group)",
            "tflops": tf, "ms": best, "flops": flops, "frac_of_bf16_peak": tf / bf16_peak,
            "peak": bf16_peak, "peak_source": f"{peak_kind} burst bf16 (MEASURED_PEAKS.json)",
            "frac_of_sustained": (tf / bf16_sust) if bf16_sust else None, "frac_of_2250": tf / 2250.0,
            "nf3_build_ms": nf3_ms, "build_then_quantize_ms": best + q_ms,
            "nf3_build_note": "mole_build_lut_nf3 (NF3 quantiser in the second GEMM's epilogue, no bf16 table) vs "
                              "mole_build_lut + mole_quantize_lut_nf3"}


def cpu_baseline(args):
    """The oracle, as it stands, on a bounded sample of the workload."""
    import oracle
    oracle.build()
    shape = inputs.SHAPES["1b"]
    V, D, N, L = shape.V, shape.D, shape.N, shape.layers
    r = np.random.default_rng(99)
    sample_T = 1024
    ids = inputs.draw_ids(r, sample_T, V, args.ids)
    uniq, inv = np.unique(ids, return_inverse=True)
    rows = inputs.normal(r, (uniq.size, N, D), 0.02, "bf16")
    Wr = inputs.normal(r, (D, N), 0.02, "bf16")
    h = inputs.normal(r, (sample_T, D), 1.0, "bf16")
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.combine(inv.astype(np.int32), h, Wr, rows)
        reps += 1
        if time.perf_counter() - t0 > 10.0 or reps >= 5000:
            break
    dt = time.perf_counter() - t0
    per_layer = sample_T * reps / dt
    return {"value": per_layer / L, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{sample_T} tokens of one 1B-shaped layer x {reps} repetitions ({dt:.1f} s); "
                      f"tokens/s through {L} layers = per-layer rate / {L}"}


if __name__ == "__main__":
    main()
