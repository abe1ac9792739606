"""Benchmark: one paged GQA decode step (kv_append + paged_decode_attention,
fused into one launch by pgd_decode_step; --unfused times the two calls) on
the Llama-3-8B-shaped workload (64 sequences, context U[512, 4096], 32 q /
8 KV heads, head_dim 128, block_size 16, bf16 KV, 64 new tokens appended).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints ONE JSON line (rank 0).  `value` is achieved HBM bandwidth in GB/s:
the algorithmic bytes of a step (every cached K/V row once per (sequence, KV
head), q in, out back, block-table entries, context lengths, append payload
read + written) divided by the device time of the step, summed over ranks.
With N > 1 (torchrun) every rank runs its own independent batch (weak
scaling, no collective on the data path); time is the max over ranks.

--impl reference times the fp64 CPU oracle on host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("paged GQA decode attention: achieved HBM GB/s (% of peak), "
          "µs per decode step")
DEFAULT_WORKLOAD = "llama3_8b_decode"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = ["paged_gqa_decode_07_b200/csrc/pgd_decode.cuh",
                  "paged_gqa_decode_07_b200/csrc/pgd_ptx.cuh",
                  "paged_gqa_decode_07_b200/csrc/pgd_launch.h",
                  "paged_gqa_decode_07_b200/csrc/pgd_decode_family.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload: str):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu
    summary, only if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        e = d.get(workload)
        if e and e.get("kernel_source_hash") == kernel_source_hash():
            return int(e["dram_bytes_per_launch"])
    except Exception:  # noqa: BLE001
        pass
    return None


def workload_desc(w) -> dict:
    return {"workload": f"{w.name}: {w.num_seqs} seqs, {w.num_tokens} context tokens "
                        f"(seed 0 draw), {w.num_q_heads} q / {w.num_kv_heads} kv heads, "
                        f"head_dim {w.head_dim}, block_size {w.block_size}, {w.kv_dtype} KV"
                        + (f", kv_append of {len(w.slot_mapping)} tokens"
                           if w.slot_mapping is not None else ""),
            "num_seqs": w.num_seqs, "context_tokens": w.num_tokens,
            "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size, "kv_dtype": w.kv_dtype}


# --------------------------------------------------------------------------- #
# clocks during the timed region                                              #
# --------------------------------------------------------------------------- #
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 3.0:
            time.sleep(0.02)

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self):
        return time.time()

    def stop(self, t_begin, t_end):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=2)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [ln for ts, ln in self.lines if t_begin - 0.05 <= ts <= t_end + 0.15]
        if not rows and self.lines:
            rows = [min(self.lines, key=lambda x: abs(x[0] - t_end))[1]]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- #
# rank aggregation                                                            #
# --------------------------------------------------------------------------- #
def reduce_over_ranks(step_bytes: int, ms_step: float, e2e_ms: float, dec_ms: float,
                      world: int, device=None) -> dict:
    """Whole-job figures over all ranks: the bytes every rank moved in one step
    are summed, each time is the maximum over ranks, and value = summed bytes
    / max step time.  Works on any initialised process group (nccl with CUDA
    tensors, gloo with CPU ones); with world == 1 it only divides."""
    import torch
    import torch.distributed as dist
    if world > 1:
        t = torch.tensor([ms_step, e2e_ms, dec_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step, e2e_ms, dec_ms = t.tolist()
        b = torch.tensor([float(step_bytes)], dtype=torch.float64, device=device)
        dist.all_reduce(b, op=dist.ReduceOp.SUM)
        total_bytes = b.item()
    else:
        total_bytes = float(step_bytes)
    return {"ms_step": ms_step, "e2e_ms": e2e_ms, "dec_ms": dec_ms, "total_bytes": total_bytes,
            "value": total_bytes / (ms_step * 1e-3) / 1e9,
            "e2e_value": total_bytes / (e2e_ms * 1e-3) / 1e9}


# --------------------------------------------------------------------------- #
# our arm                                                                     #
# --------------------------------------------------------------------------- #
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import paged_gqa_decode_07_b200 as pgd
    from workloads import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    # every rank runs its own batch: same shape (context lengths of seed 0),
    # its own block permutation and values
    w = make_workload(args.workload, seed=rank, shape_seed=0)
    ab = w.algorithmic_bytes()

    def to_dev(a, pin=False):
        import numpy as _np
        t = torch.from_numpy(_np.ascontiguousarray(a).view(_np.int16) if a.dtype == _np.uint16
                             else _np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.pin_memory() if pin else t.to(dev)

    q, k, v = to_dev(w.q), to_dev(w.k_cache), to_dev(w.v_cache)
    bt, cl = to_dev(w.block_table), to_dev(w.context_lens)
    ks = to_dev(w.k_scale) if w.k_scale is not None else None
    vs = to_dev(w.v_scale) if w.v_scale is not None else None
    has_app = w.slot_mapping is not None
    if has_app:
        kn, vn, sl = to_dev(w.k_new), to_dev(w.v_new), to_dev(w.slot_mapping)
    out = torch.empty_like(q)
    mcl = w.max_context_len
    stream = torch.cuda.current_stream()
    # a decode step whose appended tokens are each sequence's newest token runs
    # as one fused launch (pgd_decode_step); --unfused times append + decode
    fused = has_app and not args.unfused and len(w.slot_mapping) == w.num_seqs

    def step(q_, kn_, vn_, sl_, bt_, cl_, out_):
        if fused:
            pgd.decode_step(q_, kn_, vn_, k, v, bt_, cl_, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.block_size, w.scale, out_, max_context_len=mcl,
                            k_scale=ks, v_scale=vs, stream=stream)
            return
        if has_app:
            pgd.kv_append(kn_, vn_, sl_, k, v, stream=stream)
        pgd.paged_decode_attention(q_, k, v, bt_, cl_, w.num_q_heads, w.num_kv_heads,
                                   w.head_dim, w.block_size, w.scale, out_,
                                   max_context_len=mcl, k_scale=ks, v_scale=vs, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- warm-up -------------------------------------------------------------
    for _ in range(args.warmup):
        step(q, kn if has_app else None, vn if has_app else None, sl if has_app else None,
             bt, cl, out)
    torch.cuda.synchronize()
    assert pgd.get_device_error() == 0

    def decode_only():
        if fused:
            pgd.decode_step(q, kn, vn, k, v, bt, cl, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.block_size, w.scale, out, max_context_len=mcl, k_scale=ks,
                            v_scale=vs, stream=stream)
        else:
            pgd.paged_decode_attention(q, k, v, bt, cl, w.num_q_heads, w.num_kv_heads,
                                       w.head_dim, w.block_size, w.scale, out,
                                       max_context_len=mcl, k_scale=ks, v_scale=vs,
                                       stream=stream)

    # ---- timed region: K back-to-back steps, device time ---------------------
    # No event sits between launches (an event between two launches stops the
    # next launch from overlapping its set-up with the previous one's tail).
    # With one launch per step the decode kernel's average launch duration is
    # this region's time / K; the unfused mode brackets each decode launch.
    K = args.steps
    single = fused or not has_app          # one launch per step
    ev_dec = [] if single else [(torch.cuda.Event(enable_timing=True),
                                 torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local_rank) if not args.no_clocks else None
    if clocks:
        clocks.start()
    barrier()
    torch.cuda.synchronize()
    t_begin = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        if single:
            decode_only()
            continue
        pgd.kv_append(kn, vn, sl, k, v, stream=stream)
        ev_dec[i][0].record(stream)
        decode_only()
        ev_dec[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_end = time.time()
    clk = clocks.stop(t_begin, t_end) if clocks else None
    ms_total = e0.elapsed_time(e1)
    if single:
        dec_avg_ms = ms_total / K
    else:
        dec_avg_ms = sum(a.elapsed_time(b) for a, b in ev_dec) / K
    flags = pgd.get_device_error()
    # for reference: the same launch bracketed by its own events, one at a time
    iso = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(min(K, 50))]
    for a_, b_ in iso:
        a_.record(stream)
        decode_only()
        b_.record(stream)
    torch.cuda.synchronize()
    iso_ms = sum(a_.elapsed_time(b_) for a_, b_ in iso) / len(iso)

    # ---- end to end through the public API with host buffers ----------------
    hq = to_dev(w.q, pin=True)
    hbt, hcl = to_dev(w.block_table, pin=True), to_dev(w.context_lens, pin=True)
    dq, dbt, dcl = torch.empty_like(q), torch.empty_like(bt), torch.empty_like(cl)
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = [(hq, dq), (hbt, dbt), (hcl, dcl)]
    if has_app:
        hkn, hvn, hsl = to_dev(w.k_new, pin=True), to_dev(w.v_new, pin=True), \
            to_dev(w.slot_mapping, pin=True)
        dkn, dvn, dsl = torch.empty_like(kn), torch.empty_like(vn), torch.empty_like(sl)
        h2d += [(hkn, dkn), (hvn, dvn), (hsl, dsl)]
    h2d_bytes = sum(h.numel() * h.element_size() for h, _ in h2d)
    d2h_bytes = hout.numel() * hout.element_size()
    Ke = max(1, min(K, args.e2e_steps))

    def e2e_step():
        for h, d in h2d:
            d.copy_(h, non_blocking=True)
        step(dq, dkn if has_app else None, dvn if has_app else None, dsl if has_app else None,
             dbt, dcl, out)
        hout.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(Ke):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = f0.elapsed_time(f1) / Ke

    # ---- aggregate over ranks ----------------------------------------------------
    ms_step = ms_total / K
    agg = reduce_over_ranks(ab["step_total"], ms_step, e2e_ms, dec_avg_ms, world, dev)
    ms_step, e2e_ms, dec_avg_ms = agg["ms_step"], agg["e2e_ms"], agg["dec_ms"]
    value, e2e_value = agg["value"], agg["e2e_value"]
    peak, peak_kind = measured_peak()
    dec_bytes = ab["step_total"] if fused else ab["decode_total"]
    achieved = dec_bytes / (dec_avg_ms * 1e-3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        cfg = workload_desc(w)
        cfg.update({"parallelism": f"replicas x{world} (independent batch per GPU)",
                    "l2": f"inputs larger than L2 ({ab['kv'] / 1e6:.0f} MB of KV read per step "
                          f"vs {L2_BYTES / 2**20:.0f} MiB L2); no flush",
                    "global_batch": w.num_seqs * world})
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "us_per_step": round(ms_step * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.kv_dtype, "data": "synthetic (seeded N(0,1) Q/K/V, shuffled block table)",
            "config": cfg,
            "pct_of_measured_hbm": round(100 * value / world / peak, 1),
            "pct_of_nominal_8tbs": round(100 * value / world / 8000.0, 1),
            "roofline": {"bound": "hbm",
                         "kernel": "paged_decode_kernel" + (" (fused append)" if fused else ""),
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "algorithmic_bytes_per_launch": dec_bytes,
                         "avg_launch_us": round(dec_avg_ms * 1e3, 2),
                         "launch_timing": "timed region / K (one launch per step, "
                                          "back to back)" if single else
                                          "events around each decode launch",
                         "isolated_launch_us": round(iso_ms * 1e3, 2),
                         "traffic": recorded_traffic(args.workload)},
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s",
                    "us_per_step": round(e2e_ms * 1e3, 2),
                    "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                    "steps": Ke},
            "gpu_launches": K * (2 if has_app and not fused else 1),
            "fused_step": fused,
            "clocks": clk,
            "device_flags": flags,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# CPU oracle (baseline leg and reference arm)                                 #
# --------------------------------------------------------------------------- #
def _oracle_units(w):
    """(seq, kv head) units in a fixed seeded order, with their KV bytes."""
    rng = np.random.default_rng(1234)
    units = [(s, h) for s in range(w.num_seqs) for h in range(w.num_kv_heads)
             if w.context_lens[s] > 0]
    order = rng.permutation(len(units))
    return [units[i] for i in order]


def _oracle_setup(w):
    import oracle
    oracle.build_oracle()
    kc, vc = w.k_cache, w.v_cache
    if w.slot_mapping is not None:
        kc, vc = oracle.kv_append(w.k_new, w.v_new, w.slot_mapping, kc, vc, w.block_size)
    return oracle, kc, vc


def _oracle_unit(oracle, w, kc, vc, s, h):
    g = w.group
    rs = np.full(g, s, np.int32)
    rh = np.arange(h * g, h * g + g, dtype=np.int32)
    oracle.paged_decode_rows(w.q, kc, vc, w.block_table, w.context_lens, w.num_kv_heads,
                             w.scale, rs, rh, w.k_scale, w.v_scale)
    return int(w.context_lens[s]) * w.head_dim * 2 * w.elem_bytes


def cpu_baseline(w, seconds: float) -> dict:
    """Time the oracle, as it stands, on a bounded sample of the workload:
    whole (sequence, KV head) units in a fixed random order until `seconds`
    of CPU time have passed.  Value = KV bytes of the sampled units / time."""
    oracle, kc, vc = _oracle_setup(w)
    units = _oracle_units(w)
    done, nbytes = 0, 0
    t0 = time.perf_counter()
    for s, h in units:
        nbytes += _oracle_unit(oracle, w, kc, vc, s, h)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} of {len(units)} (sequence, KV head) units of the same workload "
                      f"({nbytes / 1e6:.1f} MB of K/V, {dt:.1f} s), fp64 single-threaded C",
            "host_cpus": os.cpu_count()}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from workloads import make_workload
    w = make_workload(args.workload, seed=0)
    oracle, kc, vc = _oracle_setup(w)
    units = _oracle_units(w)
    # each step: a bounded slice of the workload (whole units), sized so the
    # whole run stays within about two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    t = time.perf_counter()
    _oracle_unit(oracle, w, kc, vc, *units[0])
    per_unit = time.perf_counter() - t
    per_step = max(1, min(len(units), int(budget / max(per_unit, 1e-6))))
    pos = 0

    def step():
        nonlocal pos
        b = 0
        for _ in range(per_step):
            b += _oracle_unit(oracle, w, kc, vc, *units[pos % len(units)])
            pos += 1
        return b

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    nbytes = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    cfg = workload_desc(w)
    cfg.update({"parallelism": "host, 1 thread", "global_batch": w.num_seqs})
    sample = (f"{per_step} (sequence, KV head) unit(s) per step, fixed random order, "
              f"fp64 single-threaded C oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfg,
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="time kv_append and the decode as two launches")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE",
              file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
