"""Benchmark: one paged GQA decode step on the long-context small-batch
workload by default (4 sequences of 131072 tokens, 64 q / 8 KV heads,
head_dim 128, block_size 64, bf16 KV: 2.1 GB of K/V read per step, the
split-KV partitioning and log-sum-exp combine case).  Other workloads with
--workload; the ones that carry an append payload (llama3_8b_decode) time the
kv_append of each sequence's newest token fused into the decode launch
(pgd_decode_step), or the two calls with --unfused.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-copy-probe]

Prints ONE JSON line (rank 0).  `value` is achieved HBM bandwidth in GB/s:
the algorithmic bytes of a step (every cached K/V row once per (sequence, KV
head), q in, out back, block-table entries, context lengths, append payload
read + written) divided by the device time of the step, summed over ranks.
With N > 1 (torchrun) every rank runs its own independent batch (weak
scaling, no collective on the data path); time is the max over ranks.

--impl reference times the fp64 CPU oracle on host cores (rank 0 only).

Other rows of the path, same JSON line, each on its own workload shape:
    --q-len L --window W   decode of the L newest tokens per sequence (causal
                           among them) and/or a sliding window of W tokens
                           (pgd_paged_decode_attention_ex); the bytes count
                           the visible K/V rows only
    --math cuda_core       the decode kernel's q.k and p.V as FP32 FMAs with
                           warp-shuffle sums instead of mma.sync (comparison)
    --kvp                  one batch with every sequence's KV split along its
                           length over the N ranks: slice decode to fp32,
                           all-gather, log-sum-exp merge (strong scaling)
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
DEFAULT_WORKLOAD = "long_context"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
# The decode kernel and the host code that sets its grid and work cut: a
# committed DRAM-traffic record counts only while these are unchanged.
KERNEL_SOURCES = ["paged_gqa_decode_07_b200/csrc/pgd_decode.cuh",
                  "paged_gqa_decode_07_b200/csrc/pgd_ptx.cuh",
                  "paged_gqa_decode_07_b200/csrc/pgd_launch.h",
                  "paged_gqa_decode_07_b200/csrc/pgd_decode_family.cuh",
                  "paged_gqa_decode_07_b200/csrc/pgd_grid.h"]


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


def l2_replicas(read_bytes: int, cache_bytes: int, cap_bytes: int = 16 << 30) -> int:
    """How many copies of the K/V caches the timed loop rotates through, one
    per step, so that a cached row is read again only after at least 2x L2
    of other K/V has streamed past it (1 when one step already reads that
    much).  Capped so that the copies hold at most `cap_bytes`."""
    if read_bytes >= 2 * L2_BYTES:
        return 1
    want = -(-2 * L2_BYTES // max(1, read_bytes))
    return int(max(1, min(want, cap_bytes // max(1, cache_bytes))))


def cache_copies(w, read_bytes, T):
    """The caches (and FP8 scales) on the device, replicated per l2_replicas."""
    R = l2_replicas(read_bytes, w.k_cache.nbytes + w.v_cache.nbytes)
    ks = T(w.k_scale) if w.k_scale is not None else None
    vs = T(w.v_scale) if w.v_scale is not None else None
    return [(T(w.k_cache), T(w.v_cache)) for _ in range(R)], ks, vs


def copy_probe(dev, nbytes: int = 2 << 30, reps: int = 20) -> dict:
    """HBM copy bandwidth in this process: the best of `reps` device-to-device
    copies of an `nbytes` buffer, counting the bytes read and written."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    for _ in range(3):
        dst.copy_(src)
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src)
        b.record()
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    del src, dst
    torch.cuda.empty_cache()
    return {"gbs": round(2 * nbytes / (best * 1e-3) / 1e9, 1), "bytes_per_copy": 2 * nbytes,
            "how": f"best of {reps} device-to-device copies of {nbytes >> 30} GiB "
                   "(read + write bytes), same process, after the timed regions"}


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
def _to_torch(a, dev=None, pin=False):
    """numpy -> torch (bf16 bits stay bf16); pinned host memory or `dev`."""
    import torch
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.pin_memory() if pin else t.to(dev)


class Mode:
    """One kind of timed step.  step(inp, ev, r) runs one step on the tensors
    of `inp` (device resident) and copy r of the caches; with `ev` = (start,
    end) events it records them around the dominant kernel's launch."""
    single = True            # one launch per step: its duration = region / K
    kernel = "paged_decode_kernel"
    scaling = "weak"

    def __init__(self):
        self.inputs, self.host, self.out = {}, {}, None
        self.cfg = {}
        self.replicas = 1
        self.read_bytes = 0


def mode_step(args, w, pgd, dev, stream):
    """The decode step: kv_append of each sequence's newest token fused into
    the decode launch (pgd_decode_step), or --unfused: the two calls."""
    m = Mode()
    T = lambda a: _to_torch(a, dev)  # noqa: E731
    ab = w.algorithmic_bytes()
    caches, ks, vs = cache_copies(w, ab["kv"], T)
    has_app = w.slot_mapping is not None
    arrays = {"q": w.q, "bt": w.block_table, "cl": w.context_lens}
    if has_app:
        arrays.update(kn=w.k_new, vn=w.v_new, sl=w.slot_mapping)
    m.inputs = {n: T(a) for n, a in arrays.items()}
    m.host = {n: _to_torch(a, pin=True) for n, a in arrays.items()}
    m.out = torch_empty_like(m.inputs["q"])
    fused = has_app and not args.unfused and len(w.slot_mapping) == w.num_seqs
    mcl = w.max_context_len

    def calls(inp, r):
        """The step's library calls on input set `inp` and cache copy r,
        prepared once (argument checks and marshalling) and re-issued every
        step, as a serving loop with persistent buffers would."""
        k, v = caches[r]
        out = inp.get("out", m.out)
        app = None
        if has_app and not fused:
            app = pgd.kv_append(inp["kn"], inp["vn"], inp["sl"], k, v, stream=stream,
                                prepare=True)
        if fused:
            dec = pgd.decode_step(inp["q"], inp["kn"], inp["vn"], k, v, inp["bt"], inp["cl"],
                                  w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                  w.scale, out, max_context_len=mcl, k_scale=ks, v_scale=vs,
                                  stream=stream, prepare=True)
        else:
            dec = pgd.paged_decode_attention(inp["q"], k, v, inp["bt"], inp["cl"], w.num_q_heads,
                                             w.num_kv_heads, w.head_dim, w.block_size, w.scale,
                                             out, max_context_len=mcl, k_scale=ks, v_scale=vs,
                                             stream=stream, prepare=True)
        return app, dec

    prepared = {}

    def step(inp, ev=None, r=0):
        key = (id(inp), r)
        if key not in prepared:
            prepared[key] = calls(inp, r)
        app, dec = prepared[key]
        if app is not None:
            app()
        if ev:
            ev[0].record(stream)
        dec()
        if ev:
            ev[1].record(stream)

    m.step = step
    m.single = fused or not has_app
    m.launches = 2 if has_app and not fused else 1
    m.kernel = "paged_decode_kernel" + (" (fused append)" if fused else "")
    m.dec_bytes = ab["step_total"] if fused else ab["decode_total"]
    m.step_bytes = ab["step_total"]
    m.fused = fused
    m.replicas, m.read_bytes = len(caches), ab["kv"]
    return m


def mode_ex(args, w, pgd, dev, stream):
    """q_len query tokens per sequence and/or a sliding window
    (pgd_paged_decode_attention_ex).  The append payload, if the workload
    has one, is written once before timing, so every token is cached."""
    from workloads import multi_query
    m = Mode()
    T = lambda a: _to_torch(a, dev)  # noqa: E731
    L, W = args.q_len, args.window
    ab = w.algorithmic_bytes(L, W)
    caches, ks, vs = cache_copies(w, ab["kv"], T)
    if w.slot_mapping is not None:
        for k, v in caches:
            pgd.kv_append(T(w.k_new), T(w.v_new), T(w.slot_mapping), k, v, stream=stream)
    arrays = {"q": multi_query(w, L, seed=0), "bt": w.block_table, "cl": w.context_lens}
    m.inputs = {n: T(a) for n, a in arrays.items()}
    m.host = {n: _to_torch(a, pin=True) for n, a in arrays.items()}
    m.out = torch_empty_like(m.inputs["q"])
    mcl = w.max_context_len

    prepared = {}

    def step(inp, ev=None, r=0):
        key = (id(inp), r)
        if key not in prepared:
            k, v = caches[r]
            prepared[key] = pgd.paged_decode_attention_ex(
                inp["q"], k, v, inp["bt"], inp["cl"], w.num_q_heads, w.num_kv_heads, w.head_dim,
                w.block_size, w.scale, inp.get("out", m.out), window=W, max_context_len=mcl,
                k_scale=ks, v_scale=vs, stream=stream, prepare=True)
        if ev:
            ev[0].record(stream)
        prepared[key]()
        if ev:
            ev[1].record(stream)

    m.step, m.launches, m.fused = step, 1, False
    m.replicas, m.read_bytes = len(caches), ab["kv"]
    m.kernel = f"paged_decode_kernel (q_len {L}, window {W})"
    m.dec_bytes = m.step_bytes = ab["decode_total"]
    m.cfg = {"q_len": L, "window": W, "visible_tokens":
             int(sum(b - a for a, b in zip(*w.visible_ranges(L, W))))}
    return m


def mode_kvp(args, w, pgd, dev, stream, rank, world):
    """KV parallelism: every sequence's KV is split along its length over the
    ranks (pgd_kvp_plan); a step is this rank's slice decode
    (pgd_paged_decode_partial), the all-gather of the split results and the
    merge (pgd_merge_partials).  Total work is fixed as ranks are added."""
    import torch

    from paged_gqa_decode_07_b200 import kvp
    m = Mode()
    T = lambda a: _to_torch(a, dev)  # noqa: E731
    if w.slot_mapping is not None:
        raise SystemExit("--kvp needs a workload without an append payload")
    start, length = kvp.plan(w.context_lens, w.block_size, world, rank)
    bs, Hkv, D, e = w.block_size, w.num_kv_heads, w.head_dim, w.elem_bytes
    slice_kv = int(length.astype(np.int64).sum()) * Hkv * D * 2 * e
    caches, ks, vs = cache_copies(w, slice_kv, T)
    table = kvp.local_block_table(w.block_table, start, length, w.block_size)
    arrays = {"q": w.q, "bt": table, "cl": length}
    m.inputs = {n: T(a) for n, a in arrays.items()}
    m.host = {n: _to_torch(a, pin=True) for n, a in arrays.items()}
    dec = kvp.KVPDecoder(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                         device=dev)
    m.out = dec.out
    mcl = int(length.max(initial=0))
    rows = w.num_seqs * w.num_q_heads

    def step(inp, ev=None, r=0):
        k, v = caches[r]
        if ev:
            ev[0].record(stream)
        pgd.paged_decode_partial(inp["q"], k, v, inp["bt"], inp["cl"], w.num_q_heads,
                                 w.num_kv_heads, w.head_dim, w.block_size, w.scale,
                                 dec.o_local, dec.lse_local, max_context_len=mcl, k_scale=ks,
                                 v_scale=vs, stream=stream)
        if ev:
            ev[1].record(stream)
        kvp.gather_partials(dec.o_local, dec.lse_local, dec.o_all, dec.lse_all)
        pgd.merge_partials(dec.o_all, dec.lse_all, inp.get("out", dec.out).view(rows, w.head_dim),
                           dec.lse, stream=stream)

    blocks = int(((length.astype(np.int64) + bs - 1) // bs).sum())
    meta = blocks * 4 + w.num_seqs * 4 + (2 * Hkv * 4 if w.kv_dtype == "e4m3" else 0)
    # the slice kernel reads q, its slice and metadata, and writes fp32 o + lse
    m.dec_bytes = slice_kv + meta + rows * D * 2 + rows * (D + 1) * 4
    full = w.algorithmic_bytes()
    # the job's bytes: every K/V row once, q in and out back once, metadata
    m.step_bytes = slice_kv + meta + (full["qo"] if rank == 0 else 0)
    m.step, m.single, m.launches, m.fused = step, False, 2, False
    m.kernel = "paged_decode_kernel (fp32 split result of the rank's KV slice)"
    m.scaling = "strong"
    m.replicas, m.read_bytes = len(caches), slice_kv
    m.cfg = {"kvp_ranks": world, "exchange_bytes_per_rank": dec.exchange_bytes(),
             "slice_tokens_this_rank": int(length.sum())}
    return m


def mode_op(args, w, pgd, dev, stream):
    """One auxiliary kernel alone, on the workload's shapes:
      kv_append        N new tokens' bf16 (or E4M3) K/V rows scattered into
                       N distinct cache slots (pgd_kv_append)
      kv_append_quant  N bf16 rows quantised into an E4M3 cache
                       (pgd_kv_append_quant)
      merge            the log-sum-exp merge of P split results of every
                       (sequence, query head) row (pgd_merge_partials)
    N = --append-tokens (default: one per sequence); P = --merge-parts."""
    import torch
    m = Mode()
    rng = np.random.default_rng(77)
    Hkv, D, bs = w.num_kv_heads, w.head_dim, w.block_size
    if args.op in ("kv_append", "kv_append_quant"):
        N = args.append_tokens or w.num_seqs
        pool = max(w.num_blocks, -(-N // bs))
        if args.op == "kv_append":
            e = w.elem_bytes
            dt = torch.bfloat16 if e == 2 else torch.uint8
        else:
            e, dt = 1, torch.uint8
        k = torch.zeros((pool, Hkv, bs, D), dtype=dt, device=dev)
        v = torch.zeros_like(k)
        src_dt = torch.bfloat16 if args.op == "kv_append_quant" else dt
        host = {"kn": torch.randn((N, Hkv, D)).to(src_dt) if src_dt == torch.bfloat16 else
                torch.randint(0, 120, (N, Hkv, D), dtype=torch.uint8),
                "sl": torch.from_numpy(rng.permutation(pool * bs)[:N].astype(np.int64))}
        host["vn"] = host["kn"].flip(0).contiguous()
        ks = torch.full((Hkv,), 0.01, dtype=torch.float32, device=dev)
        m.inputs = {n: t.to(dev) for n, t in host.items()}
        m.host = {n: t.pin_memory() for n, t in host.items()}
        m.out = k
        src_e = 2 if args.op == "kv_append_quant" else e
        m.dec_bytes = m.step_bytes = 2 * N * Hkv * D * (src_e + e) + 8 * N + \
            (8 * Hkv if args.op == "kv_append_quant" else 0)
        m.read_bytes = 2 * N * Hkv * D * src_e
        prepared = {}

        def step(inp, ev=None, r=0):
            key = id(inp)
            if key not in prepared:
                if args.op == "kv_append":
                    prepared[key] = pgd.kv_append(inp["kn"], inp["vn"], inp["sl"], k, v,
                                                  stream=stream, prepare=True)
                else:
                    prepared[key] = pgd.kv_append_quant(inp["kn"], inp["vn"], inp["sl"], k, v,
                                                        ks, ks, stream=stream, prepare=True)
            if ev:
                ev[0].record(stream)
            prepared[key]()
            if ev:
                ev[1].record(stream)

        m.kernel = "kv_append_kernel" if args.op == "kv_append" else "kv_append_quant_kernel"
        m.cfg = {"op": args.op, "append_tokens": N, "pool_slots": pool * bs}
    else:
        P, rows = args.merge_parts, w.num_seqs * w.num_q_heads
        host = {"o": torch.randn((P, rows, D), dtype=torch.float32),
                "l": (torch.randn((P, rows), dtype=torch.float32) * 3)}
        m.inputs = {n: t.to(dev) for n, t in host.items()}
        m.host = {n: t.pin_memory() for n, t in host.items()}
        m.out = torch.empty((rows, D), dtype=torch.bfloat16, device=dev)
        m.dec_bytes = m.step_bytes = P * rows * (D + 1) * 4 + rows * D * 2
        m.read_bytes = P * rows * (D + 1) * 4
        prepared = {}

        def step(inp, ev=None, r=0):
            key = id(inp)
            if key not in prepared:
                prepared[key] = pgd.merge_partials(inp["o"], inp["l"], inp.get("out", m.out),
                                                   stream=stream, prepare=True)
            if ev:
                ev[0].record(stream)
            prepared[key]()
            if ev:
                ev[1].record(stream)

        m.kernel = "merge_partials_kernel"
        m.cfg = {"op": "merge", "merge_parts": P, "rows": rows}
    m.step, m.single, m.launches, m.fused = step, True, 1, False
    m.replicas = 1
    return m


def torch_empty_like(t):
    import torch
    return torch.empty_like(t)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import paged_gqa_decode_07_b200 as pgd
    from workloads import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    pgd.set_decode_math(args.math)
    if args.kvp:
        # one batch split over the ranks: the same data on every rank
        w = make_workload(args.workload, seed=0, shape_seed=0)
        m = mode_kvp(args, w, pgd, dev, stream, rank, world)
    else:
        # every rank runs its own batch: same shape (context lengths of seed
        # 0), its own block permutation and values
        w = make_workload(args.workload, seed=rank, shape_seed=0)
        if args.op:
            m = mode_op(args, w, pgd, dev, stream)
        elif args.q_len > 1 or args.window > 0:
            m = mode_ex(args, w, pgd, dev, stream)
        else:
            m = mode_step(args, w, pgd, dev, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- warm-up -------------------------------------------------------------
    R = m.replicas
    for i in range(max(args.warmup, R)):
        m.step(m.inputs, None, i % R)
    torch.cuda.synchronize()
    assert pgd.get_device_error() == 0

    # ---- timed region: K back-to-back steps, device time ---------------------
    # No event sits between launches of a one-launch step (an event between
    # two launches stops the next launch from overlapping its set-up with the
    # previous one's tail): the kernel's average launch duration is this
    # region's time / K.  Steps of several launches bracket the dominant one.
    K = args.steps
    ev_dec = [] if m.single else [(torch.cuda.Event(enable_timing=True),
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
        m.step(m.inputs, None if m.single else ev_dec[i], i % R)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_end = time.time()
    clk = clocks.stop(t_begin, t_end) if clocks else None
    ms_total = e0.elapsed_time(e1)
    if m.single:
        dec_avg_ms = ms_total / K
    else:
        dec_avg_ms = sum(a.elapsed_time(b) for a, b in ev_dec) / K
    flags = pgd.get_device_error()
    # for reference: the dominant launch bracketed by its own events, one at a time
    iso = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(min(K, 50))]
    for i, ev in enumerate(iso):
        m.step(m.inputs, ev, i % R)
    torch.cuda.synchronize()
    iso_ms = sum(a_.elapsed_time(b_) for a_, b_ in iso) / len(iso)

    # ---- end to end through the public API with host buffers ----------------
    def e2e_run():
        # Every step copies its inputs from pinned host memory (packed into one
        # buffer, one copy) and reads its output back.  As in a serving loop, the
        # input copy of step i+1 and the read-back of step i-1 run on their own
        # streams while step i decodes (inputs and outputs double-buffered); all
        # of every step's copies are inside the timed region.
        names = list(m.host.keys())
        nbytes = {n: m.host[n].numel() * m.host[n].element_size() for n in names}
        offs, total = {}, 0
        for n in names:
            offs[n] = total
            total += (nbytes[n] + 255) // 256 * 256
        hpack = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        for n in names:
            hpack[offs[n]:offs[n] + nbytes[n]].copy_(m.host[n].reshape(-1).view(torch.uint8))
        dpack = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
        bufs = []
        for b in range(2):
            views = {n: dpack[b][offs[n]:offs[n] + nbytes[n]].view(m.host[n].dtype)
                     .view(m.host[n].shape) for n in names}
            views["out"] = torch.empty_like(m.out)
            bufs.append(views)
        hout = [torch.empty(m.out.shape, dtype=m.out.dtype, pin_memory=True) for _ in range(2)]
        s_h2d = torch.cuda.Stream(device=dev)
        s_d2h = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b copied
        ev_cmp = [torch.cuda.Event() for _ in range(2)]    # step using buffer b computed
        ev_out = [torch.cuda.Event() for _ in range(2)]    # output of buffer b read back
        h2d_bytes = total
        d2h_bytes = hout[0].numel() * hout[0].element_size()
        Ke = max(1, min(K, args.e2e_steps))

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                if i >= 2:
                    s_h2d.wait_event(ev_cmp[b])            # step i-2 no longer reads buffer b
                with torch.cuda.stream(s_h2d):
                    dpack[b].copy_(hpack, non_blocking=True)
                ev_in[b].record(s_h2d)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])           # output of step i-2 read back
                m.step(bufs[b], None, i % R)
                ev_cmp[b].record(stream)
                s_d2h.wait_event(ev_cmp[b])
                with torch.cuda.stream(s_d2h):
                    hout[b].copy_(bufs[b]["out"], non_blocking=True)
                ev_out[b].record(s_d2h)

        e2e_steps(3)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(s_h2d)
        e2e_steps(Ke)
        s_d2h.wait_event(ev_cmp[(Ke - 1) % 2])
        f1.record(s_d2h)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = f0.elapsed_time(f1) / Ke
        # the kernels are deterministic: the read-back output is the resident run's
        assert torch.equal(hout[(Ke - 1) % 2].view(torch.uint8), m.out.cpu().view(torch.uint8)), \
            "end-to-end output differs from the device-resident run"
        return e2e_ms, h2d_bytes, d2h_bytes, Ke

    if args.op:
        # an auxiliary kernel alone: no end-to-end line (its result is the
        # cache or a merged output of other launches, not a step's output)
        e2e_ms, h2d_bytes, d2h_bytes, Ke = float("nan"), 0, 0, 0
    else:
        e2e_ms, h2d_bytes, d2h_bytes, Ke = e2e_run()

    # ---- aggregate over ranks ----------------------------------------------------
    ms_step = ms_total / K
    agg = reduce_over_ranks(m.step_bytes, ms_step, e2e_ms, dec_avg_ms, world, dev)
    ms_step, e2e_ms = agg["ms_step"], agg["e2e_ms"]
    value, e2e_value = agg["value"], agg["e2e_value"]
    peak, peak_kind = measured_peak()
    # the dominant kernel of this rank (rank 0 prints its own launch figures)
    achieved = m.dec_bytes / (dec_avg_ms * 1e-3) / 1e9

    probe = copy_probe(dev) if not args.no_copy_probe else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.op:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        cfg = workload_desc(w)
        cfg.update(m.cfg)
        if args.math != "tensor_core":
            cfg["math"] = args.math
        kv_mb = m.read_bytes / 1e6
        if R == 1:
            l2 = (f"inputs larger than L2 ({kv_mb:.0f} MB of KV read per step vs "
                  f"{L2_BYTES / 2**20:.0f} MiB L2); no flush")
        else:
            l2 = (f"{kv_mb:.0f} MB of KV read per step is under 2x the {L2_BYTES / 2**20:.0f} "
                  f"MiB L2: the steps rotate through {R} copies of the caches, so "
                  f"{R * kv_mb:.0f} MB of KV streams between two reads of a row; no flush")
        cfg.update({"parallelism": (f"KV parallel over {world} rank(s) (one batch, each "
                                    f"sequence split along its length)") if args.kvp else
                    f"replicas x{world} (independent batch per GPU)",
                    "l2": l2, "cache_copies": R,
                    "global_batch": w.num_seqs * (1 if args.kvp else world)})
        default_mode = not args.kvp and args.q_len == 1 and args.window == 0 and not args.op
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "us_per_step": round(ms_step * 1e3, 2),
            "higher_is_better": True, "scaling": m.scaling, "vs_baseline": None,
            "dtype": w.kv_dtype, "data": "synthetic (seeded N(0,1) Q/K/V, shuffled block table)",
            "config": cfg,
            "pct_of_measured_hbm": round(100 * value / world / peak, 1),
            "pct_of_nominal_8tbs": round(100 * value / world / 8000.0, 1),
            "pct_of_same_run_copy": round(100 * achieved / probe["gbs"], 1) if probe else None,
            "copy_probe": probe,
            "roofline": {"bound": "hbm", "kernel": m.kernel,
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "algorithmic_bytes_per_launch": m.dec_bytes,
                         "avg_launch_us": round(dec_avg_ms * 1e3, 2),
                         "launch_timing": "timed region / K (one launch per step, "
                                          "back to back)" if m.single else
                                          "events around each dominant launch",
                         "isolated_launch_us": round(iso_ms * 1e3, 2),
                         "traffic": recorded_traffic(args.workload) if default_mode else None},
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s",
                    "us_per_step": round(e2e_ms * 1e3, 2),
                    "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                    "steps": Ke,
                    "copies": "one packed H2D of the step's inputs and one D2H of its output "
                              "per step, on their own streams, overlapping the neighbouring "
                              "steps' decode (double-buffered)"} if not args.op else None,
            "gpu_launches": K * m.launches,
            "fused_step": m.fused,
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


def _oracle_unit(oracle, w, kc, vc, s, h, n_tok=None):
    """The oracle on every query row of unit (s, h); with n_tok, on the first
    n_tok tokens of the sequence only (a bounded sample).  Returns the K/V
    bytes of the unit that were read (once per unit, as the GPU arm counts)."""
    g = w.group
    rs = np.full(g, s, np.int32)
    rh = np.arange(h * g, h * g + g, dtype=np.int32)
    cl = w.context_lens
    if n_tok is not None and n_tok < int(cl[s]):
        cl = cl.copy()
        cl[s] = n_tok
    oracle.paged_decode_rows(w.q, kc, vc, w.block_table, cl, w.num_kv_heads,
                             w.scale, rs, rh, w.k_scale, w.v_scale)
    return int(cl[s]) * w.head_dim * 2 * w.elem_bytes


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
    # each step: a bounded sample of the workload, sized so that the whole run
    # (warm-up and timed steps) stays within about two minutes: whole units in
    # a fixed random order, or, when one unit alone would take longer than a
    # step's share, the first tokens of one unit
    budget = 120.0 / max(1, args.steps + args.warmup)
    s0, h0 = units[0]
    n_cal = int(min(int(w.context_lens[s0]), 4096))
    t = time.perf_counter()
    _oracle_unit(oracle, w, kc, vc, s0, h0, n_cal)
    per_token = (time.perf_counter() - t) / max(1, n_cal)
    step_tokens = max(w.block_size, int(budget / max(per_token, 1e-9)))
    pos = 0

    def step():
        nonlocal pos
        b, left = 0, step_tokens
        while left > 0:
            s_, h_ = units[pos % len(units)]
            pos += 1
            n = min(left, int(w.context_lens[s_]))
            b += _oracle_unit(oracle, w, kc, vc, s_, h_, n)
            left -= n
        return b

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    nbytes = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    cfg = workload_desc(w)
    cfg.update({"parallelism": "host, 1 thread", "global_batch": w.num_seqs})
    sample = (f"{step_tokens} context tokens of whole (sequence, KV head) units per step "
              f"(all query rows of each unit; the first tokens of a unit when it is longer), "
              f"fixed random order, fp64 single-threaded C oracle")
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
    ap.add_argument("--no-copy-probe", action="store_true",
                    help="skip the same-run HBM copy probe (4 GiB of device buffers)")
    ap.add_argument("--unfused", action="store_true",
                    help="time kv_append and the decode as two launches")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per sequence (causal among them)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window in tokens (0 = whole context)")
    ap.add_argument("--math", choices=["tensor_core", "cuda_core"], default="tensor_core",
                    help="consumer math of the decode kernel (cuda_core: FMA + warp shuffles, "
                         "bf16 head_dim 128 with <= 8 query rows per KV head)")
    ap.add_argument("--kvp", action="store_true",
                    help="split every sequence's KV over the ranks (strong scaling)")
    ap.add_argument("--op", choices=["kv_append", "kv_append_quant", "merge"], default=None,
                    help="time one auxiliary kernel alone on the workload's shapes")
    ap.add_argument("--append-tokens", type=int, default=0,
                    help="--op kv_append*: new tokens per call (default: one per sequence)")
    ap.add_argument("--merge-parts", type=int, default=8,
                    help="--op merge: split results merged per row")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.q_len < 1 or args.window < 0:
        ap.error("--q-len must be >= 1 and --window >= 0")
    if args.kvp and (args.q_len > 1 or args.window > 0 or args.unfused):
        ap.error("--kvp runs the one-token decode without append")
    if args.op and (args.kvp or args.q_len > 1 or args.window > 0 or args.unfused):
        ap.error("--op times one auxiliary kernel alone")

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
