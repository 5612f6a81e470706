"""Benchmark: decode attention (split-KV, Flash-Decoding style) on B200.

One step = one fd_decode call (split kernel + combine kernel) over one batch
of the workload, inputs resident in HBM. Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl fd|reference]

Multi-GPU, one process per GPU: under torchrun (WORLD_SIZE set, and equal to
--gpus), or, with --gpus N > 1 and no WORLD_SIZE, bench.py starts the N ranks
itself. Every rank decodes its own independent batch of the same shape (seed +
rank); nothing is exchanged on the data path, so scaling is weak and value =
sum over ranks of KV bytes / the slowest rank's device time.

At one GPU on the headline workload the line also carries per_config: every
other workload (and the 8-bit caches of the two long batch-1 ones) measured
the same way in the same run.

The reference arm (--impl reference) is the CPU oracle (fp64, host cores) on
a bounded sample of the same workload.
"""
import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import decode_attention_07_b200 as fd  # noqa: E402
from decode_attention_07_b200.configs import HEADLINE, WORKLOADS  # noqa: E402
from decode_attention_07_b200.inputs import bf16_bits, make_inputs  # noqa: E402

METRIC = "decode-attention µs/call and KV-read GB/s as % of B200 HBM peak, 1 GPU"
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024


# The sources that define the split kernel and its launch (tile sizes, ring,
# consumers, grid): DRAM traffic recorded for one hash is valid while they
# are unchanged.
SPLIT_KERNEL_SOURCES = ("fd_api.cu", "fd_merge.cuh", "fd_partition.cuh", "fd_ptx.cuh", "fd_quant.cuh",
                        "fd_split.cuh")


def kernel_source_hash() -> str:
    """Hash of the split kernel's CUDA sources (SPLIT_KERNEL_SOURCES)."""
    import hashlib
    h = hashlib.sha256()
    for name in SPLIT_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "decode_attention_07_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """Per-launch DRAM bytes (read + write) recorded in profiles/traffic.txt
    for this workload, if the kernel sources are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == workload and parts[1] == want:
                return int(parts[2]) + int(parts[3])
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed work runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ byte counts --

def byte_counts(w, lens, S, q_len=1, elem_bytes=2):
    """Algorithmic bytes of one call: K/V inside the sequences, q, and the
    outputs / workspace segments each stage writes and reads (q_len queries
    per sequence: q_len times the query and output bytes)."""
    lens = np.clip(lens.astype(np.int64), 0, w.Lmax)
    kv = int(lens.sum()) * w.Hkv * w.D * elem_bytes * 2
    q = w.B * q_len * w.Hq * w.D * 2
    seg = fd.fd_segments(w.B, w.Hkv, w.Lmax, lens.astype(np.int32), S)
    used = seg["row"] >= 0
    row_bytes = q_len * w.g * (w.D + 1) * 4
    n_whole = int(seg["whole"][used].sum())
    n_part = int(used.sum()) - n_whole
    multi_rows = len(set(seg["row"][used & (seg["whole"] == 0)].tolist()))
    empty_rows = int((lens == 0).sum()) * w.Hkv
    split_bytes = kv + q + (n_whole + n_part) * row_bytes + w.B * 4
    combine_bytes = n_part * row_bytes + (multi_rows + empty_rows) * row_bytes + w.B * 4
    return dict(kv=kv, q=q, split=split_bytes, combine=combine_bytes, total=split_bytes + combine_bytes,
                segments=n_part, whole_rows=n_whole, multi_rows=multi_rows)


def launch_bytes(w, lens_per_copy, S, q_len=1, elem_bytes=2):
    """Algorithmic bytes of one launch when the timed calls alternate over
    input copies with these lengths (ragged copies differ): the copies' mean
    of byte_counts."""
    per_copy = [byte_counts(w, lens, S, q_len, elem_bytes) for lens in lens_per_copy]
    return {k: sum(c[k] for c in per_copy) / len(per_copy) for k in per_copy[0]}


# ------------------------------------------------------------- the CPU arm --

def oracle_sample(x, budget_s=12.0, nthreads=0, collect=None):
    """Time the CPU oracle on a bounded sample of the workload: whole
    sequences (all kv heads and query heads; the oracle spreads the rows over
    the host cores), longest first, until about `budget_s` seconds of work;
    a sequence too long for the budget is cut to its first kv heads.
    Returns (kv_bytes_processed, seconds, threads, description); with a list
    `collect`, appends (b, first query head, oracle out, oracle lse) per call."""
    import oracle
    w = x.workload
    orc = oracle.default()
    quant = hasattr(x, "k8")
    elem = 1 if quant else 2
    order = np.argsort(-x.seqlens_host, kind="stable")
    done_bytes, spent, rows, threads = 0, 0.0, 0, 0
    for b in order:
        L = int(min(max(x.seqlens_host[b], 0), w.Lmax))
        if L == 0:
            continue
        # kv heads per call: enough rows to occupy the cores, few enough to stay in budget
        step = max(1, min(w.Hkv, (os.cpu_count() or 1) // max(1, w.g)))
        for j0 in range(0, w.Hkv, step):
            j1 = min(w.Hkv, j0 + step)
            qh = bf16_bits(x.q[b:b + 1, j0 * w.g:j1 * w.g])
            if quant:
                kh = x.k8[b:b + 1, j0:j1, :L].cpu().numpy()
                vh = x.v8[b:b + 1, j0:j1, :L].cpu().numpy()
                ks, vs = x.k_scale[j0:j1].cpu().numpy(), x.v_scale[j0:j1].cpu().numpy()
                t0 = time.perf_counter()
                o, lo = orc.attention_quant(qh, kh, vh, ks, vs, np.array([L], np.int32), x.scale, x.kv_type,
                                            nthreads)
            else:
                kh = bf16_bits(x.k[b:b + 1, j0:j1, :L])
                vh = bf16_bits(x.v[b:b + 1, j0:j1, :L])
                t0 = time.perf_counter()
                o, lo = orc.attention(qh, kh, vh, np.array([L], np.int32), x.scale, nthreads)
            spent += time.perf_counter() - t0
            if collect is not None:
                collect.append((int(b), j0 * w.g, o[0], lo[0]))
            threads = max(threads, orc.threads_used)
            done_bytes += (j1 - j0) * L * w.D * elem * 2
            rows += j1 - j0
            if spent >= budget_s:
                break
        if spent >= budget_s:
            break
    desc = (f"{rows} (sequence, kv-head) rows x {w.g} query heads of {w.name} seed {x.seed}"
            f"{' (' + x.kv_type + ' cache)' if quant else ''}, longest sequences first; "
            f"KV bytes of the sample / oracle seconds")
    return done_bytes, spent, threads, desc


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    x = make_inputs(w, args.seed, device="cuda" if torch.cuda.is_available() else "cpu")
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(x, budget_s=per_step)
    total_b, total_s, threads, desc = 0, 0.0, 0, ""
    for _ in range(args.steps):
        b, s, t, desc = oracle_sample(x, budget_s=per_step)
        total_b += b
        total_s += s
        threads = max(threads, t)
    gbs = total_b / total_s / 1e9
    kv_full = int(np.clip(x.seqlens_host, 0, w.Lmax).astype(np.int64).sum()) * w.Hkv * w.D * 4
    line = {
        "metric": METRIC, "impl": "reference", "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": kv_full / (gbs * 1e9) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, None, "n/a (host memory)"),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rank_seed(seed: int, rank: int) -> int:
    """Each rank decodes its own independent batch: seed + rank."""
    return int(seed) + int(rank)


def max_over_ranks(value: float, device) -> float:
    """The slowest rank's value (device time is reported as the max over
    ranks). Works on any process group: NCCL with a CUDA device, gloo on CPU."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank_step: float, steps: int, ms_max: float) -> float:
    """Weak scaling: every rank moves the same bytes per step; the job's rate
    is all ranks' bytes over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


def config_dict(w, S, l2):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "Lmax": w.Lmax,
            "ragged": w.ragged, "num_splits": S, "l2": l2, "description": w.description}


# ------------------------------------------------------------- the GPU arm --

def read_probe_gbs(dev, stream, nbytes=2 << 30, reps=10):
    """HBM read ceiling on this GPU: fd_read_probe over a buffer far larger
    than L2, CUDA events around `reps` back-to-back passes."""
    buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    for _ in range(2):
        fd.fd_read_probe(buf, sink, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fd.fd_read_probe(buf, sink, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    gbs = nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9
    timed_out = probe_timed_out(int(sink.item()))
    del buf
    torch.cuda.empty_cache()
    return None if timed_out else gbs


def probe_timed_out(sink_word: int) -> bool:
    """fd_read_probe folds data into the low 32 bits of its sink and sets the
    upper half when a bounded wait gave up (a pass that stopped early would
    report an inflated rate)."""
    return ((sink_word >> 32) & 0x7FFFFFFF) != 0


class L2Flush:
    """Evicts the caller's data from L2 between isolated calls: a write of
    twice L2's size, then a read of another buffer of twice its size, so L2
    is left holding clean lines (a timed call that starts behind the write
    alone would first pay for writing back ~L2 of dirty lines)."""

    def __init__(self, dev):
        self.w = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self, i):
        self.w.fill_(i & 255)
        self.r.sum()


def per_call_stats(call_at, dev, stream, steps, flush=None):
    """Each call timed alone with CUDA events, L2 flushed before it (outside
    the events, see L2Flush): median, p10, p90 in us."""
    flush = flush or L2Flush(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush(i)
        ev[i][0].record(stream)
        call_at(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t = np.array([a.elapsed_time(b) * 1e3 for a, b in ev])
    return {"median_us": float(np.median(t)), "p10_us": float(np.percentile(t, 10)),
            "p90_us": float(np.percentile(t, 90)), "calls": steps,
            "l2": "flushed before every call: write of 2x L2, then read of another 2x L2 (outside the events)"}


class Workspace:
    """One workload's inputs, outputs, workspace and prepared calls on this
    rank: `calls[i]` enqueues one call on input copy i (two copies rotated
    when a copy is larger than L2, so no call finds its predecessor's bytes
    in L2; one copy otherwise, with L2 flushed before every timed call)."""

    def __init__(self, w, kv, seed, dev, stream, q_len=1, paged=0, layout="HND", page_order="shuffled"):
        self.w, self.kv, self.dev, self.stream = w, kv, dev, stream
        self.quant = kv != "bf16"
        self.S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
        S, Q = self.S, q_len

        def draw(sd):
            if self.quant:
                from decode_attention_07_b200.inputs import make_quant
                return make_quant(w, kv, sd, device=dev)
            return make_inputs(w, sd, device=dev)

        xs = [draw(seed)]
        kv_per_copy = xs[0].kv_bytes()
        self.n_copies = 2 if kv_per_copy >= L2_BYTES else 1
        self.l2_note = (f"inputs larger than L2: 2 input copies of {kv_per_copy / 1e6:.0f} MB rotated"
                        if self.n_copies == 2 else
                        "L2 flushed before every timed call (write of 2x L2 then read of 2x L2, outside the events)")
        for c in range(1, self.n_copies):
            xs.append(draw(seed + 1000 * c))
        nbytes = fd.fd_workspace_bytes(w.B, w.Hq * Q, w.Hkv, w.D, w.Lmax, S)
        self.ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=dev)   # row counters start at zero
        oshape = (w.B, w.Hq) if Q == 1 else (w.B, Q, w.Hq)
        out = torch.empty(oshape + (w.D,), dtype=torch.float32, device=dev)
        lse = torch.empty(oshape, dtype=torch.float32, device=dev)
        self.out, self.lse = out, lse
        if Q > 1:
            # q_len new tokens per sequence: queries [B, q_len, Hq, D] drawn like q
            for i, x in enumerate(xs):
                g = torch.Generator(device=dev).manual_seed(seed + 77 + i)
                x.q = (torch.randn((w.B, Q, w.Hq, w.D), generator=g, device=dev) * w.sigma_q).to(torch.bfloat16)
        self.counts = launch_bytes(w, [x.seqlens_host for x in xs], S, Q, 1 if self.quant else 2)
        self.kv_bytes = sum(x.kv_bytes() for x in xs) / self.n_copies
        ws = self.ws
        if paged:
            # the same logical caches, scattered into shuffled page pools
            from decode_attention_07_b200.inputs import make_paged
            pgs = [make_paged(x, paged, layout, seed=7 + i, order=page_order) for i, x in enumerate(xs)]
            for x in xs:   # the contiguous copies are not used by the paged calls
                if self.quant:
                    x.k8 = x.v8 = None
                else:
                    x.k = x.v = None
            torch.cuda.empty_cache()
            if self.quant:
                self.calls = [fd.prepare_decode_quant_paged(x.q, pg.k_pages, pg.v_pages, x.k_scale, x.v_scale, kv,
                                                            pg.block_table, x.seqlens, x.scale, out, lse, ws, layout,
                                                            S, stream) for x, pg in zip(xs, pgs)]
            else:
                self.calls = [fd.prepare_decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens,
                                                      x.scale, out, lse, ws, layout, S, stream)
                              for x, pg in zip(xs, pgs)]
            self.pages = pgs
        elif self.quant:
            self.calls = [fd.prepare_decode_quant(x.q, x.k8, x.v8, x.k_scale, x.v_scale, kv, x.seqlens, x.scale, out,
                                                  lse, ws, S, stream) for x in xs]
        elif Q > 1:
            self.calls = [fd.prepare_decode_multi(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S, stream)
                          for x in xs]
        else:
            self.calls = [fd.prepare_decode(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S, stream) for x in xs]
        self.xs = xs
        self.flush = L2Flush(dev) if self.n_copies == 1 else None

    def call(self, i):
        self.calls[i % self.n_copies]()

    def timed(self, steps):
        """Device milliseconds of `steps` calls: back to back over the rotated
        copies (one event pair), or, for a workload that fits in L2, call by
        call with L2 flushed before each (flush outside the events)."""
        st = self.stream
        if self.flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for i in range(steps):
                self.call(i)
            e1.record(st)
            torch.cuda.synchronize(self.dev)
            return e0.elapsed_time(e1)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            self.flush(i)
            ev[i][0].record(st)
            self.call(0)
            ev[i][1].record(st)
        torch.cuda.synchronize(self.dev)
        return sum(a.elapsed_time(b) for a, b in ev)

    def parity_rows(self):
        """(b, kv head) rows checked against the oracle: the first and the
        last sequence, each with its last kv head (empty rows skipped)."""
        w = self.w
        rows = []
        for b in sorted({0, w.B - 1}):
            if int(min(max(self.xs[0].seqlens_host[b], 0), w.Lmax)) > 0:
                rows.append((b, w.Hkv - 1))
        return rows

    def parity(self, rows=None):
        """One call on input copy 0, then the oracle on `rows`: max-abs error
        on out, relative error on lse (floored at 1)."""
        import oracle
        w, x = self.w, self.xs[0]
        orc = oracle.default()
        self.calls[0]()
        torch.cuda.synchronize(self.dev)
        o_gpu, l_gpu = self.out.double().cpu().numpy(), self.lse.double().cpu().numpy()
        err_o, err_l, n = 0.0, 0.0, 0
        for b, j in rows if rows is not None else self.parity_rows():
            L = int(min(max(x.seqlens_host[b], 0), w.Lmax))
            qh = bf16_bits(x.q[b:b + 1, j * w.g:(j + 1) * w.g])
            if self.quant:
                o, lo = orc.attention_quant(qh, x.k8[b:b + 1, j:j + 1, :L].cpu().numpy(),
                                            x.v8[b:b + 1, j:j + 1, :L].cpu().numpy(), x.k_scale[j:j + 1].cpu().numpy(),
                                            x.v_scale[j:j + 1].cpu().numpy(), np.array([L], np.int32), x.scale,
                                            x.kv_type)
            else:
                o, lo = orc.attention(qh, bf16_bits(x.k[b:b + 1, j:j + 1, :L]), bf16_bits(x.v[b:b + 1, j:j + 1, :L]),
                                      np.array([L], np.int32), x.scale)
            og, lg = o_gpu[b, j * w.g:(j + 1) * w.g], l_gpu[b, j * w.g:(j + 1) * w.g]
            err_o = max(err_o, float(np.abs(og - o[0]).max()))
            fin = np.isfinite(lo[0])
            if fin.any():
                err_l = max(err_l, float((np.abs(lg[fin] - lo[0][fin]) / np.maximum(1.0, np.abs(lo[0][fin]))).max()))
            n += w.g
        return {"max_abs_err_out": err_o, "max_rel_err_lse": err_l, "rows": n,
                "tolerance": {"out_abs": 2e-3, "lse_rel": 1e-4},
                "against": "oracle (fp64): the first and last sequence, last kv head, all its query heads"}


def config_entry(args, w, kv, dev, stream, peak):
    """One workload measured like the headline, for the line's per_config
    object: back-to-back and isolated us per call, KV and algorithmic
    bandwidth, roofline fraction, and oracle parity on sampled rows."""
    wk = Workspace(w, kv, args.seed, dev, stream)
    for i in range(max(3, args.warmup)):
        wk.call(i)
    torch.cuda.synchronize(dev)
    ms = wk.timed(args.steps)
    us = ms * 1e3 / args.steps
    iso = per_call_stats(wk.call, dev, stream, max(10, min(args.steps, 20)))
    achieved = wk.counts["total"] / (us * 1e-6) / 1e9
    key = w.name + (f":{kv}" if kv != "bf16" else "")
    entry = {
        "workload": w.name, "kv_cache": kv, "num_splits": wk.S, "l2": wk.l2_note,
        "timing": "back to back over rotated copies" if wk.flush is None else "call by call, L2 flushed before each",
        "us_per_call": us, "us_per_call_isolated": iso,
        "kv_gbs": wk.kv_bytes / (us * 1e-6) / 1e9,
        "pct_of_nominal_hbm_kv": 100.0 * wk.kv_bytes / (us * 1e-6) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS, "bytes_per_launch": wk.counts["total"],
                     "traffic": measured_traffic(key)},
        "parity": wk.parity(),
        "steps": args.steps,
    }
    del wk
    torch.cuda.empty_cache()
    return key, entry


# workloads measured beside the headline in the per_config object (name, cache type)
PER_CONFIG = [("tiny_mha", "bf16"), ("gqa_128k", "bf16"), ("batch_4k", "bf16"), ("ragged_64k", "bf16"),
              ("mha_16k", "e4m3"), ("gqa_128k", "e4m3")]


def run_fd(args, w, rank, world):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    quant = args.kv != "bf16"
    Q = args.q_len
    wk = Workspace(w, args.kv, rank_seed(args.seed, rank), dev, stream, Q, args.paged, args.layout, args.page_order)
    S, n_copies, xs, out, lse, ws = wk.S, wk.n_copies, wk.xs, wk.out, wk.lse, wk.ws
    counts, kv_bytes, calls = wk.counts, wk.kv_bytes, wk.calls

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    probe = read_probe_gbs(dev, stream) if rank == 0 else None
    for i in range(max(3, args.warmup)):
        wk.call(i)
    torch.cuda.synchronize(dev)

    # ---- main timed region: K calls back to back (or, for a workload that
    # fits in L2, call by call with L2 flushed outside the events) ---------
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        t_wall = time.perf_counter()
        ms_local = wk.timed(args.steps)
        # keep the sampler on the same work for >= 1.5 s so clocks are seen under load
        t_min = time.perf_counter() + (0.0 if args.no_clock_window else 1.5)
        j = 0
        while time.perf_counter() < t_min:
            for _ in range(50):
                wk.call(j)
                j += 1
            torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t_wall
    barrier()
    ms_max = max_over_ranks(ms_local, dev)
    us_per_call = ms_max * 1e3 / args.steps
    gbs = whole_job_gbs(world, kv_bytes, args.steps, ms_max)

    per_call = per_call_stats(wk.call, dev, stream, max(10, min(args.steps, 50)))

    # ---- the two stages as separate kernels (for the per-stage split) ------
    # Each stage is timed as K back-to-back launches of that stage alone
    # (one event pair around them, per-launch average), as the fused call
    # is: the split over the rotated input copies, then the combine K times
    # over the workspace the last split left (it only reads the workspace
    # and rewrites out / lse, so repeating it is the same work each time).
    stages = None
    if not args.paged and Q == 1 and not quant:
        k_st = max(5, min(args.steps, 20))

        def timed_loop(fn):
            fn(0)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(k_st):
                fn(i)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) * 1e3 / k_st

        def split_i(i):
            x = xs[i % n_copies]
            fd.fd_split(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S, stream)

        split_us = timed_loop(split_i)
        x0 = xs[(k_st - 1) % n_copies]
        combine_us = timed_loop(lambda i: fd.fd_combine(w.B, w.Hq, w.Hkv, w.D, w.Lmax, x0.seqlens, out, lse, ws, S,
                                                         stream))
        stages = {"split_us": split_us, "combine_us": combine_us,
                  "how": f"{k_st} back-to-back launches of each stage alone, per-launch average"}

    # ---- end to end: host buffers in, host buffers out ---------------------
    e2e = None
    if not args.no_e2e and not args.paged:
        x = xs[0]
        kc, vc = (x.k8, x.v8) if quant else (x.k, x.v)
        hq, hk, hv = x.q.cpu().pin_memory(), kc.cpu().pin_memory(), vc.cpu().pin_memory()
        hs = x.seqlens.cpu().pin_memory()
        dq, dk, dv, dsq = (torch.empty_like(t) for t in (x.q, kc, vc, x.seqlens))
        if quant:   # the per-head scales travel with the cache
            hks, hvs = x.k_scale.cpu().pin_memory(), x.v_scale.cpu().pin_memory()
            dks, dvs = torch.empty_like(x.k_scale), torch.empty_like(x.v_scale)
        ho = torch.empty(tuple(out.shape), dtype=torch.float32).pin_memory()
        hl = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs) + ((hks, hvs) if quant else ()))
        d2h = ho.numel() * 4 + hl.numel() * 4
        e_steps = max(3, min(args.steps, 20))

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dsq.copy_(hs, non_blocking=True)
            if quant:
                dks.copy_(hks, non_blocking=True)
                dvs.copy_(hvs, non_blocking=True)
                fd.fd_decode_quant(dq, dk, dv, dks, dvs, args.kv, dsq, x.scale, out, lse, ws, S, stream)
            elif Q > 1:
                fd.fd_decode_multi(dq, dk, dv, dsq, x.scale, out, lse, ws, S, stream)
            else:
                fd.fd_decode_splits(dq, dk, dv, dsq, x.scale, out, lse, ws, S, stream)
            ho.copy_(out, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": whole_job_gbs(world, x.kv_bytes(), e_steps, ems), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "us_per_call": ems * 1e3 / e_steps}
        del dq, dk, dv, dsq

    status = fd.fd_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status}: {fd.fd_strerror(status)}")

    if rank != 0:
        return 0
    peak, peak_kind = peaks()
    kernel_gbs = counts["total"] / (us_per_call * 1e-6) / 1e9
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_max / args.steps, "us_per_call": us_per_call,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.kv, "data": "synthetic",
        "config": dict(config_dict(w, S, wk.l2_note), **({"kv_cache": args.kv} if quant else {}),
                       **({"paged": {"page_size": args.paged, "layout": args.layout, "page_order": args.page_order}}
                          if args.paged else {}),
                       **({"q_len": Q} if Q > 1 else {})),
        "pct_of_nominal_hbm": 100.0 * gbs / world / NOMINAL_HBM_GBS,
        "pct_of_measured_copy": 100.0 * gbs / world / peak,
        "read_probe": {"gbs": probe, "bytes": 2 << 30,
                       "kernel": "fd_read_probe (bulk copies, 1 block per SM, 128 KiB in flight)"},
        "pct_of_read_probe": 100.0 * gbs / world / probe if probe else None,
        "per_call": per_call,
        "call_bytes_gbs": world * counts["total"] * args.steps / (ms_max * 1e-3) / 1e9,
        "roofline": {"kernel": "fd_split_kernel (fused combine)" + (f", {args.kv} cache" if quant else ""),
                     "bound": "hbm", "achieved": kernel_gbs,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": kernel_gbs / peak,
                     "traffic": None if args.paged or Q > 1 else measured_traffic(w.name + (f":{args.kv}" if quant else "")),
                     "bytes_per_launch": counts["total"],
                     "us_per_launch": us_per_call,
                     "frac_of_nominal_8tbs": kernel_gbs / NOMINAL_HBM_GBS},
        "stages_alone": stages,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "wall_s": wall,
    }
    if world == 1 and not args.no_cpu_baseline and not args.paged and Q == 1:   # bf16 or 8-bit cache
        rows = []
        b, s, t, desc = oracle_sample(xs[0], budget_s=args.cpu_seconds, collect=rows)
        # parity of the timed path on the same sample: one more call on the first input copy
        calls[0]()
        torch.cuda.synchronize(dev)
        o_gpu, l_gpu = out.double().cpu().numpy(), lse.double().cpu().numpy()
        err_o, err_l = 0.0, 0.0
        for bb, h0, o_ref, l_ref in rows:
            og, lg = o_gpu[bb, h0:h0 + o_ref.shape[0]], l_gpu[bb, h0:h0 + l_ref.shape[0]]
            err_o = max(err_o, float(np.abs(og - o_ref).max()))
            fin = np.isfinite(l_ref)
            if fin.any():
                err_l = max(err_l, float((np.abs(lg[fin] - l_ref[fin]) / np.maximum(1.0, np.abs(l_ref[fin]))).max()))
        line["parity"] = {"max_abs_err_out": err_o, "max_rel_err_lse": err_l,
                          "rows": sum(r[2].shape[0] for r in rows), "tolerance": {"out_abs": 2e-3, "lse_rel": 1e-4},
                          "against": "oracle (fp64) on the cpu_baseline sample"}
        b1, s1, _, desc1 = oracle_sample(xs[0], budget_s=max(1.0, args.cpu_seconds / 4), nthreads=1)
        line["cpu_baseline"] = {"value": b / s / 1e9, "unit": "GB/s", "cores": t, "kind": "oracle",
                                "sample": desc, "seconds": s,
                                "single_thread": {"value": b1 / s1 / 1e9, "unit": "GB/s", "cores": 1,
                                                  "sample": desc1, "seconds": s1}}
    if world == 1 and not args.no_per_config and not args.paged and Q == 1 and not quant and w.name == HEADLINE:
        del wk, xs, calls, out, lse, ws
        torch.cuda.empty_cache()
        per = {}
        for name, kv in PER_CONFIG:
            key, entry = config_entry(args, WORKLOADS[name], kv, dev, stream, peak)
            per[key] = entry
            line["gpu_launches"] += args.steps
        line["per_config"] = per
        if fd.fd_device_status(stream) != 0:
            raise RuntimeError("device status after the per-config runs")
    if world == 1 and rank == 0:
        line["host_cost"] = host_cost(w)
    print(json.dumps(line), flush=True)
    return 0


def host_cost(w, calls=200):
    """Host microseconds per call of fd_decode / fd_decode_splits / fd_plan
    through the C ABI, timed by the C++ program fd_host_bench (no Python on
    the path), on this workload's shape; an empty kernel's launch beside them."""
    from decode_attention_07_b200 import build as lib_build
    exe = lib_build.HOST_BENCH
    if not os.path.exists(exe):
        return {"unavailable": "fd_host_bench is not built (python -c 'import __graft_entry__ as g; g.build()')"}
    r = subprocess.run([exe, str(w.B), str(w.Hq), str(w.Hkv), str(w.D), str(w.Lmax), str(calls)],
                       capture_output=True, text=True, timeout=300)
    if r.returncode != 0:
        return {"unavailable": f"fd_host_bench exited {r.returncode}: {r.stderr.strip()[-200:]}"}
    d = json.loads(r.stdout.strip().splitlines()[-1])
    d["how"] = "C++ through the C ABI, steady clock around CALLS back-to-back enqueues, tensor maps cached"
    return d


def run_cp(args, w, rank, world):
    """Context parallelism: one batch whose cache is sharded along its token
    positions over the `world` ranks. A step is the local split-kernel decode
    of this rank's range, the all-gather of the (out, lse) partials and their
    merge; total work is fixed as ranks are added (strong scaling)."""
    from decode_attention_07_b200 import context
    from decode_attention_07_b200.inputs import draw_seqlens
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    lo, hi = context.token_range(w.Lmax, rank, world)
    ws_ = w.with_(Lmax=hi - lo)
    lens = draw_seqlens(w, args.seed)                                     # the same batch on every rank
    local = np.clip(lens.astype(np.int64) - lo, 0, hi - lo).astype(np.int32)
    gq = torch.Generator(device=dev).manual_seed(args.seed)              # the same query on every rank
    q = (torch.randn((w.B, w.Hq, w.D), generator=gq, device=dev) * w.sigma_q).to(torch.bfloat16)
    xs = [make_inputs(ws_, args.seed + 1000 * c + rank, device=dev, seqlens=local) for c in range(2)]
    for x in xs:
        x.q = q
    n_copies = 2 if xs[0].kv_bytes() >= L2_BYTES else 1
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, ws_.Lmax)
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, ws_.Lmax, S)
    wsb = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=dev)
    part_o = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    part_l = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    all_o = torch.empty((world, w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    all_l = torch.empty((world, w.B, w.Hq), dtype=torch.float32, device=dev)
    out = torch.empty_like(part_o)
    lse = torch.empty_like(part_l)
    calls = [fd.prepare_decode(x.q, x.k, x.v, x.seqlens, x.scale, part_o, part_l, wsb, S, stream)
             for x in xs[:n_copies]]
    flush = None if n_copies == 2 else torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step(i):
        calls[i % n_copies]()
        if world > 1:
            torch.distributed.all_gather_into_tensor(all_o, part_o)
            torch.distributed.all_gather_into_tensor(all_l, part_l)
            fd.fd_merge_partials(all_o, all_l, out, lse, stream)
        else:
            fd.fd_merge_partials(part_o[None], part_l[None], out, lse, stream)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps if flush is not None else 1)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        if flush is None:
            ev[0][0].record(stream)
            for i in range(args.steps):
                step(i)
            ev[0][1].record(stream)
        else:
            for i in range(args.steps):
                flush.fill_(i & 255)
                ev[i][0].record(stream)
                step(i)
                ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ms_max = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
    status = fd.fd_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status}: {fd.fd_strerror(status)}")
    if rank != 0:
        return 0
    total_kv = int(np.clip(lens, 0, w.Lmax).astype(np.int64).sum()) * w.Hkv * w.D * 2 * 2
    gbs = total_kv * args.steps / (ms_max * 1e-3) / 1e9
    peak, peak_kind = peaks()
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_max / args.steps, "us_per_call": ms_max * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_dict(w, S, "inputs larger than L2: 2 shard copies rotated" if n_copies == 2
                                   else "L2 flushed before every timed step (256 MiB write outside the events)"),
                       parallelism=f"cp{world}", shard_tokens=hi - lo),
        "roofline": {"kernel": "whole step per rank (split kernel + all-gather + merge)", "bound": "hbm",
                     "achieved": gbs / world, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": gbs / world / peak, "traffic": None},
        "gpu_launches": args.steps * 2,
        "clocks": clocks.summary(),
        "e2e": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def launch_ranks(n: int, argv) -> int:
    """`--gpus N` outside torchrun: start N copies of this script, one per
    GPU, with RANK / LOCAL_RANK / WORLD_SIZE / MASTER_ADDR / MASTER_PORT set
    as torchrun would, and wait for all of them. Rank 0's stdout is ours;
    the others' is discarded (they print nothing). If one rank fails, the
    others are ended (by their own PIDs) and the first failure is returned."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__), *argv], env=env,
                                      stdout=None if r == 0 else subprocess.DEVNULL))
    rc = 0
    pending = list(procs)
    while pending:
        for pr in list(pending):
            code = pr.poll()
            if code is None:
                continue
            pending.remove(pr)
            if code != 0 and rc == 0:
                rc = code
                for other in pending:
                    other.terminate()
        time.sleep(0.05)
    return rc


def check_launch(world: int, rank: int) -> int:
    """`--check-launch`: the multi-rank plumbing alone, without a GPU
    workload. Every rank joins the process group (NCCL with GPUs, gloo
    without), the ranks count themselves with an all-reduce and gather their
    PIDs; rank 0 prints one JSON line."""
    t = torch.ones(1, dtype=torch.float64)
    pids = [os.getpid()]
    if world > 1:
        if torch.cuda.is_available():
            t = t.cuda()
        torch.distributed.all_reduce(t)
        pids = [None] * world
        torch.distributed.all_gather_object(pids, os.getpid())
    if rank == 0:
        print(json.dumps({"check_launch": True, "n_gpus": world, "ranks_joined": int(t.item()), "pids": pids,
                          "backend": torch.distributed.get_backend() if world > 1 else None}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fd", "reference"], default="fd")
    ap.add_argument("--config", choices=list(WORKLOADS), default=HEADLINE)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--paged", type=int, default=0, metavar="PAGE_SIZE",
                    help="read the caches from a shuffled page pool with this page size (fd_decode_paged)")
    ap.add_argument("--layout", choices=["HND", "NHD"], default="HND", help="page layout for --paged")
    ap.add_argument("--page-order", choices=["shuffled", "inorder"], default="shuffled",
                    help="--paged: pool pages in a shuffled order, or in sequence order (consecutive pages)")
    ap.add_argument("--cp", action="store_true",
                    help="context parallelism: shard the cache's tokens over the ranks (strong scaling)")
    ap.add_argument("--kv", choices=["bf16", "e4m3", "int8"], default="bf16",
                    help="key/value cache element type; e4m3 / int8 use fd_decode_quant with per-head scales")
    ap.add_argument("--q-len", type=int, default=1,
                    help="new tokens per sequence, each a query seeing the cache up to itself (fd_decode_multi)")
    ap.add_argument("--no-clock-window", action="store_true",
                    help="do not extend clock sampling past the timed region (for profiler runs)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="report the headline workload only (no per_config object)")
    ap.add_argument("--check-launch", action="store_true",
                    help="only start the ranks, join the process group and report them (no workload)")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" in os.environ:
        if int(os.environ["WORLD_SIZE"]) != args.gpus:
            ap.error(f"WORLD_SIZE={os.environ['WORLD_SIZE']} but --gpus {args.gpus}: launch one rank per GPU")
    elif args.gpus > 1:
        return launch_ranks(args.gpus, sys.argv[1:])
    if args.paged and args.q_len != 1:
        ap.error("--paged takes one query per sequence")
    if args.cp and (args.paged or args.kv != "bf16" or args.q_len != 1):
        ap.error("--cp shards a contiguous bf16 cache with one query per sequence")
    w = WORKLOADS[args.config]
    world = int(os.environ.get("WORLD_SIZE", 1))
    rank = int(os.environ.get("RANK", 0))
    if world > 1 and (args.impl == "fd" or args.check_launch):
        import datetime
        if torch.cuda.is_available():
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        elif args.check_launch:   # CPU-only check of the launcher
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            raise RuntimeError("the GPU arm needs CUDA devices")
    try:
        if args.check_launch:
            return check_launch(world, rank)
        if args.impl == "reference":
            return run_reference(args, w, rank, world)
        if args.cp:
            return run_cp(args, w, rank, world)
        return run_fd(args, w, rank, world)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
