"""Benchmark of the paired-count resident on B200.

Workload (default): the 512x512-scan, 192x192-pixel uint8 acquisition
(9.66 GB raw, counter-based synthetic Poisson counts: bright-field disk r=30
with lambda=3, lambda=0.01 outside), generated and encoded on the device.
One step is the query schedule of that workload through the C ABI:
bright-field and annular (40<=r<=90) masked sums at block_stride 1, 4 and 16,
then a 65-query drag (a full r=30 disk query followed by 64 one-pixel-shift
delta queries).  `value` is masked-sum queries per second over all ranks
with the resident already in HBM; `e2e` repeats the steps with every mask
copied in from pinned host memory and every image read back to pinned host
memory inside the timed region.

Each rank holds its own resident and runs the same schedule (independent
acquisitions, weak scaling, no data-path collective).

--impl reference times the CPU oracle (plain C, test infrastructure) on a
bounded sample of the same workload and reports the same metric.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import tempfile
import threading
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "masked_sum queries/s and raw-equivalent GB/s decoded at 512x512x192x192 vs HBM roofline"
UNIT = "queries/s"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def schedule(w: W.Workload):
    """[(label, mask uint8[P], stride, delta)] for one step."""
    q = []
    for k in w.strides:
        for name in ("bf", "adf"):
            q.append((f"{name}_k{k}", w.masks[name], k, False))
    if w.drag:
        q.append(("drag_full", w.drag[0], 1, False))
        for t in range(1, len(w.drag)):
            q.append(("drag_delta", w.drag[t], 1, True))
    return q


def stream_lengths(res, w):
    """Encoded extent of every stream, [B][P] (from the exported group tables)."""
    B, P = w.n_blocks, w.n_pixels
    lens = np.zeros((B, P), np.uint32)
    for b in range(B):
        g, _ = res.export_block(b)
        ends = np.stack([(g[:, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF for j in range(32)], axis=1)
        ends = ends.astype(np.int64)
        starts = np.concatenate([np.zeros((ends.shape[0], 1), np.int64), ends[:, :-1]], axis=1)
        lens[b] = (ends - starts).reshape(-1)[:P]
    return lens


PLAN_HEAVY, PLAN_LIGHT, PLAN_ITEM = 16, 1, 2     # the index plan's planner weights


def decompose(slots, roots, P, add, rem, pclass=None):
    """The plan's split of a query over the index layout: (items, residual pixels).
    add/rem: bool [P] pixels entering / leaving the image (a full query has no rem).
    Items are (level, id): a leaf whose every pixel enters (or every pixel leaves), or a
    root whose leaves all do so in the same direction.  In a full query with the pixel
    classes given, a leaf partly in the mask becomes an item plus its unmasked pixels
    (subtracted) when their decode weight plus PLAN_ITEM is below the masked pixels'
    (heavy pixels PLAN_HEAVY, light ones PLAN_LIGHT).  The residual pixels are decoded
    (added or subtracted); the first return holds the items."""
    real = slots < P
    px = np.where(real, slots, 0)
    a = np.where(real, add[px], True).all(axis=1)
    r = np.where(real, rem[px], True).all(axis=1) & rem.any()
    state = np.where(a, 1, np.where(r, 2, 0))
    if pclass is not None and not rem.any():
        wgt = np.where(pclass[px] != 0, PLAN_LIGHT, PLAN_HEAVY) * real
        inside = add[px] & real
        c_in = (wgt * inside).sum(axis=1)
        c_out = (wgt * (real & ~inside)).sum(axis=1)
        state = np.where((state == 0) & (PLAN_ITEM + c_out < c_in), 3, state)
    items, covered = [], np.zeros(slots.shape[0], bool)
    for i in range(len(roots) - 1):
        s = state[roots[i]:roots[i + 1]]
        if s[0] in (1, 2) and (s == s[0]).all():
            items.append((1, i))
            covered[roots[i]:roots[i + 1]] = True
        else:
            for l in range(roots[i], roots[i + 1]):
                if state[l] > 0:
                    items.append((0, l))
                    covered[l] = True
    cov = np.zeros(P, bool)
    cov[slots[covered][slots[covered] < P]] = True
    resid = (add | rem) & ~cov
    # leaves taken as item minus their unmasked pixels
    comp = np.zeros(P, bool)
    for l in np.nonzero(state == 3)[0]:
        q = slots[l][slots[l] < P]
        comp[q[~add[q]]] = True
    return items, resid | comp


def algorithmic_bytes(lens, w, sched, out_bits, idx=None):
    """Per query: encoded bytes of the decoded streams in the touched blocks + 2 B offset per stream +
    4 B group base per touched group + the image written + the 4 B list entries; with the index
    (idx = (slots, roots, bytes [B][L+R])), the residual pixels' streams plus the stored sums of
    the index items in the touched blocks and 4 B per item."""
    out = []
    prev = None
    for label, m, k, delta in sched:
        sel = m.astype(bool)
        as_delta = delta and prev is not None        # a delta with no baseline runs as a full query
        if as_delta:
            add, rem = sel & ~prev, ~sel & prev
        else:
            add, rem = sel, np.zeros_like(sel)
        prev = sel
        rows = list(range(0, w.n_blocks, k))
        items = []
        resid = add | rem
        if idx is not None and not as_delta:           # deltas take the per-pixel plan
            slots, roots, gbytes, pclass = idx
            items, resid = decompose(slots, roots, w.n_pixels, add, rem, pclass)
        pix = np.nonzero(resid)[0]
        enc = int(lens[rows][:, pix].sum(dtype=np.int64))
        groups = len(np.unique(pix // 32)) * len(rows)
        isum = 0
        if items:
            L = slots.shape[0]
            gid = np.array([g if lvl == 0 else L + g for lvl, g in items])
            isum = int(gbytes[rows][:, gid].sum(dtype=np.int64))
        img = len(rows) * 512 * out_bits // 8
        listed = np.count_nonzero(add | rem)
        raw = listed * 512 * len(rows) * (w.dtype_bits // 8)
        out.append(dict(label=label, enc=enc + isum, streams=pix.size * len(rows), items=len(items),
                        bytes=enc + 2 * pix.size * len(rows) + 4 * groups + isum + 4 * len(items) + img + 4 * pix.size,
                        raw=raw))
    return out


class Clocks:
    """SM clock and clock-event reasons sampled during the timed region: through NVML (the
    library nvidia-smi reads) every 10 ms on a background thread, else by nvidia-smi every
    200 ms into a temporary file.  Reading only: no setting of the GPU is changed."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, uuid: str | None = None, period: float = 0.010):
        self.index, self.uuid, self.period = index, uuid, period
        self.samples = []            # (sm MHz, max sm MHz, reason names)
        self.source = None
        self.proc = self.thread = None
        self.path = os.path.join(tempfile.gettempdir(), f"qem_clocks_{os.getpid()}_{index}.csv")

    def _start_nvml(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            h = None
            if self.uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid if self.uuid.startswith("GPU-")
                                                         else "GPU-" + self.uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            get_reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                           or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)

            def sample():
                bits = int(get_reasons(h))
                return (float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)), mx,
                        tuple(n for n, b in self.REASONS if bits & b))

            sample()                 # fails here if the device cannot be read
        except Exception:
            pynvml.nvmlShutdown()
            raise
        self._nvml = pynvml
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(sample())
                except Exception:
                    pass
                self._stop.wait(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        self.source = "nvml"

    def __enter__(self):
        try:
            self._start_nvml()
        except Exception:
            try:
                self.f = open(self.path, "w")
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                              "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                             stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi"
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()
            names = [n for n, _ in self.REASONS]
            for line in open(self.path):
                r = [x.strip() for x in line.split(",")]
                if len(r) < 9 or not r[1].replace(".", "").isdigit() or not r[2].replace(".", "").isdigit():
                    continue
                self.samples.append((float(r[1]), float(r[2]),
                                     tuple(names[i] for i in range(4) if r[5 + i].lower() == "active")))
            try:
                os.remove(self.path)
            except OSError:
                pass

    def summary(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        return {"sm_mhz": statistics.median(x[0] for x in self.samples),
                "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted({n for x in self.samples for n in x[2]}),
                "samples": len(self.samples), "source": self.source}


def build_resident(w, dev, torch, V, stream=None):
    """Generate the workload's counts on the device and encode them (chunked for large ones)."""
    spec = w.counter
    pc = torch.from_numpy(spec.pixel_class.astype(np.int32)).to(dev)
    cd = torch.from_numpy(spec.class_desc.astype(np.int32)).to(dev)
    th = torch.from_numpy(spec.thresholds.view(np.int64)).to(dev)
    dt = torch.uint8 if w.dtype_bits == 8 else torch.uint16
    raw_bytes = w.raw_bytes
    chunk_blocks = w.n_blocks if raw_bytes <= (24 << 30) else 1
    buf = torch.empty((chunk_blocks * 512, w.n_pixels), dtype=dt, device=dev)
    res = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), w.dtype_bits)
    t_enc = 0.0
    for b0 in range(0, w.n_blocks, chunk_blocks):
        nb = min(chunk_blocks, w.n_blocks - b0)
        V.generate_counts(buf, w.dtype_bits, spec.seed, b0 * 512, nb * 512, w.n_pixels, pc, cd, th)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        res.append(buf, nb)
        e1.record()
        torch.cuda.synchronize()
        t_enc += e0.elapsed_time(e1) / 1e3
    return res, buf, t_enc


def oracle_sample(w, n_blocks=4):
    """The oracle's sample of a workload: n_blocks blocks spread evenly over the
    acquisition (block i * B / n), regenerated on the host and encoded by the oracle.
    Returns (blocks, Encoded, encode seconds on all cores, encode seconds on one core
    for the first block)."""
    import oracle as O

    blocks = sorted({int(i * w.n_blocks // n_blocks) for i in range(n_blocks)})
    counts = [w.block_counts(b) for b in blocks]
    threads = os.cpu_count() or 1
    enc = O.Encoded(w.n_pixels, w.dtype_bits, [None] * len(blocks), [None] * len(blocks))

    def job(i):
        enc.groups[i], enc.payloads[i] = O.encode_block(counts[i], w.dtype_bits)

    from concurrent.futures import ThreadPoolExecutor

    t0 = time.perf_counter()
    with ThreadPoolExecutor(min(threads, len(blocks))) as ex:
        list(ex.map(job, range(len(blocks))))
    t_all = time.perf_counter() - t0
    t1 = time.perf_counter()
    O.encode_block(counts[0], w.dtype_bits)
    t_one = time.perf_counter() - t1
    return blocks, enc, t_all, t_one


def oracle_step(w, enc, n_sample, sched, threads):
    """One step of the schedule by the oracle over the sampled blocks: every query runs
    over them (a delta from the previous query's image) and its time per block is scaled
    to the ceil(B/k) blocks the query touches in the full acquisition.  Returns the scaled
    step time in seconds and the raw bytes the step's queries cover."""
    import oracle as O

    prev = img = None
    scaled = 0.0
    raw = 0
    w_bytes = w.dtype_bits // 8
    for label, m, k, delta in sched:
        t0 = time.perf_counter()
        if delta and prev is not None:
            img = O.resident_delta(enc, img, prev, m, None, 1, threads=threads)
        else:
            img = O.resident_masked_sum(enc, m, None, 1, threads=threads)
        scaled += (time.perf_counter() - t0) / n_sample * math.ceil(w.n_blocks / k)
        raw += int((m != 0).sum()) * 512 * math.ceil(w.n_blocks / k) * w_bytes
        prev = m
    return scaled, raw


SAMPLE_RULE = ("every query of the step runs over {n} blocks spread evenly over the acquisition ({blocks} of {B}, "
               "regenerated on the host and encoded by the oracle) and its time per block is scaled to the "
               "ceil(B/k) blocks it touches; encode time of the same blocks scaled to all B blocks")


def cpu_baseline(w, min_seconds=10.0):
    """The oracle as it stands, on the host cores, with the reference arm's sampling rule:
    queries/s of the step's schedule, raw-equivalent GB/s of those queries, encode GB/s,
    each also on one core."""
    blocks, enc, t_enc, t_enc_one = oracle_sample(w)
    sched = schedule(w)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    steps = scaled = raw = 0
    while True:
        s_, r_ = oracle_step(w, enc, len(blocks), sched, threads)
        steps += 1
        scaled += s_
        raw = r_
        if time.perf_counter() - t0 > min_seconds:
            break
    wall = time.perf_counter() - t0
    step_s = scaled / steps
    one_s, _ = oracle_step(w, enc, len(blocks), sched, 1)
    block_raw = 512 * w.n_pixels * (w.dtype_bits // 8)
    return {"value": len(sched) / step_s, "unit": UNIT, "cores": threads, "kind": "oracle", "cpu": cpu_model(),
            "raw_equiv_gbs": raw / step_s / 1e9,
            "encode_gbs": block_raw * len(blocks) / t_enc / 1e9,
            "single_core": {"value": len(sched) / one_s, "raw_equiv_gbs": raw / one_s / 1e9,
                            "encode_gbs": block_raw / t_enc_one / 1e9},
            "sample": SAMPLE_RULE.format(n=len(blocks), blocks=blocks, B=w.n_blocks)
                      + f"; {steps} steps in {wall:.1f} s of CPU time on {threads} threads"}


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo where there is one)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or platform.machine()


def kernel_source_hash():
    """SHA-256 of the device code (kernels.cu and the header it shares with the host
    side) with comments, trailing blanks and empty lines removed: a committed ncu
    capture stays tied to the code it measured, whatever happens to the comments."""
    import hashlib
    import re

    text = ""
    for name in ("kernels.cu", "qem_internal.h"):
        with open(os.path.join(ROOT, "virtual_imaging_b200", "csrc", name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        text += "\n".join(line.rstrip() for line in src.splitlines() if line.strip()) + "\n"
    return hashlib.sha256(text.encode()).hexdigest()


def workload_config(w, nq, world):
    """The workload part of the bench line's config, the same for both arms."""
    return {"workload": f"{w.name}: scan {w.scan_rows}x{w.scan_cols}, detector {w.det_rows}x{w.det_cols}, "
                        f"uint{w.dtype_bits}, counter-based Poisson"
                        + (" (BF r=30 lambda=3, outside 0.01)" if w.name == "c4" else ""),
            "queries_per_step": nq,
            "schedule": "bf/adf at block_stride " + ",".join(str(k) for k in w.strides)
                        + (f" + drag: 1 full + {len(w.drag) - 1} deltas" if w.drag else ""),
            "parallelism": f"{world} independent residents (one per GPU)"}


def run_reference(args, rank, world):
    """The oracle timed on the host cores on a bounded sample of the same workload and
    schedule (the sampling rule of SAMPLE_RULE, the same as the cpu_baseline leg)."""
    if rank != 0:
        return
    w = W.workload(args.config)
    blocks, enc, t_enc, _ = oracle_sample(w)
    sched = schedule(w)
    threads = os.cpu_count() or 1
    for _ in range(args.warmup):
        oracle_step(w, enc, len(blocks), sched, threads)
    t0 = time.perf_counter()
    tot = 0.0
    raw = 0
    for _ in range(args.steps):
        s_, raw = oracle_step(w, enc, len(blocks), sched, threads)
        tot += s_
    wall = time.perf_counter() - t0
    step_full = tot / args.steps
    value = len(sched) / step_full
    sample = (SAMPLE_RULE.format(n=len(blocks), blocks=blocks, B=w.n_blocks)
              + f"; {args.steps} timed steps took {wall:.1f} s of CPU time; ms_per_step is the scaled "
                f"full-acquisition step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_full * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8" if w.dtype_bits == 8 else "u16",
            "data": "synthetic",
            "config": workload_config(w, len(sched), world),
            "raw_equiv_gbs": raw / step_full / 1e9,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "cpu": cpu_model(),
                             "encode_gbs": 512 * w.n_pixels * (w.dtype_bits // 8) * len(blocks) / t_enc / 1e9,
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_encode(dev, torch, V):
    """Bounded encode case for ncu: the default geometry (192x192 uint8, same counts) but 16
    blocks (302 MB of raw counts, above the 126 MB L2), generated and encoded once."""
    w = W.workload("c4")
    w.scan_rows = 16
    res, buf, t_enc = build_resident(w, dev, torch, V)
    print(json.dumps({"encode_s": t_enc, "blocks": w.n_blocks}), flush=True)
    res.free()


def run_profile_case(dev, torch, V, config="c4"):
    """Small bounded case for ncu: build the resident of `config` (the default workload unless
    --config names another), then a few bright-field / annular block_stride-1 queries (the
    kernels ncu captures are the k_decode_reduce launches)."""
    w = W.workload(config)
    res, buf, t_enc = build_resident(w, dev, torch, V)
    del buf
    torch.cuda.empty_cache()
    res.build_index((w.det_rows // 2, w.det_cols // 2))
    out = torch.empty((w.n_blocks, 512), dtype=V.out_dtype(res.info()["out_bits_auto"]), device=dev)
    bf = torch.from_numpy(w.masks["bf"]).to(dev)
    adf = torch.from_numpy(w.masks["adf"]).to(dev)
    res.profile(True)
    for m in (bf, adf, bf, adf):
        res.masked_sum(m, out=out)
    # a short drag: one full query then delta queries (launches 5.. are deltas)
    for t, d in enumerate(w.drag[:6]):
        md = torch.from_numpy(d).to(dev)
        (res.masked_sum_delta if t else res.masked_sum)(md, out=out)
    # the schedule's other strides (launches 10..13: bf k4, adf k4, bf k16, adf k16)
    for k in (4, 16):
        for m in (bf, adf):
            res.masked_sum(m, block_stride=k, out=out[: -(-w.n_blocks // k)])
    # a two-block decode and one frame (k_decode_blocks, k_decode_range)
    frames = torch.empty((2 * 512, w.n_pixels), dtype=torch.uint8 if w.dtype_bits == 8 else torch.uint16, device=dev)
    res.decode_blocks(0, 2, out=frames)
    res.decode_range(777, 1)
    # launch 14: bright field with the index dropped (every disk pixel decoded pair by pair)
    res.drop_index()
    res.masked_sum(bf, out=out)
    # one centre-of-mass moment query over the bright field (k_moments)
    rr, cc = np.divmod(np.arange(w.n_pixels), w.det_cols)
    wts = torch.from_numpy(np.stack([rr - w.det_rows // 2, cc - w.det_cols // 2]).astype(np.int32)).to(dev)
    res.masked_moments(bf, wts)
    p = res.profile_read()
    print(json.dumps({"encode_s": t_enc, "kernels": p}), flush=True)
    res.free()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="c4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--saved-form", default=None, metavar="PATH",
                    help="also time writing the resident's saved form to PATH and reopening it")
    ap.add_argument("--no-index", action="store_true",
                    help="query without the interaction index (every masked pixel decoded)")
    ap.add_argument("--profile", action="store_true", help="bounded case for ncu captures")
    ap.add_argument("--profile-encode", action="store_true", help="bounded encode case for ncu captures")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import virtual_imaging_b200 as V
    from virtual_imaging_b200.series import max_over_ranks

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    if args.profile:
        run_profile_case(dev, torch, V, args.config)
        return
    if args.profile_encode:
        run_profile_encode(dev, torch, V)
        return
    w = W.workload(args.config)
    res, buf, _ = build_resident(w, dev, torch, V)
    # interaction index about the detector centre (the centre of the bright-field
    # disk and of the annulus); built by decoding every stream once
    index = None
    if not args.no_index:
        torch.cuda.synchronize()
        i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        i0.record()
        res.build_index((w.det_rows // 2, w.det_cols // 2))
        i1.record()
        torch.cuda.synchronize()
        ii = res.info()
        index = {"s": i0.elapsed_time(i1) / 1e3, "bytes": ii["index_bytes"], "leaves": ii["index_leaves"],
                 "roots": ii["index_roots"], "centre": [w.det_rows // 2, w.det_cols // 2]}
    # a second, warm encode of the same counts for the encode figure (chunked workloads keep the first)
    enc_s = None
    enc_prof = None
    if buf.shape[0] == w.n_scans:
        res2 = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), w.dtype_bits)
        res2.profile(True)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        res2.append(buf, w.n_blocks)
        e1.record()
        torch.cuda.synchronize()
        enc_s = e0.elapsed_time(e1) / 1e3
        enc_prof = {k: round(v[1], 3) for k, v in res2.profile_read().items() if v[0]}
        res2.free()
    # block decode leg (16 blocks)
    nd = min(16, w.n_blocks)
    frames = torch.empty((nd * 512, w.n_pixels), dtype=buf.dtype, device=dev)
    res.decode_blocks(0, nd, out=frames)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record()
    res.decode_blocks(0, nd, out=frames, wait=False)
    d1.record()
    torch.cuda.synchronize()
    dec_s = d0.elapsed_time(d1) / 1e3
    res.finish()
    ok_frames = bool(torch.equal(frames, buf[: nd * 512])) if buf.shape[0] >= nd * 512 else None
    del frames
    del buf
    torch.cuda.empty_cache()

    info = res.info()
    out_bits = info["out_bits_auto"]
    sched = schedule(w)
    masks = [torch.from_numpy(m.astype(np.uint8)).to(dev) for (_, m, _, _) in sched]
    outs = {}
    for label, m, k, d in sched:
        rows = -(-w.n_blocks // k)
        outs.setdefault(k, torch.empty((rows, 512), dtype=V.out_dtype(out_bits), device=dev))

    def step(ms=masks):
        for (label, m, k, delta), md in zip(sched, ms):
            fn = res.masked_sum_delta if delta else res.masked_sum
            fn(md, block_stride=k, out=outs[k], wait=False)

    # the first query after the build, timed alone: the cold figure
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    c0.record()
    res.masked_sum(masks[0], block_stride=sched[0][2], out=outs[sched[0][2]], wait=False)
    c1.record()
    torch.cuda.synchronize()
    cold = (sched[0][0], c0.elapsed_time(c1))
    for _ in range(args.warmup):
        step()
    res.finish()
    # one more untimed step with the library's own counters: the streams its
    # decode listed, to check the count behind the algorithmic bytes
    try:
        res.counters()
        step()
        res.finish()
        streams_kernel = int(res.counters()[1])
    except V.QemError:
        streams_kernel = None
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # timed region of `value`: the queries alone (per-kernel events would sit
    # between the plan and decode launches of every query and cost ~0.8 ms per
    # step, so they are taken in the second timed pass below)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        dev_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        dev_uuid = None
    with Clocks(local, dev_uuid) as clk:
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    res.finish()
    t = e0.elapsed_time(e1) / 1e3
    t = max_over_ranks(t, device=dev)

    # second timed pass of the same schedule with CUDA events around every
    # kernel launch (on the launching stream): per-kernel durations for the
    # roofline and the breakdown
    res.profile(True)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    for _ in range(args.steps):
        step()
    p1.record()
    torch.cuda.synchronize()
    res.finish()
    t_prof = p0.elapsed_time(p1) / 1e3
    prof = res.profile_read()
    res.profile(False)

    # end to end: each step's masks go up from pinned host memory in one copy, every
    # query writes its own image, and each image comes back to pinned host memory as
    # soon as its query has finished, overlapping the queries after it (one 71 MB
    # read-back per step at the end of the step slowed the next step's queries by
    # ~15 %; spread over the step it costs ~2 %).  Uploads and read-backs run on two
    # copy streams of their own (opposite directions), so the next step's upload
    # does not queue behind this step's read-backs.  Two sets of device buffers are
    # used in turn; a step waits until the read-backs of the set it is about to
    # overwrite have finished.
    P = w.n_pixels
    nq_ = len(sched)
    host_masks = torch.from_numpy(np.stack([m.astype(np.uint8) for (_, m, _, _) in sched])).pin_memory()
    img_elems = [(-(-w.n_blocks // k)) * 512 for (_, _, k, _) in sched]
    img_off = np.concatenate([[0], np.cumsum(img_elems)])
    odt = V.out_dtype(out_bits)
    sets = []
    for _ in range(2):
        dmask = torch.empty((nq_, P), dtype=torch.uint8, device=dev)
        dimg = torch.empty(int(img_off[-1]), dtype=odt, device=dev)
        himg = torch.empty(int(img_off[-1]), dtype=odt).pin_memory()
        views = [dimg[int(img_off[i]):int(img_off[i + 1])].view(-1, 512) for i in range(nq_)]
        sets.append({"mask": dmask, "img": dimg, "host": himg, "views": views, "free": None})
    h2d = host_masks.numel()
    d2h = int(img_off[-1]) * sets[0]["img"].element_size()
    comp_st = torch.cuda.current_stream(dev)
    up_st = torch.cuda.Stream(device=dev)
    down_st = torch.cuda.Stream(device=dev)
    turn = [0]

    def e2e_step():
        S = sets[turn[0]]
        turn[0] ^= 1
        if S["free"] is not None:
            # the read-backs of this set two steps ago (the last of them follows that
            # step's last query, the last reader of its masks) have finished
            up_st.wait_event(S["free"])
            comp_st.wait_event(S["free"])
        with torch.cuda.stream(up_st):
            S["mask"].copy_(host_masks, non_blocking=True)
        up = torch.cuda.Event()
        up.record(up_st)
        comp_st.wait_event(up)
        for i, (label, m, k, delta) in enumerate(sched):
            fn = res.masked_sum_delta if delta else res.masked_sum
            fn(S["mask"][i], block_stride=k, out=S["views"][i], wait=False, stream=comp_st)
            done = torch.cuda.Event()
            done.record(comp_st)
            down_st.wait_event(done)
            with torch.cuda.stream(down_st):
                S["host"][int(img_off[i]):int(img_off[i + 1])].copy_(S["img"][int(img_off[i]):int(img_off[i + 1])],
                                                                     non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(down_st)
        S["free"] = ev

    e2e_step()
    res.finish()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        e2e_step()
    comp_st.wait_stream(down_st)
    f1.record()
    torch.cuda.synchronize()
    res.finish()
    te = f0.elapsed_time(f1) / 1e3
    te = max_over_ranks(te, device=dev)
    # the read-back images are the queries' results: the last step's first image
    # against a fresh query of the same mask
    last = sets[turn[0] ^ 1]
    lbl0, m0_, k0_, _ = sched[0]
    ref0 = res.masked_sum(torch.from_numpy(m0_.astype(np.uint8)).to(dev), block_stride=k0_,
                          out_bits=out_bits).cpu()
    e2e_exact = bool(torch.equal(last["host"][: int(img_off[1])].view(-1, 512), ref0))

    # fused moments (centre-of-mass numerators and denominator) over the bright-field
    # disk and the annulus, stride 1: every masked pixel decoded, 10 back to back
    rr, cc = np.divmod(np.arange(w.n_pixels), w.det_cols)
    wts = torch.from_numpy(np.stack([rr - w.det_rows // 2, cc - w.det_cols // 2]).astype(np.int32)).to(dev)
    mom_out = torch.empty((3, w.n_blocks, 512), dtype=torch.int64, device=dev)
    mom = {}
    for name in ("bf", "adf"):
        md = torch.from_numpy(w.masks[name].astype(np.uint8)).to(dev)
        res.masked_moments(md, wts, out=mom_out)
        torch.cuda.synchronize()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record()
        for _ in range(10):
            res.masked_moments(md, wts, out=mom_out, wait=False)
        m1.record()
        torch.cuda.synchronize()
        res.finish()
        mom[f"{name}_k1_ms"] = m0.elapsed_time(m1) / 10

    saved = None
    if args.saved_form:
        torch.cuda.synchronize()
        s0 = time.perf_counter()
        res.save(args.saved_form)
        s1 = time.perf_counter()
        back = V.Resident.load(args.saved_form)
        torch.cuda.synchronize()
        s2 = time.perf_counter()
        fbytes = os.path.getsize(args.saved_form)
        same = all(np.array_equal(a, b) for b0 in (0, w.n_blocks - 1)
                   for a, b in zip(res.export_block(b0), back.export_block(b0)))
        back.free()
        os.remove(args.saved_form)
        saved = {"file_bytes": fbytes, "save_s": s1 - s0, "load_s": s2 - s1, "blocks_checked_equal": same}

    # per-query breakdown (separate, untimed for `value`)
    lens = stream_lengths(res, w)
    idx = None
    if index is not None:
        slots, roots = res.index_layout()
        codes = res.index_desc() >> 30
        gbytes = np.where(codes > 0, 512 << np.maximum(codes.astype(np.int64) - 1, 0), 0)
        idx = (slots, roots, gbytes, res.pixel_classes())
    ab = algorithmic_bytes(lens, w, sched, out_bits, idx)
    # per query: the median of 20 warm passes over the schedule, each query timed
    # alone (events around the call, synchronised after it)
    per_query = {}
    for _ in range(20):
        for (label, m, k, delta), md, a in zip(sched, masks, ab):
            q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fn = res.masked_sum_delta if delta else res.masked_sum
            q0.record()
            fn(md, block_stride=k, out=outs[k], wait=False)
            q1.record()
            torch.cuda.synchronize()
            d = per_query.setdefault(label, {"ms": [], "enc_bytes": a["enc"], "raw_bytes": a["raw"]})
            d["ms"].append(q0.elapsed_time(q1))
    res.finish()
    for label, d in per_query.items():
        d["runs"] = len(d["ms"])
        d["ms"] = statistics.median(d["ms"])
        if label == cold[0]:
            d["cold_ms"] = cold[1]
        d["raw_equiv_gbs"] = d["raw_bytes"] / (d["ms"] / 1e3) / 1e9
        d["enc_gbs"] = d["enc_bytes"] / (d["ms"] / 1e3) / 1e9

    hbm, peak_kind = peaks()

    # single diffraction frames: one-scan range decodes at 20 scans spread over the
    # acquisition, each timed alone; the first is checked against a block decode
    odt_counts = torch.uint8 if w.dtype_bits == 8 else torch.uint16
    fr = torch.empty((1, w.n_pixels), dtype=odt_counts, device=dev)
    f_scans = [int(x) for x in np.linspace(0, w.n_scans - 1, 20)]
    res.decode_range(f_scans[0], 1, out=fr)
    f_exact = bool(torch.equal(fr[0], res.decode_blocks(f_scans[0] // 512, 1)[f_scans[0] % 512]))
    f_ms = []
    for sc in f_scans:
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record()
        res.decode_range(sc, 1, out=fr, wait=False)
        q1.record()
        torch.cuda.synchronize()
        f_ms.append(q0.elapsed_time(q1))
    res.finish()
    frame = {"ms": statistics.median(f_ms), "ms_max": max(f_ms), "runs": len(f_ms), "exact": f_exact,
             "gcounts_per_s": w.n_pixels / (statistics.median(f_ms) / 1e3) / 1e9}

    # dense dark field (every pixel outside the bright-field disk) three ways: the
    # cached total minus the complement (qem_masked_sum_complement), the interaction
    # index, and (below, without the index) the plain decode of every masked pixel
    df_m = torch.from_numpy((1 - w.masks["bf"]).astype(np.uint8)).to(dev)
    o_df = torch.empty((w.n_blocks, 512), dtype=V.out_dtype(out_bits), device=dev)
    torch.cuda.synchronize()
    tb0 = time.perf_counter()
    res.masked_sum_complement(df_m, out=o_df)
    t_total_build = time.perf_counter() - tb0

    def med_ms(fn, n=20):
        xs = []
        for _ in range(n):
            q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            q0.record()
            fn()
            q1.record()
            torch.cuda.synchronize()
            xs.append(q0.elapsed_time(q1))
        res.finish()
        return statistics.median(xs)

    df_comp = med_ms(lambda: res.masked_sum_complement(df_m, out=o_df, wait=False))
    img_comp = o_df.clone()
    df_idx = med_ms(lambda: res.masked_sum(df_m, out=o_df, wait=False))
    dense_df = {"pixels": int(df_m.sum().item()), "complement_ms": df_comp,
                "index_ms": df_idx if index is not None else None, "total_build_s": t_total_build,
                "exact_vs_index": bool(torch.equal(img_comp, o_df))}

    # decode only: the same schedule with the interaction index dropped, so every
    # masked pixel of every query is decoded (timed without and with per-kernel events,
    # as `value` and the roofline are), and bf/adf k=1 alone (median of 20)
    decode_only = None
    if index is not None:
        res.drop_index()
        step()
        res.finish()
        torch.cuda.synchronize()
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0.record()
        for _ in range(args.steps):
            step()
        n1.record()
        torch.cuda.synchronize()
        res.finish()
        t_ni = n0.elapsed_time(n1) / 1e3
        res.profile(True)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        res.finish()
        prof_ni = res.profile_read()
        res.profile(False)
        ab_ni = algorithmic_bytes(lens, w, sched, out_bits, None)
        bytes_ni = sum(a["bytes"] for a in ab_ni)
        n_dni, ms_dni = prof_ni["decode_reduce"]
        q_ni = {}
        for (label, m, k, delta), md, a in zip(sched, masks, ab_ni):
            if label not in ("bf_k1", "adf_k1"):
                continue
            qs = []
            for _ in range(20):
                q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                q0.record()
                res.masked_sum(md, block_stride=k, out=outs[k], wait=False)
                q1.record()
                torch.cuda.synchronize()
                qs.append(q0.elapsed_time(q1))
            res.finish()
            ms = statistics.median(qs)
            q_ni[label] = {"ms": round(ms, 4), "runs": len(qs), "enc_gbs": round(a["enc"] / (ms / 1e3) / 1e9, 1),
                           "hbm_frac_enc": round(a["enc"] / (ms / 1e3) / 1e9 / hbm, 4),
                           "raw_equiv_gbs": round(a["raw"] / (ms / 1e3) / 1e9, 1)}
        dense_df["plain_ms"] = med_ms(lambda: res.masked_sum(df_m, out=o_df, wait=False))
        ach_ni = bytes_ni * args.steps / (ms_dni / 1e3) / 1e9 if ms_dni > 0 else None
        decode_only = {"value": nq_ * args.steps / t_ni, "unit": UNIT, "ms_per_step": t_ni / args.steps * 1e3,
                       "queries": q_ni,
                       "roofline": {"achieved": ach_ni, "peak": hbm, "unit": "GB/s",
                                    "frac": ach_ni / hbm if ach_ni else None, "kernel": "k_decode_reduce",
                                    "avg_launch_ms": ms_dni / max(1, n_dni),
                                    "algorithmic_bytes_per_launch": bytes_ni * args.steps / max(1, n_dni)},
                       "note": "interaction index dropped: every masked pixel of every query decoded"}

    # DRAM traffic per decode launch from a committed ncu capture, if it was taken on
    # this exact kernel source (else null)
    traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "k_decode_reduce_c4_traffic.json")) as f:
            tj = json.load(f)
        if args.config == "c4" and tj.get("kernel_source_hash") == kernel_source_hash():
            traffic = tj["schedule_bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        traffic = None
    n_dec, ms_dec = prof["decode_reduce"]
    bytes_step = sum(a["bytes"] for a in ab)
    raw_step = sum(a["raw"] for a in ab)
    achieved = bytes_step * args.steps / (ms_dec / 1e3) / 1e9 if ms_dec > 0 else None
    launches = sum(prof[k][0] for k in ("plan", "decode_reduce", "finalize"))
    clocks = clk.summary()

    nq = len(sched)
    line = {
        "metric": METRIC, "value": world * nq * args.steps / t, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8" if w.dtype_bits == 8 else "u16", "data": "synthetic",
        "config": {**workload_config(w, nq, world),
                   "l2": (f"no flush between steps; each step reads {bytes_step / 1e9:.2f} GB of encoded streams, "
                          f"offsets, index sums and images ({'above' if bytes_step > 126e6 else 'below'} the 126 MB L2), but single launches read "
                          f"{min(a['bytes'] for a in ab) / 1e6:.1f}-{max(a['bytes'] for a in ab) / 1e6:.1f} MB "
                          f"(below it) and consecutive queries share streams (bf at stride 4 and 16 reads a "
                          f"subset of bf at stride 1; a drag delta's leaving pixels were read by the previous "
                          f"query), so per-query figures are partly served from L2"),
                   "launch_bytes_mb": {lbl: round(a["bytes"] / 1e6, 2) for (lbl, _, _, _), a in zip(sched, ab)},
                   "resident_bytes": info["payload_bytes"] + info["group_bytes"], "raw_bytes": w.raw_bytes},
        "raw_equiv_gbs": world * raw_step * args.steps / t / 1e9,
        "e2e": {"value": world * nq * args.steps / te, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "images_checked": e2e_exact},
        "gpu_launches": int(launches),
        "accounting": {"streams_per_step_decoded": streams_kernel,
                       "streams_per_step_counted": int(sum(a["streams"] for a in ab))},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": (achieved / hbm) if achieved else None, "traffic": traffic,
                     "kernel": "k_decode_reduce", "peak_kind": peak_kind,
                     "avg_launch_ms": ms_dec / max(1, n_dec), "launches": n_dec,
                     "algorithmic_bytes_per_launch": bytes_step * args.steps / max(1, n_dec)},
        "queries": {k: {"ms": round(v["ms"], 4), "runs": v["runs"], "raw_equiv_gbs": round(v["raw_equiv_gbs"], 1),
                        "enc_gbs": round(v["enc_gbs"], 1), "hbm_frac_enc": round(v["enc_gbs"] / hbm, 4),
                        **({"cold_ms": round(v["cold_ms"], 4)} if "cold_ms" in v else {})}
                    for k, v in per_query.items()},
        "kernels_ms_per_step": {k: v[1] / args.steps for k, v in prof.items() if v[0]},
        "profiled_pass_ms_per_step": t_prof * 1e3 / args.steps,
        # encode: wall time of one qem_encode_append of the whole acquisition into a
        # fresh resident (arena and scratch allocation included), and its kernels alone
        "encode": {"gbs_raw": (w.raw_bytes / enc_s / 1e9) if enc_s else None, "s": enc_s, "kernels_ms": enc_prof,
                   "kernel_gbs_raw": (w.raw_bytes / (sum(enc_prof.values()) / 1e3) / 1e9) if enc_prof else None,
                   "hbm_frac": ((w.raw_bytes + info["payload_bytes"] + info["group_bytes"]) / enc_s / 1e9 / hbm)
                   if enc_s else None},
        "index": index,
        "saved_form": saved,
        "moments": mom,
        "decode_blocks": {"blocks": nd, "s": dec_s, "gcounts_per_s": nd * 512 * w.n_pixels / dec_s / 1e9,
                          "exact": ok_frames},
        "frame": frame,
        "dense_df": dense_df,
        "decode_only": decode_only,
        "resident": {"payload_bytes": info["payload_bytes"], "forms": info["form_count"],
                     "bits_per_count": 8 * info["payload_bytes"] / (w.n_scans * w.n_pixels)},
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    res.free()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
