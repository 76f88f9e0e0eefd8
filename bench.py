"""Benchmark of the MXFP4 block quantizer hot path on B200.

One step = one pass of the whole hot path over the sweep workload
(8192 x 28672 bf16, N(0,1) with 0.1% outliers x100, seed 5 + rank):
  rows RNE quantize, columns SR quantize, fused double quantization,
  dequantize of the row layout, Hadamard-rotate + rows SR quantize,
plus one oscillation-tracker step (with its synthetic update) on the
tracker workload (4096 x 4096 fp32 master weight).
Metric: GB/s of algorithmic bytes in+out (whole job), with % of the measured
HBM peak per kernel. Inputs are larger than L2 (470 MB and 268 MB against a
126 MB L2), so no flush is needed between steps.

--impl reference times the CPU oracle on a bounded sample of the same
workload (one 32-row band per op); it is the reported baseline.
Multi-GPU (torchrun): every rank runs the same step on its own data
(weak scaling, no collective on the data path); the timed region is the max
over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SWEEP = (8192, 28672)
OSC = (4096, 4096)
SEED = 5

# Algorithmic bytes per element (in + out), per op.
BYTES_PER_ELEM = {
    "quant_rows_rne": 2 + 0.5 + 1 / 32,
    "quant_cols_sr": 2 + 0.5 + 1 / 32,
    "double_quant": 2 + 2 * (0.5 + 1 / 32),
    "dequant_rows": 0.5 + 1 / 32 + 2,
    "rht_quant_sr": 2 + 0.5 + 1 / 32,
    "osc_update": 8,
    "osc_step": 28,
}
# ... of which read (the rest is written): the DRAM read counter of a kernel
# compares with these (a ratio above 1 means re-reads); writes can still sit
# in L2 when a kernel ends, so the write counter reads low.
READ_BYTES_PER_ELEM = {
    "quant_rows_rne": 2, "quant_cols_sr": 2, "double_quant": 2,
    "dequant_rows": 0.5 + 1 / 32, "rht_quant_sr": 2, "osc_update": 4, "osc_step": 16,
}
OP_ELEMS = {k: SWEEP[0] * SWEEP[1] for k in BYTES_PER_ELEM}
OP_ELEMS["osc_update"] = OP_ELEMS["osc_step"] = OSC[0] * OSC[1]
# Kernels outside the step that --only can still run inside it, alone, for
# a profiler capture (rows SR quantization of the sweep).
PROFILE_ONLY_OPS = {"quant_rows_sr": 2 + 0.5 + 1 / 32}


# Further operations built beyond the step (Q-EMA), timed on their own.
NEXT_OPS = {"qema_quant": (4 + 4 + 4 + 0.5 + 1 / 32, (4096, 14336)),
            # Y = Q_D(X) Q_D(W)^T: X the sweep, W a second 8192-row tensor
            "gemm_mxf4": (None, (8192, 8192, 28672)),
            # the same with X quantized in the GEMM's load stage, against
            # quantize + blocked scales + GEMM, for W's first N rows
            "gemm_quant_a": (None, (256, 512, 1024, 8192))}


def alg_bytes(op):
    per = BYTES_PER_ELEM[op] if op in BYTES_PER_ELEM else PROFILE_ONLY_OPS[op]
    return per * OP_ELEMS.get(op, SWEEP[0] * SWEEP[1])


STEP_BYTES = sum(alg_bytes(op) for op in BYTES_PER_ELEM)
STEP_ELEMS = sum(OP_ELEMS.values())


def rank_seed(rank):
    """Each rank quantizes its own seeded sweep (replicas, weak scaling)."""
    return SEED + rank


def reduce_max(value, world, device=None):
    """Max over ranks of a float (the timed region's duration)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_step, steps, elapsed_ms_max):
    """Whole-job GB/s: all ranks' algorithmic bytes over the slowest rank."""
    return world * bytes_per_step * steps / (elapsed_ms_max * 1e-3) / 1e9


# Sources of each op's kernel: a DRAM traffic figure in
# profiles/dram_traffic.txt holds while the digest of these files is unchanged.
_COMMON_SOURCES = ("mxfp4_device.cuh", "launch.cuh")
OP_SOURCES = {
    "quant_rows_rne": ("quantize.cu",) + _COMMON_SOURCES,
    "quant_cols_sr": ("quantize.cu",) + _COMMON_SOURCES,
    "double_quant": ("quantize.cu",) + _COMMON_SOURCES,
    "dequant_rows": ("quantize.cu",) + _COMMON_SOURCES,
    "rht_quant_sr": ("rht.cu", "tc_common.cuh") + _COMMON_SOURCES,
    "osc_update": ("osc.cu",) + _COMMON_SOURCES,
    "osc_step": ("osc.cu",) + _COMMON_SOURCES,
}


def kernel_source_digest(op):
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "mxfp4_block_quantization_quantizer_b200", "csrc")
    for name in OP_SOURCES[op]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:12]


def measured_traffic(op):
    """(dram read bytes, dram write bytes) of one full-size launch of op from
    profiles/dram_traffic.txt (an ncu capture of that launch), or None when
    the op's kernel sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    digest = kernel_source_digest(op)
    for line in lines:
        parts = line.split()
        if len(parts) >= 4 and parts[0] == op and parts[3] == "src=" + digest:
            return float(parts[1]), float(parts[2])
    return None


def measured_fp4_peak():
    """Dense FP4 tensor peak: the measured bf16 GEMM burst x 4 (the nominal
    fp4/bf16 ratio, 9 / 2.25 PFLOP/s); 1.59 PFLOP/s bf16 if unmeasured."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 4"
    except Exception:
        return 4.0 * 1590.0, "fallback bf16 x 4"


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default="",
                    help="comma-separated ops to run (profiling); default all")
    ap.add_argument("--rows", type=int, default=SWEEP[0],
                    help="rows of the sweep workload (profiling a smaller case)")
    ap.add_argument("--gemm", default="",
                    help="M,N,K: time only the MXFP4 GEMM at that shape "
                         "(profiling); prints one line")
    ap.add_argument("--gemm-fused", action="store_true",
                    help="with --gemm: the GEMM that quantizes bf16 A in its "
                         "load stage (mxfp4_gemm_quantize_a)")
    return ap.parse_args()


def run_gemm_only(args):
    """The MXFP4 GEMM alone on ROWS quantizations of two seeded N(0,1)
    tensors [M, K] and [N, K] (profiling a case of a chosen size)."""
    import numpy as np
    import torch

    import mxfp4_block_quantization_quantizer_b200 as m
    from mxfp4_block_quantization_quantizer_b200 import workloads as W

    M, N, K = (int(v) for v in args.gemm.split(","))
    dev = torch.device("cuda", 0)
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    xa = to(W.normal_bf16(M, K, 11))
    ac, as_ = m.quantize(xa, m.ROWS, m.RNE)
    bc, bs = m.quantize(to(W.normal_bf16(N, K, 12)), m.ROWS, m.RNE)
    ab, bb = m.scales_to_blocked(as_), m.scales_to_blocked(bs)
    out = torch.empty(M, N, dtype=torch.float32, device=dev)
    if args.gemm_fused:
        run = lambda: m.gemm_quantize_a(xa, bc, bb, out=out)  # noqa: E731
    else:
        run = lambda: m.gemm(ac, ab, bc, bb, K, out=out)  # noqa: E731
    for _ in range(args.warmup):
        run()
    evs = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize(dev)
    d = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e-3
    peak, kind = measured_fp4_peak()
    tf = 2.0 * M * N * K / d / 1e12
    print(json.dumps({"profile_run": True,
                      "op": "gemm_quant_a" if args.gemm_fused else "gemm_mxf4",
                      "shape": [M, N, K],
                      "us": d * 1e6, "TFLOP_s": tf, "frac": tf / peak,
                      "peak_kind": kind}), flush=True)


def config_block(args, world):
    return {"workload": "sweep 8192x28672 bf16 N(0,1)+0.1% x100 outliers "
                        "[rows RNE, cols SR, double quant, dequant rows, "
                        "RHT+rows SR] + oscillation tracker step on 4096x4096 "
                        "fp32 master weight",
            "shape": list(SWEEP), "osc_shape": list(OSC), "seed": SEED,
            "sr_seed": SEED, "rht_sign_seed": 2, "osc_threshold": 4.0,
            "l2": "inputs larger than L2 (470 MB, 268 MB); no flush",
            "parallelism": "replicas x%d (weak, no collective)" % world}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def cpu_sample_step(x_band, w_band, osc_state, row0):
    """One step of the oracle on a sample: a 32-row band of the sweep for
    each op, and a 16-row band of the tracker workload. Returns bytes."""
    import oracle as O
    C = x_band.shape[1]
    n = x_band.size
    O.quantize(x_band, O.ROWS, O.RNE, 0, row0=row0)
    O.quantize(x_band, O.COLS, O.SR, SEED, row0=row0)
    O.double_quantize(x_band, SEED, row0=row0)
    c, s = O.quantize(x_band, O.ROWS, O.RNE, 0, row0=row0)
    O.dequantize(c, s, 32, C)
    O.rht_quantize(x_band, 2, O.SR, SEED, row0=row0)
    w, ws, dw, dq = osc_state
    O.osc_synthetic_update(w, SEED, 0, row0=0)
    O.osc_step(w, ws, dw, dq)
    nb = 0.0
    for op in ("quant_rows_rne", "quant_cols_sr", "double_quant", "dequant_rows",
               "rht_quant_sr"):
        nb += BYTES_PER_ELEM[op] * n
    nb += (BYTES_PER_ELEM["osc_update"] + BYTES_PER_ELEM["osc_step"]) * w.size
    return nb, n * 5 + w.size * 2


def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline_sample(x_np, w_np, max_seconds=20.0):
    band = np.ascontiguousarray(x_np[:32])
    wb = np.ascontiguousarray(w_np[:16])
    state = (wb.copy(), wb.copy(), np.zeros_like(wb), np.zeros_like(wb))
    t0 = time.perf_counter()
    total_b, total_e, reps = 0.0, 0, 0
    while True:
        b, e = cpu_sample_step(band, wb, state, 0)
        total_b += b
        total_e += e
        reps += 1
        if time.perf_counter() - t0 > max_seconds or reps >= 50:
            break
    dt = time.perf_counter() - t0
    return {"value": total_b / dt / 1e9, "unit": "GB/s", "cores": 1,
            "kind": "oracle", "cpu": cpu_model(), "host_cores": os.cpu_count(),
            "sample": "%d reps of one 32x28672 band of the sweep per op (rows RNE, "
                      "cols SR, double quant, dequant, RHT+SR) and a 16x4096 band "
                      "of the tracker (update + step); single thread, %.1f s"
                      % (reps, dt),
            "gelem_s": total_e / dt / 1e9}


def _oracle_band_worker(args):
    """One process's share of the all-cores baseline: the sample step on its
    own 32-row band, repeated `reps` times. Returns (bytes, elements, s)."""
    x_band, w_band, reps = args
    state = (w_band.copy(), w_band.copy(), np.zeros_like(w_band),
             np.zeros_like(w_band))
    t0 = time.perf_counter()
    nb = ne = 0
    for _ in range(reps):
        b, e = cpu_sample_step(x_band, w_band, state, 0)
        nb += b
        ne += e
    return nb, ne, time.perf_counter() - t0


def cpu_baseline_all_cores(x_np, w_np, reps=8):
    """The same oracle, row-block parallel over every host core (spawned
    processes, one 32-row band each): whole-job bytes over wall time."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    cores = os.cpu_count() or 1
    bands = [(np.ascontiguousarray(x_np[32 * (i % (x_np.shape[0] // 32)):][:32]),
              np.ascontiguousarray(w_np[:16]), reps) for i in range(cores)]
    warm = [(b[0], b[1], 1) for b in bands]
    # spawn (never fork after CUDA); a dead worker raises instead of hanging
    with ProcessPoolExecutor(cores, mp_context=mp.get_context("spawn")) as ex:
        list(ex.map(_oracle_band_worker, warm, timeout=300))  # start-up
        t0 = time.perf_counter()
        res = list(ex.map(_oracle_band_worker, bands, timeout=600))
        dt = time.perf_counter() - t0
    nb = sum(r[0] for r in res)
    ne = sum(r[1] for r in res)
    return {"value": nb / dt / 1e9, "unit": "GB/s", "cores": cores,
            "cpu": cpu_model(),
            "kind": "oracle",
            "sample": "%d processes x %d reps of the one-band sample step "
                      "(each its own 32x28672 band), %.1f s wall" % (cores, reps, dt),
            "gelem_s": ne / dt / 1e9}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mxfp4_block_quantization_quantizer_b200 import workloads as W
    x = W.normal_bf16(64, SWEEP[1], SEED, 0.001, 100.0)
    w = W.osc_w(seed=3, rows=16, cols=OSC[1])
    band = np.ascontiguousarray(x[:32])
    state = (w.copy(), w.copy(), np.zeros_like(w), np.zeros_like(w))
    for _ in range(args.warmup):
        cpu_sample_step(band, w, state, 0)
    t0 = time.perf_counter()
    nb = ne = 0
    for _ in range(args.steps):
        b, e = cpu_sample_step(band, w, state, 0)
        nb += b
        ne += e
    dt = time.perf_counter() - t0
    value = nb / dt / 1e9
    line = {"impl": "reference", "metric": "MXFP4 quantize GB/s (bytes in+out)",
            "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": config_block(args, 1),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "cpu": cpu_model(),
                             "sample": "each step: one 32x28672 band of the sweep "
                                       "per op and a 16x4096 tracker band"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gelem_s": ne / dt / 1e9}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for line in out.strip().splitlines():
            p = [s.strip() for s in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import mxfp4_block_quantization_quantizer_b200 as m
    from mxfp4_block_quantization_quantizer_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    m.lib()

    # inputs (seeded numpy), uploaded once
    R, C = args.rows, SWEEP[1]
    x_np = W.sweep(seed=rank_seed(rank), rows=R)
    w_np = W.osc_w(seed=3 + rank)
    u8 = lambda *s: torch.empty(s, dtype=torch.uint8, device=dev)  # noqa: E731

    def buffers():
        """Device inputs and outputs of one step (the e2e loop uses two)."""
        return {
            "x": torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev),
            "w": torch.from_numpy(w_np).to(dev),
            "rows": (u8(R, C // 2), u8(R, C // 32)),
            "cols": (u8(C, R // 2), u8(C, R // 32)),
            "dq": (u8(R, C // 2), u8(R, C // 32), u8(C, R // 2), u8(C, R // 32)),
            "rht": (u8(R, C // 2), u8(R, C // 32), None),
            "y": torch.empty(R, C, dtype=torch.bfloat16, device=dev),
            "nflag": torch.zeros(1, dtype=torch.int64, device=dev),
        }

    def outputs(b):
        return [*b["rows"], *b["cols"], *b["dq"], b["y"], b["rht"][0],
                b["rht"][1], b["w"], b["nflag"]]

    buf0 = buffers()
    # tracker state (stays on the device across steps)
    ws, dwt, dqt = buf0["w"].clone(), torch.zeros_like(buf0["w"]), torch.zeros_like(buf0["w"])

    ops = [o for o in BYTES_PER_ELEM if not args.only or o in args.only.split(",")]
    ops += [o for o in PROFILE_ONLY_OPS if o in args.only.split(",")]
    if (R, C) != SWEEP:
        for o in ops:
            if o not in ("osc_update", "osc_step"):
                OP_ELEMS[o] = R * C
    stream = torch.cuda.current_stream(dev)
    ev = {op: [] for op in ops}
    step_no = [0]

    def step(record, b=buf0):
        t = step_no[0]
        step_no[0] += 1
        pairs = []
        cur = torch.cuda.current_stream(dev)

        def timed(op, fn):
            if op not in ops:
                return
            if record:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(cur)
                fn()
                e1.record(cur)
                pairs.append((op, e0, e1))
            else:
                fn()

        x, w = b["x"], b["w"]
        timed("quant_rows_rne", lambda: m.quantize(x, m.ROWS, m.RNE, 0, out=b["rows"]))
        timed("quant_rows_sr", lambda: m.quantize(x, m.ROWS, m.SR, SEED, out=b["rows"]))
        timed("quant_cols_sr", lambda: m.quantize(x, m.COLS, m.SR, SEED, out=b["cols"]))
        timed("double_quant", lambda: m.double_quantize(x, SEED, out=b["dq"]))
        timed("dequant_rows", lambda: m.dequantize(b["rows"][0], b["rows"][1], R, C, out=b["y"]))
        timed("rht_quant_sr", lambda: m.rht_quantize(x, 2, m.SR, SEED, out=b["rht"]))
        timed("osc_update", lambda: m.osc_synthetic_update(w, 3, t % 200))
        timed("osc_step", lambda: m.osc_step(w, ws, dwt, dqt, window_end=(t % 200 == 199),
                                             n_flagged=b["nflag"]))
        return pairs

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)
    all_pairs = []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(args.steps):
        all_pairs.extend(step(True))
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    for op, a, b in all_pairs:
        ev[op].append(a.elapsed_time(b))
    elapsed_ms = reduce_max(elapsed_ms, world, dev)

    # further operations: Q-EMA on an fp32 master weight, timed alone
    next_ops = {}
    if not args.only:
        qR, qC = NEXT_OPS["qema_quant"][1]
        qw = torch.from_numpy(W.master_w(seed=7 + rank, rows=qR, cols=qC)).to(dev)
        qe = torch.from_numpy(W.master_w(seed=8 + rank, rows=qR, cols=qC)).to(dev)
        qout = (u8(qR, qC // 2), u8(qR, qC // 32))
        for _ in range(args.warmup):
            m.qema_quantize(qw, qe, 0.998, out=qout)
        qev = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            m.qema_quantize(qw, qe, 0.998, out=qout)
            b.record(stream)
            qev.append((a, b))
        torch.cuda.synchronize(dev)
        d = statistics.mean(a.elapsed_time(b) for a, b in qev) * 1e-3
        d = reduce_max(d, world, dev)
        nbytes = NEXT_OPS["qema_quant"][0] * qR * qC
        next_ops["qema_quant"] = {"us": d * 1e6, "GB_s": nbytes / d / 1e9,
                                  "bytes": nbytes, "shape": [qR, qC],
                                  "launches": args.steps}
        del qw, qe, qout

        # the overflow-aware scale rule on the sweep: rows RNE, double
        # quantization, rotation + SR (the step's ops with the other rule)
        def timed_alone(fn):
            for _ in range(args.warmup):
                fn()
            tev = []
            for _ in range(args.steps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                tev.append((a, b))
            torch.cuda.synchronize(dev)
            return reduce_max(statistics.mean(a.elapsed_time(b) for a, b in tev) * 1e-3,
                              world, dev)

        oout = (u8(R, C // 2), u8(R, C // 32))
        dout = (u8(R, C // 2), u8(R, C // 32), u8(C, R // 2), u8(C, R // 32))
        for name, step_op, fn in (
                ("quant_rows_sr", "quant_rows_rne",
                 lambda: m.quantize(buf0["x"], m.ROWS, m.SR, SEED, out=oout)),
                ("quant_rows_rne_oas", "quant_rows_rne",
                 lambda: m.quantize(buf0["x"], m.ROWS, m.RNE, out=oout, oas=True)),
                ("double_quant_oas", "double_quant",
                 lambda: m.double_quantize(buf0["x"], SEED, out=dout, oas=True)),
                ("rht_quant_sr_oas", "rht_quant_sr",
                 lambda: m.rht_quantize(buf0["x"], 2, m.SR, SEED, out=oout + (None,),
                                        oas=True))):
            d = timed_alone(fn)
            nbytes = BYTES_PER_ELEM[step_op] * R * C
            next_ops[name] = {"us": d * 1e6, "GB_s": nbytes / d / 1e9, "bytes": nbytes,
                              "shape": [R, C], "launches": args.steps}
        del oout, dout

        # the tracker's window-end step (flag, snap, reset: k_osc_step with
        # the window end) on the tracker workload, on copies of its state
        ow, ows = buf0["w"].clone(), ws.clone()
        odw, odq = dwt.clone(), dqt.clone()
        nfl = torch.zeros(1, dtype=torch.int64, device=dev)
        d = timed_alone(lambda: m.osc_step(ow, ows, odw, odq, window_end=True, n_flagged=nfl))
        nbytes = (BYTES_PER_ELEM["osc_step"] + 4) * OSC[0] * OSC[1]  # w is written too
        next_ops["osc_step_window_end"] = {"us": d * 1e6, "GB_s": nbytes / d / 1e9,
                                           "bytes": nbytes, "shape": list(OSC),
                                           "launches": args.steps}
        # Q-Ramping on the tracker workload: an iteration inside the tracking
        # window (46 B/element) and one outside it (22 B/element)
        qd = (ow * 1e-4).contiguous()
        qacc = torch.zeros_like(ow)
        qfl = torch.zeros(OSC, dtype=torch.uint8, device=dev)
        for name, it, per in (("qramp_step_tracking", 5, 46), ("qramp_step", 35, 22)):
            d = timed_alone(lambda: m.qramp_step(ow, qd, ows, odw, odq, qacc, qfl, it,
                                                 track_iters=30, k1=16.0, k2=5))
            nbytes = per * OSC[0] * OSC[1]
            next_ops[name] = {"us": d * 1e6, "GB_s": nbytes / d / 1e9, "bytes": nbytes,
                              "shape": list(OSC), "launches": args.steps}
        del ow, ows, odw, odq, nfl, qd, qacc, qfl
        # the rotation of fp32 inputs (the in-register butterfly kernel) on
        # the fp32 master weight, rounding SR
        fR, fC = NEXT_OPS["qema_quant"][1]
        fw = torch.from_numpy(W.master_w(seed=7 + rank, rows=fR, cols=fC)).to(dev)
        fout = (u8(fR, fC // 2), u8(fR, fC // 32), None)
        d = timed_alone(lambda: m.rht_quantize(fw, 2, m.SR, SEED, out=fout))
        nbytes = (4 + 0.5 + 1 / 32) * fR * fC
        next_ops["rht_quant_sr_f32"] = {"us": d * 1e6, "GB_s": nbytes / d / 1e9,
                                        "bytes": nbytes, "shape": [fR, fC],
                                        "launches": args.steps}
        del fw, fout

        # MXFP4 GEMM on the block-scaled tensor cores, consuming the step's
        # ROWS codes of the sweep as the activation operand
        gM, gN, gK = NEXT_OPS["gemm_mxf4"][1]
        if (R, C) == (gM, gK):
            w2 = torch.from_numpy(W.normal_bf16(gN, gK, 6 + rank).view(np.int16)).view(
                torch.bfloat16).to(dev)
            bc, bs = m.quantize(w2, m.ROWS, m.RNE)
            del w2
            ac, as_ = m.quantize(buf0["x"], m.ROWS, m.RNE)
            ab, bb = m.scales_to_blocked(as_), m.scales_to_blocked(bs)
            gout = torch.empty(gM, gN, dtype=torch.float32, device=dev)
            for _ in range(args.warmup):
                m.gemm(ac, ab, bc, bb, gK, out=gout)
            gev = []
            for _ in range(args.steps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                m.gemm(ac, ab, bc, bb, gK, out=gout)
                b.record(stream)
                gev.append((a, b))
            torch.cuda.synchronize(dev)
            d = statistics.mean(a.elapsed_time(b) for a, b in gev) * 1e-3
            d = reduce_max(d, world, dev)
            flops = 2.0 * gM * gN * gK
            peak, kind = measured_fp4_peak()
            next_ops["gemm_mxf4"] = {"us": d * 1e6, "TFLOP_s": flops / d / 1e12,
                                     "flops": flops, "shape": [gM, gN, gK],
                                     "launches": args.steps, "peak_TFLOP_s": peak,
                                     "peak_kind": kind,
                                     "frac": flops / d / 1e12 / peak}
            # the activation quantized inside the GEMM (one launch) against
            # quantize + blocked scales + GEMM (three), for W's first N rows
            qout = (u8(gM, gK // 2), u8(gM, gK // 32))
            qblk = u8(-(-gM // 128) * 128, -(-(gK // 32) // 4) * 4)
            for nn in NEXT_OPS["gemm_quant_a"][1]:
                bcn = bc[:nn]
                bbn = m.scales_to_blocked(bs[:nn])
                outn = torch.empty(gM, nn, dtype=torch.float32, device=dev)
                d_fused = timed_alone(lambda: m.gemm_quantize_a(buf0["x"], bcn, bbn, out=outn))

                def two_step():
                    m.quantize(buf0["x"], m.ROWS, m.RNE, out=qout)
                    m.scales_to_blocked(qout[1], out=qblk)
                    m.gemm(qout[0], qblk, bcn, bbn, gK, out=outn)
                d_two = timed_alone(two_step)
                flops = 2.0 * gM * nn * gK
                next_ops["gemm_quant_a_n%d" % nn] = {
                    "us": d_fused * 1e6, "two_step_us": d_two * 1e6,
                    "speedup_vs_two_step": d_two / d_fused,
                    "TFLOP_s": flops / d_fused / 1e12, "shape": [gM, nn, gK],
                    "launches": args.steps,
                    "x_read_GB_s": 2.0 * gM * gK / d_fused / 1e9}
                if nn == NEXT_OPS["gemm_quant_a"][1][0]:
                    # the same with stochastic rounding (a gradient operand)
                    d_fs = timed_alone(lambda: m.gemm_quantize_a(buf0["x"], bcn, bbn, m.SR,
                                                                 SEED, out=outn))

                    def two_step_sr():
                        m.quantize(buf0["x"], m.ROWS, m.SR, SEED, out=qout)
                        m.scales_to_blocked(qout[1], out=qblk)
                        m.gemm(qout[0], qblk, bcn, bbn, gK, out=outn)
                    d_ts = timed_alone(two_step_sr)
                    next_ops["gemm_quant_a_sr_n%d" % nn] = {
                        "us": d_fs * 1e6, "two_step_us": d_ts * 1e6,
                        "speedup_vs_two_step": d_ts / d_fs, "shape": [gM, nn, gK],
                        "launches": args.steps}
                del bcn, bbn, outn
            del qout, qblk
            del ac, as_, bc, bs, ab, bb, gout

    # end to end: pinned host input -> device -> kernels -> host results
    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"profile_run": True, "ops": ops,
                              "ms": elapsed_ms / args.steps,
                              "ops_us": {op: 1e3 * statistics.mean(ev[op])
                                         for op in ops},
                              "next_ops": next_ops}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    # Double-buffered: step t's uploads, kernels and downloads run on three
    # streams, so the uploads of step t+1 and the downloads of step t-1
    # overlap step t (PCIe moves both directions at once).
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    w_host = torch.from_numpy(w_np).pin_memory()
    bufs = [buf0, buffers()]
    host_outs = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outputs(buf0)]
    h2d = x_host.numel() * 2 + w_host.numel() * 4
    d2h = sum(o.numel() * o.element_size() for o in outputs(buf0))
    s_up, s_run, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    for e in ev_run + ev_down:
        e.record(stream)

    def e2e_step(t):
        k = t % 2
        b = bufs[k]
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_run[k])    # step t-2 finished reading x
            s_up.wait_event(ev_down[k])   # and its w went out
            b["x"].copy_(x_host, non_blocking=True)
            b["w"].copy_(w_host, non_blocking=True)
            ev_up[k].record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_up[k])
            s_run.wait_event(ev_down[k])  # step t-2's outputs are out
            step(False, b)
            ev_run[k].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_run[k])
            for h, o in zip(host_outs, outputs(b)):
                h.copy_(o, non_blocking=True)
            ev_down[k].record(s_down)

    for t in range(2):
        e2e_step(t)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_up)
    for t in range(args.e2e_steps):
        e2e_step(t)
    s_up.wait_stream(s_down)
    e_end.record(s_up)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_end)
    e2e_ms = reduce_max(e2e_ms, world, dev)
    if world > 1:
        dist.barrier()

    if rank == 0:
        peak, peak_kind = measured_peaks()
        per_op = {}
        for op in ops:
            d = statistics.mean(ev[op]) * 1e-3
            ach = alg_bytes(op) / d / 1e9
            per_op[op] = {"us": d * 1e6, "GB_s": ach, "frac": ach / peak,
                          "bytes": alg_bytes(op)}
        dom = max(per_op, key=lambda k: per_op[k]["us"])
        step_s = elapsed_ms * 1e-3 / args.steps
        value = job_gbs(world, STEP_BYTES, args.steps, elapsed_ms)
        measured = measured_traffic(dom)
        traffic = None if measured is None else measured[0] + measured[1]
        read_ratio = (None if measured is None else
                      measured[0] / (READ_BYTES_PER_ELEM[dom] * OP_ELEMS[dom]))
        line = {
            "metric": "MXFP4 quantize GB/s (bytes in+out)",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": config_block(args, world),
            "gelem_s": world * STEP_ELEMS / step_s / 1e9,
            "hbm_frac": value / world / peak,
            "roofline": {"bound": "hbm", "kernel": dom,
                         "achieved": per_op[dom]["GB_s"], "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": per_op[dom]["frac"], "traffic": traffic,
                         "dram_read_over_alg_read": read_ratio},
            "ops": per_op,
            "e2e": {"value": job_gbs(world, STEP_BYTES, args.e2e_steps, e2e_ms),
                    "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "next_ops": {k: (dict(v, frac=v["GB_s"] / peak) if "GB_s" in v else v)
                         for k, v in next_ops.items()},
            "gpu_launches": len(ops) * args.steps,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline_sample(x_np, w_np)
            line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(x_np, w_np)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.gemm:
        run_gemm_only(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
