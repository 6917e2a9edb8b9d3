"""Benchmark of the NVFP4 hot path: one linear layer's forward + backward
step at the 8B-shaped workload, every quantization and all three GEMMs on the
device through the C ABI.

A step (one batch, one rank):
  1. X  [8192, 4096]  -> Four Over Six, 1D row blocks          (fprop A)
  2. W  [14336, 4096] -> Four Over Six, 16x16 2D blocks        (fprop B)
  3. fprop  Y  = X W^T            8192 x 14336, K = 4096, bf16 out
  4. dY [8192, 14336] -> MS-EDEN (or RHT+SR), rows and columns (dgrad A, wgrad A)
  5. W  -> rotated RTN along the output features (columns)     (dgrad B)
  6. dgrad  dX = dY W             8192 x 4096,  K = 14336
  7. X  -> rotated RTN along the tokens (columns)              (wgrad B)
  8. wgrad  dW = dY^T X           14336 x 4096, K = 8192
The rotated operands of a backward GEMM share one seed, so the Hadamard
rotations cancel in the product.

`value` = the three GEMMs' algorithmic FLOPs / device time of the whole step
(quantization included), summed over ranks (weak scaling: every rank runs its
own batch; no data-path collective).  Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--bwd-mode eden|sr]
  python bench.py --impl reference ...   # the CPU oracle, bounded sample
"""
import argparse
import functools
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 quantize Gelem/s & % HBM roofline; NVFP4 GEMM TFLOPS & % FP4 peak"
TOKENS, HIDDEN, OUT = 8192, 4096, 14336
BWD_NAMES = {"eden": "MS-EDEN", "sr": "RHT+SR", "sr_hw": "RHT+hardware SR"}


def workload(bwd_mode="eden"):
    return ("linear fwd+bwd, 8B-shaped: X 8192x4096 (4/6 1D), W 14336x4096 (4/6 2D), "
            f"dY 8192x14336 ({BWD_NAMES[bwd_mode]} rows+cols), fprop/dgrad/wgrad NVFP4 GEMMs, bf16 out")
FP4_PER_BF16 = 4.0   # nominal dense FP4 / BF16 tensor throughput on B200 (9 / 2.25 PFLOP/s)
FP4_DATASHEET_TFLOPS = 9000.0   # B200 dense FP4, datasheet
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

ROW, COL, B2D, RHT, GEMM = 0x1, 0x2, 0x4, 0x40, 0x20
RTN, FOUR_SIX, RHT_SR, MS_EDEN, RHT_SR_HW = 0, 1, 2, 3, 4
BWD_MODES = {"eden": MS_EDEN, "sr": RHT_SR, "sr_hw": RHT_SR_HW}


def gemm_flops():
    return 2.0 * TOKENS * OUT * HIDDEN * 3


# (name, elements, algorithmic bytes per element) of the step's quantize calls
def quant_calls():
    return [("X 4/6 rows", TOKENS * HIDDEN, 2 + 0.5 + 1 / 16),
            ("W 4/6 2D", OUT * HIDDEN, 2 + 0.5 + 1 / 16),
            ("dY rows+cols", TOKENS * OUT, 2 + 2 * (0.5 + 1 / 16)),
            ("W rotated cols", OUT * HIDDEN, 2 + 0.5 + 1 / 16),
            ("X rotated cols", TOKENS * HIDDEN, 2 + 0.5 + 1 / 16)]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK), "fallback"


# --------------------------------------------------------------------------
# distributed plumbing (one process per GPU; CPU tests drive it with gloo)
# --------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x, device=None):
    """Max of a host float over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, device=None):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, _, r in rows for n, v in zip(names, r) if v.lower().startswith("active")})
        loaded = [c for c, _, _ in rows if c > 0.5 * rows[0][1]] or [c for c, _, _ in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": rows[0][1], "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------
def carve(buf, shapes):
    """Consecutive row-major views of the given shapes in a 1-D buffer."""
    views, o = [], 0
    for r, c in shapes:
        views.append(buf[o:o + r * c].view(r, c))
        o += r * c
    return views


class LayerStep:
    """Pre-allocated buffers and the C-ABI call sequence of one step."""

    def __init__(self, x, w, dy, bwd_mode, device, shared_amax=True, results=None):
        import torch
        from nvfp4_block_quantization_amax_b200 import api
        self.api = api
        self.x, self.w, self.dy = x, w, dy
        self.bwd = bwd_mode
        # shared_amax: one nvfp4_amax pass per weight / activation gives the
        # plain amax of its forward quantization and the rotated-column amax
        # of its backward partner; otherwise each call runs its own amax pass
        self.shared_amax = shared_amax
        self.amax = {k: torch.zeros(3, dtype=torch.float32, device=device) for k in ("x", "w")}
        T, H = x.shape
        O = w.shape[0]
        self.plan = [  # (tensor, mode, flags)
            ("x", FOUR_SIX, ROW | GEMM),
            ("w", FOUR_SIX, ROW | B2D | GEMM),
            ("dy", bwd_mode, ROW | COL | GEMM),
            ("w_rot", RTN, COL | RHT | GEMM),
            ("x_rot", RTN, COL | RHT | GEMM),
        ]
        src = {"x": x, "w": w, "dy": dy, "w_rot": w, "x_rot": x}
        self.src = src
        self.out = {}
        self.ws = {}
        for name, mode, flags in self.plan:
            t = src[name]
            self.out[name] = api.alloc_outputs(t.shape[0], t.shape[1], flags, device)
            self.ws[name] = api.workspace_for(t.shape[0], t.shape[1], flags, device)
        # results: optionally one contiguous bf16 buffer holding Y, dX, dW
        if results is None:
            results = torch.empty(T * O + T * H + O * H, dtype=torch.bfloat16, device=device)
        self.y, self.dx, self.dw = carve(results, [(T, O), (T, H), (O, H)])
        self.results = results
        self.ev = None

    def quantize(self, name, mode, flags, seed, sid, amax=None):
        self.api.nvfp4_quantize(self.src[name], mode, flags, seed=seed, stream_id=sid, out=self.out[name],
                                workspace=self.ws[name], amax=amax)

    def run(self, step, timers=None):
        """One step.  timers: dict call name -> list of (start, end) CUDA
        events (quantize calls are named q_*, GEMMs fprop / dgrad / wgrad)."""
        api = self.api
        seed = 1000 * (step + 1)   # a new rotation and noise per step
        mark = (lambda k: _Mark(timers, k)) if timers is not None else (lambda k: _NoMark())
        sa = self.shared_amax
        ax, aw = self.amax["x"], self.amax["w"]
        with mark("q_x"):
            if sa:
                api.nvfp4_amax(self.x, COL | RHT, seed=seed, out=ax)
            self.quantize("x", FOUR_SIX, ROW | GEMM, 0, 0, amax=ax if sa else None)
        with mark("q_w"):
            if sa:
                api.nvfp4_amax(self.w, COL | RHT, seed=seed, out=aw)
            self.quantize("w", FOUR_SIX, ROW | B2D | GEMM, 0, 1, amax=aw if sa else None)
        qx, qw = self.out["x"], self.out["w"]
        with mark("fprop"):
            api.nvfp4_gemm(qx.codes_row, qx.scales_row, qx.alpha_row, qw.codes_row, qw.scales_row, qw.alpha_row,
                           out=self.y)
        with mark("q_dy"):
            self.quantize("dy", self.bwd, ROW | COL | GEMM, seed, 0)
        with mark("q_w_rot"):
            self.quantize("w_rot", RTN, COL | RHT | GEMM, seed, 1, amax=aw if sa else None)
        qd, qwr = self.out["dy"], self.out["w_rot"]
        with mark("dgrad"):
            api.nvfp4_gemm(qd.codes_row, qd.scales_row, qd.alpha_row, qwr.codes_col, qwr.scales_col,
                           qwr.alpha_col, out=self.dx)
        with mark("q_x_rot"):
            self.quantize("x_rot", RTN, COL | RHT | GEMM, seed, 2, amax=ax if sa else None)
        qxr = self.out["x_rot"]
        with mark("wgrad"):
            api.nvfp4_gemm(qd.codes_col, qd.scales_col, qd.alpha_col, qxr.codes_col, qxr.scales_col,
                           qxr.alpha_col, out=self.dw)

    def shapes(self):
        """(name, elements, algorithmic bytes per element) of the quantize
        calls and (name, M, N, K) of the GEMMs."""
        T, H = self.x.shape
        O = self.w.shape[0]
        one = 2 + 0.5 + 1 / 16
        quant = [("q_x", T * H, one), ("q_w", O * H, one), ("q_dy", T * O, 2 + 2 * (0.5 + 1 / 16)),
                 ("q_w_rot", O * H, one), ("q_x_rot", T * H, one)]
        gemms = [("fprop", T, O, H), ("dgrad", T, H, O), ("wgrad", O, H, T)]
        return quant, gemms


GEMM_CALLS = ("fprop", "dgrad", "wgrad")
QUANT_CALLS = ("q_x", "q_w", "q_dy", "q_w_rot", "q_x_rot")


class _NoMark:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


class _Mark:
    def __init__(self, timers, key):
        self.timers, self.key = timers, key

    def __enter__(self):
        import torch
        self.s = torch.cuda.Event(enable_timing=True)
        self.s.record()
        return self

    def __exit__(self, *a):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.timers.setdefault(self.key, []).append((self.s, e))
        return False


def gemm_traffic_record():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    src = os.path.join(ROOT, "nvfp4_block_quantization_amax_b200", "csrc", "gemm.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    g = d.get("gemm", {})
    return g.get("dram_bytes_per_launch") if g.get("source_sha256_16") == h else None


QUANT_SOURCES = ("quantize.cu", "nvfp4_device.cuh", "tile.cuh", "launch.cuh")


def quantizer_issue_record():
    """Per-kernel instruction counts of the step's quantizer launches from the
    committed ncu summary, if it was taken on the current quantizer sources
    (else None)."""
    p = os.path.join(ROOT, "profiles", "quantizer_issue.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    csrc = os.path.join(ROOT, "nvfp4_block_quantization_amax_b200", "csrc")
    h = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read() for f in QUANT_SOURCES)).hexdigest()[:16]
    return d if d.get("source_sha256_16") == h else None


def quantize_roofline(rec, quant_ms, sm_mhz, n_sm, hbm_gbs):
    """The quantizer against its floors: per kernel the larger of its issue
    time (warp instructions / (SMs x 4 schedulers x the sampled SM clock))
    and its HBM time (algorithmic bytes / HBM peak), summed over the step's
    kernels, against the step's measured quantizer time."""
    rate = n_sm * 4 * sm_mhz * 1e6
    issue = [k["warp_instructions"] / rate for k in rec["kernels"]]
    mem = [k["algorithmic_bytes"] / (hbm_gbs * 1e9) for k in rec["kernels"]]
    floor = sum(max(a, b) for a, b in zip(issue, mem))
    return {"bound": "per kernel max(issue, hbm)", "floor_us": round(floor * 1e6, 1),
            "achieved_us": round(quant_ms * 1e3, 1), "frac": floor / (quant_ms * 1e-3),
            "issue_floor_us": round(sum(issue) * 1e6, 1), "hbm_floor_us": round(sum(mem) * 1e6, 1),
            "sm_mhz": sm_mhz, "kernels": len(issue),
            "instructions": "ncu smsp__inst_executed.sum per kernel, profiles/quantizer_issue.json"}


class L2Flush:
    """Overwrites a 256 MiB buffer (twice L2) between timed calls so no
    timed call starts with its inputs in L2."""

    def __init__(self, device):
        import torch
        self.buf = torch.empty(64 << 20, dtype=torch.int32, device=device)

    def __call__(self):
        self.buf.fill_(1)


def time_call(fn, iters, flush=None, warm=1):
    """Median device time (ms) of fn() over `iters` calls, CUDA events on the
    current stream, L2 overwritten before every call when flush is given."""
    import torch
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(iters):
        if flush is not None:
            flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        ts.append((s, e))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ts)


MODE_NAMES = {RTN: "rtn", FOUR_SIX: "four_six", RHT_SR: "rht_sr", MS_EDEN: "ms_eden", RHT_SR_HW: "rht_sr_hw"}
SP, PROVIDED = 0x8, 0x10


def quant_bytes_per_elem(flags):
    """Algorithmic bytes per element of one quantize call: the bf16 read once,
    codes and scales of every requested orientation."""
    n_or = bool(flags & ROW) + bool(flags & COL)
    if flags & B2D:
        return 2 + 0.5 * n_or + n_or / 256
    return 2 + n_or * (0.5 + 1 / 16)


def quantize_modes_table(api, tensors, hbm, flush, iters=7):
    """Every mode x orientation on the given tensors: the whole call (two
    passes), the single-pass call, and the quantize kernel alone (alpha
    provided); microseconds and the fraction of HBM bandwidth by algorithmic
    bytes."""
    import torch
    table = {}
    for label, t, modes, extra in tensors:
        R, C = t.shape
        out = api.alloc_outputs(R, C, ROW | COL | extra, t.device)
        ws = api.workspace_for(R, C, ROW | COL | SP, t.device)
        alpha = torch.full((1,), 1e-3, dtype=torch.float32, device=t.device)
        entry = {}
        for mode in modes:
            per = {}
            for oname, of in (("rows", ROW), ("cols", COL), ("dual", ROW | COL)):
                flags = of | extra
                us, frac = [], []
                for variant in ("two_pass", "single_pass", "kernel_alone"):
                    if variant == "two_pass":
                        fn = lambda: api.nvfp4_quantize(t, mode, flags, seed=5, out=out, workspace=ws)
                    elif variant == "single_pass":
                        fn = lambda: api.nvfp4_quantize(t, mode, flags | SP, seed=5, out=out, workspace=ws)
                    else:
                        fn = lambda: api.nvfp4_quantize(t, mode, flags, seed=5, alpha=alpha, out=out, workspace=ws)
                    ms = time_call(fn, iters, flush)
                    us.append(round(ms * 1e3, 2))
                    frac.append(round(R * C * quant_bytes_per_elem(flags) / (ms * 1e-3) / 1e9 / hbm, 4))
                per[oname] = {"us": us, "frac_hbm": frac}
            entry[MODE_NAMES[mode]] = per
        table[label] = entry
        del out, ws
    return table


def sweep_table(api, hbm, flush, device):
    """The size sweep: bf16 4096 x N, every mode, rows and rows + columns,
    two-pass vs single-pass amax; Gelem/s and fraction of HBM bandwidth."""
    import torch
    from nvfp4_block_quantization_amax_b200 import synthetic
    res = {}
    for n in synthetic.SWEEP_N:
        x = synthetic.device_sweep(n, seed=n, device=device)
        out = api.alloc_outputs(4096, n, ROW | COL, device)
        ws = api.workspace_for(4096, n, ROW | COL | SP, device)
        iters = 10 if n <= 16384 else 3
        per = {}
        for mode in MODE_NAMES:
            row = {}
            for oname, of in (("rows", ROW), ("dual", ROW | COL)):
                g, f = [], []
                for sp in (0, SP):
                    ms = time_call(lambda: api.nvfp4_quantize(x, mode, of | sp, seed=3, out=out, workspace=ws),
                                   iters, flush)
                    g.append(round(4096 * n / (ms * 1e-3) / 1e9, 1))
                    f.append(round(4096 * n * quant_bytes_per_elem(of) / (ms * 1e-3) / 1e9 / hbm, 4))
                row[oname] = {"gelem_s": g, "frac_hbm": f}
            per[MODE_NAMES[mode]] = row
        res[f"4096x{n}"] = per
        del x, out, ws
        torch.cuda.empty_cache()
    return res


def step_breakdown(step, steps, hbm, fp4_peak):
    """Run `steps` steps with every call timed; per call: average us and its
    roofline fraction (quantize: algorithmic bytes vs HBM; GEMM: 2MNK vs the
    FP4 peak)."""
    import torch
    timers = {}
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        step.run(100 + i, timers)
    e.record()
    torch.cuda.synchronize()
    ms_step = s.elapsed_time(e) / steps
    quant, gemms = step.shapes()
    calls = []
    for name, n, bpe in quant:
        us = 1e3 * sum(a.elapsed_time(b) for a, b in timers[name]) / steps
        calls.append({"call": name, "us": round(us, 2), "bound": "hbm",
                      "frac": round(n * bpe / (us * 1e-6) / 1e9 / hbm, 4)})
    flops = 0.0
    for name, M, N, K in gemms:
        us = 1e3 * sum(a.elapsed_time(b) for a, b in timers[name]) / steps
        flops += 2.0 * M * N * K
        calls.append({"call": name, "us": round(us, 2), "bound": "tensor",
                      "frac": round(2.0 * M * N * K / (us * 1e-6) / 1e12 / fp4_peak, 4)})
    return {"ms_per_step": ms_step, "gemm_tflops_per_step_time": flops / (ms_step * 1e-3) / 1e12, "calls": calls}


def run_device(args, rank, world, local_rank):
    import torch
    from nvfp4_block_quantization_amax_b200 import _lib, synthetic
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    _lib.load()
    layer = synthetic.fwd_bwd_8b(seed=17 * rank)
    x, w, dy = (layer[k].to(device) for k in ("x", "w", "dy"))
    bwd = BWD_MODES[args.bwd_mode]
    step = LayerStep(x, w, dy, bwd, device, shared_amax=not args.amax_per_call)

    # --- device-resident timing ---
    for i in range(args.warmup):
        step.run(i)
    torch.cuda.synchronize()
    barrier(device)
    timers = {}
    launches0 = _lib.nvfp4_launch_count()
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        barrier(device)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for i in range(args.steps):
            step.run(args.warmup + i, timers)
        end.record()
        torch.cuda.synchronize()
        barrier(device)
    launches = _lib.nvfp4_launch_count() - launches0
    ms_local = start.elapsed_time(end) / args.steps
    clocks = clk.summary()
    ms = max_over_ranks(ms_local, device)
    gemm_ms = sum(s.elapsed_time(e) for k in GEMM_CALLS for s, e in timers[k]) / (3 * args.steps)
    quant_ms = sum(s.elapsed_time(e) for k in QUANT_CALLS for s, e in timers[k]) / args.steps

    # --- end to end: pinned host inputs in, results back to pinned host ---
    # Every step copies its inputs in and its results out; the copies run on
    # their own streams (one per direction) and overlap the compute of the
    # neighbouring steps, two sets of device buffers taking turns.  A step's
    # inputs X, W, dY sit in one buffer and its results Y, dX, dW in another,
    # so each direction is one copy per step (measured about 2% faster than
    # three copies each way).
    T_, H_ = x.shape
    O_ = w.shape[0]
    in_shapes, out_shapes = [(T_, H_), (O_, H_), (T_, O_)], [(T_, O_), (T_, H_), (O_, H_)]
    n_in, n_out = sum(r * c for r, c in in_shapes), sum(r * c for r, c in out_shapes)
    h_in = torch.empty(n_in, dtype=torch.bfloat16).pin_memory()
    for v, t in zip(carve(h_in, in_shapes), (x, w, dy)):
        v.copy_(t.cpu())
    h_out = torch.empty(n_out, dtype=torch.bfloat16).pin_memory()
    # 32 steps: the one pipeline fill and drain in the timed region weighs 1/32
    e2e_steps = max(4, min(args.steps, 32))
    sets = []
    for _ in range(2):
        d_in = torch.empty(n_in, dtype=torch.bfloat16, device=device)
        sets.append((LayerStep(*carve(d_in, in_shapes), bwd, device, shared_amax=not args.amax_per_call,
                               results=torch.empty(n_out, dtype=torch.bfloat16, device=device)), d_in))
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    comp = torch.cuda.current_stream(device)

    def e2e_run(n, first):
        done_compute, done_out = [None, None], [None, None]
        for i in range(n):
            k = i % 2
            b, d_in = sets[k]
            with torch.cuda.stream(s_in):
                if done_compute[k] is not None:   # the set's previous step has read its inputs
                    s_in.wait_event(done_compute[k])
                d_in.copy_(h_in, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            comp.wait_event(e_in)
            if done_out[k] is not None:           # its previous results have left the device
                comp.wait_event(done_out[k])
            b.run(first + i)
            e_c = torch.cuda.Event()
            e_c.record(comp)
            done_compute[k] = e_c
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                h_out.copy_(b.results, non_blocking=True)
                e_o = torch.cuda.Event()
                e_o.record(s_out)
                done_out[k] = e_o
        return done_out

    e2e_run(2, 0)
    torch.cuda.synchronize()
    barrier(device)
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record(s_in)
    e2e_run(e2e_steps, 0)
    for st in (comp, s_in):
        s_out.wait_stream(st)
    e2.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2) / e2e_steps, device)
    barrier(device)
    del sets

    total_flops = sum_over_ranks(gemm_flops(), device)
    peaks, src = load_peaks()
    hbm = peaks["hbm_gbs"]
    # the GEMM is timed inside a step of a few milliseconds repeated for well
    # under the seconds a sustained figure needs: the burst peak applies
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    gemm_tflops = 2.0 * TOKENS * OUT * HIDDEN / (gemm_ms * 1e-3) / 1e12
    q_elems = sum(n for _, n, _ in quant_calls())
    q_bytes = sum(n * b for _, n, b in quant_calls())
    q_gelem = q_elems / (quant_ms * 1e-3) / 1e9
    q_gbs = q_bytes / (quant_ms * 1e-3) / 1e9
    traffic = gemm_traffic_record()
    h2d = h_in.numel() * h_in.element_size()
    d2h = h_out.numel() * h_out.element_size()
    per_call = {k: round(1e3 * sum(s.elapsed_time(e) for s, e in timers[k]) / args.steps, 2)
                for k in QUANT_CALLS + GEMM_CALLS}
    result = {
        "metric": METRIC,
        "value": total_flops / (ms * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1 x e2m1 -> f32 (GEMM), f32 (quantizer)",
        "data": "synthetic (seeded; shapes and distributions of the pages' 8B workload)",
        "config": {"workload": workload(args.bwd_mode), "tokens": TOKENS, "hidden": HIDDEN, "out_features": OUT,
                   "bwd_mode": args.bwd_mode, "parallelism": f"replicas x{world} (weak)",
                   "amax": "per call" if args.amax_per_call else
                           "one nvfp4_amax pass per X and W (plain + rotated columns) shared by their forward "
                           "and backward quantize calls; dY's own two-pass call",
                   "l2": "inputs larger than L2: 419 MB of bf16 per step; sub-benchmarks overwrite a 256 MiB "
                         "buffer before every timed call"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": traffic,
                     "kernel": "nvfp4_gemm_pair_kernel (avg of fprop, dgrad, wgrad)",
                     "peak_source": f"{src} bf16 burst x {FP4_PER_BF16:g} (nominal FP4/BF16 ratio)",
                     "peak_datasheet": FP4_DATASHEET_TFLOPS,
                     "frac_datasheet": gemm_tflops / FP4_DATASHEET_TFLOPS},
        "quantize": {"gelem_s": q_gelem, "alg_gbs": q_gbs, "frac_hbm": q_gbs / hbm,
                     "ms_per_step": quant_ms, "hbm_peak_gbs": hbm,
                     "note": "algorithmic bytes: bf16 read once + codes + scales per orientation"},
        "gemm": {"tflops": gemm_tflops, "frac_fp4_peak": gemm_tflops / fp4_peak,
                 "frac_datasheet": gemm_tflops / FP4_DATASHEET_TFLOPS, "ms_per_gemm": gemm_ms},
        "per_call_us": per_call,
        "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
                "note": "every step's inputs copied in from pinned host memory and its results copied back; "
                        "copies on one stream per direction overlap the neighbouring steps' compute"},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    qrec = quantizer_issue_record()
    if qrec is not None and clocks.get("sm_mhz"):
        n_sm = torch.cuda.get_device_properties(device).multi_processor_count
        result["quantize_roofline"] = quantize_roofline(qrec, quant_ms, clocks["sm_mhz"], n_sm, hbm)
    else:
        result["quantize_roofline"] = None
    del h_in, h_out
    if not args.no_extras:
        result.update(run_extras(args, step, x, w, dy, device, hbm, fp4_peak))
    return result


def run_extras(args, step, x, w, dy, device, hbm, fp4_peak):
    """The sub-benchmarks of the JSON line: every quantize mode on the 8B
    tensors, the 4096 x N sweep, the 12B-shaped step, the GEMMs timed alone
    (NVFP4 and MXFP4)."""
    import torch
    from nvfp4_block_quantization_amax_b200 import synthetic
    api = step.api
    flush = L2Flush(device)
    extras = {}
    all_modes = list(MODE_NAMES)
    extras["quantize_modes"] = {
        "columns": ["two_pass (amax + quantize)", "single_pass", "kernel_alone (alpha provided)"],
        "timing": "CUDA events, L2 overwritten before each call, median of 7",
        "bytes": "algorithmic: bf16 read once + codes + scales per orientation",
        **quantize_modes_table(api, [("X 8192x4096", x, all_modes, 0), ("dY 8192x14336", dy, all_modes, 0),
                                     ("W 14336x4096 2D", w, [RTN, FOUR_SIX], B2D)], hbm, flush)}
    # GEMMs alone (burst): the step's NVFP4 operands, and MXFP4 ones of the fprop shape
    qx, qw = step.out["x"], step.out["w"]
    ms = time_call(lambda: api.nvfp4_gemm(qx.codes_row, qx.scales_row, qx.alpha_row, qw.codes_row, qw.scales_row,
                                          qw.alpha_row, out=step.y), 20, flush)
    fl = 2.0 * TOKENS * OUT * HIDDEN
    extras["nvfp4_gemm_alone"] = {"shape": "8192x14336x4096", "us": round(ms * 1e3, 2),
                                  "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / fp4_peak,
                                  "frac_datasheet": fl / (ms * 1e-3) / 1e12 / FP4_DATASHEET_TFLOPS}
    mx_x = api.mxfp4_quantize(x, ROW | GEMM)
    mx_w = api.mxfp4_quantize(w, ROW | GEMM)
    ms = time_call(lambda: api.mxfp4_gemm(mx_x.codes_row, mx_x.scales_row, mx_w.codes_row, mx_w.scales_row,
                                          out=step.y), 20, flush)
    extras["mxfp4_gemm"] = {"shape": "8192x14336x4096", "us": round(ms * 1e3, 2),
                            "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / fp4_peak,
                            "frac_datasheet": fl / (ms * 1e-3) / 1e12 / FP4_DATASHEET_TFLOPS}
    del mx_x, mx_w
    # the 12B-hybrid-shaped step: tokens 16384, hidden 5120, FFN 20480
    s = synthetic.STEP_12B
    lay = synthetic.device_layer(s["tokens"], s["hidden"], s["ffn"], seed=12, device=device)
    st12 = LayerStep(lay["x"], lay["w"], lay["dy"], BWD_MODES[args.bwd_mode], device,
                     shared_amax=not args.amax_per_call)
    for i in range(3):
        st12.run(i)
    torch.cuda.synchronize()
    extras["step12b"] = {"workload": "12B-hybrid-shaped linear fwd+bwd: X 16384x5120, W 20480x5120, "
                                     f"dY 16384x20480 ({BWD_NAMES[args.bwd_mode]}), one stream",
                         **step_breakdown(st12, 20, hbm, fp4_peak)}
    del st12, lay
    torch.cuda.empty_cache()
    extras["sweep"] = {"timing": "CUDA events, L2 overwritten before each call, median of 10 (3 for N >= 65536)",
                       "columns": ["two_pass", "single_pass"],
                       "data": "device-drawn N(0,1) with 0.1% channel outliers x50 (torch CUDA generator)",
                       **sweep_table(api, hbm, flush, device)}
    return extras


# --------------------------------------------------------------------------
# the CPU oracle on a bounded sample of the same step
# --------------------------------------------------------------------------
@functools.lru_cache(maxsize=4)
def _sample_tensors(budget_rows):
    from nvfp4_block_quantization_amax_b200 import synthetic
    return (synthetic.bf16_bits(synthetic.normal_with_channel_outliers(budget_rows * 16, HIDDEN, seed=0)),
            synthetic.bf16_bits(synthetic.weight(budget_rows * 16, HIDDEN, seed=1)),
            synthetic.bf16_bits(synthetic.laplace_with_spikes(budget_rows * 16, OUT, seed=2)))


def oracle_sample(budget_rows=64, gemm_rows=16, gemm_cols=16, bwd_mode="eden"):
    """Time the oracle on a sample of every part of the step and extrapolate
    to one full step.  Returns (step_seconds_extrapolated, sample description,
    threads)."""
    import numpy as np
    import oracle
    from nvfp4_block_quantization_amax_b200 import synthetic
    rng = np.random.default_rng(0)
    xb, wb, dyb = _sample_tensors(budget_rows)
    bwd = BWD_MODES[bwd_mode]
    t_total = 0.0
    parts = []

    def timed(fn):
        t0 = time.perf_counter()
        r = fn()
        return time.perf_counter() - t0, r

    # quantize parts: sample tensors of (budget_rows*16) rows, scaled by rows
    for name, bits, mode, flags, full_rows in [
            ("X 4/6 rows", xb, FOUR_SIX, ROW, TOKENS), ("W 4/6 2D", wb, FOUR_SIX, ROW | B2D, OUT),
            ("dY rows+cols", dyb, bwd, ROW | COL, TOKENS), ("W rot cols", wb, RTN, COL | RHT, OUT),
            ("X rot cols", xb, RTN, COL | RHT, TOKENS)]:
        dt, _ = timed(lambda: oracle.quantize(bits, mode, flags, seed=1))
        scale = full_rows / bits.shape[0]
        t_total += dt * scale
        parts.append(f"{name}: {bits.shape[0]}x{bits.shape[1]}")
    # GEMM parts: FP64 reference on gemm_rows x gemm_cols outputs at full K
    for (M, N, K) in [(TOKENS, OUT, HIDDEN), (TOKENS, HIDDEN, OUT), (OUT, HIDDEN, TOKENS)]:
        A = rng.integers(0, 256, (gemm_rows, K // 2), dtype=np.uint8)
        B = rng.integers(0, 256, (gemm_cols, K // 2), dtype=np.uint8)
        sA = rng.integers(0x28, 0x48, (gemm_rows, K // 16), dtype=np.uint8)
        sB = rng.integers(0x28, 0x48, (gemm_cols, K // 16), dtype=np.uint8)
        dt, _ = timed(lambda: oracle.gemm_f64(A, sA, 1.0, B, sB, 1.0, gemm_rows, gemm_cols, K))
        t_total += dt * (M * N) / (gemm_rows * gemm_cols)
        parts.append(f"GEMM {gemm_rows}x{gemm_cols} of {M}x{N}, K={K}")
    threads = omp_threads()
    desc = ("oracle timed on " + "; ".join(parts) + "; each part scaled to the full step by its element count "
            "(extrapolated)")
    return t_total, desc, threads


def _gomp():
    import ctypes
    import oracle
    oracle.lib()   # loads the oracle and with it the OpenMP runtime it links
    try:
        return ctypes.CDLL("libgomp.so.1")
    except OSError:
        return None


def omp_threads():
    g = _gomp()
    return int(g.omp_get_max_threads()) if g is not None else 1


class single_threaded:
    """Run the oracle's OpenMP regions on one thread inside the block."""

    def __enter__(self):
        self.g = _gomp()
        self.n = omp_threads()
        if self.g is not None:
            self.g.omp_set_num_threads(1)
        return self

    def __exit__(self, *a):
        if self.g is not None:
            self.g.omp_set_num_threads(self.n)
        return False


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    t_step = []
    desc = threads = None
    # each step is a bounded sample: 1024-row slices for a short run, fewer
    # rows (down to 16) when many steps are asked for, so that the whole run
    # stays within a few minutes
    budget_rows = max(1, min(64, (64 * 32) // (args.warmup + args.steps)))
    for i in range(args.warmup + args.steps):
        dt, desc, threads = oracle_sample(budget_rows=budget_rows, bwd_mode=args.bwd_mode)
        if i >= args.warmup:
            t_step.append(dt)
    s = statistics.mean(t_step)
    v = gemm_flops() / s / 1e12
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer, f64 GEMM (CPU oracle)",
            "data": "synthetic", "config": {"workload": workload(args.bwd_mode), "bwd_mode": args.bwd_mode},
            "extrapolated": True,
            "note": "each step times the oracle on bounded slices of the step and scales every part to the "
                    "full step by its element count: ms_per_step is an extrapolation, not a measured run",
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
                             "extrapolated": True},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline_line(bwd_mode):
    dt, desc, threads = oracle_sample(bwd_mode=bwd_mode)
    with single_threaded():
        dt1, desc1, _ = oracle_sample(budget_rows=16, bwd_mode=bwd_mode)
    return {"value": gemm_flops() / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": desc, "extrapolated": True, "step_seconds_extrapolated": dt,
            "single_thread": {"value": gemm_flops() / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                              "sample": desc1, "extrapolated": True, "step_seconds_extrapolated": dt1}}


KERNEL_CASES = ("gemm_fprop", "gemm_dgrad", "gemm_wgrad", "quant_x", "quant_w2d", "quant_dy", "quant_dy_sr",
                "quant_dy_sr_hw", "quant_w_rot", "quant_x_rot", "mx_dy", "mx_gemm_fprop")


def run_kernel_case(name, iters=3):
    """Run one C-ABI call of the step a few times on its full-size inputs
    (the small, single-kernel command that profiler captures use)."""
    import torch
    from nvfp4_block_quantization_amax_b200 import synthetic
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    layer = synthetic.fwd_bwd_8b(seed=0)
    x, w, dy = (layer[k].to(device) for k in ("x", "w", "dy"))
    step = LayerStep(x, w, dy, MS_EDEN, device)
    step.run(0)  # produce every operand once
    torch.cuda.synchronize()
    api = step.api
    qx, qw, qd, qwr, qxr = (step.out[k] for k in ("x", "w", "dy", "w_rot", "x_rot"))
    mx = {}
    if name == "mx_gemm_fprop":   # MXFP4 operands of the fprop GEMM (GEMM scale layout)
        mx["x"] = api.mxfp4_quantize(x, ROW | GEMM)
        mx["w"] = api.mxfp4_quantize(w, ROW | GEMM)
    calls = {
        "gemm_fprop": lambda: api.nvfp4_gemm(qx.codes_row, qx.scales_row, qx.alpha_row, qw.codes_row,
                                             qw.scales_row, qw.alpha_row, out=step.y),
        "gemm_dgrad": lambda: api.nvfp4_gemm(qd.codes_row, qd.scales_row, qd.alpha_row, qwr.codes_col,
                                             qwr.scales_col, qwr.alpha_col, out=step.dx),
        "gemm_wgrad": lambda: api.nvfp4_gemm(qd.codes_col, qd.scales_col, qd.alpha_col, qxr.codes_col,
                                             qxr.scales_col, qxr.alpha_col, out=step.dw),
        "quant_x": lambda: step.quantize("x", FOUR_SIX, ROW | GEMM, 0, 0),
        "quant_w2d": lambda: step.quantize("w", FOUR_SIX, ROW | B2D | GEMM, 0, 1),
        "quant_dy": lambda: step.quantize("dy", MS_EDEN, ROW | COL | GEMM, 7, 0),
        "quant_dy_sr": lambda: step.quantize("dy", RHT_SR, ROW | COL | GEMM, 7, 0),
        "quant_dy_sr_hw": lambda: step.quantize("dy", RHT_SR_HW, ROW | COL | GEMM, 7, 0),
        "quant_w_rot": lambda: step.quantize("w_rot", RTN, COL | RHT | GEMM, 7, 1),
        "quant_x_rot": lambda: step.quantize("x_rot", RTN, COL | RHT | GEMM, 7, 2),
        "mx_dy": lambda: api.mxfp4_quantize(dy, ROW | COL | RHT, seed=7),
        "mx_gemm_fprop": lambda: api.mxfp4_gemm(mx["x"].codes_row, mx["x"].scales_row, mx["w"].codes_row,
                                                mx["w"].scales_row, out=step.y),
    }
    for _ in range(iters):
        calls[name]()
    torch.cuda.synchronize()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--bwd-mode", choices=sorted(BWD_MODES), default="eden")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--amax-per-call", action="store_true",
                    help="every quantize call runs its own amax pass (default: one nvfp4_amax pass per X and W "
                         "serves their forward and rotated backward quantizations)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sub-benchmarks (per-mode table, sweep, 12B step, GEMMs alone)")
    ap.add_argument("--kernel-case", choices=KERNEL_CASES,
                    help="run one call of the step a few times and exit (for profiler captures)")
    args = ap.parse_args(argv)
    if args.kernel_case:
        run_kernel_case(args.kernel_case)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        r = run_reference(args)
        if r is not None:
            print(json.dumps(r), flush=True)
        return 0
    rank, world, local_rank = dist_env()
    init_dist("nccl" if world > 1 else "gloo")
    res = run_device(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_line(args.bwd_mode)
        print(json.dumps(res), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
