"""Benchmark of binarized-QK top-N attention (HAD + BinaryAttention) on B200.

Default workload: the long-sequence stress configuration with HAD's top-N
selection (B2 H16 n16384 d64 bf16 -- a 1024x1024 image at 8x8 patches --
relative-position bias 255x255 per head, top-1920 per query, float softmax and
A.V), the largest single-GPU configuration of the metric.  Other workloads are
selected with --workload.  A "step" is one pass of the whole hot path over one
batch: channel means + sign/pack of Q and K (+ int8 V), bias tables, scores,
logits, top-N, softmax, A.V, output.  Metric: queries/s = valid (batch, head,
query) rows per second over all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Timing: W untimed warm-up steps; K timed steps, each bracketed by CUDA events
on the launching stream, with an L2 flush (a 256 MiB write, larger than the
126 MB L2) between steps outside the events; barrier + synchronize on both
sides; the reported time is the max over ranks.  A step replays two CUDA graphs
captured from the library's two stages (had_attention_prepare /
had_attention_prepared) on that stream; the fused kernel's own time comes from
the events between them.

Roofline of the fused kernel (the method's own definition): the slower of its
algorithmic HBM bytes at the measured copy bandwidth and its score contraction
(2 d int8 ops per valid score) at the int8 tensor-pipe peak; the fraction is
that time over the measured kernel time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "binary-QK top-N attention queries/sec on 1 B200; % of roofline (HBM or int pipe)"
UNIT = "queries/s"

# (workload name, N, mode) per bench workload id
WORKLOADS = {
    "deit": ("deit", 0, "u8i8"),
    "deit_dense_bias": ("deit_dense_bias", 0, "u8i8"),
    "tiny": ("tiny", 15, "float"),
    "bert": ("bert", 30, "float"),
    "t5_128": ("t5_128", 15, "float"),
    "t5_256": ("t5_256", 30, "float"),
    "t5_512": ("t5_512", 60, "float"),
    "t5_1024": ("t5_1024", 120, "float"),
    "stress_topn": ("stress", 1920, "float"),
    "stress_u8i8": ("stress", 0, "u8i8"),
    # head dim 128 (the BinaryAttention kernel benchmark's head dim)
    "deit_d128": ("deit_d128", 0, "u8i8"),
    # 4-bit V (uint8 A x per-channel 4-bit V, two codes per byte)
    "deit_u8i4": ("deit", 0, "u8i4"),
    "stress_u8i4": ("stress", 0, "u8i4"),
    "stress_topn_u8i4": ("stress", 1920, "u8i4"),
    "t5_1024_d128": ("t5_1024_d128", 120, "float"),
    # the library's dense comparison mode: standard bf16 attention on the unbinarized inputs
    "deit_dense_ref": ("deit", 0, "ref"),
    "t5_1024_dense_ref": ("t5_1024", 0, "ref"),
    "stress_dense_ref": ("stress", 0, "ref"),
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
        "fallback"


HEAD_STAGE_BYTES = 128 * 1024  # heads up to this size are prepared by one kernel from shared memory


def launches_per_step(n: int, elem: int, mode: str, has_bias: bool, dense_bias: bool = False, d: int = 64) -> int:
    """Kernels one prepare + attend step launches: the sign/pack stage (one
    kernel for short heads, which also builds relative-position bias tables;
    otherwise statistics, their per-head finalization and the pack, plus the
    bias range and the table fill), the range and tables of a dense bias
    matrix (two kernels), the hi/lo split of an fp32 V (float mode), and the
    fused attention."""
    rel = has_bias and not dense_bias
    k = 1 if (d == 64 and n * 64 * elem <= HEAD_STAGE_BYTES) else 3 + (2 if rel else 0)
    if dense_bias:
        k += 2
    if mode == "float" and elem == 4:
        k += 1
    return k + 1


def relpos_table_launches(gh: int, gw: int) -> int:
    """Kernels that build a relative-position table's extended tables outside the
    prepare stage (the fused projection, the dense comparison mode): one CTA per
    head for tables of at most 8192 extended entries, else the range and a fill
    over many CTAs per head.  The extended size is E = 3T + 3K_x rounded up to 4,
    T = (2gh - 1) S, K_x = (gh - 1) S + gw, S the smallest row stride >= 2gw - 1
    with S = gw (mod 32)."""
    S = 2 * gw - 1
    while S % 32 != gw % 32:
        S += 1
    T, Kx = (2 * gh - 1) * S, (gh - 1) * S + gw
    E = (3 * T + 3 * Kx + 3) // 4 * 4
    return 1 if E <= 8192 else 2


# Issue-limited CUDA-core rate of one B200: 148 SMs x 4 schedulers x 32 lanes x
# 1965 MHz (clocks.max.sm), one lane-operation per lane per clock.  A derived
# ceiling for the diagnostic ALU roofline, not a measured peak.
ALU_PEAK_TOPS = 148 * 4 * 32 * 1.965e9 / 1e12

# tensor-pipe dense rates relative to bf16 (the nominal 4.5 / 2.25 PFLOP/s of int8 / bf16)
INT8_PER_BF16 = 2.0


def score_tensor_ops(valid_scores: int, d: int = 64) -> float:
    """Operations of the score contraction on the tensor pipe: one d-element
    +-1 int8 dot product per valid (query, key) pair = 2 d ops."""
    return 2.0 * d * valid_scores


def method_roofline(kbytes: float, tensor_ops: float, kernel_ms: float, hbm_gbs: float, i8_tops: float) -> dict:
    """The fused kernel's roofline as the method defines it: the slower of its
    algorithmic HBM bytes at the measured bandwidth and its score contraction at
    the int8 tensor-pipe peak.  frac = that time / the measured kernel time."""
    t_hbm = kbytes / (hbm_gbs * 1e9)
    t_tc = tensor_ops / (i8_tops * 1e12)
    t = kernel_ms * 1e-3
    if t_tc >= t_hbm:
        return {"bound": "tensor", "achieved": tensor_ops / t / 1e12, "peak": i8_tops, "unit": "TOPS (int8)",
                "frac": t_tc / t, "t_roof_ms": t_tc * 1e3, "t_hbm_ms": t_hbm * 1e3, "t_tensor_ms": t_tc * 1e3}
    return {"bound": "hbm", "achieved": kbytes / t / 1e9, "peak": hbm_gbs, "unit": "GB/s", "frac": t_hbm / t,
            "t_roof_ms": t_hbm * 1e3, "t_hbm_ms": t_hbm * 1e3, "t_tensor_ms": t_tc * 1e3}


def alu_ops_per_score(mode: str, N: int, n: int, has_bias: bool) -> float:
    """CUDA-core operations per valid (query, key) pair that the fused kernel's
    formulation cannot avoid (address arithmetic, loop control and the tensor-core
    work not counted).  Dense (N = 0 or N >= n): the weight of a score is a
    level-table lookup, times an exp(bias) lookup when there is a bias; uint8
    mode needs the normalizer first, so it computes the weight twice (sum, then
    scale-round-convert and a quarter of a byte pack); float mode sums in the
    same pass and packs half a bf16 pair.  Top-N without a bias: one histogram
    increment, then lookup, tie test, select and the pack.  Top-N with a bias:
    one histogram increment (on one tile in eight when a row has 64 tiles or
    more: the sampled level pass), the float-binned pass (bias load, logit FMA,
    the saturating bin map, the address, increment) and the output pass
    (load, FMA, two compares, exp as FFMA + ex2, select, pack)."""
    dense = N == 0 or N >= n
    quant = mode in ("u8i8", "u8i4")
    if dense:
        if quant:
            w = 3.0 if has_bias else 1.0
            return (w + 1.0) + (w + 2.25)
        return (3.0 if has_bias else 1.0) + 1.0 + 0.5
    if not has_bias:
        return 1.0 + (3.0 + (2.25 if quant else 0.5))
    return (0.125 if -(-n // 64) >= 64 else 1.0) + 6.0 + 7.5


def kernel_bytes_per_token(mode: str, v_bytes: int, o_bytes: int, d: int = 64) -> int:
    """Algorithmic bytes per valid token of the fused kernel.

    Reads the packed sign bits of Q and K (d / 8 B each), V (float mode,
    d * v_bytes), int8 V (d bytes) or 4-bit V (d / 2 bytes), and writes O
    (d * o_bytes).
    The comparison mode ("ref") reads the bf16 Q, K and V and writes O.
    """
    if mode == "ref":
        return 3 * d * v_bytes + d * o_bytes
    v = d if mode == "u8i8" else d // 2 if mode == "u8i4" else d * v_bytes
    return d // 8 + d // 8 + v + d * o_bytes


def path_bytes_per_token(mode: str, in_bytes: int, o_bytes: int, d: int = 64) -> int:
    """Algorithmic bytes per token of the whole path: read Q, K, V once, write and
    read back the packed bits (and the int8 or 4-bit V in the uint8 modes), write O once."""
    if mode == "ref":
        return 3 * d * in_bytes + d * o_bytes
    b = 3 * d * in_bytes + 2 * (d // 8) * 2 + d * o_bytes
    if mode == "u8i8":
        b += 2 * d
    elif mode == "u8i4":
        b += d
    return b


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The max of a per-rank scalar over all ranks of the process group (the
    value itself without one).  Every multi-GPU time is reported this way."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank processes `units_per_rank` per step (weak
    scaling), and the job takes the slowest rank's time."""
    return units_per_rank * world * steps / (total_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons; only the samples
    whose timestamps fall inside the timed region are summarized."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clk", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.period)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    @staticmethod
    def _stamp(txt):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(txt.strip(), fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self, t0=None, t1=None):
        """Stop sampling; summarize the samples taken in [t0, t1] (wall-clock
        seconds since the epoch), or all of them without a window."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, n_all = [], None, set(), 0
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 10:
                    continue
                n_all += 1
                ts = self._stamp(f[0])
                if t0 is not None and (ts is None or ts < t0 or ts > t1):
                    continue
                try:
                    sm.append(float(f[2]))
                    smax = float(f[3])
                except ValueError:
                    continue
                for k, v in zip(self.NAMES, f[6:10]):
                    if v.lower().startswith("active"):
                        reasons.add(k)
            os.unlink(self.path)
        except Exception:
            pass
        if not sm:
            return None
        loaded = [x for x in sm if smax is None or x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "period_ms": self.period}


# ----------------------------------------------------------------------------- the oracle on the host cores

def _oracle_bias(oracle, w):
    if w.bias is None:
        return None
    if isinstance(w.bias, workloads.DenseBias):
        return oracle.DenseBias(w.bias.table)
    return oracle.RelPosBias(w.bias.table, w.bias.gh, w.bias.gw, w.bias.prefix)


def _bias_desc(w):
    if w.bias is None:
        return None
    if isinstance(w.bias, workloads.DenseBias):
        return f"dense {w.bias.table.shape[1]}x{w.bias.table.shape[2]}/head"
    return f"relpos {w.bias.table.shape[1]}x{w.bias.table.shape[2]}/head, prefix {w.bias.prefix}"


def _oracle_call_s(w, N, mode, rows):
    """Seconds of one oracle call over the given query rows (plus its whole-workload
    prelude: channel means, sign bits and int8 V of every head)."""
    import oracle
    b = _oracle_bias(oracle, w)
    t0 = time.perf_counter()
    if mode == "ref":
        oracle.dense_attention(w.Q, w.K, w.V, seqlens=w.seqlens, bias=b, rows=rows)
    else:
        oracle.attention(w.Q, w.K, w.V, N=N, mode={"u8i8": 1, "u8i4": 2}.get(mode, 0), seqlens=w.seqlens, bias=b,
                         rows=rows)
    return time.perf_counter() - t0


def _valid_rows(w):
    rows = []
    for bh in range(w.B * w.H):
        L = w.n if w.seqlens is None else int(w.seqlens[bh // w.H])
        rows.append(np.arange(bh * w.n, bh * w.n + L, dtype=np.int64))
    return np.concatenate(rows)


def oracle_rate(prelude_s: float, row_s: float, total_rows: int) -> float:
    """Whole-workload oracle rate from its two measured parts: the prelude (run
    once per workload) and the per-row time (the slope over sampled rows)."""
    return total_rows / (prelude_s + row_s * total_rows)


def _oracle_parts(w, N, mode, budget_s, seed):
    """Prelude seconds (a call with no rows) and per-row seconds (slope between
    two seeded samples of m and 2m rows), with m sized to the budget."""
    allrows = _valid_rows(w)
    rng = np.random.default_rng(seed)
    pre = min(_oracle_call_s(w, N, mode, np.zeros(0, np.int64)) for _ in range(2))
    probe = np.sort(rng.choice(allrows, size=min(len(allrows), 256), replace=False))
    t = _oracle_call_s(w, N, mode, probe)
    per_row = max(t - pre, 1e-9) / len(probe)
    m = int(max(256, min(len(allrows) // 2, (budget_s / 3.0) / per_row)))
    r1 = np.sort(rng.choice(allrows, size=m, replace=False))
    r2 = np.sort(rng.choice(allrows, size=min(len(allrows), 2 * m), replace=False))
    t1, t2 = _oracle_call_s(w, N, mode, r1), _oracle_call_s(w, N, mode, r2)
    per_row = max((t1 + t2 - 2.0 * pre) / (len(r1) + len(r2)), 1e-12)
    return pre, per_row, (len(r1), len(r2)), len(allrows)


def cpu_baseline(w, N, mode, budget_s=15.0):
    """The oracle as it stands, on the host cores: whole-workload queries/s from
    its prelude time and its per-row time over a bounded seeded sample."""
    import oracle
    pre, per_row, sampled, total = _oracle_parts(w, N, mode, budget_s, 99)
    return {"value": oracle_rate(pre, per_row, total), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"two seeded samples of {sampled[0]} and {sampled[1]} of the {total} query rows of {w.name}; "
                      f"prelude (means, "
                      f"sign bits, int8 V of every head) {pre:.3f} s once, {per_row * 1e3:.4f} ms per row; "
                      f"value extrapolated to all {total} rows"}


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands on the host cores.  Each step runs
    the oracle's prelude and a bounded seeded sample of rows; the value is the
    whole-workload rate from the prelude time and the per-row slope."""
    if rank != 0:
        return 0
    import oracle
    name, N, mode = WORKLOADS[args.workload]
    w = workloads.by_name(name)
    allrows = _valid_rows(w)
    rng = np.random.default_rng(7)
    pre = min(_oracle_call_s(w, N, mode, np.zeros(0, np.int64)) for _ in range(2))
    probe = np.sort(rng.choice(allrows, size=min(len(allrows), 256), replace=False))
    per_row = max(_oracle_call_s(w, N, mode, probe) - pre, 1e-9) / len(probe)
    budget = 90.0 / max(1, args.steps + args.warmup)
    per_step = int(max(64, min(len(allrows), (budget - pre) / per_row)))
    times = []
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(allrows, size=per_step, replace=False))
        dt = _oracle_call_s(w, N, mode, rows)
        if s >= args.warmup:
            times.append(dt)
    per_row = max((sum(times) - len(times) * pre) / (len(times) * per_step), 1e-12)
    value = oracle_rate(pre, per_row, len(allrows))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, N, mode),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{per_step} seeded query rows of {w.name} per step (+ the prelude); "
                                       f"prelude {pre:.3f} s, {per_row * 1e3:.4f} ms per row; value extrapolated "
                                       f"to all {len(allrows)} rows"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _sliced(w, args):
    """The first --batch sequences and --heads heads of a workload (a smaller case of
    the same kernel variant, for profiler captures); the whole workload by default."""
    B = args.batch or w.B
    H = args.heads or w.H
    if B == w.B and H == w.H:
        return w
    bias = w.bias
    if bias is not None:
        bias = type(bias)(bias.table[:H], *[getattr(bias, f) for f in ("gh", "gw", "prefix") if hasattr(bias, f)])
    cut = lambda x: np.ascontiguousarray(x[:B, :H])  # noqa: E731
    return workloads.Workload(f"{w.name}_slice_b{B}_h{H}", B, H, w.n, w.d, w.dtype, cut(w.Q), cut(w.K), cut(w.V),
                              None if w.seqlens is None else w.seqlens[:B], bias, w.passes, w.seed, w.recipe)


def _config(w, N, mode):
    tag = "dense_ref" if mode == "ref" else f"{'dense' if N == 0 else f'top{N}'}_{mode}"
    return {"workload": f"{w.name}_{tag}", "B": w.B, "H": w.H, "n": w.n,
            "d": w.d, "N": N, "mode": mode, "in_dtype": w.dtype, "seed": w.seed,
            "bias": _bias_desc(w),
            "seqlens": None if w.seqlens is None else "U{32..256} per sequence",
            "l2": "flushed between timed steps (256 MiB write)"}


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world, local_rank):
    import torch
    import binarized_qk_sparse_b200 as had

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
    name, N, mode = WORKLOADS[args.workload]
    w = _sliced(workloads.by_name(name), args)
    bf16 = w.dtype == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float32

    def dev_t(x):
        return torch.from_numpy(x).to(tdt).to(dev)

    Q, K, V = dev_t(w.Q), dev_t(w.K), dev_t(w.V)
    seq = None if w.seqlens is None else torch.from_numpy(w.seqlens).to(dev)
    bias = None
    if isinstance(w.bias, workloads.DenseBias):
        bias = had.DenseBias(torch.from_numpy(w.bias.table).to(dev))
    elif w.bias is not None:
        bias = had.RelPosBias(torch.from_numpy(w.bias.table).to(dev), w.bias.gh, w.bias.gw, w.bias.prefix)
    O = torch.empty_like(V)
    ref = mode == "ref"
    if ref:
        ws_bytes = max(16, had.had_dense_reference_workspace_size(Q, seq, bias))
    else:
        ws_bytes = had.had_attention_workspace_size(Q, N, mode, seq, bias)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    L = had.lib()
    import ctypes
    shp = had.make_shape(Q, seq)
    bstruct = None if bias is None else ctypes.byref(had._bias_c(bias))
    mcode = had._MODES[mode] if not ref else 0
    sp = ctypes.c_void_p(stream.cuda_stream)

    def prepare():
        if ref:
            return
        st = L.had_attention_prepare(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                     ctypes.c_void_p(V.data_ptr()), ctypes.byref(shp), bstruct, N, mcode,
                                     ctypes.c_void_p(ws.data_ptr()), ws_bytes, sp)
        if st:
            raise had.HadError(st, "had_attention_prepare")

    def attend():
        if ref:
            st = L.had_dense_reference_mode(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                            ctypes.c_void_p(V.data_ptr()), ctypes.byref(shp), bstruct, 0,
                                            ctypes.c_void_p(O.data_ptr()), had._dtype_code(O),
                                            ctypes.c_void_p(ws.data_ptr()), ws_bytes, sp)
            if st:
                raise had.HadError(st, "had_dense_reference_mode")
            return
        st = L.had_attention_prepared(ctypes.c_void_p(V.data_ptr()), ctypes.byref(shp), bstruct, None, None, N, mcode,
                                      ctypes.c_void_p(O.data_ptr()), had._dtype_code(O),
                                      ctypes.c_void_p(ws.data_ptr()), ws_bytes, sp)
        if st:
            raise had.HadError(st, "had_attention_prepared")

    # the tensor pipe's int8 and bf16 MMA rates on this GPU (probe kernel, before the workload)
    probe_i8, _ = had.had_probe_mma_rate("i8", 40000)      # ~2.6 ms per launch
    probe_bf16, _ = had.had_probe_mma_rate("bf16", 20000)

    if ref:  # the bias tables (range + tables for a dense matrix) and the kernel
        kernels_per_step = 1 + (0 if bias is None else (2 if isinstance(w.bias, workloads.DenseBias)
                                                        else relpos_table_launches(w.bias.gh, w.bias.gw)))
    else:
        kernels_per_step = launches_per_step(w.n, Q.element_size(), mode, bias is not None,
                                             isinstance(w.bias, workloads.DenseBias), w.d)
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    clocks.start()  # nvidia-smi takes a moment to start: launched before the warm-up
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            prepare()
            attend()
        stream.synchronize()
        assert had.had_get_device_status() == had.HAD_OK
        # each step replays two CUDA graphs captured from the same calls (the prepare
        # stage, then the fused kernel), so that the host's per-call work (argument
        # marshalling, tensor-map encoding, launch) never leaves the GPU idle inside
        # the timed steps; the graphs hold exactly the kernels a call launches
        g_prep, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_prep, stream=stream):
            prepare()
        with torch.cuda.graph(g_attn, stream=stream):
            attend()
        g_prep.replay()
        g_attn.replay()
        stream.synchronize()
        assert had.had_get_device_status() == had.HAD_OK

        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        wall0 = time.time()
        for s in range(args.steps):
            flush.zero_()
            ev[s][0].record(stream)
            g_prep.replay()
            ev[s][1].record(stream)
            g_attn.replay()
            ev[s][2].record(stream)
        torch.cuda.synchronize()
        wall1 = time.time()
        if dist is not None:
            dist.barrier()
    clk = clocks.stop(wall0, wall1)
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    queries = w.valid_tokens
    value = whole_job_rate(queries, world, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    # e2e: the host-array entry point, every step -- it copies the step's Q, K, V
    # (and seqlens, bias table) in from pinned host memory and O out, in chunks of
    # the batch that overlap copy-in, compute and copy-out
    hQ, hK, hV = Q.cpu().pin_memory(), K.cpu().pin_memory(), V.cpu().pin_memory()
    hO = torch.empty_like(O, device="cpu").pin_memory()
    hseq = None if seq is None else seq.cpu()
    hbias = None
    if isinstance(bias, had.DenseBias):
        hbias = had.DenseBias(bias.table.cpu().pin_memory())
    elif bias is not None:
        hbias = had.RelPosBias(bias.table.cpu().pin_memory(), bias.gh, bias.gw, bias.prefix)
    if not ref:
        host_ws = torch.empty(had.had_attention_host_workspace_size(hQ, N, mode, hseq, hbias), dtype=torch.uint8,
                              device=dev)
    e2e_steps = max(3, min(args.steps, 30))
    h2d = 3 * Q.numel() * Q.element_size() + (0 if hseq is None else hseq.numel() * 4) + \
        (0 if hbias is None else hbias.table.numel() * 4)
    d2h = O.numel() * O.element_size()
    with torch.cuda.stream(stream):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for s in range(e2e_steps + 2):
            if s == 2:
                e0.record(stream)
            if ref:  # no host entry point: copies in, the call, the copy out, on the same stream
                Q.copy_(hQ, non_blocking=True)
                K.copy_(hK, non_blocking=True)
                V.copy_(hV, non_blocking=True)
                if hbias is not None:
                    bias.table.copy_(hbias.table, non_blocking=True)
                attend()
                hO.copy_(O, non_blocking=True)
            else:
                had.had_attention_host(hQ, hK, hV, N=N, mode=mode, seqlens=hseq, bias=hbias, out=hO,
                                       workspace=host_ws, stream=stream, synchronize=False)
        e1.record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, dev)

    if rank != 0:
        return 0
    peaks, peak_kind = _peaks()
    attn_avg_ms = statistics.mean(attn_ms)
    kbytes = kernel_bytes_per_token(mode, 2 if bf16 else 4, O.element_size(), w.d) * queries
    if bias is not None:
        kbytes += w.bias.table.nbytes
    if ref:  # standard attention: the bf16 QK^T and P.V contractions at the bf16 peak
        tc_ops = 2.0 * score_tensor_ops(w.valid_scores(), w.d)
        tc_peak = max(peaks["bf16_tflops"], probe_bf16)
        peak_txt = f"bf16 = max({peak_kind} burst {peaks['bf16_tflops']} TFLOP/s, probe {probe_bf16:.0f})"
    else:
        tc_ops = score_tensor_ops(w.valid_scores(), w.d)
        tc_peak = max(INT8_PER_BF16 * peaks["bf16_tflops"], probe_i8)
        peak_txt = (f"int8 = max({INT8_PER_BF16:g} x {peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s, "
                    f"probe {probe_i8:.0f} TOPS)")
    roof = method_roofline(kbytes, tc_ops, attn_avg_ms, peaks["hbm_gbs"], tc_peak)
    if ref:
        roof["unit"] = roof["unit"].replace("int8", "bf16")
    traffic = None
    tr_path = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tr_path):
        with open(tr_path) as f:
            traffic = json.load(f).get(args.workload)
    roof.update({"traffic": traffic, "kernel": "k_attn_tc (fused score/top-N/softmax/A.V)",
                 "avg_launch_ms": attn_avg_ms, "algorithmic_bytes_per_launch": kbytes,
                 "tensor_ops_per_launch": tc_ops,
                 "peak_kind": f"{peak_txt}; HBM {peak_kind} {peaks['hbm_gbs']} GB/s"})
    ops_per_score = 0.0 if ref else alu_ops_per_score(mode, N, w.n, bias is not None)
    alu_ops = ops_per_score * w.valid_scores()
    alu_achieved = alu_ops / (attn_avg_ms * 1e-3) / 1e12
    pbytes = path_bytes_per_token(mode, 2 if bf16 else 4, O.element_size(), w.d) * queries
    path_achieved = pbytes / (ms_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": mode if mode in ("u8i8", "u8i4") else ("bf16" if bf16 else "f32"),
        "data": "synthetic", "config": _config(w, N, mode),
        "parallelism": f"replicas x{world} (no collective)",
        "launch": "each step replays CUDA graphs of the two library calls (prepare, attend)",
        "score_ops_per_s": whole_job_rate(w.valid_scores(), world, args.steps, total_ms),
        "roofline": roof,
        "tensor_pipe_probe": {"i8_tops": probe_i8, "bf16_tflops": probe_bf16,
                              "kernel": "k_probe_mma: M128 N256 tcgen05.mma back to back, operands in shared memory"},
        "roofline_alu": {"bound": "alu", "achieved": alu_achieved, "peak": ALU_PEAK_TOPS, "unit": "Tlane-op/s",
                         "frac": alu_achieved / ALU_PEAK_TOPS, "ops_per_valid_score": ops_per_score,
                         "peak_kind": "derived issue ceiling: 148 SMs x 4 schedulers x 32 lanes x 1965 MHz; "
                                      "ops per score are this library's own count (diagnostic)"},
        "roofline_path": {"bound": "hbm", "achieved": path_achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": path_achieved / peaks["hbm_gbs"], "algorithmic_bytes_per_step": pbytes},
        "e2e": {"value": whole_job_rate(queries, world, 1, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": kernels_per_step * args.steps,
        "clocks": clk,
        "timed_region_s": wall1 - wall0,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, N, mode)
    print(json.dumps(line), flush=True)
    return 0


QKV_WORKLOAD = "deit_qkv"


def run_qkv(args, rank, world, local_rank):
    """DeiT's attention from its inputs' projection (B64 n197, model width 768, 12
    heads, relative-position bias, dense uint8 A x int8 V): the fused path
    (had_qkv_prepare: the projection with Q and K binarized in its epilogue, then the
    fused attention) against the unfused one on the same box (a cuBLAS projection,
    the copy into [B, H, n, d] heads, the library's prepare stage, the same attention).
    One JSON line; the fused path is the line's value."""
    import ctypes
    import torch
    import binarized_qk_sparse_b200 as had
    from binarized_qk_sparse_b200 import _build
    _build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    X, W, H, bw, _ = workloads.deit_qkv()
    B, n, Dm = X.shape
    d, N, mode = 64, 0, "u8i8"
    Xd = torch.from_numpy(X).to(torch.bfloat16).to(dev)
    Wd = torch.from_numpy(W).to(torch.bfloat16).to(dev)
    bias = had.RelPosBias(torch.from_numpy(bw.table).to(dev), bw.gh, bw.gw, bw.prefix)
    L = had.lib()
    shp = had.had_shape(B, H, n, d, had.HAD_BF16, None)
    bst = had._bias_c(bias)
    bs = ctypes.byref(bst)
    mcode = had._MODES[mode]
    sp_stream = torch.cuda.Stream(device=dev)
    sp = ctypes.c_void_p(sp_stream.cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    ws_q = torch.empty(L.had_qkv_workspace_size(ctypes.byref(shp), Dm, N, mcode, bs), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(L.had_attention_workspace_size(ctypes.byref(shp), N, mcode, bs), dtype=torch.uint8, device=dev)
    V = torch.empty((B, H, n, d), dtype=torch.bfloat16, device=dev)
    O = torch.empty_like(V)
    Pj = torch.empty((B * n, 3 * H * d), dtype=torch.bfloat16, device=dev)
    Qh, Kh, Vh = (torch.empty((B, H, n, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    O2 = torch.empty_like(V)

    def ok(st, what):
        if st:
            raise had.HadError(st, what)

    def fused_prep():
        ok(L.had_qkv_prepare(ptr(Xd), ptr(Wd), ctypes.byref(shp), Dm, bs, N, mcode, ptr(V), ptr(ws_q), ws_q.numel(),
                             sp), "had_qkv_prepare")

    def fused_attend():
        ok(L.had_attention_prepared(ptr(V), ctypes.byref(shp), bs, None, None, N, mcode, ptr(O), had._dtype_code(O),
                                    ptr(ws_q), ws_q.numel(), sp), "had_attention_prepared")

    def unfused_prep():
        torch.matmul(Xd.view(B * n, Dm), Wd.t(), out=Pj)
        Pv = Pj.view(B, n, 3, H, d)
        for tns, k in ((Qh, 0), (Kh, 1), (Vh, 2)):
            tns.copy_(Pv[:, :, k].permute(0, 2, 1, 3))
        ok(L.had_attention_prepare(ptr(Qh), ptr(Kh), ptr(Vh), ctypes.byref(shp), bs, N, mcode, ptr(ws_a),
                                   ws_a.numel(), sp), "had_attention_prepare")

    def unfused_attend():
        ok(L.had_attention_prepared(ptr(Vh), ctypes.byref(shp), bs, None, None, N, mcode, ptr(O2),
                                    had._dtype_code(O2), ptr(ws_a), ws_a.numel(), sp), "had_attention_prepared")

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    probe_i8, _ = had.had_probe_mma_rate("i8", 40000)
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    clocks.start()
    graphs = {}
    with torch.cuda.stream(sp_stream):
        for _ in range(max(3, args.warmup)):
            fused_prep(); fused_attend(); unfused_prep(); unfused_attend()
        sp_stream.synchronize()
        assert had.had_get_device_status() == had.HAD_OK
        for name, fn in (("fp", fused_prep), ("fa", fused_attend), ("up", unfused_prep), ("ua", unfused_attend)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=sp_stream):
                fn()
            graphs[name] = g
        for g in graphs.values():
            g.replay()
        sp_stream.synchronize()

        def timed(gp, ga):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                   torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
            torch.cuda.synchronize()
            w0 = time.time()
            for s_ in range(args.steps):
                flush.zero_()
                ev[s_][0].record(sp_stream)
                gp.replay()
                ev[s_][1].record(sp_stream)
                ga.replay()
                ev[s_][2].record(sp_stream)
            torch.cuda.synchronize()
            w1 = time.time()
            return ([e[0].elapsed_time(e[2]) for e in ev], [e[0].elapsed_time(e[1]) for e in ev],
                    [e[1].elapsed_time(e[2]) for e in ev], w0, w1)

        f_step, f_prep, f_att, wall0, wall1 = timed(graphs["fp"], graphs["fa"])
        u_step, u_prep, u_att, _, _ = timed(graphs["up"], graphs["ua"])
        # e2e: X from pinned host memory, the fused path, O back, every step
        hX = Xd.cpu().pin_memory()
        hO = torch.empty_like(O, device="cpu").pin_memory()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(3, min(args.steps, 30))
        for s_ in range(e2e_steps + 2):
            if s_ == 2:
                e0.record(sp_stream)
            Xd.copy_(hX, non_blocking=True)
            graphs["fp"].replay()
            graphs["fa"].replay()
            hO.copy_(O, non_blocking=True)
        e1.record(sp_stream)
        sp_stream.synchronize()
    clk = clocks.stop(wall0, wall1)
    diff = (O.float() - O2.float()).abs().max().item()  # the two paths, for the record
    if rank != 0:
        return 0
    peaks, peak_kind = _peaks()
    queries = B * H * n
    f_ms = max_over_ranks(sum(f_step), None) / args.steps
    att_ms = sum(f_att) / args.steps
    flop = 2.0 * B * n * Dm * 3 * H * d
    i8 = max(probe_i8, INT8_PER_BF16 * peaks["bf16_tflops"])
    kb = kernel_bytes_per_token(mode, 2, 2, d) * queries + bw.table.nbytes
    roof = method_roofline(kb, score_tensor_ops(B * H * n * n, d), att_ms, peaks["hbm_gbs"], i8)
    roof.update({"traffic": None, "kernel": "k_attn_tc (fused score/top-N/softmax/A.V)", "avg_launch_ms": att_ms})
    line = {
        "metric": METRIC, "value": whole_job_rate(queries, world, args.steps, sum(f_step)), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": f_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8i8", "data": "synthetic",
        "config": {"workload": f"deit_qkv_b{B}_h{H}_n{n}_dm{Dm}_dense_{mode}", "B": B, "H": H, "n": n, "d": d,
                   "Dm": Dm, "N": N, "mode": mode, "in_dtype": "bf16", "seed": 9,
                   "bias": "relpos 27x27/head, prefix 1", "seqlens": None,
                   "l2": "flushed between timed steps (256 MiB write)"},
        "launch": "each step replays CUDA graphs of the two library calls (projection + prepare, attend)",
        "qkv": {"fused_prep_ms": sum(f_prep) / args.steps, "attn_ms": att_ms,
                "unfused_ms_per_step": sum(u_step) / args.steps, "unfused_prep_ms": sum(u_prep) / args.steps,
                "unfused_attn_ms": sum(u_att) / args.steps,
                "projection_gflop": flop / 1e9,
                "fused_prep_tflops": flop / (sum(f_prep) / args.steps * 1e-3) / 1e12,
                "max_abs_diff_fused_vs_unfused_O": diff,
                "unfused": "cuBLAS bf16 projection (torch.matmul), copy into [B,H,n,d] heads, had_attention_prepare"},
        "roofline": roof,
        "e2e": {"value": queries / (e0.elapsed_time(e1) / e2e_steps * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": X.size * 2, "d2h_bytes_per_step": O.numel() * 2},
        "gpu_launches": args.steps * (6 + relpos_table_launches(bw.gh, bw.gw)),  # k_xsum, k_xmean, k_mu, k_qkv_tc, the bias tables, k_vcodes, k_attn_tc
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=80)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="stress_topn", choices=sorted(WORKLOADS) + [QKV_WORKLOAD])
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="run the first B sequences only (profiler captures)")
    ap.add_argument("--heads", type=int, default=0, help="run the first H heads only (profiler captures)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload == QKV_WORKLOAD:
        if world > 1:
            import torch
            torch.cuda.set_device(local_rank)
        return run_qkv(args, rank, 1, local_rank)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            return run_gpu(args, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
    return run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
