"""Throughput of the exact unpacked integer GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path on the q_proj-shaped workload (X 2048x4096 bf16 per-token RTN,
W 4096x4096 bf16 per-output-channel RTN, p = 0.95, beta = 15, b = 5, Mix): percentile + RTN of X and W,
plan, unpack, tcgen05 int8 GEMM with fold-back and dequantisation.  `value` is the effective TOPS of
the original-shape product, 2*M*N*K / step time, with inputs resident in HBM; `e2e` is the same through
the C ABI with the inputs copied from pinned host memory and C (int32) plus Cf (fp32) copied back inside
the timed region, the copies pipelined against the compute on their own streams.  Between timed steps L2 is flushed by writing 256 MB.  The dominant kernel (the GEMM)
is timed with CUDA events on its stream for the roofline.  With --gpus N > 1 every rank runs its own
replica (the path has no data exchange); time is the max over ranks.

--impl reference times the CPU oracle (the reference arm of this build) on a bounded sample of the same
workload on the host cores.  --workload training_triple times instead the forward, input-gradient and
weight-gradient GEMMs of one linear layer with per-tensor RTN, and --workload heavy_tokens activations
whose heavy hitters sit in channels and tokens (one GPU; no end-to-end or CPU arm).  --strategy picks
the unpack strategy (mix by default).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "effective TOPS of exact unpacked int GEMM (orig. shape) and % of B200 INT8 peak"
UNIT = "TOPS"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), \
            float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of `values` over all ranks (the slowest rank decides a step's time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def throughput(ops_per_step: float, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput in TOPS: every rank runs `steps` steps of `ops_per_step` operations."""
    return ops_per_step * world * steps / (total_ms * 1e-3) / 1e12


def _workload():
    g = workloads.q_proj()[0]
    return g


def _config(g, extra=None, strategy="mix"):
    name = workloads.STRATEGY_NAMES[STRATEGIES[strategy]]
    c = {"workload": f"q_proj-shaped X {g.M}x{g.K} bf16 per-token RTN x W {g.K}x{g.N} bf16 "
                     f"per-channel RTN, p={g.p}, beta={g.beta}, b={g.b}, {name[0].upper() + name[1:]}",
         "M": g.M, "K": g.K, "N": g.N, "b": g.b, "beta": g.beta, "p": g.p, "strategy": strategy,
         "l2": "flushed between timed steps (256 MB write)"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class Clocks:
    """SM clock and clock-event reasons of one GPU, read (never set) every few milliseconds on a host
    thread through NVML while the timed region runs, so that even a short region gets samples.  The
    GPU is found by its UUID, since NVML numbers GPUs without regard to CUDA_VISIBLE_DEVICES."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device, period_s: float = 0.004):
        self.device = device
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.handle = None
        self.error = None

    def _handle(self, nv):
        import torch
        try:
            u = str(torch.cuda.get_device_properties(self.device).uuid)
            for cand in (u, "GPU-" + u):
                try:
                    return nv.nvmlDeviceGetHandleByUUID(cand)
                except Exception:
                    pass
        except Exception:
            pass
        if nv.nvmlDeviceGetCount() == 1:
            return nv.nvmlDeviceGetHandleByIndex(0)
        raise RuntimeError("GPU not identified in NVML")

    def _run(self, nv):
        import time as _t
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, rs))
            except Exception as e:  # keep what was read so far
                self.error = str(e)
                return
            _t.sleep(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.handle = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._run, args=(nv,), daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
            self._thread = None
        return self

    def __exit__(self, *a):
        if getattr(self, "_thread", None) is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "error": self.error}
        sm = [s for s, _ in self.samples]
        seen = 0
        for _, r in self.samples:
            seen |= int(r)
        reasons = sorted(name for bit, name in self.REASONS.items() if seen & bit)
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML"}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
class Path:
    """Preallocated buffers and one step of the path on the current device."""

    def __init__(self, imq, torch, g, X, W, strategy=0, cache_weights=False):
        self.imq, self.torch, self.g = imq, torch, g
        self.strategy = strategy
        self.cached = cache_weights
        self.plan = None  # the kept plan of the cached-weight mode
        dev = X.device
        self.X, self.W = X, W
        M, K, N = g.M, g.K, g.N
        t = torch
        self.Xint = t.empty((M, K), dtype=t.int16, device=dev)
        self.Wint = t.empty((N, K), dtype=t.int16, device=dev)  # W quantised straight into B^T
        self.dX = t.empty(M, dtype=t.float32, device=dev)
        self.dW = t.empty(N, dtype=t.float32, device=dev)
        self.mx = [t.empty(n, dtype=t.int32, device=dev) for n in (M, K, K, N)]
        self.C = t.empty((M, N), dtype=t.int32, device=dev)
        self.Cf = t.empty((M, N), dtype=t.float32, device=dev)
        self.ws = None
        self.info = None
        self.launches = 0
        # the two quantisers are independent: X's (the shorter) runs on a second stream, joined before the
        # plan, so that it fills the SMs that W's column quantiser leaves idle in its last wave
        self.aux = t.cuda.Stream(device=dev)
        self.ev_fork = t.cuda.Event()
        self.ev_join = t.cuda.Event()

    def prepare_cache(self):
        """Cached-weight mode, before any timing: W quantised per output channel, the plan made with
        the activations' column maxima widened to the largest value of the same level (R^L - 1, so later
        batches with the same heavy channels stay covered), B'^T unpacked once and kept."""
        imq, g, t = self.imq, self.g, self.torch
        imq.imq_rtn_quantize(self.X, imq.IMQ_PER_ROW, g.p, g.beta, Xint=self.Xint, delta=self.dX,
                             want_qval=False, rowmax=self.mx[0], colmax=self.mx[1])
        imq.imq_rtn_quantize(self.W, imq.IMQ_PER_COL, g.p, g.beta, Xint=self.Wint, delta=self.dW,
                             want_qval=False, rowmax=self.mx[2], colmax=self.mx[3], trans_out=True)
        R = 1 << (g.b - 1)
        cm = self.mx[1].cpu().numpy().astype(np.int64)
        lv = np.ones_like(cm)
        q = cm // R
        while (q > 0).any():
            lv += q > 0
            q //= R
        widened = t.from_numpy(np.minimum(R ** lv - 1, 32767).astype(np.int32)).to(self.X.device)
        self.plan = imq.imq_plan(self.Xint, self.Wint, g.b, self.strategy, transB=True,
                                 maxes=(self.mx[0], widened, self.mx[2], self.mx[3]))
        I = self.plan.info
        self.Au = t.empty((I["M_unp"], I["K_unp"]), dtype=t.int8, device=self.X.device)
        _, self.Bu = imq.imq_unpack(self.plan, self.Xint, self.Wint, A_unp=self.Au)
        if I["acc_bits"] != 32:
            self.C = t.empty((g.M, g.N), dtype=t.int64, device=self.X.device)
        self.info = I
        t.cuda.synchronize()

    def step(self, gemm_events=None, X=None, W=None, C=None, Cf=None):
        """One pass of the path on the current stream; X, W in and C, Cf out default to the Path's own
        buffers (the end-to-end loop passes double-buffered ones)."""
        imq, g = self.imq, self.g
        X = self.X if X is None else X
        W = self.W if W is None else W
        C = self.C if C is None else C
        Cf = self.Cf if Cf is None else Cf
        if self.cached:
            # fused per-row RTN + unpack of X into the kept plan's layout, then the GEMM with the kept B'
            imq.imq_rtn_quantize_unpack(self.plan, X, g.p, g.beta, A_unp=self.Au, deltaA=self.dX)
            if gemm_events is not None:
                gemm_events[0].record()
            imq.imq_gemm_unpacked(self.plan, self.Au, self.Bu, self.dX, imq.IMQ_PER_ROW, self.dW, imq.IMQ_PER_COL,
                                  C=C, Cf=Cf)
            if gemm_events is not None:
                gemm_events[1].record()
            self.launches = 2
            return
        main = self.torch.cuda.current_stream()
        self.ev_fork.record(main)
        self.aux.wait_event(self.ev_fork)
        imq.imq_rtn_quantize(X, imq.IMQ_PER_ROW, g.p, g.beta, Xint=self.Xint, delta=self.dX,
                             want_qval=False, rowmax=self.mx[0], colmax=self.mx[1], stream=self.aux)
        imq.imq_rtn_quantize(W, imq.IMQ_PER_COL, g.p, g.beta, Xint=self.Wint, delta=self.dW,
                             want_qval=False, rowmax=self.mx[2], colmax=self.mx[3], trans_out=True)
        self.ev_join.record(self.aux)
        main.wait_event(self.ev_join)
        # plan and unpack in one host call (the unpack queued right behind the plan's last kernel)
        plan, Au, Bu = imq.imq_plan_unpack(self.Xint, self.Wint, g.b, self.strategy, transB=True, maxes=self.mx,
                                           workspace=self.ws)
        I = plan.info
        if Au is None:
            # first step, or a plan larger than the workspace: size it, then unpack
            self.ws = imq.workspace_for(plan, self.X.device)
            Au, Bu = imq.workspace_views(plan, self.ws)
            imq.imq_unpack(plan, self.Xint, self.Wint, A_unp=Au, B_unp_t=Bu)
        if gemm_events is not None:
            gemm_events[0].record()
        imq.imq_gemm_unpacked(plan, Au, Bu, self.dX, imq.IMQ_PER_ROW, self.dW, imq.IMQ_PER_COL, C=C, Cf=Cf)
        if gemm_events is not None:
            gemm_events[1].record()
        self.info = I
        # kernels of this library launched by the step (the launch list of the same step shows them):
        # 2 quantisers, each followed by the reduction of its per-CTA line maxima; the level kernel; the
        # maps kernel; 2 unpack kernels (int16 rows: they also zero the unused OUTER lines); the GEMM
        self.launches = 4 + 1 + (1 if I["K_unp"] > 0 else 0) + 2 + 1
        if self.strategy == imq.IMQ_HYBRID:
            self.launches += 4  # the hybrid's count (both operands' outer lines are stored rows), histogram,
            # choice and level kernels
        plan.destroy()


def _rows_unpack(line_is_row, K, K_unp):
    """True when the library unpacks int16 lines with its staged-row kernel (the condition of its launcher:
    stored rows, the line and the block metadata within shared memory)."""
    Kr = (K + 15) // 16 * 16
    nw = min(8, (64 * 1024) // (Kr * 2))
    if nw < 1:
        nw = 1 if (192 * 1024) // (Kr * 2) >= 1 else 0
    return bool(line_is_row) and nw >= 1 and K_unp // 16 <= 4096 and nw * Kr * 2 + (K_unp // 16) * 5 <= 200 * 1024


class GemmPath:
    """One pass of the path for one workloads.Gemm (stored operands with their quantisation groups and
    transposes) on the current device: RTN of A and B, plan with the quantisers' maxima over logical
    lines, unpack into a workspace, GEMM with fold-back and dequantisation."""

    def __init__(self, imq, torch, g, A, B, strategy=0):
        self.imq, self.torch, self.g, self.A, self.B = imq, torch, g, A, B
        self.strategy = strategy
        t, dev = torch, A.device
        self.Ai = t.empty(tuple(A.shape), dtype=t.int16, device=dev)
        self.Bi = t.empty(tuple(B.shape), dtype=t.int16, device=dev)
        ng = lambda gran, shp: 1 if gran == imq.IMQ_PER_TENSOR else (shp[0] if gran == imq.IMQ_PER_ROW else shp[1])
        self.dA = t.empty(ng(g.qa, A.shape), dtype=t.float32, device=dev)
        self.dB = t.empty(ng(g.qb, B.shape), dtype=t.float32, device=dev)
        self.mA = [t.empty(n, dtype=t.int32, device=dev) for n in A.shape]  # stored rows, stored columns
        self.mB = [t.empty(n, dtype=t.int32, device=dev) for n in B.shape]
        self.C = None
        self.Cf = t.empty((g.M, g.N), dtype=t.float32, device=dev)
        self.ws = None
        self.info = None

    def step(self, gemm_events=None):
        imq, g = self.imq, self.g
        imq.imq_rtn_quantize(self.A, g.qa, g.p, g.beta, Xint=self.Ai, delta=self.dA, want_qval=False,
                             rowmax=self.mA[0], colmax=self.mA[1])
        imq.imq_rtn_quantize(self.B, g.qb, g.p, g.beta, Xint=self.Bi, delta=self.dB, want_qval=False,
                             rowmax=self.mB[0], colmax=self.mB[1])
        # maxima over LOGICAL lines: a transposed operand's stored rows are its logical columns
        a_row, a_col = (self.mA[1], self.mA[0]) if g.transA else (self.mA[0], self.mA[1])
        b_row, b_col = (self.mB[1], self.mB[0]) if g.transB else (self.mB[0], self.mB[1])
        plan = imq.imq_plan(self.Ai, self.Bi, g.b, self.strategy, g.transA, g.transB,
                            maxes=(a_row, a_col, b_row, b_col))
        I = plan.info
        need = I["workspace_bytes"]
        if self.ws is None or self.ws.numel() < need + 1024:
            self.ws = self.torch.empty(need + 1024, dtype=self.torch.int8, device=self.A.device)
        if self.C is None or (self.C.dtype == self.torch.int32) != (I["acc_bits"] == 32):
            self.C = self.torch.empty((g.M, g.N), device=self.A.device,
                                      dtype=self.torch.int32 if I["acc_bits"] == 32 else self.torch.int64)
        na = I["M_unp"] * I["K_unp"]
        a_off = (-self.ws.data_ptr()) % 1024
        b_off = a_off + (na + 1023) // 1024 * 1024
        Au = self.ws[a_off:a_off + na].view(I["M_unp"], I["K_unp"])
        Bu = self.ws[b_off:b_off + I["N_unp"] * I["K_unp"]].view(I["N_unp"], I["K_unp"])
        imq.imq_unpack(plan, self.Ai, self.Bi, A_unp=Au, B_unp_t=Bu)
        if gemm_events is not None:
            gemm_events[0].record()
        imq.imq_gemm_unpacked(plan, Au, Bu, self.dA, g.gA, self.dB, g.gB, C=self.C, Cf=self.Cf)
        if gemm_events is not None:
            gemm_events[1].record()
        self.info = I
        # kernels of this library launched by the step: per quantiser its kernel and the reduction of its
        # per-CTA line maxima, plus for a per-tensor bf16 group the init and two histogram + select passes;
        # the level and maps kernels (and those of the hybrid choice); 2 unpack kernels; the zeroing
        # launches counted above; the GEMM
        quant = lambda gran: 7 if gran == imq.IMQ_PER_TENSOR else 2
        # a zeroing launch per OUTER operand unless its int16 lines are stored rows, which the row unpack
        # kernel stages and zeroes itself
        outer = (int(bool(I["dir_a"] & imq.IMQ_DIR_OUTER) and not _rows_unpack(not g.transA, I["K"], I["K_unp"])) +
                 int(bool(I["dir_b"] & imq.IMQ_DIR_OUTER) and not _rows_unpack(g.transB, I["K"], I["K_unp"])))
        hybrid = 0
        if self.strategy == imq.IMQ_HYBRID:
            # histogram, choice and levels, plus one count kernel for operands whose outer lines are
            # stored rows and two for operands whose outer lines are stored columns
            rows_outer = [not g.transA, g.transB]
            hybrid = 3 + (1 if any(rows_outer) else 0) + (2 if not all(rows_outer) else 0)
        self.launches = (quant(g.qa) + quant(g.qb) + 1 + (1 if I["K_unp"] > 0 else 0) + hybrid + 2 + outer + 1)
        plan.destroy()


STRATEGIES = {"mix": workloads.MIX, "row_row": workloads.ROW_ROW, "row_col": workloads.ROW_COL,
              "col_row": workloads.COL_ROW, "col_col": workloads.COL_COL, "joint": workloads.MIX_JOINT,
              "hybrid": workloads.HYBRID}

GEMM_WORKLOADS = {
    "training_triple": (workloads.training_triple,
                        "training triple of one linear layer: forward X.W, dgrad dY.W^T, wgrad dY^T.X (X 16384x512, "
                        "W 512x2048, dY 16384x2048 bf16), per-tensor RTN p=0.95 beta=31, b=5"),
    "heavy_tokens": (workloads.heavy_tokens,
                     "X 2048x4096 bf16 with 6 heavy channels and 4 heavy tokens, per-tensor RTN, x W 4096x4096 "
                     "bf16 per-channel RTN, p=0.95, beta=15, b=8"),
}


def run_gemms(args):
    """--workload training_triple | heavy_tokens: one step is the whole path (RTN of both operands, plan,
    unpack, GEMM) for each GEMM of the workload, with the strategy --strategy names."""
    import torch

    import bit_integer_gemm_b200 as imq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    imq.lib()
    make, desc = GEMM_WORKLOADS[args.workload]
    strategy = STRATEGIES[args.strategy]
    gems = make()
    dev_of = {}
    for g in gems:
        for st in (g.A, g.B):
            if st.name not in dev_of:
                dev_of[st.name] = torch.from_numpy(st.data.view(np.int16)).to(dev).view(torch.bfloat16)
    paths = [GemmPath(imq, torch, g, dev_of[g.A.name], dev_of[g.B.name], strategy) for g in gems]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        for pth in paths:
            pth.step()
    torch.cuda.synchronize()
    if imq.imq_device_status() != imq.IMQ_OK:
        raise RuntimeError("device status not OK after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    gev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in paths]
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    with Clocks(dev) as clk:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record()
            for pth, ev in zip(paths, gev[k]):
                pth.step(ev)
            ends[k].record()
        torch.cuda.synchronize()
    total_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends))
    n = len(paths)
    gemm_ms = [gev[k][i][0].elapsed_time(gev[k][i][1]) for k in range(args.steps) for i in range(n)]
    ops = sum(2.0 * g.M * g.N * g.K for g in gems)
    value = throughput(ops, 1, args.steps, total_ms)
    exec_ops = sum(2.0 * p.info["M_unp"] * p.info["N_unp"] * p.info["K_unp"] for p in paths)
    gemm_total_ms = sum(gemm_ms) / args.steps
    bf16_burst, _, _, src = _peaks()
    int8_peak = 2.0 * bf16_burst
    achieved = exec_ops / (gemm_total_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic (seeded, bf16)",
        "config": {"workload": f"{desc}, {workloads.STRATEGY_NAMES[strategy]}",
                   "strategy": args.strategy,
                   "l2": "flushed between timed steps (256 MB write)",
                   "gemms": [{"name": g.name, "M": g.M, "K": g.K, "N": g.N, "ratio": round(p.info["ratio"], 4),
                              "dir_a": p.info["dir_a"], "dir_b": p.info["dir_b"], "M_unp": p.info["M_unp"],
                              "N_unp": p.info["N_unp"], "K_unp": p.info["K_unp"],
                              "gemm_ms": round(sum(gemm_ms[i::n]) / args.steps, 4)}
                             for i, (g, p) in enumerate(zip(gems, paths))]},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(int8_peak, 1), "unit": "TOPS",
                     "frac": round(achieved / int8_peak, 4), "traffic": None,
                     "kernel": f"k_gemm, the {n} launch(es) of a step together", "peak_source": f"{src} bf16 burst x2"},
        "e2e": None,
        "gpu_launches": args.steps * sum(p.launches for p in paths),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    import bit_integer_gemm_b200 as imq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    imq.lib()

    g = _workload()
    Xh = torch.from_numpy(g.A.data.view(np.int16)).view(torch.bfloat16)
    Wh = torch.from_numpy(g.B.data.view(np.int16)).view(torch.bfloat16)
    X = Xh.to(dev)
    W = Wh.to(dev)
    path = Path(imq, torch, g, X, W, STRATEGIES[args.strategy], cache_weights=args.cache_weights)
    if args.cache_weights:
        path.prepare_cache()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        path.step()
    torch.cuda.synchronize()
    if imq.imq_device_status() != imq.IMQ_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ---- device-resident timed region ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with Clocks(dev) as clk:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record()
            path.step(gev[k])
            ends[k].record()
        torch.cuda.synchronize()
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    gemm_ms = [a.elapsed_time(b) for a, b in gev]
    total_ms = sum(step_ms)
    launches = path.launches * args.steps

    # ---- end to end through the C ABI with host buffers ----
    # Every step copies its X and W from pinned host memory and reads C and Cf back.  The copies run on
    # their own streams, double-buffered, so that step k+1's upload and step k-1's download overlap
    # step k's compute; the time is from the first upload's start to the last download's end.
    Xp = Xh.pin_memory()
    Wp = Wh.pin_memory()
    Cp = [torch.empty((g.M, g.N), dtype=path.C.dtype).pin_memory() for _ in range(2)]
    Cfp = [torch.empty((g.M, g.N), dtype=torch.float32).pin_memory() for _ in range(2)]
    Xd = [X, torch.empty_like(X)]
    Wd = [W, torch.empty_like(W)]
    Cd = [path.C, torch.empty_like(path.C)]
    Cfd = [path.Cf, torch.empty_like(path.Cf)]
    s_comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done = [ev() for _ in range(args.steps)]
    comp_done = [ev() for _ in range(args.steps)]
    out_done = [ev() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_start.record(s_in)
    for k in range(args.steps):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])  # step k-2 has read this input slot
            Xd[b].copy_(Xp, non_blocking=True)
            if not path.cached:  # a cached weight stays resident as its unpacked B'
                Wd[b].copy_(Wp, non_blocking=True)
            in_done[k].record(s_in)
        s_comp.wait_event(in_done[k])
        if k >= 2:
            s_comp.wait_event(out_done[k - 2])  # step k-2's result has been read from this slot
        path.step(X=Xd[b], W=Wd[b], C=Cd[b], Cf=Cfd[b])
        comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            Cp[b].copy_(Cd[b], non_blocking=True)
            Cfp[b].copy_(Cfd[b], non_blocking=True)
            out_done[k].record(s_out)
    t_end.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = t_start.elapsed_time(t_end)
    if imq.imq_device_status() != imq.IMQ_OK:
        raise RuntimeError("device status not OK after the timed steps")

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist if world > 1 else None, dev)

    I = path.info
    ops = 2.0 * g.M * g.N * g.K
    value = throughput(ops, world, args.steps, total_ms)
    e2e_value = throughput(ops, world, args.steps, e2e_ms)
    bf16_burst, bf16_sus, hbm, src = _peaks()
    int8_peak = 2.0 * bf16_burst  # dense int8 = 2 x dense bf16 on B200 (nominal 4.5 vs 2.25 PFLOP/s)
    exec_ops = 2.0 * I["M_unp"] * I["N_unp"] * I["K_unp"]
    gemm_avg_ms = sum(gemm_ms) / len(gemm_ms)
    achieved = exec_ops / (gemm_avg_ms * 1e-3) / 1e12
    traffic = _traffic_from_profiles()
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic (seeded, bf16)",
        "config": _config(g, {"parallelism": f"replicas x{world}", "ratio": round(I["ratio"], 4),
                              "dir_a": I["dir_a"], "dir_b": I["dir_b"], "M_unp": I["M_unp"],
                              "N_unp": I["N_unp"], "K_unp": I["K_unp"], "acc_bits": I["acc_bits"],
                              "pct_int8_peak_effective": round(100 * value / world / int8_peak, 2),
                              **({"weights": "quantised, planned and unpacked once before timing; per step: fused "
                                             "per-row RTN + unpack of X, GEMM"} if args.cache_weights else {})},
                          args.strategy),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(achieved / int8_peak, 4), "traffic": traffic,
                     "kernel": "k_gemm (tcgen05 kind::i8)", "peak_source": f"{src} bf16 burst x2",
                     "gemm_ms": round(gemm_avg_ms, 4), "exec_ops_per_launch": exec_ops},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT,
                "h2d_bytes_per_step": 2 * g.M * g.K + (0 if path.cached else 2 * g.K * g.N),
                "d2h_bytes_per_step": (path.C.element_size() + 4) * g.M * g.N,
                "how": ("every step uploads X" + ("" if path.cached else ", W") + " from pinned host memory "
                        "and reads C, Cf back; uploads, compute and downloads on three streams, double-"
                        "buffered, timed from the first upload to the last download; no L2 flush (inputs "
                        "arrive from the host each step, per-step working set above L2)")},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(g, target_s=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# the oracle on the host (cpu_baseline and the reference arm)
# ------------------------------------------------------------------------------------------------
def _oracle_sample(g, rows: int, qW=None, nthreads: int = 0):
    """Definition tier of the oracle on `rows` rows of X: RTN of those rows (per token), RTN of W (per
    channel; once, passed in when already done), the direct int64 product (on `nthreads` host threads,
    0 = all) and the dequantisation."""
    import oracle
    t0 = time.perf_counter()
    if qW is None:
        qW = oracle.rtn_quantize(oracle.as_f32(g.B.data, "bf16"), oracle.PER_COL, g.p, g.beta)
    xs = oracle.as_f32(g.A.data[:rows], "bf16")
    xi, dx, _ = oracle.rtn_quantize(xs, oracle.PER_ROW, g.p, g.beta)
    C = oracle.gemm_i64(xi, qW[0], nthreads)
    oracle.dequant(C, dx, oracle.PER_ROW, qW[1], oracle.PER_COL)
    return time.perf_counter() - t0, qW


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(g, target_s=15.0):
    probe_rows = 8
    t_probe, qW = _oracle_sample(g, probe_rows)
    t_small, _ = _oracle_sample(g, probe_rows, qW)
    rows = int(max(probe_rows, min(g.M, probe_rows * target_s / max(t_small, 1e-3))))
    t_w0 = time.perf_counter()
    import oracle
    qW = oracle.rtn_quantize(oracle.as_f32(g.B.data, "bf16"), oracle.PER_COL, g.p, g.beta)
    t_w = time.perf_counter() - t_w0
    t_rows, _ = _oracle_sample(g, rows, qW)
    t = t_w + t_rows
    ops = 2.0 * rows * g.N * g.K
    # the same per-row work on one host thread, on the probe's rows (W's RTN already done)
    t_one, _ = _oracle_sample(g, probe_rows, qW, nthreads=1)
    one = 2.0 * probe_rows * g.N * g.K / t_one / 1e12
    return {"value": round(ops / t / 1e12, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"{rows} of {g.M} rows of X: RTN of those rows + RTN of all of W + int64 product + "
                      f"dequant; {t:.1f} s on the host", "seconds": round(t, 2),
            "single_thread": {"value": round(one, 6), "unit": UNIT,
                              "sample": f"{probe_rows} rows of X (RTN + int64 product + dequant, W quantised "
                                        f"before), one host thread, {t_one:.2f} s"}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    g = _workload()
    import oracle
    qW = oracle.rtn_quantize(oracle.as_f32(g.B.data, "bf16"), oracle.PER_COL, g.p, g.beta)
    # size one step (a bounded sample of rows) so that warm-up + steps take about a minute
    t8, _ = _oracle_sample(g, 8, qW)
    per_step = 60.0 / max(1, args.steps + args.warmup)
    rows = int(max(8, min(g.M, 8 * per_step / max(t8, 1e-3))))
    for _ in range(args.warmup):
        _oracle_sample(g, rows, qW)
    times = [_oracle_sample(g, rows, qW)[0] for _ in range(args.steps)]
    total = sum(times)
    ops = 2.0 * rows * g.N * g.K
    value = ops * args.steps / total / 1e12
    sample = (f"{rows} of {g.M} rows of X per step: RTN of those rows + int64 product + dequant "
              f"(W quantised once before timing)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic (seeded, bf16)", "config": _config(g, {"parallelism": "host cores"}, args.strategy),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _gemm_source_sha1():
    import hashlib
    h = hashlib.sha1()
    for name in ("gemm.cu", "common.cuh"):
        with open(os.path.join(ROOT, "bit_integer_gemm_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_from_profiles():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when the GEMM's source has
    changed since those counters were taken (the summary records the hash of the source it measured)."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("source_sha1") != _gemm_source_sha1():
            return None
        return rec.get("bytes_per_launch")
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--workload", choices=["q_proj"] + sorted(GEMM_WORKLOADS), default="q_proj",
                    help="q_proj: the headline step (default); training_triple: the three GEMMs of one "
                         "quantised-training step of a linear layer; heavy_tokens: activations with heavy "
                         "channels and heavy tokens (the last two: one GPU, no end-to-end or CPU arms)")
    ap.add_argument("--strategy", choices=sorted(STRATEGIES), default="mix",
                    help="unpack strategy of the plans (default mix)")
    ap.add_argument("--cache-weights", action="store_true",
                    help="q_proj only: inference with a static weight -- W quantised, planned and unpacked "
                         "once before timing; each step is the fused per-row RTN + unpack of X and the GEMM")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in GEMM_WORKLOADS:
        run_gemms(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
