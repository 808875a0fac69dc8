"""Throughput of the exact unpacked integer GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole path over one batch of the workload: percentile + RTN of every input
matrix, plan, unpack, tcgen05 int8 GEMM with fold-back and dequantisation, for every GEMM of the
workload.  The default workload is the LLaMA-7B MLP-shaped one, the largest single-GPU configuration:
gate and up X 2048x4096 . W 4096x11008, then down H 2048x11008 . W 11008x4096 (bf16 inputs, per-token
RTN of X and H, per-output-channel RTN of the weights, p = 0.95, beta = 31, b = 4, Mix).  Others:
q_proj (X 2048x4096 . W 4096x4096, beta = 15, b = 5), attention (32 heads of Q.K^T and P.V, seq 2048,
head dim 128, beta = 15, b = 5), wgrad (dY^T . X, 16384 tokens, 2048 x 512 outputs, per-tensor RTN,
beta = 31, the sweep over b in {3,4,5,8} and the five strategies), training_triple, heavy_tokens.

`value` is the effective TOPS of the original-shape products, sum 2*M*N*K / step time, with inputs
resident in HBM; between timed steps L2 is flushed by writing 256 MB.  `e2e` is the same metric through
the C ABI with every input copied from pinned host memory and every C (int32/int64) and Cf (fp32)
copied back inside the timed region, pipelined on their own streams.  The dominant kernel (the GEMM) is
timed with CUDA events on its stream for the roofline.  With --gpus N > 1 every rank runs its own
replica (the path has no data exchange); time is the max over ranks.

--impl reference times the CPU oracle (this build's reference arm) on a bounded sample of the same
workload on the host cores.  --strategy picks the unpack strategy (mix by default; wgrad sweeps its
own).  --cache-weights (q_proj only): the weight is quantised, planned and unpacked once before timing.
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

STRATEGIES = {"mix": workloads.MIX, "row_row": workloads.ROW_ROW, "row_col": workloads.ROW_COL,
              "col_row": workloads.COL_ROW, "col_col": workloads.COL_COL, "joint": workloads.MIX_JOINT,
              "hybrid": workloads.HYBRID}

# name -> (factory, description, uses --strategy)
WORKLOADS = {
    "mlp": (workloads.mlp, "LLaMA-7B MLP-shaped: gate and up X 2048x4096 . W 4096x11008, down H 2048x11008 . "
                           "W 11008x4096, bf16, per-token RTN (X, H) and per-output-channel RTN (W), p=0.95, "
                           "beta=31, b=4", True),
    "q_proj": (workloads.q_proj, "LLaMA-7B q_proj-shaped X 2048x4096 . W 4096x4096, bf16, per-token / "
                                 "per-channel RTN, p=0.95, beta=15, b=5", True),
    "attention": (workloads.attention, "attention, batch 1, 32 heads, seq 2048, head dim 128: Q.K^T (Q per row, "
                                       "K per token) then P.V (P = softmax of N(0,3^2) logits per row, V per "
                                       "column), bf16, p=0.95, beta=15, b=5", True),
    "wgrad": (workloads.wgrad, "weight gradient dY^T . X, dY 16384x2048 Student-t(3), X 16384x512 with 4 "
                               "outlier channels, per-tensor RTN, p=0.95, beta=31; the sweep b in {3,4,5,8} x "
                               "{mix, row/row, row/col, col/row, col/col}", False),
    "training_triple": (workloads.training_triple, "training triple of one linear layer: forward X.W, dgrad "
                                                   "dY.W^T, wgrad dY^T.X (X 16384x512, W 512x2048, dY "
                                                   "16384x2048 bf16), per-tensor RTN p=0.95 beta=31, b=5", True),
    "heavy_tokens": (workloads.heavy_tokens, "X 2048x4096 bf16 with 6 heavy channels and 4 heavy tokens, per-"
                                             "tensor RTN, . W 4096x4096 bf16 per-channel RTN, p=0.95, beta=15, "
                                             "b=8", True),
}


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


def gemm_list(name: str, strategy: str):
    """The GEMMs of a workload, each with the strategies a step runs it with: [(Gemm, strategy)]."""
    make, _, uses_strategy = WORKLOADS[name]
    out = []
    for g in make():
        for st in (g.strategies if not uses_strategy else [STRATEGIES[strategy]]):
            out.append((g, st))
    return out


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
def quant_spec(g, side):
    """How one operand of GEMM g is quantised: (stored name, granularity, trans_out, plan transpose flag).
    A weight B stored K x N and quantised per output channel goes straight into the N x K layout
    (trans_out), whose rows the unpacker reads fastest; the plan then takes it with transB."""
    if side == "A":
        return g.A.name, g.qa, False, g.transA
    if g.qb == workloads.PER_COL and not g.transB:
        return g.B.name, g.qb, True, True
    return g.B.name, g.qb, False, g.transB


class Step:
    """One pass of the path over every GEMM of a workload on the current device.  Each distinct
    (input, granularity) is quantised once per step (X feeds both MLP GEMMs), the quantisers alternate
    between two streams, then every GEMM is planned and unpacked (one host call each, the next plan's
    host round trip overlapping the previous unpack on the device) and the GEMMs run in order."""

    def __init__(self, imq, torch, gems, inputs):
        self.imq, self.torch = imq, torch
        self.gems = gems  # [(Gemm, strategy)]
        self.inputs = inputs  # stored name -> device tensor
        t = torch
        dev = next(iter(inputs.values())).device
        self.dev = dev
        self.q = {}  # (name, gran, trans_out) -> dict(xint, delta, rowmax, colmax)
        for g, _ in gems:
            for side in ("A", "B"):
                name, gran, tr, _ = quant_spec(g, side)
                key = (name, gran, tr)
                if key in self.q:
                    continue
                x = inputs[name]
                r, c = x.shape
                ng = 1 if gran == imq.IMQ_PER_TENSOR else (r if gran == imq.IMQ_PER_ROW else c)
                self.q[key] = dict(xint=None, shape=(c, r) if tr else (r, c), delta=t.empty(ng, dtype=t.float32, device=dev),
                                   rowmax=t.empty(r, dtype=t.int32, device=dev), colmax=t.empty(c, dtype=t.int32, device=dev),
                                   gran=gran, tr=tr, name=name, p=g.p, beta=g.beta)
        self.wide_checked = False
        self.ws = [None] * len(gems)
        self.C = [None] * len(gems)
        self.Cf = [t.empty((g.M, g.N), dtype=t.float32, device=dev) for g, _ in gems]
        self.infos = [None] * len(gems)
        self.aux = t.cuda.Stream(device=dev)
        self.ev_fork = t.cuda.Event()
        self.ev_join = t.cuda.Event()
        self.n_events = len(gems)

    def _choose_widths(self, inputs):
        """Once, before any timing: int16 quantised values unless an input's values leave int16 (the
        quantiser then reports IMQ_ERR_RANGE), and both operands of a GEMM in int32 when either is."""
        imq, t = self.imq, self.torch
        wide = set()
        for key, j in self.q.items():
            x = inputs[j["name"]]
            tmp = t.empty(j["shape"], dtype=t.int16, device=self.dev)
            imq.imq_rtn_quantize(x, j["gran"], j["p"], j["beta"], Xint=tmp, delta=j["delta"], want_qval=False,
                                 rowmax=j["rowmax"], colmax=j["colmax"], trans_out=j["tr"])
            st = imq.imq_device_status(clear=True)
            if st == imq.IMQ_ERR_RANGE:
                wide.add(key)
            elif st != imq.IMQ_OK:
                raise imq.ImqError(st, "imq_rtn_quantize")
        changed = True
        while changed:
            changed = False
            for g, _ in self.gems:
                ka, kb = quant_spec(g, "A")[:3], quant_spec(g, "B")[:3]
                if (ka in wide) != (kb in wide):
                    wide.update((ka, kb))
                    changed = True
        for key, j in self.q.items():
            j["xint"] = t.empty(j["shape"], dtype=t.int32 if key in wide else t.int16, device=self.dev)
        self.wide_checked = True

    def _quantise(self, inputs):
        imq, t = self.imq, self.torch
        if not self.wide_checked:
            self._choose_widths(inputs)
        main = t.cuda.current_stream()
        self.ev_fork.record(main)
        self.aux.wait_event(self.ev_fork)
        # the longest jobs first, alternating streams
        jobs = sorted(self.q.values(), key=lambda j: -inputs[j["name"]].numel())
        for k, j in enumerate(jobs):
            x = inputs[j["name"]]
            imq.imq_rtn_quantize(x, j["gran"], j["p"], j["beta"], Xint=j["xint"], delta=j["delta"],
                                 want_qval=False, rowmax=j["rowmax"], colmax=j["colmax"], trans_out=j["tr"],
                                 stream=self.aux if k % 2 else None)
        self.ev_join.record(self.aux)
        main.wait_event(self.ev_join)

    def step(self, gemm_events=None, inputs=None, outputs=None):
        imq, t = self.imq, self.torch
        inputs = self.inputs if inputs is None else inputs
        self._quantise(inputs)
        plans = []
        for i, (g, strategy) in enumerate(self.gems):
            na, ga, tra, ta = quant_spec(g, "A")
            nb, gb, trb, tb = quant_spec(g, "B")
            qa, qb = self.q[(na, ga, tra)], self.q[(nb, gb, trb)]
            # maxima over LOGICAL lines: rowmax / colmax are over the stored input's rows / columns
            a_row, a_col = (qa["colmax"], qa["rowmax"]) if g.transA else (qa["rowmax"], qa["colmax"])
            b_row, b_col = (qb["colmax"], qb["rowmax"]) if g.transB else (qb["rowmax"], qb["colmax"])
            plan, Au, Bu = imq.imq_plan_unpack(qa["xint"], qb["xint"], g.b, strategy, ta, tb,
                                               maxes=(a_row, a_col, b_row, b_col), workspace=self.ws[i])
            if Au is None:
                # first step, or a plan larger than the workspace: size it, then unpack
                self.ws[i] = imq.workspace_for(plan, self.dev)
                Au, Bu = imq.workspace_views(plan, self.ws[i])
                imq.imq_unpack(plan, qa["xint"], qb["xint"], A_unp=Au, B_unp_t=Bu)
            I = plan.info
            if self.C[i] is None or (self.C[i].dtype == t.int32) != (I["acc_bits"] == 32):
                self.C[i] = t.empty((g.M, g.N), dtype=t.int32 if I["acc_bits"] == 32 else t.int64, device=self.dev)
            plans.append((plan, Au, Bu, qa, qb))
            self.infos[i] = I
        for i, ((g, _), (plan, Au, Bu, qa, qb)) in enumerate(zip(self.gems, plans)):
            C = self.C[i] if outputs is None else outputs[i][0]
            Cf = self.Cf[i] if outputs is None else outputs[i][1]
            if gemm_events is not None:
                gemm_events[i][0].record()
            imq.imq_gemm_unpacked(plan, Au, Bu, qa["delta"], g.gA, qb["delta"], g.gB, C=C, Cf=Cf)
            if gemm_events is not None:
                gemm_events[i][1].record()
        for plan, *_ in plans:
            plan.destroy()


class AttentionStep:
    """One pass of the path over an attention layer (32 heads): the heads' Q, K and P stacked head-major
    and V as seq x (heads * dim), each quantised by one call (per row: per head and token; V per column:
    per head and dim, straight into the (heads * dim) x seq layout), then Q.K^T and P.V each planned,
    unpacked and multiplied as one batch (imq_plan_batched: one host round trip for all heads; one
    unpack launch per operand; one GEMM launch over every head's tiles)."""

    def __init__(self, imq, torch, gems, inputs):
        self.imq, self.torch = imq, torch
        self.gems = gems
        self.heads = len(gems) // 2
        g_qk, g_pv = gems[0][0], gems[1][0]
        self.g_qk, self.g_pv = g_qk, g_pv
        self.inputs = inputs
        t = torch
        dev = next(iter(inputs.values())).device
        self.dev = dev
        H, S, D = self.heads, g_qk.M, g_qk.K
        self.S, self.D = S, D
        self.q = {}
        # (name, granularity, trans_out, stored shape of the quantised matrix)
        specs = {"Q": (imq.IMQ_PER_ROW, False, (H * S, D)), "K": (imq.IMQ_PER_ROW, False, (H * S, D)),
                 "P": (imq.IMQ_PER_ROW, False, (H * S, S)), "V": (imq.IMQ_PER_COL, True, (H * D, S))}
        for name, (gran, tr, shape) in specs.items():
            x = inputs[name]
            ng = x.shape[0] if gran == imq.IMQ_PER_ROW else x.shape[1]
            self.q[name] = dict(gran=gran, tr=tr, shape=shape, xint=None,
                                delta=t.empty(ng, dtype=t.float32, device=dev),
                                rowmax=t.empty(x.shape[0], dtype=t.int32, device=dev),
                                colmax=t.empty(x.shape[1], dtype=t.int32, device=dev))
        self.ws = [None, None]
        self.C = [None, None]
        self.Cf = [t.empty((H, S, S), dtype=t.float32, device=dev), t.empty((H, S, D), dtype=t.float32, device=dev)]
        self.infos = [None] * len(gems)
        self.aux = t.cuda.Stream(device=dev)
        self.ev_fork = t.cuda.Event()
        self.ev_join = t.cuda.Event()
        self.n_events = 2

    def _widths(self, inputs):
        imq, t = self.imq, self.torch
        wide = set()
        for name, j in self.q.items():
            tmp = t.empty(j["shape"], dtype=t.int16, device=self.dev)
            imq.imq_rtn_quantize(inputs[name], j["gran"], self.g_qk.p, self.g_qk.beta, Xint=tmp, delta=j["delta"],
                                 want_qval=False, rowmax=j["rowmax"], colmax=j["colmax"], trans_out=j["tr"])
            st = imq.imq_device_status(clear=True)
            if st == imq.IMQ_ERR_RANGE:
                wide.add(name)
            elif st != imq.IMQ_OK:
                raise imq.ImqError(st, "imq_rtn_quantize")
        for a, b in (("Q", "K"), ("P", "V")):  # both operands of a GEMM share the integer dtype
            if a in wide or b in wide:
                wide.update((a, b))
        for name, j in self.q.items():
            j["xint"] = t.empty(j["shape"], dtype=t.int32 if name in wide else t.int16, device=self.dev)

    def step(self, gemm_events=None, inputs=None, outputs=None):
        imq, t = self.imq, self.torch
        inputs = self.inputs if inputs is None else inputs
        if self.q["Q"]["xint"] is None:
            self._widths(inputs)
        main = t.cuda.current_stream()
        self.ev_fork.record(main)
        self.aux.wait_event(self.ev_fork)
        for k, name in enumerate(("P", "V", "Q", "K")):
            j = self.q[name]
            imq.imq_rtn_quantize(inputs[name], j["gran"], self.g_qk.p, self.g_qk.beta, Xint=j["xint"],
                                 delta=j["delta"], want_qval=False, rowmax=j["rowmax"], colmax=j["colmax"],
                                 trans_out=j["tr"], stream=self.aux if k % 2 else None)
        self.ev_join.record(self.aux)
        main.wait_event(self.ev_join)
        H, S, D = self.heads, self.S, self.D
        batches = []
        for i, (a, bname, g, N) in enumerate((("Q", "K", self.g_qk, S), ("P", "V", self.g_pv, D))):
            qa, qb = self.q[a], self.q[bname]
            batch = imq.imq_plan_batched(qa["xint"], qb["xint"], H, S, g.K, N, g.b, self.gems[2 * i][1], transB=True)
            _, need = batch.workspace_layout()
            if self.ws[i] is None or self.ws[i].numel() < need + 1024:
                self.ws[i] = t.empty(need + 1024, dtype=t.uint8, device=self.dev)
            imq.imq_unpack_batched(batch, qa["xint"], qb["xint"], self.ws[i], strideA=S * qa["xint"].shape[1],
                                   strideB=N * qb["xint"].shape[1])
            wide = any(batch[h].info["acc_bits"] == 64 for h in range(H))
            if self.C[i] is None or (self.C[i].dtype == t.int64) != wide:
                self.C[i] = t.empty((H, S, N), dtype=t.int64 if wide else t.int32, device=self.dev)
            for h in range(H):
                self.infos[2 * h + i] = batch[h].info
            batches.append((batch, qa, qb, N))
        for i, (batch, qa, qb, N) in enumerate(batches):
            C = self.C[i] if outputs is None else outputs[i][0]
            Cf = self.Cf[i] if outputs is None else outputs[i][1]
            if gemm_events is not None:
                gemm_events[i][0].record()
            imq.imq_gemm_unpacked_batched(batch, self.ws[i], qa["delta"], S, imq.IMQ_PER_ROW, qb["delta"], N,
                                          imq.IMQ_PER_COL, C, Cf)
            if gemm_events is not None:
                gemm_events[i][1].record()
        for batch, *_ in batches:
            batch.destroy()


def attention_inputs(gems):
    """The attention workload's per-head matrices stacked the way AttentionStep quantises them."""
    qk = [g for g, _ in gems if g.name.startswith("attn_qk")]
    pv = [g for g, _ in gems if g.name.startswith("attn_pv")]
    return {"Q": np.concatenate([g.A.data for g in qk]), "K": np.concatenate([g.B.data for g in qk]),
            "P": np.concatenate([g.A.data for g in pv]), "V": np.concatenate([g.B.data for g in pv], axis=1)}


def count_launches(torch, fn):
    """Kernels of this library (namespace imq) that one call of fn launches, counted from a CUDA activity
    trace of that call (torch.profiler), outside any timed region."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    n = 0
    names = {}
    for e in prof.events():
        if getattr(e, "device_type", None) is not None and "CUDA" in str(e.device_type) and "imq::" in e.name:
            n += 1
            short = e.name.split("(")[0].replace("void ", "")
            names[short] = names.get(short, 0) + 1
    return n, names


class CachedPath:
    """The q_proj step with a kept weight (--cache-weights): W quantised per output channel, planned with
    the activations' column maxima widened to the largest value of the same level (imq_level_cover, so
    later batches with the same heavy channels stay covered) and unpacked once, before any timing; each
    step is the fused per-row RTN + unpack of X into the kept plan's layout and the GEMM."""

    def __init__(self, imq, torch, g, X, W, strategy=0, cache_weights=True):
        self.imq, self.torch, self.g = imq, torch, g
        self.strategy = strategy
        self.plan = None
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
        self.info = None

    def prepare_cache(self):
        imq, g, t = self.imq, self.g, self.torch
        imq.imq_rtn_quantize(self.X, imq.IMQ_PER_ROW, g.p, g.beta, Xint=self.Xint, delta=self.dX,
                             want_qval=False, rowmax=self.mx[0], colmax=self.mx[1])
        imq.imq_rtn_quantize(self.W, imq.IMQ_PER_COL, g.p, g.beta, Xint=self.Wint, delta=self.dW,
                             want_qval=False, rowmax=self.mx[2], colmax=self.mx[3], trans_out=True)
        widened = imq.imq_level_cover(self.mx[1], g.b)
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
        """One step on the current stream; X in and C, Cf out default to the path's own buffers."""
        imq, g = self.imq, self.g
        X = self.X if X is None else X
        C = self.C if C is None else C
        Cf = self.Cf if Cf is None else Cf
        imq.imq_rtn_quantize_unpack(self.plan, X, g.p, g.beta, A_unp=self.Au, deltaA=self.dX)
        if gemm_events is not None:
            gemm_events[0].record()
        imq.imq_gemm_unpacked(self.plan, self.Au, self.Bu, self.dX, imq.IMQ_PER_ROW, self.dW, imq.IMQ_PER_COL,
                              C=C, Cf=Cf)
        if gemm_events is not None:
            gemm_events[1].record()


# ------------------------------------------------------------------------------------------------
# the run
# ------------------------------------------------------------------------------------------------
def _to_dev(torch, st, dev):
    return torch.from_numpy(np.ascontiguousarray(st.data).view(np.int16)).to(dev).view(torch.bfloat16)


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

    gems = gemm_list(args.workload, args.strategy)
    if args.workload == "attention":
        arrays = attention_inputs(gems)
    else:
        arrays = {}
        for g, _ in gems:
            for st in (g.A, g.B):
                arrays.setdefault(st.name, st.data)
    host = {n: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) for n, a in arrays.items()}
    inputs = {n: h.to(dev) for n, h in host.items()}
    cached = args.cache_weights
    if cached:
        if args.workload != "q_proj":
            raise SystemExit("--cache-weights applies to the q_proj workload only")
        g0 = gems[0][0]
        path = CachedPath(imq, torch, g0, inputs[g0.A.name], inputs[g0.B.name], gems[0][1], cache_weights=True)
        path.prepare_cache()
        run_step = lambda ev=None: path.step(None if ev is None else ev[0])
    else:
        path = (AttentionStep if args.workload == "attention" else Step)(imq, torch, gems, inputs)
        run_step = lambda ev=None: path.step(ev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if imq.imq_device_status() != imq.IMQ_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ---- device-resident timed region ----
    n = 1 if cached else path.n_events
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    gev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with Clocks(dev) as clk:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record()
            run_step(gev[k])
            ends[k].record()
        torch.cuda.synchronize()
    barrier()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    gemm_ms = [[gev[k][i][0].elapsed_time(gev[k][i][1]) for k in range(args.steps)] for i in range(n)]

    # ---- end to end through the C ABI with host buffers ----
    # Every step copies its inputs from pinned host memory and reads every C and Cf back.  The copies run
    # on their own streams, double-buffered, so that step k+1's upload and step k-1's download overlap
    # step k's compute; the time is from the first upload's start to the last download's end.
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    up_names = [nm for nm in inputs if not (cached and nm == gems[0][0].B.name)]  # a cached weight stays resident
    pin_in = {nm: host[nm].pin_memory() for nm in up_names}
    slots_in = [dict(inputs), {nm: torch.empty_like(inputs[nm]) if nm in up_names else inputs[nm] for nm in inputs}]
    if cached:
        outs0 = [(path.C, path.Cf)]
    else:
        outs0 = list(zip(path.C, path.Cf))
    slots_out = [outs0, [(torch.empty_like(c), torch.empty_like(cf)) for c, cf in outs0]]
    pin_out = [[(torch.empty(c.shape, dtype=c.dtype).pin_memory(), torch.empty(cf.shape, dtype=cf.dtype).pin_memory())
                for c, cf in outs0] for _ in range(2)]
    s_comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    comp_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    out_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_start.record(s_in)
    for k in range(e2e_steps):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])  # step k-2 has read this input slot
            for nm in up_names:
                slots_in[b][nm].copy_(pin_in[nm], non_blocking=True)
            in_done[k].record(s_in)
        s_comp.wait_event(in_done[k])
        if k >= 2:
            s_comp.wait_event(out_done[k - 2])  # step k-2's results have been read from this slot
        if cached:
            g0 = gems[0][0]
            path.step(None, X=slots_in[b][g0.A.name], C=slots_out[b][0][0], Cf=slots_out[b][0][1])
        else:
            path.step(None, inputs=slots_in[b], outputs=slots_out[b])
        comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            for (c, cf), (pc, pcf) in zip(slots_out[b], pin_out[b]):
                pc.copy_(c, non_blocking=True)
                pcf.copy_(cf, non_blocking=True)
            out_done[k].record(s_out)
    t_end.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = t_start.elapsed_time(t_end)
    if imq.imq_device_status() != imq.IMQ_OK:
        raise RuntimeError("device status not OK after the timed steps")
    h2d = sum(host[nm].numel() * 2 for nm in up_names)
    d2h = sum(c.numel() * c.element_size() + cf.numel() * 4 for c, cf in outs0)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist if world > 1 else None, dev)

    # kernels of this library in one step, from a CUDA activity trace of one more step (not timed)
    try:
        per_step, by_kernel = count_launches(torch, run_step)
    except Exception as e:  # keep the measurement; the count is then unknown
        per_step, by_kernel = None, {"error": str(e)[:200]}

    ops = float(sum(g.ops for g, _ in gems))
    value = throughput(ops, world, args.steps, total_ms)
    e2e_value = throughput(ops, world, e2e_steps, e2e_ms)
    bf16_burst, bf16_sus, hbm, src = _peaks()
    int8_peak = 2.0 * bf16_burst  # dense int8 = 2 x dense bf16 on B200 (nominal 4.5 vs 2.25 PFLOP/s)
    infos = [path.info] if cached else path.infos
    exec_ops = [2.0 * I["M_unp"] * I["N_unp"] * I["K_unp"] for I in infos]
    gemm_avg = [sum(v) / len(v) for v in gemm_ms]
    achieved = sum(exec_ops) / (sum(gemm_avg) * 1e-3) / 1e12
    if len(gemm_avg) != len(infos):
        # one GEMM launch covers several problems (the batched attention layer): per-problem times are
        # the launch's time shared in proportion to executed work, for the per-GEMM listing only
        per_launch = len(infos) // len(gemm_avg)
        shares = []
        for li, t in enumerate(gemm_avg):
            idx = [k for k in range(len(infos)) if k % len(gemm_avg) == li]
            tot = sum(exec_ops[k] for k in idx) or 1.0
            shares.append({k: t * exec_ops[k] / tot for k in idx})
        gemm_avg = [shares[k % len(gemm_avg)][k] for k in range(len(infos))]
        assert per_launch >= 1
    _, desc, uses_strategy = WORKLOADS[args.workload]
    per_gemm = []
    for (g, st), I, t in zip(gems, infos, gemm_avg):
        per_gemm.append({"name": g.name, "M": g.M, "K": g.K, "N": g.N, "b": g.b,
                         "strategy": workloads.STRATEGY_NAMES[st], "ratio": round(I["ratio"], 4),
                         "dir_a": I["dir_a"], "dir_b": I["dir_b"], "M_unp": I["M_unp"], "N_unp": I["N_unp"],
                         "K_unp": I["K_unp"], "acc_bits": I["acc_bits"], "gemm_ms": round(t, 4),
                         "exec_TOPS": round(2.0 * I["M_unp"] * I["N_unp"] * I["K_unp"] / (t * 1e-3) / 1e12, 1)})
    config = {"workload": args.workload + ": " + desc + (f", {workloads.STRATEGY_NAMES[STRATEGIES[args.strategy]]}"
                                                       if uses_strategy else ""),
              "strategy": args.strategy if uses_strategy else "sweep", "parallelism": f"replicas x{world}",
              "l2": "flushed between timed steps (256 MB write)", "ops_per_step": ops,
              "pct_int8_peak_effective": round(100 * value / world / int8_peak, 2),
              "gemms": per_gemm if len(per_gemm) <= 24 else per_gemm[:2] + [{"...": len(per_gemm) - 4}] + per_gemm[-2:]}
    if cached:
        config["weights"] = ("quantised, planned and unpacked once before timing; per step: fused per-row RTN + "
                             "unpack of X, GEMM")
    traffic = _traffic_from_profiles(args.workload, cached)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic (seeded, bf16)",
        "config": config,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(achieved / int8_peak, 4), "traffic": traffic,
                     "kernel": f"k_gemm (tcgen05 kind::i8), the {n} launch(es) of a step together",
                     "peak_source": f"{src} bf16 burst x2", "gemm_ms": round(sum(gemm_avg), 4),
                     "exec_ops_per_step": sum(exec_ops)},
        "roofline_hbm": _hbm_roofline(args.workload, path, gemm_ms, hbm) if args.workload == "attention" else None,
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "how": ("every step uploads its inputs from pinned host memory and reads every C and Cf back; "
                        "uploads, compute and downloads on three streams, double-buffered, timed from the first "
                        "upload to the last download; no L2 flush (inputs arrive from the host each step)")},
        "gpu_launches": None if per_step is None else per_step * args.steps,
        "gpu_launches_per_step": by_kernel,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(gems, target_s=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# the oracle on the host (cpu_baseline and the reference arm)
# ------------------------------------------------------------------------------------------------
def _logical_f32(st, trans):
    import oracle
    x = oracle.as_f32(st.data, st.dtype)
    return np.ascontiguousarray(x.T) if trans else x


class OracleSample:
    """The definition tier of the oracle on a sub-block of every distinct product of the workload:
    RTN of the sampled output rows of A (only those rows when A is quantised per row, all of A per
    tensor), RTN of the sampled output columns of B likewise, the direct int64 product of the block and
    its dequantisation.  GEMMs that differ only in b or strategy share one exact product (the definition
    does not depend on them), so each distinct product is computed once."""

    def __init__(self, gems):
        seen, self.gems = set(), []
        for g, _ in gems:
            key = (g.A.name, g.B.name, g.qa, g.qb, g.transA, g.transB, g.p, g.beta)
            if key not in seen:
                seen.add(key)
                self.gems.append(g)
        self.logical = {}
        self.qcache = {}

    def _A(self, g):
        k = ("A", g.A.name, g.transA)
        if k not in self.logical:
            self.logical[k] = _logical_f32(g.A, g.transA)
        return self.logical[k]

    def _B(self, g):
        k = ("B", g.B.name, g.transB)
        if k not in self.logical:
            self.logical[k] = _logical_f32(g.B, g.transB)
        return self.logical[k]

    def run(self, frac, nthreads=0):
        """Runs the sample covering `frac` of every product's rows and columns; returns (seconds, ops,
        fixed): `fixed` is the part of the seconds spent quantising whole matrices per tensor, which does
        not shrink with the sample (made once, on the first run, and counted in every run's seconds)."""
        import oracle
        t0 = time.perf_counter()
        ops = fixed = spent = 0.0
        for g in self.gems:
            A, B = self._A(g), self._B(g)
            r = max(1, int(round(g.M * frac)))
            c = max(1, int(round(g.N * frac)))
            if g.gA == oracle.PER_ROW:
                ai, da, _ = oracle.rtn_quantize(A[:r], oracle.PER_ROW, g.p, g.beta)
            else:
                tc = time.perf_counter()
                (ai, da), tq = self._per_tensor(("A", g.A.name, g.transA, g.p, g.beta), A, g)
                spent += time.perf_counter() - tc
                fixed += tq
                ai = ai[:r]
            if g.gB == oracle.PER_COL:
                bi, db, _ = oracle.rtn_quantize(np.ascontiguousarray(B[:, :c]), oracle.PER_COL, g.p, g.beta)
            else:
                tc = time.perf_counter()
                (bi, db), tq = self._per_tensor(("B", g.B.name, g.transB, g.p, g.beta), B, g)
                spent += time.perf_counter() - tc
                fixed += tq
                bi = np.ascontiguousarray(bi[:, :c])
            C = oracle.gemm_i64(ai, bi, nthreads)
            oracle.dequant(C, da, g.gA, db, g.gB)
            ops += 2.0 * r * c * g.K
        # the whole-matrix quantisations count with the time they took when first made
        return time.perf_counter() - t0 - spent + fixed, ops, fixed

    def _per_tensor(self, key, X, g):
        """The per-tensor quantisation of a whole matrix and the seconds it took, computed once: it does not
        depend on the sample, so later runs reuse it and count its measured time."""
        import oracle
        if key not in self.qcache:
            tq = time.perf_counter()
            xi, d, _ = oracle.rtn_quantize(X, oracle.PER_TENSOR, g.p, g.beta)
            self.qcache[key] = ((xi, d), time.perf_counter() - tq)
        return self.qcache[key]

    def full_ops(self):
        return sum(2.0 * g.M * g.N * g.K for g in self.gems)

    def rate(self, seconds, ops, fixed, frac):
        """Throughput of the whole products in ops/s.  Without per-tensor quantisation it is the sample's
        own rate.  With it, the whole-matrix quantisations (timed in full) plus the rest of the sample's
        time scaled up by 1 / frac^2 (its product's share of the full products; the per-line quantisations
        grow only as frac, so the estimate is on the slow side) stand for the full products' time."""
        if fixed <= 0.0:
            return ops / seconds
        return self.full_ops() / (fixed + (seconds - fixed) / (frac * frac))


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _sample_frac(s, target_s, nthreads=0):
    """The sampled fraction of rows and columns whose oracle run takes about target_s or less (besides the
    per-tensor quantisations of whole matrices, made once): doubled from 1/256 while a run takes under a
    quarter of the target, then scaled as if the time grew with the square of the fraction (the product's
    share; the per-line quantisations grow more slowly, so the run only gets shorter than the target)."""
    f = 1.0 / 256
    t, _, fixed = s.run(f, nthreads)
    t -= fixed  # the per-tensor quantisations do not grow with the sample
    while t < target_s / 4 and f < 1.0:
        f = min(1.0, 2 * f)
        t, _, fixed = s.run(f, nthreads)
        t -= fixed
    return float(min(1.0, f * (target_s / max(t, 1e-6)) ** 0.5))


def cpu_baseline(gems, target_s=15.0):
    s = OracleSample(gems)
    frac = _sample_frac(s, target_s)
    t, ops, fixed = s.run(frac)
    f1 = 1.0 / 256
    t1, ops1, fixed1 = s.run(f1, nthreads=1)
    per_tensor = (f"; the per-tensor quantisation of whole matrices ({fixed:.1f} s) counted in full and the rest "
                  f"scaled to the whole products") if fixed > 0 else ""
    return {"value": round(s.rate(t, ops, fixed, frac) / 1e12, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"{frac:.4f} of the output rows and of the output columns of each of the {len(s.gems)} "
                      f"distinct products: RTN of those lines (the whole matrix where quantised per tensor) + "
                      f"int64 product of the block + dequant; {t:.1f} s on the host, {ops / 1e9:.2f} GOP"
                      + per_tensor,
            "seconds": round(t, 2),
            "single_thread": {"value": round(s.rate(t1, ops1, fixed1, f1) / 1e12, 6), "unit": UNIT,
                              "sample": f"{f1:.4f} of the rows and columns, one host thread, {t1:.2f} s"}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    gems = gemm_list(args.workload, args.strategy)
    s = OracleSample(gems)
    # one step is a bounded sample sized so that warm-up + steps take about a minute
    frac = _sample_frac(s, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        s.run(frac)
    runs = [s.run(frac) for _ in range(args.steps)]
    total = sum(r[0] for r in runs)
    value = s.rate(total, runs[0][1] * args.steps, sum(r[2] for r in runs), frac) / 1e12
    _, desc, uses_strategy = WORKLOADS[args.workload]
    sample = (f"{frac:.4f} of the output rows and columns of each distinct product per step: RTN of those lines "
              f"(whole matrix where per tensor) + int64 product + dequant"
              + ("; whole-matrix quantisations counted in full, the rest scaled to the whole products"
                 if any(r[2] > 0 for r in runs) else ""))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic (seeded, bf16)",
            "config": {"workload": args.workload + ": " + desc, "parallelism": "host cores",
                       "strategy": args.strategy if uses_strategy else "sweep"},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _hbm_roofline(workload, path, gemm_ms, hbm):
    """For the attention layer, whose Q.K^T (inner dimension 128) writes far more bytes than it computes:
    the GEMM launches graded on bytes -- the unpacked operands read once and C and Cf written once, over
    the launch time -- against the measured copy bandwidth."""
    out = []
    for i, t in enumerate(gemm_ms):
        infos = path.infos[i::len(gemm_ms)]
        C, Cf = path.C[i], path.Cf[i]
        nbytes = sum(I["M_unp"] * I["K_unp"] + I["N_unp"] * I["K_unp"] for I in infos) + \
            C.numel() * C.element_size() + Cf.numel() * 4
        ms = sum(t) / len(t)
        out.append({"gemm": ["Q.K^T", "P.V"][i], "bytes": nbytes, "ms": round(ms, 4),
                    "achieved": round(nbytes / (ms * 1e-3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)})
    return out


def _gemm_source_sha1():
    import hashlib
    h = hashlib.sha1()
    for name in ("gemm.cu", "common.cuh", "plan.cu"):
        with open(os.path.join(ROOT, "bit_integer_gemm_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_from_profiles(workload, cached):
    """DRAM bytes per step of the GEMM launches from the committed ncu summary of this workload, or None
    when there is none or the GEMM's source or the plan's layout code has changed since those counters were
    taken (the summary records the hash of the sources it measured)."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec.get(workload + ("_cached" if cached else ""))
        if not ent or ent.get("source_sha1") != _gemm_source_sha1():
            return None
        return ent.get("bytes_per_step")
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--e2e-steps", type=int, default=10, help="steps of the end-to-end measurement (3 or more)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mlp",
                    help="mlp: the headline step (default, the largest single-GPU configuration)")
    ap.add_argument("--strategy", choices=sorted(STRATEGIES), default="mix",
                    help="unpack strategy of the plans (default mix; the wgrad sweep runs its own five)")
    ap.add_argument("--cache-weights", action="store_true",
                    help="q_proj only: inference with a static weight -- W quantised, planned and unpacked "
                         "once before timing; each step is the fused per-row RTN + unpack of X and the GEMM")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
