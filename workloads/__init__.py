"""Seeded synthetic inputs shaped like the GEMMs the IM-Unpack summary page reports on.

This module is shared by the tests, the benchmark and the oracle checks.  It draws random matrices and
rounds them to bfloat16; it holds none of the quantisation, planning, unpacking or GEMM arithmetic.

The page ("IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers", atlas.scime.ai
summary; measured-effects table and "Limitations") reports unpack ratios on LLaMA-7B linear-layer and
attention GEMMs and trains ViT / RoBERTa / T5 with quantised GEMMs.  Those tensors and datasets are not
available, so each workload below is a synthetic stand-in with the same shapes and with heavy hitters
planted the way the page describes them (a few entries far outside the bulk, concentrated in channels):

  tiny       A 64x128, B 128x64 fp32 N(0,1); 82 (1% of 8192) of the 128 entries on two inner indices
             of A, and 82 of B's, scaled x50.  Seed 0.
  q_proj     X 2048x4096 N(0,1), 6 channels x60; W 4096x4096 N(0,0.02^2), 8389 (0.05%) distinct
             positions x30.  bf16.  Seed 1.
  mlp        X as q_proj; W_gate, W_up 4096x11008 and W_down 11008x4096 as q_proj's W (0.05% x30);
             H 2048x11008 N(0,1) with 11 channels (0.1%) x100.  bf16.  Seed 2.
  attention  32 heads; per head Q, K 2048x128 N(0,1) with 4 shared dims x20; logits 2048x2048
             N(0,3^2), P = row softmax in fp32; V 2048x128 N(0,1).  bf16.  Head h uses seed [3, h].
  wgrad      dY 16384x2048 Student-t(3) drawn as N(0,1)/sqrt(chi2_3/3); X 16384x512 N(0,1) with 4
             columns x50.  bf16.  Seed 4.

Two more are built from the same pieces: the quantised-training triple of one linear layer (seed 5 for
its weight) and heavy_tokens (seed 6), activations with heavy hitters in some channels AND some tokens.

Matrices are returned as numpy arrays: float32 for 'f32', bfloat16 bit patterns in uint16 for 'bf16'.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

PER_TENSOR, PER_ROW, PER_COL = 0, 1, 2
MIX, ROW_ROW, ROW_COL, COL_ROW, COL_COL, MIX_JOINT, HYBRID = 0, 1, 2, 3, 4, 5, 6
STRATEGY_NAMES = {MIX: "mix", ROW_ROW: "row/row", ROW_COL: "row/col", COL_ROW: "col/row",
                  COL_COL: "col/col", MIX_JOINT: "joint mix", HYBRID: "hybrid"}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest with ties to even; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


@dataclass
class Stored:
    """One stored (row-major) matrix: float32 values or bf16 bit patterns."""
    name: str
    data: np.ndarray
    dtype: str  # 'f32' | 'bf16'

    @property
    def shape(self):
        return self.data.shape


@dataclass
class Gemm:
    """C = A * B on stored matrices.  transA: A is stored K x M; transB: B is stored N x K.
    qa / qb: quantisation groups over the STORED matrix (PER_TENSOR / PER_ROW / PER_COL)."""
    name: str
    A: Stored
    B: Stored
    transA: bool
    transB: bool
    qa: int
    qb: int
    p: float
    beta: int
    b: int
    strategies: list = field(default_factory=lambda: [MIX])

    @property
    def M(self):
        return self.A.shape[1] if self.transA else self.A.shape[0]

    @property
    def K(self):
        return self.A.shape[0] if self.transA else self.A.shape[1]

    @property
    def N(self):
        return self.B.shape[0] if self.transB else self.B.shape[1]

    @property
    def gA(self):
        """Granularity of A's scales on the LOGICAL A: PER_TENSOR or PER_ROW (per output row)."""
        if self.qa == PER_TENSOR:
            return PER_TENSOR
        rowwise = (self.qa == PER_ROW) != self.transA
        return PER_ROW if rowwise else PER_COL

    @property
    def gB(self):
        """Granularity of B's scales on the LOGICAL B: PER_TENSOR or PER_COL (per output column)."""
        if self.qb == PER_TENSOR:
            return PER_TENSOR
        colwise = (self.qb == PER_COL) != self.transB
        return PER_COL if colwise else PER_ROW

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _scatter_scale(rng, x, frac, factor):
    n = int(round(frac * x.size))
    pos = rng.choice(x.size, n, replace=False)
    x.reshape(-1)[pos] *= np.float32(factor)
    return x


def _channels_scale(rng, x, count, factor):
    ch = rng.choice(x.shape[1], count, replace=False)
    x[:, ch] *= np.float32(factor)
    return x


def tiny() -> list:
    rng = np.random.default_rng(0)
    A = _normal(rng, (64, 128))
    B = _normal(rng, (128, 64))
    inner = rng.choice(128, 2, replace=False)
    n_hh = int(round(0.01 * A.size))
    cand_a = [(i, t) for t in inner for i in range(64)]
    for k in rng.choice(len(cand_a), n_hh, replace=False):
        A[cand_a[k]] *= np.float32(50)
    cand_b = [(t, j) for t in inner for j in range(64)]
    for k in rng.choice(len(cand_b), n_hh, replace=False):
        B[cand_b[k]] *= np.float32(50)
    return [Gemm("tiny", Stored("A", A, "f32"), Stored("B", B, "f32"), False, False, PER_TENSOR,
                 PER_TENSOR, 0.95, 15, 5)]


def _bf(name, x):
    return Stored(name, f32_to_bf16_bits(x), "bf16")


def q_proj() -> list:
    rng = np.random.default_rng(1)
    X = _channels_scale(rng, _normal(rng, (2048, 4096)), 6, 60)
    W = _scatter_scale(rng, _normal(rng, (4096, 4096), 0.02), 0.0005, 30)
    return [Gemm("q_proj", _bf("X", X), _bf("W", W), False, False, PER_ROW, PER_COL, 0.95, 15, 5)]


def mlp() -> list:
    rng = np.random.default_rng(2)
    X = _bf("X", _channels_scale(rng, _normal(rng, (2048, 4096)), 6, 60))
    Wg = _bf("W_gate", _scatter_scale(rng, _normal(rng, (4096, 11008), 0.02), 0.0005, 30))
    Wu = _bf("W_up", _scatter_scale(rng, _normal(rng, (4096, 11008), 0.02), 0.0005, 30))
    H = _bf("H", _channels_scale(rng, _normal(rng, (2048, 11008)), 11, 100))
    Wd = _bf("W_down", _scatter_scale(rng, _normal(rng, (11008, 4096), 0.02), 0.0005, 30))
    mk = lambda n, a, b: Gemm(n, a, b, False, False, PER_ROW, PER_COL, 0.95, 31, 4)
    return [mk("mlp_gate", X, Wg), mk("mlp_up", X, Wu), mk("mlp_down", H, Wd)]


def attention_head(h: int, seq: int = 2048, dim: int = 128) -> list:
    rng = np.random.default_rng([3, h])
    Q = _normal(rng, (seq, dim))
    Kt = _normal(rng, (seq, dim))
    dims = rng.choice(dim, 4, replace=False)
    Q[:, dims] *= np.float32(20)
    Kt[:, dims] *= np.float32(20)
    logits = _normal(rng, (seq, seq), 3.0)
    logits -= logits.max(axis=1, keepdims=True)
    P = np.exp(logits)
    P /= P.sum(axis=1, keepdims=True)
    V = _normal(rng, (seq, dim))
    q, k, p, v = _bf(f"Q{h}", Q), _bf(f"K{h}", Kt), _bf(f"P{h}", P.astype(np.float32)), _bf(f"V{h}", V)
    return [Gemm(f"attn_qk_h{h}", q, k, False, True, PER_ROW, PER_ROW, 0.95, 15, 5),
            Gemm(f"attn_pv_h{h}", p, v, False, False, PER_ROW, PER_COL, 0.95, 15, 5)]


def attention(heads: int = 32) -> list:
    out = []
    for h in range(heads):
        out += attention_head(h)
    return out


def wgrad() -> list:
    rng = np.random.default_rng(4)
    z = rng.standard_normal((16384, 2048), dtype=np.float32)
    chi = rng.chisquare(3, (16384, 2048)).astype(np.float32)
    dY = z / np.sqrt(chi / np.float32(3))
    X = _channels_scale(rng, _normal(rng, (16384, 512)), 4, 50)
    gem = []
    for b in (3, 4, 5, 8):
        gem.append(Gemm(f"wgrad_b{b}", _bf("dY", dY), _bf("X", X), True, False, PER_TENSOR,
                        PER_TENSOR, 0.95, 31, b, [MIX, ROW_ROW, ROW_COL, COL_ROW, COL_COL]))
    return gem


def training_triple(b: int = 5) -> list:
    """The three GEMMs of one quantised-training step of a linear layer Y = X W (X 16384 x 512, W 512 x
    2048, the weight-gradient layer's shapes): forward X.W, input gradient dY.W^T (W as stored, transB)
    and weight gradient dY^T.X (dY as stored, transA), each operand quantised per tensor with p = 0.95,
    beta = 31.  dY and X are the weight-gradient workload's (seed 4); W, which that workload lacks, is
    drawn like the projection weights (N(0, 0.02), 0.05 % of entries x30) from seed 5."""
    w = wgrad()[0]
    dY, X = w.A, w.B
    rng = np.random.default_rng(5)
    W = _bf("W", _scatter_scale(rng, _normal(rng, (512, 2048), 0.02), 0.0005, 30))
    mk = lambda n, a, bb, ta, tb: Gemm(n, a, bb, ta, tb, PER_TENSOR, PER_TENSOR, 0.95, 31, b, [MIX])
    return [mk("train_forward", X, W, False, False), mk("train_dgrad", dY, W, False, True),
            mk("train_wgrad", dY, X, True, False)]


def heavy_tokens(b: int = 8) -> list:
    """Activations whose heavy hitters sit in a few channels AND a few tokens, the structure that pure
    row or pure column unpacking both handle badly (the page prints no such workload; this is a
    stand-in for it): X 2048 x 4096 N(0,1) with 6 channels x60 (as q_proj) and 4 tokens x60 outside
    those channels, quantised per tensor; W 4096 x 4096 N(0, 0.02^2) per output channel, no planted
    heavy hitters.  p = 0.95, beta = 15 and b = 8: the b-bit bound 127 is 8.5 beta, so only the planted
    heavy hitters leave it.  bf16.  Seed 6."""
    rng = np.random.default_rng(6)
    X = _normal(rng, (2048, 4096))
    ch = rng.choice(4096, 6, replace=False)
    X[:, ch] *= np.float32(60)
    rows = rng.choice(2048, 4, replace=False)
    other = np.setdiff1d(np.arange(4096), ch)
    X[np.ix_(rows, other)] *= np.float32(60)
    W = _normal(rng, (4096, 4096), 0.02)
    return [Gemm("heavy_tokens", _bf("X", X), _bf("W", W), False, False, PER_TENSOR, PER_COL, 0.95, 15, b,
                 [MIX, HYBRID])]


CONFIGS = {"tiny": tiny, "q_proj": q_proj, "mlp": mlp, "attention": attention, "wgrad": wgrad,
           "training_triple": training_triple, "heavy_tokens": heavy_tokens}


def rows_and_cols_case(rng, M, K, N, big=5000, dense_rows=1, dense_cols=1, scatter=0.02):
    """Small random integer operands whose heavy hitters sit in a few whole rows AND a few whole columns
    of each matrix (plus a scattered fraction): entries in [-20, 20], heavy ones up to +-big.  A has
    `dense_rows` heavy rows and `dense_cols` heavy columns (in a random half of the rows); B likewise."""
    out = []
    for rows, cols in ((M, K), (K, N)):
        X = rng.integers(-20, 21, size=(rows, cols)).astype(np.int64)
        for r in rng.choice(rows, size=min(dense_rows, rows), replace=False):
            X[r, :] = rng.integers(-big, big + 1, size=cols)
        for c in rng.choice(cols, size=min(dense_cols, cols), replace=False):
            sel = rng.random(rows) < 0.5
            X[sel, c] = rng.integers(-big, big + 1, size=int(sel.sum()))
        mask = rng.random(X.shape) < scatter
        X[mask] = rng.integers(-big, big + 1, size=int(mask.sum()))
        out.append(X)
    return out[0], out[1]


def random_case(rng, M, K, N, big=5000, frac=0.1):
    """Small random integer GEMM operands with heavy hitters: entries mostly in [-20, 20], a fraction
    `frac` of them up to +-big.  Used for brute-force checks."""
    A = rng.integers(-20, 21, size=(M, K)).astype(np.int64)
    B = rng.integers(-20, 21, size=(K, N)).astype(np.int64)
    for X in (A, B):
        mask = rng.random(X.shape) < frac
        X[mask] = rng.integers(-big, big + 1, size=int(mask.sum()))
    return A, B
