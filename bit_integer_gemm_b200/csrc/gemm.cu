// gemm.cu -- the low-bit integer GEMM on the unpacked operands with the fold-back epilogue (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Approach": the original integer GEMM is reproduced exactly by low bit-width integer GEMMs
// followed by bit-shift scaling and accumulation.
//
// Design (B200).  One launch runs a table of problems (one unpacked GEMM each: a single plan, or every
// head of a batched attention layer) as a persistent kernel with one CTA per SM, or one CTA pair per two
// SMs when A' has more than one 128-row block (cta_group::2: a 256 x bn tile, each CTA loading its own
// 128 rows of A' and its bn/2 rows of B'^T).  Its work units are (problem, output tile, K split):
//   warp 0      TMA producer: 128 x 128-byte boxes of A' and bn x 128-byte (bn/2 per CTA of a pair)
//               boxes of B'^T, 128-byte swizzle, into a ring of 6 (pair) or 4 stages (mbarrier
//               complete_tx); no multicast -- every CTA loads its own boxes.
//   warp 1      MMA issuer (one thread of the leading CTA): tcgen05.mma kind::i8, M = 256 (pair) or 128,
//               N = bn, K = 32, s8 x s8 -> s32 in tensor memory (TMEM); commits free the stages and
//               hand the accumulator to the epilogue (multicast to both CTAs of a pair).
//   warps 2..   epilogue, 8 warps for int32 values (two per TMEM lane quarter) or 4 for int64: Horner
//               rescales in TMEM, fold-back, dequantisation, stores.
// The inner dimension of a problem is a sequence of exponent groups whose products carry the weight R^e.
// A unit runs its pieces of them (the plan's steps, cut at the unit's K-split boundaries) in descending
// e into one 256-column TMEM slot; between two pieces of a chunk the epilogue multiplies the slot by
// R^(e_prev - e) in place (Horner's rule); at the end of a chunk, or of the unit's K range, it drains
// the slot into C with the shift of its last group.  Every slot value stays below 2^31: a Horner state
// times R^e is a sum of digit products over a subset of the inner triples, and any such sum is bounded
// by the plan's bound sum_t max|A[:,t]| * max|B[t,:]| (all digits of an entry share its sign), which
// the plan checks against R^e before letting a group join a chunk.
// Two units run interleaved, piece by piece, one per TMEM slot, so that the epilogue works on one slot
// while the tensor cores run the other.  Drain: each epilogue warp owns one TMEM lane quarter = one
// group of 32 unpacked rows of A; a 32-column chunk is one group of 32 unpacked columns of B.  Column
// levels of B are folded inside each thread's registers, the values are transposed through a swizzled
// shared buffer, and row levels of A are folded from consecutive rows of that buffer while every lane
// stores along a row of C.  Without a K split the first drain of a tile writes C and the last also
// writes Cf; with one, the drains add into C atomically (integer sums are exact in any order) after
// the launcher has zeroed it, and a second small kernel writes Cf from the finished C.
// Every mbarrier wait is bounded (common.cuh): a stuck pipeline ends the kernel with IMQ_ERR_TIMEOUT.
#include <string.h>

#include <mutex>
#include <type_traits>
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

// Per CTA: 128 accumulator rows x up to BN columns.  The tile width bn (a multiple of 32, at most BN)
// is chosen per launch so that the tiles spread evenly over the SMs; each TMEM slot spans BN columns.
constexpr int BM = 128, BN = 256, BK = 128;
constexpr int NCHUNK = BN / 32;  // 32-column chunks of a full-width slot
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr int kMaxSplits = 16;   // K splits of one output tile
constexpr int kMaxPieces = kMaxJobs + kMaxSplits;  // a split boundary cuts at most one step in two
constexpr int kMaxProbs = 64;    // problems of one launch (larger batches take several launches)
constexpr int kMaxInlineOrder = 2048;  // tile columns whose order a single-problem launch carries inline

// Epilogue shape per accumulation width: with int32 values two warps share each TMEM lane quarter (each
// takes every other chunk), with int64 values one warp per quarter (its transpose buffer is twice as
// large).  Either way the transpose buffers take 32 KB.
template <bool kWide>
struct Epi {
  static constexpr int kWarps = kWide ? 4 : 8;
  static constexpr int kPerQuarter = kWarps / 4;
  static constexpr int kChunks = NCHUNK / kPerQuarter;  // chunks of a slot per warp
  static constexpr int kThreads = 64 + 32 * kWarps;
  using T = typename std::conditional<kWide, int64_t, int32_t>::type;
  static_assert(kWarps * 32 * 32 * sizeof(T) == 32768, "transpose buffers");
};

// One problem: its operands' tensor maps, its tiles and K splits, its pieces and the fold-back and
// dequantisation data of its epilogue.  Pieces of split s are [split_off[s], split_off[s + 1]).
struct alignas(64) GemmProb {
  CUtensorMap tmA, tmB;
  int32_t tiles_m, tiles_n, splits, n_pieces;
  // tile column order: the k-th column of tiles in schedule order is order[order_off + k] (order_off < 0:
  // k), the order array being GemmLaunch::order for a single problem and the int32 array after the problem
  // table for a table launch.  With B unpacked OUTER its line groups are sorted by level class, so tiles of
  // different classes cover the same output columns; the order interleaves them by position, so that the
  // tiles completing a 32-byte sector of C and Cf run at about the same time.
  int32_t order_off;
  int32_t split_off[kMaxSplits + 1];
  int32_t pc_kb0[kMaxPieces];    // first 128-deep k-block of the piece
  int32_t pc_nkb[kMaxPieces];    // its k-blocks
  int8_t pc_first[kMaxPieces];   // the piece opens a chunk: its first MMA overwrites the slot
  int8_t pc_after[kMaxPieces];   // >= 0: Horner shift of the slot after the piece; -1: drain
  int8_t pc_dshift[kMaxPieces];  // shift of the drained value (e of the piece's group times b-1)
  int8_t pc_dfirst[kMaxPieces];  // the drain is the tile's first: it writes C without reading it
  int8_t pc_dlast[kMaxPieces];   // the drain is the tile's last: it also writes Cf
  int32_t bm1;
  int32_t a_outer, b_outer;
  const int32_t* srcA;
  const int32_t* grpA_L;
  const int32_t* grpA_n;
  int64_t n_grp_a;  // row groups of A' (the last tile may hold fewer than BM / 32)
  const int32_t* srcB;
  const int32_t* grpB_L;
  const int32_t* grpB_n;
  int64_t n_grp_b;
  int64_t M, N;
  const float* dA;
  const float* dB;
  int32_t dA_per_row, dB_per_col;
  void* C;
  int32_t c64;
  int64_t ldc;
  float* Cf;
  int64_t ldcf;
};

// What every unit of a launch shares.  A single problem travels inline (`one`, read from the parameter
// space); a batch of problems is a table in device memory (`probs`).
struct GemmLaunch {
  int32_t bn;      // tile width (columns of C' per tile), a multiple of 32 in [32, BN]
  int32_t nchunk;  // bn / 32
  int32_t nprob;
  int32_t atomic;     // drains add into C atomically (a K-split launch); Cf is written afterwards
  int32_t sched_off;  // slot 1 trails slot 0 by this many pieces (see Order)
  int32_t unit_off[kMaxProbs + 1];  // first unit of each problem
  int32_t* status;
  uint64_t timeout_ns;
  const GemmProb* probs;  // nullptr: the problem is `one`
  GemmProb one;
  int32_t order[kMaxInlineOrder];  // the single problem's tile column order (see GemmProb::order_off)
};
// kernel parameters above 4 KB need CUDA 12.1 or later; the limit there is 32 764 bytes
static_assert(sizeof(GemmLaunch) <= 32764, "GEMM parameters exceed the kernel parameter limit");

// Tile geometry.  One CTA: a 128 x 256 tile, A 128 rows and B 256 rows (of B'^T) per k-block, 4
// stages.  CTA pair (cta_group::2): a 256 x 256 tile, each CTA loading its own 128 rows of A and its
// 128 of the 256 rows of B, so that a k-block costs each SM 32 KB instead of 48 KB; 6 stages.
template <bool kPair>
struct Geo {
  static constexpr int kTM = kPair ? 2 * BM : BM;  // rows of A' per tile
  static constexpr int kBRows = kPair ? BN / 2 : BN;  // B stage rows at the full tile width
  static constexpr int kStages = kPair ? 6 : 4;
  static constexpr int kAStage = BM * BK;  // bytes
  static constexpr int kBStage = kBRows * BK;
  static constexpr size_t kA = 0;
  static constexpr size_t kB = kA + (size_t)kStages * kAStage;
  static constexpr size_t kScratch = kB + (size_t)kStages * kBStage;  // epilogue transpose buffers
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr size_t kBars = kScratch + 32768;
  static constexpr size_t kMisc = kBars + (2 * kStages + 5) * 8;  // tmem base, abort flag
  static constexpr size_t kOut = kMisc + 16;  // per epilogue warp: the drain's output fields (a table launch)
  static constexpr size_t kEnd = kOut + 8 * 64;
  static constexpr size_t kBytes = kEnd + 1024;  // slack for 1024-byte alignment of the base
  static_assert(kBytes <= 232448, "shared memory budget");
};

// A work unit: problem, output tile (mt, nt), K split s, and its pieces [pc0, pc0 + npc).
struct Unit {
  const GemmProb* pb;
  int mt, nt, pc0, npc;
};

// kMulti: the problems are a table in device memory; otherwise the one problem is read from the
// parameter space (the single-problem launch keeps its fields in the constant bank).
template <bool kMulti>
__device__ __forceinline__ const GemmProb* prob_at(const GemmLaunch& L, int p) {
  if constexpr (kMulti)
    return L.probs + p;
  else
    return &L.one;
}

template <bool kMulti>
__device__ __forceinline__ const GemmProb* prob_of(const GemmLaunch& L, int u) {
  int p = 0;
  if constexpr (kMulti)
    while (p + 1 < L.nprob && u >= L.unit_off[p + 1]) ++p;
  return prob_at<kMulti>(L, p);
}

// Units of problem p are unit_off[p] .. unit_off[p + 1] - 1, the K splits of one tile adjacent.
template <bool kMulti>
__device__ Unit unit_of(const GemmLaunch& L, int u) {
  int p = 0;
  if constexpr (kMulti)
    while (p + 1 < L.nprob && u >= L.unit_off[p + 1]) ++p;
  const GemmProb* pb = prob_at<kMulti>(L, p);
  const int local = u - L.unit_off[p];
  const int s = local % pb->splits, tile = local / pb->splits;
  Unit r;
  r.pb = pb;
  r.mt = tile % pb->tiles_m;
  r.nt = tile / pb->tiles_m;
  if (pb->order_off >= 0) {
    if constexpr (kMulti)
      r.nt = reinterpret_cast<const int32_t*>(L.probs + L.nprob)[pb->order_off + r.nt];
    else
      r.nt = L.order[pb->order_off + r.nt];
  }
  r.pc0 = pb->split_off[s];
  r.npc = pb->split_off[s + 1] - r.pc0;
  return r;
}

// The order in which a CTA (pair) runs the pieces of its units.  Its units p = 0, 1, 2, ... (global
// unit first + p * stride) alternate between the two TMEM slots (slot p % 2); each slot runs its units'
// pieces in sequence, and between two pieces of a slot the epilogue works on it (a Horner rescale or a
// drain) while the tensor cores run the other slot's piece.  Slot 1 trails slot 0 by `off` pieces, so
// that a drain (the long epilogue event) overlaps a long piece of the other slot instead of a short
// one: slot 0's j0-th piece runs before slot 1's j1-th while j0 <= j1 + off.  Producer, MMA issuer and
// epilogue walk the same order.
template <bool kMulti>
struct Order {
  const GemmLaunch* L;
  int first, stride, count, off;
  // per slot (0 and 1, kept in named fields so that they stay in registers): local unit index, piece
  // within it, pieces done, and the unit's first piece and piece count
  int p0, p1, k0, k1, j0, j1, a0, a1, n0, n1;
  __device__ void load(int p, int& a, int& n) const {
    if (p < count) {
      const Unit u = unit_of<kMulti>(*L, first + p * stride);
      a = u.pc0;
      n = u.npc;
    }
  }
  __device__ Order(const GemmLaunch& l, int first_, int stride_, int count_)
      : L(&l), first(first_), stride(stride_), count(count_), off(l.sched_off), p0(0), p1(1), k0(0), k1(0), j0(0),
        j1(0), a0(0), a1(0), n0(1), n1(1) {
    load(0, a0, n0);
    load(1, a1, n1);
  }
  __device__ bool done() const { return p0 >= count && p1 >= count; }
  // next (slot, global unit index, piece index into its problem's tables)
  __device__ void next(int& slot, int& unit, int& pc) {
    slot = (p1 >= count || (p0 < count && j0 <= j1 + off)) ? 0 : 1;
    if (slot == 0) {
      unit = first + p0 * stride;
      pc = a0 + k0;
      ++j0;
      if (++k0 == n0) {
        k0 = 0;
        p0 += 2;
        load(p0, a0, n0);
      }
    } else {
      unit = first + p1 * stride;
      pc = a1 + k1;
      ++j1;
      if (++k1 == n1) {
        k1 = 0;
        p1 += 2;
        load(p1, a1, n1);
      }
    }
  }
};

// x * 2^k in the two's-complement type T, through the unsigned type (the plan's bounds guarantee the
// exact result fits T).
template <typename T>
__device__ __forceinline__ T shl(T x, int k) {
  using U = typename std::make_unsigned<T>::type;
  return (T)((U)x << k);
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > timeout_ns) return false;
  return true;
}

// Transpose buffer index: row r, column c, XOR-swizzled so that both a row sweep and a column sweep of
// the warp hit 32 different banks.
__device__ __forceinline__ int sw(int r, int c) { return r * 32 + (c ^ r); }

// Column fold of one 32-column chunk holding 32/L columns of level L, shifted, into the transpose
// buffer: row `lane`, column s = sum_l R^l v[s L + l] * 2^shift.
template <int L, typename T>
__device__ __forceinline__ void fold_store(const uint32_t (&v)[32], T* scr, int lane, int bm1, int shift) {
#pragma unroll
  for (int s = 0; s < 32 / L; ++s) {
    T a = 0;
#pragma unroll
    for (int l = 0; l < L; ++l) a += shl<T>((T)(int32_t)v[s * L + l], l * bm1);
    scr[sw(lane, s)] = shl<T>(a, shift);
  }
}

// The same for levels 9..31 (three columns at most), through the buffer to avoid dynamic register
// indexing.  Each lane reads back only its own row.
template <typename T>
__device__ __forceinline__ void fold_store_deep(const uint32_t (&v)[32], T* scr, int lane, int LB, int nB, int bm1,
                                                int shift) {
#pragma unroll
  for (int k = 0; k < 32; ++k) scr[sw(lane, k)] = (T)(int32_t)v[k];
  T w0 = 0, w1 = 0, w2 = 0;
  for (int l = 0; l < LB; ++l) {
    w0 += shl<T>(scr[sw(lane, l)], l * bm1);
    if (nB > 1) w1 += shl<T>(scr[sw(lane, LB + l)], l * bm1);
    if (nB > 2) w2 += shl<T>(scr[sw(lane, 2 * LB + l)], l * bm1);
  }
  scr[sw(lane, 0)] = shl<T>(w0, shift);
  scr[sw(lane, 1)] = shl<T>(w1, shift);
  scr[sw(lane, 2)] = shl<T>(w2, shift);
}

// Per-warp drain metadata of one tile, fetched before the accumulator is ready.  Lane t holds output
// row t of the warp's row group (its index in C and its dequantisation scale).  In the store phase of a
// chunk with nB output columns, lane t writes column s = t % nB of the rows r0 = t / nB, r0 + per, ...
// (per = 32 / nB rows at a time), so that all lanes store even when nB < 32.  NC = chunks of this warp.
template <int NC>
struct DrainMeta {
  int LA, nA;
  int32_t my_row;
  float my_sa;
  int32_t pk[NC];   // per chunk: nB | LB << 6 | s << 12 | r0 << 18 | per << 24 (r0 = 63: idle lane)
  int32_t col[NC];  // the output column of this lane's s in each chunk
  float sb[NC];     // its dequantisation scale
};

__device__ __forceinline__ int pk_nB(int32_t pk) { return pk & 63; }
__device__ __forceinline__ int pk_LB(int32_t pk) { return (pk >> 6) & 63; }
__device__ __forceinline__ int pk_s(int32_t pk) { return (pk >> 12) & 63; }
__device__ __forceinline__ int pk_r0(int32_t pk) { return (pk >> 18) & 63; }
__device__ __forceinline__ int pk_per(int32_t pk) { return (pk >> 24) & 63; }

// Chunks of warp h (of PQ warps on the quarter): h, h + PQ, h + 2 PQ, ...  row0: the first row of A'
// in this CTA's accumulator.  `scales`: the drain writes Cf (its scales are fetched).
template <int NC, int PQ>
__device__ __forceinline__ void drain_prepare(const GemmProb& g, int nchunk, int64_t row0, int nt, int q, int h,
                                              int lane, bool scales, DrainMeta<NC>& m) {
  int64_t my_row;
  if (g.a_outer) {
    const int64_t grp = row0 / 32 + q;
    m.LA = grp < g.n_grp_a ? g.grpA_L[grp] : 1;
    m.nA = grp < g.n_grp_a ? g.grpA_n[grp] : 0;
    my_row = lane < m.nA ? g.srcA[grp * 32 + (int64_t)lane * m.LA] : 0;
  } else {
    m.LA = 1;
    const int64_t r0 = row0 + q * 32;
    const int64_t rem = g.M - r0;
    m.nA = rem <= 0 ? 0 : (rem < 32 ? (int)rem : 32);
    my_row = lane < m.nA ? r0 + lane : 0;
  }
  m.my_row = (int32_t)my_row;
  m.my_sa = (scales && g.Cf && lane < m.nA) ? g.dA[g.dA_per_row ? my_row : 0] : 0.0f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = h + PQ * i;
    const int64_t gc = (int64_t)nt * nchunk + c;
    int LB = 1, nB = 0;
    if (c >= nchunk) {
      // beyond this launch's tile width: nothing to store
    } else if (g.b_outer) {
      LB = gc < g.n_grp_b ? g.grpB_L[gc] : 1;
      nB = gc < g.n_grp_b ? g.grpB_n[gc] : 0;
    } else {
      const int64_t rem = g.N - gc * 32;
      nB = rem <= 0 ? 0 : (rem < 32 ? (int)rem : 32);
    }
    int s = 0, r0 = 63, per = 1;
    if (nB > 0) {
      per = 32 / nB;
      s = lane % nB;
      r0 = lane / nB;
      if (r0 >= per) r0 = 63;
    }
    m.pk[i] = nB | (LB << 6) | (s << 12) | (r0 << 18) | (per << 24);
    m.col[i] = 0;
    if (r0 != 63) m.col[i] = g.b_outer ? g.srcB[gc * 32 + (int64_t)s * LB] : (int32_t)(gc * 32 + s);
  }
#pragma unroll
  for (int i = 0; i < NC; ++i)
    m.sb[i] = (scales && g.Cf && pk_r0(m.pk[i]) != 63) ? g.dB[g.dB_per_col ? m.col[i] : 0] : 0.0f;
}

// Releases a slot to the MMA issuer: a local arrive, or for a CTA pair an arrive on the leading CTA's
// barrier (acce_bar is then its shared::cluster address).
template <bool kPair>
__device__ __forceinline__ void release_slot(uint32_t acce_bar) {
  if constexpr (kPair)
    mbar_arrive_cluster(acce_bar);
  else
    mbar_arrive(acce_bar);
}

// Drains this warp's chunks of one TMEM slot (its 32 lanes) into C: fold, shift, then write (first),
// add (a later drain of the same tile), or add atomically (atomic: several K splits share the tile).
// `last` (never with atomic): also writes Cf.
// The problem's output fields, read once per drain into registers (a problem table in global memory could
// alias the drain's own stores as far as the compiler knows, which would reload them at every store).
struct DrainOut {
  void* C;
  float* Cf;
  int64_t ldc, ldcf;
  int32_t c64, bm1;
};

template <typename T, int NC, int PQ, bool kPair>
__device__ __forceinline__ void drain_slot(const DrainOut& g, uint32_t tbase, uint32_t acce_bar, int lane, int h,
                                           bool first, bool last, bool atomic, int shift, T* scr,
                                           const DrainMeta<NC>& m) {
  uint32_t v[32];
  tmem_ld32(tbase + h * 32, v);
#pragma unroll 1
  for (int i = 0; i < NC; ++i) {
    tmem_wait_ld();
    // dynamic indexing of the unrolled metadata arrays is avoided by a uniform select
    int32_t pk = 0, mycol = 0;
    float sb = 0.0f;
#pragma unroll
    for (int k = 0; k < NC; ++k)
      if (k == i) {
        pk = m.pk[k];
        mycol = m.col[k];
        sb = m.sb[k];
      }
    const int LB = pk_LB(pk), nB = pk_nB(pk);
    const int nA = m.nA, LA = m.LA;
    const bool work = nB > 0 && nA > 0;
    // 1. fold the column levels of B inside the registers (row = lane = unpacked row) into the buffer
    if (work) {
      switch (LB) {
        case 1: fold_store<1, T>(v, scr, lane, g.bm1, shift); break;
        case 2: fold_store<2, T>(v, scr, lane, g.bm1, shift); break;
        case 3: fold_store<3, T>(v, scr, lane, g.bm1, shift); break;
        case 4: fold_store<4, T>(v, scr, lane, g.bm1, shift); break;
        case 5: fold_store<5, T>(v, scr, lane, g.bm1, shift); break;
        case 6: fold_store<6, T>(v, scr, lane, g.bm1, shift); break;
        case 7: fold_store<7, T>(v, scr, lane, g.bm1, shift); break;
        case 8: fold_store<8, T>(v, scr, lane, g.bm1, shift); break;
        default: fold_store_deep<T>(v, scr, lane, LB, nB, g.bm1, shift);
      }
    }
    // 2. the registers are free: this warp's next chunk streams in while this one is stored; after the
    //    last chunk the slot is released to the MMA warp
    if (i + 1 < NC) {
      tmem_ld32(tbase + (h + PQ * (i + 1)) * 32, v);
    } else {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release_slot<kPair>(acce_bar);
    }
    __syncwarp();
    // 3. lane (r0, s) stores column s of output rows r0, r0 + per, ...; the row levels of A (OUTER
    //    unpacking) are folded here, from LA consecutive rows of the buffer.  The trip count is uniform
    //    so that every lane takes part in the shuffles of the row metadata.
    if (work) {
      const int s = pk_s(pk), per = pk_per(pk), r0 = pk_r0(pk);
      const int iters = (nA + per - 1) / per;
#pragma unroll 2
      for (int it = 0; it < iters; ++it) {
        const int t = r0 + it * per;
        const int src = t < 32 ? t : 0;
        const int64_t row = __shfl_sync(0xffffffffu, m.my_row, src);
        const float sa = __shfl_sync(0xffffffffu, m.my_sa, src);
        if (t < nA) {
          T val;
          if (LA == 1) {
            val = scr[sw(t, s)];
          } else {
            val = 0;
            for (int l = 0; l < LA; ++l) val += shl<T>(scr[sw(t * LA + l, s)], l * g.bm1);
          }
          if (g.C) {
            if (g.c64) {
              int64_t* cp = static_cast<int64_t*>(g.C) + row * g.ldc + mycol;
              if (atomic) {
                atomicAdd(reinterpret_cast<unsigned long long*>(cp), (unsigned long long)(int64_t)val);
              } else {
                if (!first) val += (T)*cp;
                *cp = (int64_t)val;
              }
            } else {
              int32_t* cp = static_cast<int32_t*>(g.C) + row * g.ldc + mycol;
              if (atomic) {
                atomicAdd(cp, (int32_t)val);
              } else {
                if (!first) val += (T)*cp;
                *cp = (int32_t)val;
              }
            }
          }
          if (last && g.Cf)
            g.Cf[row * g.ldcf + mycol] =
                __fmul_rn(sizeof(T) == 8 ? __ll2float_rn((long long)val) : __int2float_rn((int)val),
                          __fmul_rn(sa, sb));
        }
      }
    }
    __syncwarp();
  }
}

// Acquire, for the tensor-map proxy, a map that a host copy wrote into device memory.
__device__ __forceinline__ void tensormap_acquire(const void* p) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(p))
               : "memory");
}

template <bool kWide, bool kPair, bool kMulti>
__global__ void __launch_bounds__(Epi<kWide>::kThreads, 1) k_gemm(const __grid_constant__ GemmLaunch L) {
  using G = Geo<kPair>;
  using E = Epi<kWide>;
  using T = typename E::T;
  constexpr int STAGES = G::kStages;
  constexpr int A_STAGE = G::kAStage, B_STAGE = G::kBStage;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + G::kA;
  uint8_t* sB = base + G::kB;
  T* scratch = reinterpret_cast<T*>(base + G::kScratch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + G::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + G::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + G::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + STAGES);
  const uint32_t accf0 = smem_addr(bars + 2 * STAGES), acce0 = smem_addr(bars + 2 * STAGES + 2);
  const uint32_t drain_bar = smem_addr(bars + 2 * STAGES + 4);
  constexpr uint32_t kCols = 2 * BN;  // two accumulator slots
  // CTA pair: rank 0 leads (issues the MMAs, owns the barriers both CTAs' loads and epilogues signal)
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(accf0 + 8 * s, 1);
      mbar_init(acce0 + 8 * s, E::kWarps * (kPair ? 2 : 1));  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    // the maps of a problem table were written by a host copy: acquire them for the TMA unit
    for (int p = 0; p < L.nprob; ++p) {
      const GemmProb* pb = prob_at<kMulti>(L, p);
      if (kMulti) {
        tensormap_acquire(&pb->tmA);
        tensormap_acquire(&pb->tmB);
      }
      if (p < 4) {
        tma_prefetch_desc(&pb->tmA);
        tma_prefetch_desc(&pb->tmB);
      }
    }
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_addr(tmem_holder), kCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(tmem_holder), kCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // the peer's barriers must be initialised before any load or arrive reaches them
  if constexpr (kPair)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_units = L.unit_off[L.nprob];
  // the units of this CTA (or pair): first + p * stride, p = 0 .. count - 1
  const int first = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int stride = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int count = first < num_units ? (num_units - first + stride - 1) / stride : 0;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // rows of B'^T this CTA loads per k-block (half the tile width for a pair) and their bytes
      const int32_t b_rows = kPair ? L.bn / 2 : L.bn;
      const uint32_t b_bytes = (uint32_t)b_rows * BK;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 2;
      Order<kMulti> ord(L, first, stride, count);
      while (!ord.done()) {
        int slot, u, pc;
        ord.next(slot, u, pc);
        const Unit un = unit_of<kMulti>(L, u);
        const GemmProb& g = *un.pb;
        const int32_t ya = un.mt * G::kTM + (int32_t)rank * BM, yb = un.nt * L.bn + (int32_t)rank * b_rows;
        const int32_t kb0 = g.pc_kb0[pc], nkb = g.pc_nkb[pc];
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, L.status, L.timeout_ns)) goto producer_done;
          const uint32_t fb = full0 + 8 * stage;
          const int32_t kx = (kb0 + kb) * BK;
          if constexpr (kPair) {
            // both CTAs' bytes complete the leader's barrier, which expects them all
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * (A_STAGE + b_bytes));
            const uint32_t lfb = mapa_shared(fb, 0);
            tma_load_2d_pair(smem_addr(sA + (size_t)stage * A_STAGE), &g.tmA, kx, ya, lfb);
            tma_load_2d_pair(smem_addr(sB + (size_t)stage * B_STAGE), &g.tmB, kx, yb, lfb);
          } else {
            mbar_arrive_expect_tx(fb, A_STAGE + b_bytes);
            tma_load_2d(smem_addr(sA + (size_t)stage * A_STAGE), &g.tmA, kx, ya, fb);
            tma_load_2d(smem_addr(sB + (size_t)stage * B_STAGE), &g.tmB, kx, yb, fb);
          }
          issued[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      // every issued copy must land before the CTA may exit.  In a pair the leader's full barriers
      // complete only with both CTAs' bytes, so the leader's wait covers the peer's copies as well.
      if (!kPair || rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (issued[s] != 2) drain_wait(full0 + 8 * s, issued[s], L.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_i8(G::kTM, (uint32_t)L.bn);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t empty_waits[2] = {0, 0};
      Order<kMulti> ord(L, first, stride, count);
      while (!ord.done()) {
        int slot, u, pc;
        ord.next(slot, u, pc);
        const GemmProb& g = *prob_of<kMulti>(L, u);
        // the epilogue (of both CTAs) has finished the previous event of this slot
        if (!mbar_wait(acce0 + 8 * slot, (empty_waits[slot] & 1u) ^ 1u, abort_flag, L.status, L.timeout_ns))
          goto mma_done;
        ++empty_waits[slot];
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)slot * BN;
        const bool firstp = g.pc_first[pc] != 0;
        const int32_t nkb = g.pc_nkb[pc];
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, L.status, L.timeout_ns)) goto mma_done;
          tc_fence_after();
          const uint64_t adesc = smem_desc_k_sw128(smem_addr(sA + (size_t)stage * A_STAGE));
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sB + (size_t)stage * B_STAGE));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // 32 bytes further along K inside the 128-byte swizzled row: +2 in the address field
            const uint32_t acc = (firstp && kb == 0 && kk == 0) ? 0u : 1u;
            if constexpr (kPair)
              mma_i8_pair(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, acc);
            else
              mma_i8(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, acc);
          }
          // the stage is free again in both CTAs once these MMAs have read it
          if constexpr (kPair)
            mma_commit_pair_mc(empty0 + 8 * stage, 0x3);
          else
            mma_commit(empty0 + 8 * stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if constexpr (kPair)
          mma_commit_pair_mc(accf0 + 8 * slot, 0x3);
        else
          mma_commit(accf0 + 8 * slot);
      }
    mma_done:
      // every issued MMA must complete before tensor memory is released
      if constexpr (kPair)
        mma_commit_pair(drain_bar);
      else
        mma_commit(drain_bar);
      drain_wait(drain_bar, 0, L.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    constexpr int PQ = E::kPerQuarter, NC = E::kChunks;
    const int ew = warp - 2;       // epilogue warp 0 .. kWarps-1
    const int q = warp & 3;        // TMEM lane quarter this warp may access = row group of the tile
    const int h = ew / 4;          // which of the quarter's warps: chunks h, h + PQ, ...
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    T* scr = scratch + ew * 32 * 32;  // this warp's transpose buffer (XOR-swizzled rows of 32)
    DrainOut* wout = reinterpret_cast<DrainOut*>(base + G::kOut) + ew;
    // where a released slot is signalled: this CTA's barrier, or the leader's for a pair
    const uint32_t rel0 = kPair ? mapa_shared(acce0, 0) : acce0;
    const uint32_t rel1 = kPair ? mapa_shared(acce0 + 8, 0) : acce0 + 8;
    const bool atomic = L.atomic != 0;
    uint32_t full_waits[2] = {0, 0};
    Order<kMulti> ord(L, first, stride, count);
    while (!ord.done()) {
      int slot, u, pc;
      ord.next(slot, u, pc);
      const Unit un = unit_of<kMulti>(L, u);
      const GemmProb& g = *un.pb;
      DrainMeta<NC> meta;
      const bool drain = g.pc_after[pc] < 0;
      const bool last = !atomic && g.pc_dlast[pc] != 0;
      if (drain) {
        // metadata of the tile first: its loads overlap the wait for the accumulator
        const int64_t row0 = (int64_t)un.mt * G::kTM + (int64_t)rank * BM;
        drain_prepare<NC, PQ>(g, L.nchunk, row0, un.nt, q, h, lane, last, meta);
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(accf0 + 8 * slot, full_waits[slot] & 1u, abort_flag, L.status, L.timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++full_waits[slot];
      if (!ok) goto epi_done;
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_off + (uint32_t)slot * BN;
      const uint32_t rel = slot ? rel1 : rel0;
      if (!drain) {
        // Horner step: slot *= R^(e_prev - e), in place.  The plan bounds the result by 2^31, so
        // a shift of 31 or more only meets zeros.
        const int sh = g.pc_after[pc];
        // two register buffers: the next chunk's load is in flight while this one is shifted and stored
        uint32_t v0[32], v1[32];
        tmem_ld32(tbase + h * 32, v0);
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          uint32_t(&cur)[32] = (i & 1) ? v1 : v0;
          uint32_t(&nxt)[32] = (i & 1) ? v0 : v1;
          tmem_wait_ld();
          if (i + 1 < NC) tmem_ld32(tbase + (h + PQ * (i + 1)) * 32, nxt);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) cur[jj] = sh < 31 ? (cur[jj] << sh) : 0u;
          tmem_st32(tbase + (h + PQ * i) * 32, cur);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_slot<kPair>(rel);
      } else {
        if constexpr (kMulti) {
          // from the table into this warp's shared slot, read from there by the stores
          if (lane == 0) *wout = DrainOut{g.C, g.Cf, g.ldc, g.ldcf, g.c64, g.bm1};
          __syncwarp();
          drain_slot<T, NC, PQ, kPair>(*wout, tbase, rel, lane, h, g.pc_dfirst[pc] != 0, last, atomic,
                                       g.pc_dshift[pc], scr, meta);
        } else {
          const DrainOut out{g.C, g.Cf, g.ldc, g.ldcf, g.c64, g.bm1};
          drain_slot<T, NC, PQ, kPair>(out, tbase, rel, lane, h, g.pc_dfirst[pc] != 0, last, atomic, g.pc_dshift[pc],
                                       scr, meta);
        }
      }
    }
  epi_done:;
  }
  tc_fence_before();
  // neither CTA of a pair leaves (or releases tensor memory) while the other may still reach it
  if constexpr (kPair)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, kCols);
    else
      tmem_dealloc(tmem_base, kCols);
  }
}

// K-split launches: C of every problem is zeroed before the GEMM adds into it, and Cf is written from the
// finished C afterwards with the epilogue's rounding (fl(fl(C) * fl(deltaA * deltaB))).  blockIdx.y =
// problem; grid-stride over its rows and columns.
__global__ void __launch_bounds__(256) k_zero_c(const GemmProb* __restrict__ probs, const GemmProb one) {
  const GemmProb& g = probs ? probs[blockIdx.y] : one;
  if (!g.C) return;
  const int64_t n = g.M * g.N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / g.N, c = i - r * g.N;
    if (g.c64)
      static_cast<int64_t*>(g.C)[r * g.ldc + c] = 0;
    else
      static_cast<int32_t*>(g.C)[r * g.ldc + c] = 0;
  }
}

__global__ void __launch_bounds__(256) k_dequant_c(const GemmProb* __restrict__ probs, const GemmProb one) {
  const GemmProb& g = probs ? probs[blockIdx.y] : one;
  if (!g.Cf || !g.C) return;
  const int64_t n = g.M * g.N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / g.N, c = i - r * g.N;
    const float sa = g.dA[g.dA_per_row ? r : 0], sb = g.dB[g.dB_per_col ? c : 0];
    const float v = g.c64 ? __ll2float_rn((long long)static_cast<const int64_t*>(g.C)[r * g.ldc + c])
                          : __int2float_rn(static_cast<const int32_t*>(g.C)[r * g.ldc + c]);
    g.Cf[r * g.ldcf + c] = __fmul_rn(v, __fmul_rn(sa, sb));
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D int8 K-major tensor map: `rows` lines of `k` bytes, boxes of box_rows x 128 bytes, 128B swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int64_t k, int64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)k};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Makespan, in SM cycles, of the piece order of a CTA with `units` units of `n` pieces each (the pieces
// of one unit) when slot 1 trails by `off` pieces: a piece occupies the tensor cores for 2 bn cycles per
// 128-deep k-block (M=128, N=256, K=32 in 128 cycles per SM), and the epilogue event after it (done in
// order) takes `rescale` or `drain` cycles.  A slot's next piece waits for the slot's previous event.
// Used only to pick `off`.
double simulate_order(const GemmProb& g, int bn, int pc0, int n, int units, int off, double rescale, double drain) {
  const int len0 = ((units + 1) / 2) * n, len1 = (units / 2) * n;
  double mma_free = 0.0, epi_free = 0.0, slot_ready[2] = {0.0, 0.0};
  int j0 = 0, j1 = 0;
  for (int e = 0; e < len0 + len1; ++e) {
    int slot, j;
    if (j1 >= len1 || (j0 < len0 && j0 <= j1 + off)) {
      slot = 0;
      j = j0++;
    } else {
      slot = 1;
      j = j1++;
    }
    const int k = pc0 + j % n;
    const double start = mma_free > slot_ready[slot] ? mma_free : slot_ready[slot];
    const double end = start + 2.0 * bn * g.pc_nkb[k];
    mma_free = end;
    const double ev_start = epi_free > end ? epi_free : end;
    epi_free = ev_start + (g.pc_after[k] >= 0 ? rescale : drain);
    slot_ready[slot] = epi_free;
  }
  return mma_free > epi_free ? mma_free : epi_free;
}

// The pieces of a plan's steps for S K-splits: split s takes k-blocks [s T / S, (s+1) T / S) of the
// tile's k-blocks in step order (T in all).  A piece opens a chunk when its step does, and also when it
// opens its split; it ends in a drain when its step does, and also when it ends its split (the slot then
// holds a Horner state whose shift is that of the piece's group).  Shifts are clamped to 63: a larger
// one only meets zeros, since the product fits int64.
bool build_pieces(const imq_plan_t* pl, int S, GemmProb* g) {
  int64_t T = 0;
  for (int k = 0; k < pl->n_steps; ++k) T += pl->step_klen[k] / BK;
  if (S < 1 || S > kMaxSplits || (S > 1 && T < S)) return false;
  int n = 0;
  int first_drain = -1, last_drain = -1;
  for (int s = 0; s < S; ++s) {
    const int64_t b0 = T * s / S, b1 = T * (s + 1) / S;
    g->split_off[s] = n;
    int64_t cum = 0;
    for (int k = 0; k < pl->n_steps; ++k) {
      const int64_t nk = pl->step_klen[k] / BK, k0 = pl->step_k0[k] / BK;
      const int64_t lo = b0 > cum ? b0 : cum, hi = b1 < cum + nk ? b1 : cum + nk;
      if (lo < hi) {
        if (n >= kMaxPieces) return false;
        const bool opens = n == g->split_off[s];
        const bool ends_split = hi == b1;
        g->pc_kb0[n] = (int32_t)(k0 + (lo - cum));
        g->pc_nkb[n] = (int32_t)(hi - lo);
        g->pc_first[n] = (int8_t)(opens || (pl->step_first[k] && lo == cum));
        const int dsh = pl->step_drain_shift[k] < 63 ? pl->step_drain_shift[k] : 63;
        g->pc_dshift[n] = (int8_t)dsh;
        if (ends_split || pl->step_after[k] < 0) {
          g->pc_after[n] = -1;
        } else {
          g->pc_after[n] = (int8_t)(pl->step_after[k] < 63 ? pl->step_after[k] : 63);
        }
        g->pc_dfirst[n] = 0;
        g->pc_dlast[n] = 0;
        if (g->pc_after[n] < 0) {
          if (first_drain < 0) first_drain = n;
          last_drain = n;
        }
        ++n;
      }
      cum += nk;
    }
  }
  g->split_off[S] = n;
  g->n_pieces = n;
  g->splits = S;
  // without a split the tile's first drain writes C and its last also writes Cf
  if (S == 1 && first_drain >= 0) {
    g->pc_dfirst[first_drain] = 1;
    g->pc_dlast[last_drain] = 1;
  }
  return true;
}

template <bool kWide, bool kPair, bool kMulti>
imq_status launch_k_gemm(int grid, const GemmLaunch& L, cudaStream_t st) {
  auto kern = k_gemm<kWide, kPair, kMulti>;
  const size_t smem = Geo<kPair>::kBytes;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)Epi<kWide>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kPair ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kPair ? 1 : 0;  // single CTAs launch without a cluster
  IMQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, L));
  return IMQ_OK;
}

// Checks one problem's arguments; *skip when it has nothing for the GEMM kernel (empty output, or an
// empty inner dimension whose outputs are zeroed here).
imq_status check_spec(const GemmSpec& s, bool* skip, cudaStream_t st) {
  const imq_plan_t* pl = s.plan;
  const imq_plan_info& I = pl->info;
  *skip = true;
  if (!s.C && !s.Cf) return IMQ_ERR_ARG;
  if (s.C && s.ct != IMQ_I32 && s.ct != IMQ_I64) return IMQ_ERR_ARG;
  if (s.C && s.ldc < I.N) return IMQ_ERR_ARG;
  if (s.Cf && (s.ldcf < I.N || !s.dA || !s.dB)) return IMQ_ERR_ARG;
  if (s.Cf && s.gA != IMQ_PER_TENSOR && s.gA != IMQ_PER_ROW) return IMQ_ERR_ARG;
  if (s.Cf && s.gB != IMQ_PER_TENSOR && s.gB != IMQ_PER_COL) return IMQ_ERR_ARG;
  if (s.C && s.ct == IMQ_I32 && I.acc_bits > 32) return IMQ_ERR_RANGE;
  if (!s.C && pl->n_chunks > 1) return IMQ_ERR_ARG;  // several chunks of a tile accumulate in C
  if (I.M == 0 || I.N == 0) return IMQ_OK;
  const size_t esz = s.ct == IMQ_I64 ? 8 : 4;
  if (I.K_unp == 0) {
    if (s.C) IMQ_CUDA_TRY(cudaMemset2DAsync(s.C, (size_t)s.ldc * esz, 0, (size_t)I.N * esz, (size_t)I.M, st));
    if (s.Cf) IMQ_CUDA_TRY(cudaMemset2DAsync(s.Cf, (size_t)s.ldcf * 4, 0, (size_t)I.N * 4, (size_t)I.M, st));
    return IMQ_OK;
  }
  if (!s.Au || !s.Bu) return IMQ_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(s.Au) & 15) || (reinterpret_cast<uintptr_t>(s.Bu) & 15)) return IMQ_ERR_ARG;
  *skip = false;
  return IMQ_OK;
}

// One launch over `n` problems (n <= kMaxProbs, each checked and non-empty).
imq_status launch_group(const GemmSpec* const* specs, int n, DeviceState* ds, cudaStream_t st) {
  // a CTA pair per 256 x bn tile whenever some A' has more than one 128-row block
  bool pair = false, wide = false, all_c = true;
  for (int i = 0; i < n; ++i) {
    const imq_plan_info& I = specs[i]->plan->info;
    pair = pair || (I.M_unp > BM && ds->num_sms >= 2);
    // int64 accumulation in the epilogue whenever the output is int64 or the bound exceeds int32
    wide = wide || (specs[i]->C && specs[i]->ct == IMQ_I64) || I.acc_bits > 32;
    all_c = all_c && specs[i]->C != nullptr;
  }
  const int tm = pair ? Geo<true>::kTM : Geo<false>::kTM;
  const int max_units = pair ? ds->num_sms / 2 : ds->num_sms;
  // tile width: the fewest columns per SM over the busiest unit, ceil(tiles / units) * bn (a tile's
  // tensor-core time is proportional to bn), plus a per-tile cost worth 96 columns (operand re-reads,
  // the epilogue's fixed work, the pipeline's start and end) so that narrower tiles are taken only
  // where they add parallelism (fewer tiles than units) or save a whole wave
  int bn = BN;
  {
    double best = 0.0;
    for (int c = BN; c >= 128; c -= 32) {
      int64_t tiles = 0;
      for (int i = 0; i < n; ++i) {
        const imq_plan_info& I = specs[i]->plan->info;
        tiles += ((I.M_unp + tm - 1) / tm) * ((I.N_unp + c - 1) / c);
      }
      const int64_t units = tiles < max_units ? tiles : max_units;
      const int64_t waves = (tiles + units - 1) / units;
      const double cost = (double)waves * (c + 96);
      if (c == BN || cost < best) {
        best = cost;
        bn = c;
      }
    }
  }
  int64_t tiles = 0, kblocks = 0;
  for (int i = 0; i < n; ++i) {
    const imq_plan_info& I = specs[i]->plan->info;
    tiles += ((I.M_unp + tm - 1) / tm) * ((I.N_unp + bn - 1) / bn);
    int64_t T = 0;
    for (int k = 0; k < specs[i]->plan->n_steps; ++k) T += specs[i]->plan->step_klen[k] / BK;
    kblocks = (i == 0 || T < kblocks) ? T : kblocks;
  }
  // K splits when the tiles leave units idle: as many as fill the units, each split keeping at least 16
  // k-blocks (a drain costs about as much as 16 k-blocks of MMAs); only with C given (the splits add
  // into it)
  int S = 1;
  if (all_c && tiles < max_units) {
    S = (int)(max_units / tiles);
    if (S > kMaxSplits) S = kMaxSplits;
    while (S > 1 && kblocks / S < 16) --S;
  }

  // tile column orders of the problems with B unpacked OUTER: columns sorted by the mean position of their
  // line groups (stable), all problems' orders in one upload
  std::vector<int32_t> orders;
  std::vector<int64_t> order_off((size_t)n, -1);
  for (int i = 0; i < n; ++i) {
    const imq_plan_t* pl = specs[i]->plan;
    std::vector<float> gpos;
    const int64_t tn = (pl->info.N_unp + bn - 1) / bn;
    if (tn < 2 || !b_group_positions(pl, &gpos)) continue;
    const int64_t gpt = bn / 32;  // line groups per tile column
    std::vector<std::pair<float, int32_t>> key((size_t)tn);
    for (int64_t t = 0; t < tn; ++t) {
      double sum = 0.0;
      int64_t cnt = 0;
      for (int64_t g = t * gpt; g < (t + 1) * gpt && g < (int64_t)gpos.size(); ++g, ++cnt) sum += gpos[(size_t)g];
      key[(size_t)t] = {cnt ? (float)(sum / (double)cnt) : 1.0f, (int32_t)t};
    }
    std::stable_sort(key.begin(), key.end(),
                     [](const std::pair<float, int32_t>& x, const std::pair<float, int32_t>& y) { return x.first < y.first; });
    order_off[(size_t)i] = (int64_t)orders.size();
    for (const auto& kv : key) orders.push_back(kv.second);
  }

  GemmLaunch* Lp = new GemmLaunch;
  GemmLaunch& L = *Lp;
  memset(&L, 0, sizeof(L));
  std::vector<GemmProb> tab(n > 1 ? n : 0);
  int32_t units = 0;
  for (int i = 0; i < n; ++i) {
    const GemmSpec& s = *specs[i];
    const imq_plan_t* pl = s.plan;
    const imq_plan_info& I = pl->info;
    GemmProb& g = n > 1 ? tab[i] : L.one;
    memset(&g, 0, sizeof(g));
    g.tiles_m = (int32_t)((I.M_unp + tm - 1) / tm);
    g.tiles_n = (int32_t)((I.N_unp + bn - 1) / bn);
    g.order_off = (int32_t)order_off[(size_t)i];
    if (n == 1 && g.order_off >= 0) {
      // a single problem carries its order in the parameters, when it fits
      if ((int64_t)orders.size() <= kMaxInlineOrder)
        memcpy(L.order, orders.data(), sizeof(int32_t) * orders.size());
      else
        g.order_off = -1;
    }
    if (!build_pieces(pl, S, &g)) {
      delete Lp;
      return IMQ_ERR_UNSUPPORTED;
    }
    if (!make_map(&g.tmA, s.Au, I.K_unp, I.M_unp, BM) ||
        !make_map(&g.tmB, s.Bu, I.K_unp, I.N_unp, (uint32_t)(pair ? bn / 2 : bn))) {
      delete Lp;
      return IMQ_ERR_CUDA;
    }
    g.bm1 = I.b - 1;
    g.a_outer = (I.dir_a & IMQ_DIR_OUTER) != 0;
    g.b_outer = (I.dir_b & IMQ_DIR_OUTER) != 0;
    g.srcA = pl->srcA;
    g.grpA_L = pl->grpA_L;
    g.grpA_n = pl->grpA_n;
    g.n_grp_a = pl->n_grp_a;
    g.srcB = pl->srcB;
    g.grpB_L = pl->grpB_L;
    g.grpB_n = pl->grpB_n;
    g.n_grp_b = pl->n_grp_b;
    g.M = I.M;
    g.N = I.N;
    g.dA = s.dA;
    g.dB = s.dB;
    g.dA_per_row = s.gA == IMQ_PER_ROW;
    g.dB_per_col = s.gB == IMQ_PER_COL;
    g.C = s.C;
    g.c64 = s.C != nullptr && s.ct == IMQ_I64;
    g.ldc = s.ldc;
    g.Cf = s.Cf;
    g.ldcf = s.ldcf;
    L.unit_off[i] = units;
    units += g.tiles_m * g.tiles_n * g.splits;
  }
  L.unit_off[n] = units;
  L.bn = bn;
  L.nchunk = bn / 32;
  L.nprob = n;
  L.atomic = S > 1;
  L.status = ds->status;
  L.timeout_ns = kTimeoutNs;
  const GemmProb& g0 = n > 1 ? tab[0] : L.one;
  const int ctas = units < max_units ? units : max_units;
  const int grid = pair ? 2 * ctas : ctas;
  // the trailing offset of slot 1 with the shortest modelled makespan for the busiest CTA (pieces of
  // problem 0's first split); the event costs are rough per-tile figures of the epilogue (a rescale is
  // one TMEM read and write of the slot, a drain also folds and stores it, half as fast with int64
  // values and half the warps)
  {
    const int per = (units + ctas - 1) / ctas;
    const double rescale = wide ? 3000.0 : 1500.0, drain = wide ? 28000.0 : 14000.0;
    const int npc = g0.split_off[1] - g0.split_off[0];
    double best = simulate_order(g0, bn, 0, npc, per, 0, rescale, drain);
    L.sched_off = 0;
    for (int off = 1; off < npc && off <= 16; ++off) {
      const double t = simulate_order(g0, bn, 0, npc, per, off, rescale, drain);
      if (t < best) {
        best = t;
        L.sched_off = off;
      }
    }
  }
  imq_status s = IMQ_OK;
  GemmProb* dtab = nullptr;
  if (n > 1) {
    // the problem table, then the problems' tile column orders (int32), in one upload
    std::vector<char> blob(sizeof(GemmProb) * (size_t)n + sizeof(int32_t) * orders.size());
    memcpy(blob.data(), tab.data(), sizeof(GemmProb) * (size_t)n);
    if (!orders.empty()) memcpy(blob.data() + sizeof(GemmProb) * (size_t)n, orders.data(), sizeof(int32_t) * orders.size());
    void* d = nullptr;
    s = upload_table(blob.data(), blob.size(), &d, st);
    dtab = static_cast<GemmProb*>(d);
    L.probs = dtab;
  }
  if (s == IMQ_OK && L.atomic) {
    const dim3 zg((unsigned)(ds->num_sms * 2), (unsigned)n);
    k_zero_c<<<zg, 256, 0, st>>>(L.probs, L.one);
    if (cudaGetLastError() != cudaSuccess) s = IMQ_ERR_CUDA;
  }
  if (s == IMQ_OK) {
    if (n > 1) {
      if (wide)
        s = pair ? launch_k_gemm<true, true, true>(grid, L, st) : launch_k_gemm<true, false, true>(grid, L, st);
      else
        s = pair ? launch_k_gemm<false, true, true>(grid, L, st) : launch_k_gemm<false, false, true>(grid, L, st);
    } else {
      if (wide)
        s = pair ? launch_k_gemm<true, true, false>(grid, L, st) : launch_k_gemm<true, false, false>(grid, L, st);
      else
        s = pair ? launch_k_gemm<false, true, false>(grid, L, st) : launch_k_gemm<false, false, false>(grid, L, st);
    }
  }
  if (s == IMQ_OK && L.atomic) {
    const dim3 zg((unsigned)(ds->num_sms * 2), (unsigned)n);
    k_dequant_c<<<zg, 256, 0, st>>>(L.probs, L.one);
    if (cudaGetLastError() != cudaSuccess) s = IMQ_ERR_CUDA;
  }
  if (dtab) cudaFreeAsync(dtab, st);
  delete Lp;
  return s;
}

}  // namespace

imq_status launch_gemm_multi(const GemmSpec* specs, int n, cudaStream_t st) {
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  std::vector<const GemmSpec*> live;
  for (int i = 0; i < n; ++i) {
    bool skip = true;
    s = check_spec(specs[i], &skip, st);
    if (s != IMQ_OK) return s;
    if (!skip) live.push_back(specs + i);
  }
  for (size_t i = 0; i < live.size(); i += kMaxProbs) {
    const int m = (int)(live.size() - i < (size_t)kMaxProbs ? live.size() - i : (size_t)kMaxProbs);
    s = launch_group(live.data() + i, m, ds, st);
    if (s != IMQ_OK) return s;
  }
  return IMQ_OK;
}

imq_status launch_gemm(const imq_plan_t* pl, const int8_t* Au, const int8_t* Bu, const float* dA, imq_gran gA,
                       const float* dB, imq_gran gB, void* C, imq_dtype ct, int64_t ldc, float* Cf,
                       int64_t ldcf, cudaStream_t st) {
  GemmSpec s{pl, Au, Bu, dA, gA, dB, gB, C, ct, ldc, Cf, ldcf};
  return launch_gemm_multi(&s, 1, st);
}

}  // namespace imq
