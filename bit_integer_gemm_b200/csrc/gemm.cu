// gemm.cu -- the low-bit integer GEMM on the unpacked operands with the fold-back epilogue (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Approach": the original integer GEMM is reproduced exactly by low bit-width integer GEMMs
// followed by bit-shift scaling and accumulation.
//
// Design (B200, one CTA per SM, persistent over 128 x 256 output tiles of the unpacked problem):
//   warp 0      TMA producer: 128 x 128-byte tiles of A' and 256 x 128-byte tiles of B'^T, 128-byte
//               swizzle, into a 4-stage shared-memory ring (mbarrier complete_tx).
//   warp 1      MMA issuer (one thread): tcgen05.mma.cta_group::1.kind::i8, M=128 N=256 K=32,
//               s8 x s8 -> s32 accumulators in tensor memory (TMEM).
//   warps 2-5   epilogue: Horner rescales in TMEM, fold-back, dequantisation, stores.
// The inner dimension is a sequence of exponent groups whose products carry the weight R^e.  A tile runs
// them in descending e as steps into one 256-column TMEM slot; between two steps of a chunk the
// epilogue multiplies the slot by R^(e_prev - e) in place (Horner's rule), at the end of a chunk it
// drains the slot into C.  The plan proves every slot value stays below 2^31 (one chunk whenever the
// product fits int32; chunks end only where the bound forces it, and their drains accumulate in C).
// Two tiles run interleaved, step by step, one per TMEM slot: while the epilogue rescales or drains one
// tile's slot, the tensor cores work on the other tile.
// Drain: each epilogue warp owns one TMEM lane quarter = one group of 32 unpacked rows of A; a 32-column
// chunk is one group of 32 unpacked columns of B.  Column levels of B are folded inside each thread's
// registers, row levels of A across the lanes with shuffles, and the folded values are transposed
// through shared memory so that every global access is coalesced along a row of C.
// Every mbarrier wait is bounded (common.cuh): a stuck pipeline ends the kernel with IMQ_ERR_TIMEOUT.
#include <string.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

// Per CTA: 128 accumulator rows x up to BN columns.  The tile width bn (a multiple of 32, at most BN)
// is chosen per launch so that the tiles spread evenly over the SMs; each TMEM slot spans BN columns.
constexpr int BM = 128, BN = 256, BK = 128;
constexpr int NCHUNK = BN / 32;  // 32-column chunks of a full-width slot
constexpr uint64_t kTimeoutNs = 4000000000ull;

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

struct GemmArgs {
  int32_t tiles_m, tiles_n;
  int32_t bn;      // tile width (columns of C' per tile), a multiple of 32 in [32, BN]
  int32_t nchunk;  // bn / 32
  int32_t n_steps;
  int32_t sched_off;  // slot 1 trails slot 0 by this many steps (see the order below)
  int32_t step_kb0[kMaxJobs];
  int32_t step_nkb[kMaxJobs];
  int8_t step_first[kMaxJobs];   // the step opens a chunk: its first MMA overwrites the slot
  int8_t step_after[kMaxJobs];   // >= 0: Horner shift of the slot after the step; -1: drain
  int8_t step_dshift[kMaxJobs];  // shift of the drained value (e of the chunk's last group times b-1)
  int8_t step_dfirst[kMaxJobs];  // the drain is the tile's first: it writes C without reading it
  int8_t step_dlast[kMaxJobs];   // the drain is the tile's last: it also writes Cf
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
  int32_t* status;
  uint64_t timeout_ns;
};

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
  static constexpr size_t kEnd = kMisc + 16;
  static constexpr size_t kBytes = kEnd + 1024;  // slack for 1024-byte alignment of the base
  static_assert(kBytes <= 232448, "shared memory budget");
};

// The order in which a CTA runs the steps of its tiles.  Its tiles p = 0, 1, 2, ... alternate between
// the two TMEM slots (slot p % 2); each slot runs its tiles' steps in sequence, and between two steps of
// a slot the epilogue works on it (a Horner rescale or a drain) while the tensor cores run the other
// slot's step.  Slot 1 trails slot 0 by `off` steps, so that a drain (the long epilogue event) overlaps
// a long step of the other slot instead of a short one: slot 0's step j0 runs before slot 1's step j1
// while j0 <= j1 + off.  Producer, MMA issuer and epilogue walk the same order.
struct Order {
  int len0, len1, off, n_steps;
  int j0, j1;
  __device__ Order(int my_tiles, int n_steps_, int off_)
      : len0(((my_tiles + 1) / 2) * n_steps_), len1((my_tiles / 2) * n_steps_), off(off_), n_steps(n_steps_),
        j0(0), j1(0) {}
  __device__ int total() const { return len0 + len1; }
  // next (slot, local tile p, step k)
  __device__ void next(int& slot, int& p, int& k) {
    int j;
    if (j1 >= len1 || (j0 < len0 && j0 <= j1 + off)) {
      slot = 0;
      j = j0++;
    } else {
      slot = 1;
      j = j1++;
    }
    p = 2 * (j / n_steps) + slot;
    k = j % n_steps;
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
// in this CTA's accumulator.
template <int NC, int PQ>
__device__ __forceinline__ void drain_prepare(const GemmArgs& g, int64_t row0, int nt, int q, int h, int lane,
                                              bool last, DrainMeta<NC>& m) {
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
  m.my_sa = (last && g.Cf && lane < m.nA) ? g.dA[g.dA_per_row ? my_row : 0] : 0.0f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = h + PQ * i;
    const int64_t gc = (int64_t)nt * g.nchunk + c;
    int LB = 1, nB = 0;
    if (c >= g.nchunk) {
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
    m.sb[i] = (last && g.Cf && pk_r0(m.pk[i]) != 63) ? g.dB[g.dB_per_col ? m.col[i] : 0] : 0.0f;
}

// Drains this warp's chunks of one TMEM slot (its 32 lanes) into C: fold, shift, write or add.
// Releases a slot to the MMA issuer: a local arrive, or for a CTA pair an arrive on the leading CTA's
// barrier (acce_bar is then its shared::cluster address).
template <bool kPair>
__device__ __forceinline__ void release_slot(uint32_t acce_bar) {
  if constexpr (kPair)
    mbar_arrive_cluster(acce_bar);
  else
    mbar_arrive(acce_bar);
}

template <typename T, int NC, int PQ, bool kPair>
__device__ __forceinline__ void drain_slot(const GemmArgs& g, uint32_t tbase, uint32_t acce_bar, int lane, int h,
                                           bool first, bool last, int shift, T* scr, const DrainMeta<NC>& m) {
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
              if (!first) val += (T)*cp;
              *cp = (int64_t)val;
            } else {
              int32_t* cp = static_cast<int32_t*>(g.C) + row * g.ldc + mycol;
              if (!first) val += (T)*cp;
              *cp = (int32_t)val;
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

template <bool kWide, bool kPair>
__global__ void __launch_bounds__(Epi<kWide>::kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ GemmArgs g) {
  using L = Geo<kPair>;
  using E = Epi<kWide>;
  using T = typename E::T;
  constexpr int STAGES = L::kStages;
  constexpr int A_STAGE = L::kAStage, B_STAGE = L::kBStage;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + L::kA;
  uint8_t* sB = base + L::kB;
  T* scratch = reinterpret_cast<T*>(base + L::kScratch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);

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
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
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
  const int num_tiles = g.tiles_m * g.tiles_n;
  // the tiles of this CTA (or pair): unit + p * units, p = 0 .. my_tiles - 1
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int my_tiles = (num_tiles - unit + units - 1) / units;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // rows of B'^T this CTA loads per k-block (half the tile width for a pair) and their bytes
      const int32_t b_rows = kPair ? g.bn / 2 : g.bn;
      const uint32_t b_bytes = (uint32_t)b_rows * BK;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 2;
      Order ord(my_tiles, g.n_steps, g.sched_off);
      for (int e = 0; e < ord.total(); ++e) {
        int slot, p, k;
        ord.next(slot, p, k);
        const int tile = unit + p * units;
        const int mt = tile % g.tiles_m, nt = tile / g.tiles_m;
        const int32_t ya = mt * L::kTM + (int32_t)rank * BM, yb = nt * g.bn + (int32_t)rank * b_rows;
        for (int kb = 0; kb < g.step_nkb[k]; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, g.status, g.timeout_ns)) goto producer_done;
          const uint32_t fb = full0 + 8 * stage;
          const int32_t kx = (g.step_kb0[k] + kb) * BK;
          if constexpr (kPair) {
            // both CTAs' bytes complete the leader's barrier, which expects them all
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * (A_STAGE + b_bytes));
            const uint32_t lfb = mapa_shared(fb, 0);
            tma_load_2d_pair(smem_addr(sA + (size_t)stage * A_STAGE), &tmA, kx, ya, lfb);
            tma_load_2d_pair(smem_addr(sB + (size_t)stage * B_STAGE), &tmB, kx, yb, lfb);
          } else {
            mbar_arrive_expect_tx(fb, A_STAGE + b_bytes);
            tma_load_2d(smem_addr(sA + (size_t)stage * A_STAGE), &tmA, kx, ya, fb);
            tma_load_2d(smem_addr(sB + (size_t)stage * B_STAGE), &tmB, kx, yb, fb);
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
          if (issued[s] != 2) drain_wait(full0 + 8 * s, issued[s], g.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_i8(L::kTM, (uint32_t)g.bn);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t empty_waits[2] = {0, 0};
      Order ord(my_tiles, g.n_steps, g.sched_off);
      for (int e = 0; e < ord.total(); ++e) {
        int slot, p, k;
        ord.next(slot, p, k);
        (void)p;
        // the epilogue (of both CTAs) has finished the previous event of this slot
        if (!mbar_wait(acce0 + 8 * slot, (empty_waits[slot] & 1u) ^ 1u, abort_flag, g.status, g.timeout_ns))
          goto mma_done;
        ++empty_waits[slot];
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)slot * BN;
        const bool first = g.step_first[k] != 0;
        for (int kb = 0; kb < g.step_nkb[k]; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, g.status, g.timeout_ns)) goto mma_done;
          tc_fence_after();
          const uint64_t adesc = smem_desc_k_sw128(smem_addr(sA + (size_t)stage * A_STAGE));
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sB + (size_t)stage * B_STAGE));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // 32 bytes further along K inside the 128-byte swizzled row: +2 in the address field
            const uint32_t acc = (first && kb == 0 && kk == 0) ? 0u : 1u;
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
      drain_wait(drain_bar, 0, g.timeout_ns);
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
    // where a released slot is signalled: this CTA's barrier, or the leader's for a pair
    const uint32_t rel0 = kPair ? mapa_shared(acce0, 0) : acce0;
    const uint32_t rel1 = kPair ? mapa_shared(acce0 + 8, 0) : acce0 + 8;
    uint32_t full_waits[2] = {0, 0};
    Order ord(my_tiles, g.n_steps, g.sched_off);
    for (int e = 0; e < ord.total(); ++e) {
      int slot, p, k;
      ord.next(slot, p, k);
      DrainMeta<NC> meta;
      const bool drain = g.step_after[k] < 0;
      if (drain) {
        // metadata of the tile first: its loads overlap the wait for the accumulator
        const int tile = unit + p * units;
        const int64_t row0 = (int64_t)(tile % g.tiles_m) * L::kTM + (int64_t)rank * BM;
        drain_prepare<NC, PQ>(g, row0, tile / g.tiles_m, q, h, lane, g.step_dlast[k] != 0, meta);
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(accf0 + 8 * slot, full_waits[slot] & 1u, abort_flag, g.status, g.timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++full_waits[slot];
      if (!ok) goto epi_done;
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_off + (uint32_t)slot * BN;
      const uint32_t rel = slot ? rel1 : rel0;
      if (!drain) {
        // Horner step: slot *= R^(e_prev - e), in place.  The plan bounds the result by 2^31, so
        // a shift of 31 or more only meets zeros.
        const int sh = g.step_after[k];
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
        drain_slot<T, NC, PQ, kPair>(g, tbase, rel, lane, h, g.step_dfirst[k] != 0, g.step_dlast[k] != 0,
                                     g.step_dshift[k], scr, meta);
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

// Makespan, in SM cycles, of the step order of a CTA with `tiles` tiles when slot 1 trails by `off` steps:
// a step occupies the tensor cores for 2 bn cycles per 128-deep k-block (M=128, N=256, K=32 in 128
// cycles per SM), and the epilogue event after it (done in step order) takes `rescale` or `drain` cycles.  A
// slot's next step waits for the slot's previous event.  Used only to pick `off`.
double simulate_order(const GemmArgs& g, int tiles, int off, double rescale, double drain) {
  const int n = g.n_steps;
  const int len0 = ((tiles + 1) / 2) * n, len1 = (tiles / 2) * n;
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
    const int k = j % n;
    const double start = mma_free > slot_ready[slot] ? mma_free : slot_ready[slot];
    const double end = start + 2.0 * g.bn * g.step_nkb[k];
    mma_free = end;
    const double ev_start = epi_free > end ? epi_free : end;
    epi_free = ev_start + (g.step_after[k] >= 0 ? rescale : drain);
    slot_ready[slot] = epi_free;
  }
  return mma_free > epi_free ? mma_free : epi_free;
}

template <bool kWide, bool kPair>
imq_status launch_k_gemm(int grid, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                         cudaStream_t st) {
  auto kern = k_gemm<kWide, kPair>;
  const size_t smem = Geo<kPair>::kBytes;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
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
  IMQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, tmA, tmB, g));
  return IMQ_OK;
}

}  // namespace

imq_status launch_gemm(const imq_plan_t* pl, const int8_t* Au, const int8_t* Bu, const float* dA, imq_gran gA,
                       const float* dB, imq_gran gB, void* C, imq_dtype ct, int64_t ldc, float* Cf,
                       int64_t ldcf, cudaStream_t st) {
  const imq_plan_info& I = pl->info;
  if (!C && !Cf) return IMQ_ERR_ARG;
  if (C && ct != IMQ_I32 && ct != IMQ_I64) return IMQ_ERR_ARG;
  if (C && ldc < I.N) return IMQ_ERR_ARG;
  if (Cf && (ldcf < I.N || !dA || !dB)) return IMQ_ERR_ARG;
  if (Cf && gA != IMQ_PER_TENSOR && gA != IMQ_PER_ROW) return IMQ_ERR_ARG;
  if (Cf && gB != IMQ_PER_TENSOR && gB != IMQ_PER_COL) return IMQ_ERR_ARG;
  if (C && ct == IMQ_I32 && I.acc_bits > 32) return IMQ_ERR_RANGE;
  if (!C && pl->n_chunks > 1) return IMQ_ERR_ARG;  // several chunks of a tile accumulate in C
  if (I.M == 0 || I.N == 0) return IMQ_OK;
  const size_t esz = ct == IMQ_I64 ? 8 : 4;
  if (I.K_unp == 0) {
    if (C) IMQ_CUDA_TRY(cudaMemset2DAsync(C, (size_t)ldc * esz, 0, (size_t)I.N * esz, (size_t)I.M, st));
    if (Cf) IMQ_CUDA_TRY(cudaMemset2DAsync(Cf, (size_t)ldcf * 4, 0, (size_t)I.N * 4, (size_t)I.M, st));
    return IMQ_OK;
  }
  if (!Au || !Bu) return IMQ_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(Au) & 15) || (reinterpret_cast<uintptr_t>(Bu) & 15)) return IMQ_ERR_ARG;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;

  // a CTA pair per 256 x 256 tile whenever A' has more than one 128-row block
  const bool pair = I.M_unp > BM && ds->num_sms >= 2;
  const int tm = pair ? Geo<true>::kTM : Geo<false>::kTM;
  CUtensorMap tmA, tmB;
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.tiles_m = (int32_t)((I.M_unp + tm - 1) / tm);
  // tile width: the fewest columns per SM over the busiest unit, ceil(tiles / units) * bn (a tile's
  // tensor-core time is proportional to bn), plus a per-tile cost worth 96 columns (operand re-reads,
  // the epilogue's fixed work, the pipeline's start and end) so that narrower tiles are taken only
  // where they add parallelism (fewer tiles than units) or save a whole wave
  {
    const int max_units = pair ? ds->num_sms / 2 : ds->num_sms;
    double best = 0.0;
    for (int bn = BN; bn >= 128; bn -= 32) {
      const int64_t tn = (I.N_unp + bn - 1) / bn;
      const int64_t tiles = tn * g.tiles_m;
      const int64_t units = tiles < max_units ? tiles : max_units;
      const int64_t waves = (tiles + units - 1) / units;
      const double cost = (double)waves * (bn + 96);
      if (bn == BN || cost < best) {
        best = cost;
        g.bn = bn;
      }
    }
  }
  g.nchunk = g.bn / 32;
  g.tiles_n = (int32_t)((I.N_unp + g.bn - 1) / g.bn);
  if (!make_map(&tmA, Au, I.K_unp, I.M_unp, BM) ||
      !make_map(&tmB, Bu, I.K_unp, I.N_unp, (uint32_t)(pair ? g.bn / 2 : g.bn)))
    return IMQ_ERR_CUDA;
  g.n_steps = pl->n_steps;
  int first_drain = -1, last_drain = -1;
  for (int k = 0; k < pl->n_steps; ++k) {
    g.step_kb0[k] = (int32_t)(pl->step_k0[k] / BK);
    g.step_nkb[k] = (int32_t)(pl->step_klen[k] / BK);
    g.step_first[k] = (int8_t)pl->step_first[k];
    g.step_after[k] = (int8_t)pl->step_after[k];
    g.step_dshift[k] = (int8_t)pl->step_drain_shift[k];
    if (pl->step_after[k] < 0) {
      if (first_drain < 0) first_drain = k;
      last_drain = k;
    }
  }
  if (first_drain >= 0) g.step_dfirst[first_drain] = 1;
  if (last_drain >= 0) g.step_dlast[last_drain] = 1;
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
  g.dA = dA;
  g.dB = dB;
  g.dA_per_row = gA == IMQ_PER_ROW;
  g.dB_per_col = gB == IMQ_PER_COL;
  g.C = C;
  g.c64 = C != nullptr && ct == IMQ_I64;
  g.ldc = ldc;
  g.Cf = Cf;
  g.ldcf = ldcf;
  g.status = ds->status;
  g.timeout_ns = kTimeoutNs;

  const int num_tiles = g.tiles_m * g.tiles_n;
  // one CTA per SM (a pair per two SMs), never more CTAs (pairs) than tiles
  const int max_units = pair ? ds->num_sms / 2 : ds->num_sms;
  const int units = num_tiles < max_units ? num_tiles : max_units;
  const int grid = pair ? 2 * units : units;
  // int64 accumulation in the epilogue whenever the output is int64 or the bound exceeds int32
  const bool wide = g.c64 || I.acc_bits > 32;
  // the trailing offset of slot 1 with the shortest modelled makespan for the busiest CTA; the event
  // costs are rough per-tile figures of the epilogue (a rescale is one TMEM read and write of the slot,
  // a drain also folds and stores it, half as fast with int64 values and half the warps)
  {
    const int tiles = (num_tiles + units - 1) / units;
    const double rescale = wide ? 3000.0 : 1500.0, drain = wide ? 28000.0 : 14000.0;
    double best = simulate_order(g, tiles, 0, rescale, drain);
    g.sched_off = 0;
    for (int off = 1; off < g.n_steps && off <= 16; ++off) {
      const double t = simulate_order(g, tiles, off, rescale, drain);
      if (t < best) {
        best = t;
        g.sched_off = off;
      }
    }
  }
  if (wide) return pair ? launch_k_gemm<true, true>(grid, tmA, tmB, g, st) : launch_k_gemm<true, false>(grid, tmA, tmB, g, st);
  return pair ? launch_k_gemm<false, true>(grid, tmA, tmB, g, st) : launch_k_gemm<false, false>(grid, tmA, tmB, g, st);
}

}  // namespace imq
