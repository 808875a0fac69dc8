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

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;  // bytes
constexpr int B_STAGE = BN * BK;
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct GemmArgs {
  int32_t tiles_m, tiles_n;
  int32_t n_steps;
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

struct Smem {
  static constexpr size_t kA = 0;
  static constexpr size_t kB = kA + (size_t)STAGES * A_STAGE;
  // per epilogue warp: a 32 x 32 transpose buffer of up to 8-byte values, XOR-swizzled
  static constexpr size_t kScratch = kB + (size_t)STAGES * B_STAGE;
  static constexpr size_t kRows = kScratch + EPI_WARPS * 32 * 32 * 8;  // per epilogue warp: WarpRows
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr size_t kBars = kRows + EPI_WARPS * 256;
  static constexpr size_t kMisc = kBars + (2 * STAGES + 5) * 8;  // tmem base, abort flag
  static constexpr size_t kEnd = kMisc + 16;
  static constexpr size_t kBytes = kEnd + 1024;  // slack for 1024-byte alignment of the base
};

// x * 2^k in the two's-complement type T, through the unsigned type (the plan's bounds guarantee the
// exact result fits T).
template <typename T>
__device__ __forceinline__ T shl(T x, int k) {
  using U = typename std::make_unsigned<T>::type;
  return (T)((U)x << k);
}

// Column fold of one 32-column chunk holding 32/L columns of level L: w[s] = sum_l R^l v[s L + l].
template <int L, typename T>
__device__ __forceinline__ void fold_cols(const uint32_t (&v)[32], T (&w)[32], int bm1) {
#pragma unroll
  for (int s = 0; s < 32 / L; ++s) {
    T a = 0;
#pragma unroll
    for (int l = 0; l < L; ++l) a += shl<T>((T)(int32_t)v[s * L + l], l * bm1);
    w[s] = a;
  }
}

__device__ __forceinline__ int32_t shfl_t(int32_t x, int src) { return __shfl_sync(0xffffffffu, x, src); }
__device__ __forceinline__ int64_t shfl_t(int64_t x, int src) {
  const int lo = __shfl_sync(0xffffffffu, (int)(uint32_t)(uint64_t)x, src);
  const int hi = __shfl_sync(0xffffffffu, (int)(uint32_t)((uint64_t)x >> 32), src);
  return (int64_t)(((uint64_t)(uint32_t)hi << 32) | (uint32_t)lo);
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > timeout_ns) return false;
  return true;
}

// Per-warp drain metadata of one tile, fetched before the accumulator is ready: row offsets and row
// scales in shared memory, column indices and column scales in registers.  In the store phase of a
// chunk with nB output columns, lane t writes column s = t % nB of the rows r0 = t / nB, r0 + per, ...
// (per = 32 / nB rows at a time), so that all lanes store even when nB < 32.
struct DrainMeta {
  int LA, nA;
  int32_t pk[BN / 32];   // per chunk: nB | LB << 6 | s << 12 | r0 << 18 | per << 24 (r0 = 63: idle lane)
  int32_t col[BN / 32];  // the output column of this lane's s in each chunk
  float sb[BN / 32];     // its dequantisation scale
};

__device__ __forceinline__ int pk_nB(int32_t pk) { return pk & 63; }
__device__ __forceinline__ int pk_LB(int32_t pk) { return (pk >> 6) & 63; }
__device__ __forceinline__ int pk_s(int32_t pk) { return (pk >> 12) & 63; }
__device__ __forceinline__ int pk_r0(int32_t pk) { return (pk >> 18) & 63; }
__device__ __forceinline__ int pk_per(int32_t pk) { return (pk >> 24) & 63; }

struct WarpRows {       // shared memory, per epilogue warp
  int32_t row[32];      // the output row lane t holds after the row fold
  float sa[32];         // its dequantisation scale
};

// Transpose buffer index: row r, column c, XOR-swizzled so that both a row sweep and a column sweep of
// the warp hit 32 different banks.
__device__ __forceinline__ int sw(int r, int c) { return r * 32 + (c ^ r); }

__device__ __forceinline__ void drain_prepare(const GemmArgs& g, int mt, int nt, int q, int lane, bool last,
                                              DrainMeta& m, WarpRows* wr) {
  int64_t my_row;
  if (g.a_outer) {
    const int64_t grp = (int64_t)mt * (BM / 32) + q;
    m.LA = grp < g.n_grp_a ? g.grpA_L[grp] : 1;
    m.nA = grp < g.n_grp_a ? g.grpA_n[grp] : 0;
    my_row = lane < m.nA ? g.srcA[grp * 32 + (int64_t)lane * m.LA] : 0;
  } else {
    m.LA = 1;
    const int64_t r0 = (int64_t)mt * BM + q * 32;
    const int64_t rem = g.M - r0;
    m.nA = rem <= 0 ? 0 : (rem < 32 ? (int)rem : 32);
    my_row = lane < m.nA ? r0 + lane : 0;
  }
  wr->row[lane] = (int32_t)my_row;
  wr->sa[lane] = (last && g.Cf && lane < m.nA) ? g.dA[g.dA_per_row ? my_row : 0] : 0.0f;
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    const int64_t gc = (int64_t)nt * (BN / 32) + c;
    int LB = 1, nB = 0;
    if (g.b_outer) {
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
    m.pk[c] = nB | (LB << 6) | (s << 12) | (r0 << 18) | (per << 24);
    m.col[c] = 0;
    if (r0 != 63) m.col[c] = g.b_outer ? g.srcB[gc * 32 + (int64_t)s * LB] : (int32_t)(gc * 32 + s);
  }
#pragma unroll
  for (int c = 0; c < BN / 32; ++c)
    m.sb[c] = (last && g.Cf && pk_r0(m.pk[c]) != 63) ? g.dB[g.dB_per_col ? m.col[c] : 0] : 0.0f;
  __syncwarp();
}

// Drains one TMEM slot (this warp's 32 lanes) into C: fold, shift, write or add.
template <typename T>
__device__ __forceinline__ void drain_slot(const GemmArgs& g, uint32_t tbase, uint32_t acce_bar, int lane, bool first,
                                           bool last, int shift, T* scr, const DrainMeta& m, const WarpRows* wr) {
  uint32_t v[32];
  tmem_ld32(tbase, v);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    tmem_wait_ld();
    uint32_t cur[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) cur[k] = v[k];
    if (c + 1 < BN / 32) {
      tmem_ld32(tbase + (c + 1) * 32, v);  // the next chunk streams in while this one is folded
    } else {
      // the slot is fully read: the MMA warp may reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar);
    }
    // dynamic indexing of the unrolled metadata arrays is avoided by a uniform select
    int32_t pk = 0, mycol = 0;
    float sb = 0.0f;
#pragma unroll
    for (int k = 0; k < BN / 32; ++k)
      if (k == c) {
        pk = m.pk[k];
        mycol = m.col[k];
        sb = m.sb[k];
      }
    const int LB = pk_LB(pk), nB = pk_nB(pk);
    const int nA = m.nA, LA = m.LA;
    if (nB == 0 || nA == 0) continue;
    // 1. fold the column levels of B inside the registers (lane = unpacked row)
    T w[32];
    switch (LB) {
      case 1: fold_cols<1>(cur, w, g.bm1); break;
      case 2: fold_cols<2>(cur, w, g.bm1); break;
      case 3: fold_cols<3>(cur, w, g.bm1); break;
      case 4: fold_cols<4>(cur, w, g.bm1); break;
      case 5: fold_cols<5>(cur, w, g.bm1); break;
      case 6: fold_cols<6>(cur, w, g.bm1); break;
      case 7: fold_cols<7>(cur, w, g.bm1); break;
      case 8: fold_cols<8>(cur, w, g.bm1); break;
      default: {
        // levels 9..31 (three columns at most): fold through the transpose buffer
#pragma unroll
        for (int k = 0; k < 32; ++k) scr[sw(lane, k)] = (T)(int32_t)cur[k];
        __syncwarp();
#pragma unroll
        for (int s2 = 0; s2 < 3; ++s2) {
          T a = 0;
          if (s2 < nB)
            for (int l = 0; l < LB; ++l) a += shl<T>(scr[sw(lane, s2 * LB + l)], l * g.bm1);
          w[s2] = a;
        }
        __syncwarp();
      }
    }
    // 2. fold the row levels of A across the lanes: lane t gathers lanes t LA + l
    if (g.a_outer && LA > 1) {
#pragma unroll
      for (int s2 = 0; s2 < 32; ++s2) {
        if (s2 < nB) {
          T a = 0;
          for (int l = 0; l < LA; ++l) {
            const int src = lane * LA + l;
            a += shl<T>(shfl_t(w[s2], src < 32 ? src : 31), l * g.bm1);
          }
          w[s2] = a;
        }
      }
    }
    // 3. transpose through shared memory: scr[row][column]
#pragma unroll
    for (int s2 = 0; s2 < 32; ++s2)
      if (s2 < nB) scr[sw(lane, s2)] = shl<T>(w[s2], shift);
    __syncwarp();
    // 4. lane (r0, s) stores column s of rows r0, r0 + per, ...: each row of C takes nB neighbouring
    //    lanes, and all 32 / nB rows of a pass go out in one instruction
    {
      const int s = pk_s(pk), per = pk_per(pk);
#pragma unroll 4
      for (int r = pk_r0(pk); r < nA; r += per) {
        T val = scr[sw(r, s)];
        const int64_t row = wr->row[r];
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
                        __fmul_rn(wr->sa[r], sb));
      }
    }
    __syncwarp();
  }
}

template <bool kWide>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ GemmArgs g) {
  using L = Smem;
  using T = typename std::conditional<kWide, int64_t, int32_t>::type;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + L::kA;
  uint8_t* sB = base + L::kB;
  T* scratch = reinterpret_cast<T*>(base + L::kScratch);
  WarpRows* wrows = reinterpret_cast<WarpRows*>(base + L::kRows);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + STAGES);
  const uint32_t accf0 = smem_addr(bars + 2 * STAGES), acce0 = smem_addr(bars + 2 * STAGES + 2);
  const uint32_t drain_bar = smem_addr(bars + 2 * STAGES + 4);
  constexpr uint32_t kCols = 2 * BN;  // two accumulator slots

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(accf0 + 8 * s, 1);
      mbar_init(acce0 + 8 * s, EPI_WARPS);  // one arrival per epilogue warp
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
    tmem_alloc(smem_addr(tmem_holder), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = g.tiles_m * g.tiles_n;
  // this CTA's tiles blockIdx.x + i * gridDim.x, taken in pairs (one per TMEM slot)
  const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 2;
      for (int p = 0; p < my_tiles; p += 2) {
        const int npair = my_tiles - p < 2 ? my_tiles - p : 2;
        for (int k = 0; k < g.n_steps; ++k) {
          for (int x = 0; x < npair; ++x) {
            const int tile = blockIdx.x + (p + x) * gridDim.x;
            const int mt = tile % g.tiles_m, nt = tile / g.tiles_m;
            for (int kb = 0; kb < g.step_nkb[k]; ++kb) {
              if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, g.status, g.timeout_ns)) goto producer_done;
              const uint32_t fb = full0 + 8 * stage;
              mbar_arrive_expect_tx(fb, A_STAGE + B_STAGE);
              const int32_t kx = (g.step_kb0[k] + kb) * BK;
              tma_load_2d(smem_addr(sA + (size_t)stage * A_STAGE), &tmA, kx, mt * BM, fb);
              tma_load_2d(smem_addr(sB + (size_t)stage * B_STAGE), &tmB, kx, nt * BN, fb);
              issued[stage] = phase;
              if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
        }
      }
    producer_done:
      // every issued copy must land before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] != 2) drain_wait(full0 + 8 * s, issued[s], g.timeout_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t empty_waits[2] = {0, 0};
      for (int p = 0; p < my_tiles; p += 2) {
        const int npair = my_tiles - p < 2 ? my_tiles - p : 2;
        for (int k = 0; k < g.n_steps; ++k) {
          for (int slot = 0; slot < npair; ++slot) {
            // the epilogue has finished the previous event of this slot (a rescale or a drain)
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
                mma_i8(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (first && kb == 0 && kk == 0) ? 0u : 1u);
              }
              mma_commit(empty0 + 8 * stage);
              if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
              }
            }
            mma_commit(accf0 + 8 * slot);
          }
        }
      }
    mma_done:
      // every issued MMA must complete before TMEM is released
      mma_commit(drain_bar);
      drain_wait(drain_bar, 0, g.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access = row group of the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    T* scr = scratch + q * 32 * 32;  // this warp's transpose buffer (XOR-swizzled rows of 32)
    uint32_t full_waits[2] = {0, 0};
    for (int p = 0; p < my_tiles; p += 2) {
      const int npair = my_tiles - p < 2 ? my_tiles - p : 2;
      for (int k = 0; k < g.n_steps; ++k) {
        for (int slot = 0; slot < npair; ++slot) {
          DrainMeta meta;
          const bool drain = g.step_after[k] < 0;
          if (drain) {
            // metadata of the tile first: its loads overlap the wait for the accumulator
            const int tile = blockIdx.x + (p + slot) * gridDim.x;
            drain_prepare(g, tile % g.tiles_m, tile / g.tiles_m, q, lane, g.step_dlast[k] != 0, meta, wrows + q);
          }
          int ok = 1;
          if (lane == 0) ok = mbar_wait(accf0 + 8 * slot, full_waits[slot] & 1u, abort_flag, g.status, g.timeout_ns) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++full_waits[slot];
          if (!ok) goto epi_done;
          tc_fence_after();
          const uint32_t tbase = tmem_base + lane_off + (uint32_t)slot * BN;
          if (g.step_after[k] >= 0) {
            // Horner step: slot *= R^(e_prev - e), in place.  The plan bounds the result by 2^31, so
            // a shift of 31 or more only meets zeros.
            const int sh = g.step_after[k];
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
              uint32_t v[32];
              tmem_ld32(tbase + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int jj = 0; jj < 32; ++jj) v[jj] = sh < 31 ? (v[jj] << sh) : 0u;
              tmem_st32(tbase + c * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce0 + 8 * slot);
          } else {
            drain_slot<T>(g, tbase, acce0 + 8 * slot, lane, g.step_dfirst[k] != 0, g.step_dlast[k] != 0,
                          g.step_dshift[k], scr, meta, wrows + q);
          }
        }
      }
    }
  epi_done:;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kCols);
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

  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, Au, I.K_unp, I.M_unp, BM) || !make_map(&tmB, Bu, I.K_unp, I.N_unp, BN)) return IMQ_ERR_CUDA;

  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.tiles_m = (int32_t)((I.M_unp + BM - 1) / BM);
  g.tiles_n = (int32_t)((I.N_unp + BN - 1) / BN);
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
  g.a_outer = I.dir_a == IMQ_DIR_OUTER;
  g.b_outer = I.dir_b == IMQ_DIR_OUTER;
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
  const int grid = num_tiles < ds->num_sms ? num_tiles : ds->num_sms;
  const size_t smem = Smem::kBytes;
  // int64 accumulation in the epilogue whenever the output is int64 or the bound exceeds int32
  if (g.c64 || I.acc_bits > 32) {
    IMQ_CUDA_TRY(cudaFuncSetAttribute(k_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    k_gemm<true><<<grid, NUM_THREADS, smem, st>>>(tmA, tmB, g);
  } else {
    IMQ_CUDA_TRY(cudaFuncSetAttribute(k_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    k_gemm<false><<<grid, NUM_THREADS, smem, st>>>(tmA, tmB, g);
  }
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

static_assert(Smem::kBytes <= 232448, "shared memory budget");

}  // namespace imq
