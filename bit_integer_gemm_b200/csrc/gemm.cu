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
//   warps 2-5   epilogue: tcgen05.ld of the accumulators, fold-back, shift, accumulation into C,
//               dequantisation.
// The inner dimension is a sequence of exponent groups whose products carry the weight R^e.  Each group
// of each tile is one accumulation job; jobs alternate between two 256-column TMEM slots, so the MMAs of
// job n+1 run while the epilogue drains job n (also across tiles).  The epilogue folds the OUTER lines
// of a job back with their level weights, shifts by e*(b-1) and adds the result into C (the first job of
// a tile writes, later ones read-modify-write the tile they own; the last also writes the fp32 copy).
// Every partial sum is a partial sum of the exact product, so it is bounded by the plan's bound: int32
// when that is below 2^31, int64 otherwise.  The plan splits a group along K when its raw s32
// accumulator could overflow.
// Every mbarrier wait is bounded (common.cuh): a stuck pipeline ends the kernel with IMQ_ERR_TIMEOUT.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;  // bytes
constexpr int B_STAGE = BN * BK;
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct GemmArgs {
  int32_t tiles_m, tiles_n;
  int32_t n_jobs;
  int32_t job_kb0[kMaxJobs];
  int32_t job_nkb[kMaxJobs];
  int8_t job_shift[kMaxJobs];
  int32_t bm1;
  int32_t a_outer, b_outer;
  const int32_t* srcA;
  const int32_t* grpA_L;
  const int32_t* grpA_n;
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
  static constexpr size_t kStage = kB + (size_t)STAGES * B_STAGE;  // int32 [128][32], XOR-swizzled
  static constexpr size_t kRsrc = kStage + (size_t)BM * 32 * 4;
  static constexpr size_t kCsrc = kRsrc + BM * 4;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr size_t kBars = kCsrc + 32 * 4;
  static constexpr size_t kMisc = kBars + (2 * STAGES + 5) * 8;  // tmem base, abort flag, epilogue flag
  static constexpr size_t kEnd = kMisc + 16;
  static constexpr size_t kBytes = kEnd + 1024;  // slack for 1024-byte alignment of the base
};

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > timeout_ns) return false;
  return true;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ GemmArgs g) {
  using L = Smem;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base + L::kA;
  uint8_t* sB = base + L::kB;
  int32_t* stg = reinterpret_cast<int32_t*>(base + L::kStage);
  int32_t* s_rsrc = reinterpret_cast<int32_t*>(base + L::kRsrc);
  int32_t* s_csrc = reinterpret_cast<int32_t*>(base + L::kCsrc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L::kMisc + 4);
  volatile int* epi_ok = reinterpret_cast<volatile int*>(base + L::kMisc + 8);

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
      mbar_init(acce0 + 8 * s, EPI_THREADS);
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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 2;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int mt = tile % g.tiles_m, nt = tile / g.tiles_m;
        for (int j = 0; j < g.n_jobs; ++j) {
          for (int kb = 0; kb < g.job_nkb[j]; ++kb) {
            if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, g.status, g.timeout_ns)) goto producer_done;
            const uint32_t fb = full0 + 8 * stage;
            mbar_arrive_expect_tx(fb, A_STAGE + B_STAGE);
            const int32_t x = (g.job_kb0[j] + kb) * BK;
            tma_load_2d(smem_addr(sA + (size_t)stage * A_STAGE), &tmA, x, mt * BM, fb);
            tma_load_2d(smem_addr(sB + (size_t)stage * B_STAGE), &tmB, x, nt * BN, fb);
            issued[stage] = phase;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
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
      uint32_t job_count = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        for (int j = 0; j < g.n_jobs; ++j, ++job_count) {
          const uint32_t slot = job_count & 1u;
          // the epilogue has drained the job this slot held before
          if (!mbar_wait(acce0 + 8 * slot, (empty_waits[slot] & 1u) ^ 1u, abort_flag, g.status, g.timeout_ns))
            goto mma_done;
          ++empty_waits[slot];
          tc_fence_after();
          const uint32_t d = tmem_base + slot * BN;
          for (int kb = 0; kb < g.job_nkb[j]; ++kb) {
            if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, g.status, g.timeout_ns)) goto mma_done;
            tc_fence_after();
            const uint64_t adesc = smem_desc_k_sw128(smem_addr(sA + (size_t)stage * A_STAGE));
            const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sB + (size_t)stage * B_STAGE));
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
              // 32 bytes further along K inside the 128-byte swizzled row: +2 in the address field
              mma_i8(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb == 0 && k == 0) ? 0u : 1u);
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
    mma_done:
      // every issued MMA must complete before TMEM is released
      mma_commit(drain_bar);
      drain_wait(drain_bar, 0, g.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;   // 0..127
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;     // accumulator row owned by this thread
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t full_waits[2] = {0, 0};
    uint32_t job_count = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mt = tile % g.tiles_m, nt = tile / g.tiles_m;
      // source rows of this tile
      int LA, nA;
      if (g.a_outer) {
        LA = g.grpA_L[mt];
        nA = g.grpA_n[mt];
        if (et < nA) s_rsrc[et] = g.srcA[(int64_t)mt * BM + (int64_t)et * LA];
      } else {
        LA = 1;
        const int64_t rem = g.M - (int64_t)mt * BM;
        nA = rem < BM ? (int)rem : BM;
        if (et < nA) s_rsrc[et] = mt * BM + et;
      }
      for (int j = 0; j < g.n_jobs; ++j, ++job_count) {
        const uint32_t slot = job_count & 1u;
        // one thread waits and all 128 take its answer, so every epilogue thread passes the same named
        // barriers even when a wait gives up
        if (et == 0)
          *epi_ok = mbar_wait(accf0 + 8 * slot, full_waits[slot] & 1u, abort_flag, g.status, g.timeout_ns) ? 1 : 0;
        named_bar_sync(1, EPI_THREADS);
        const bool ok = *epi_ok != 0;
        named_bar_sync(1, EPI_THREADS);
        ++full_waits[slot];
        if (!ok) goto epi_done;
        tc_fence_after();
        const bool first = j == 0, last = j == g.n_jobs - 1;
        const int64_t mul = (int64_t)1 << g.job_shift[j];
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_base + lane_off + slot * BN + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) stg[row * 32 + (jj ^ lane)] = (int32_t)v[jj];
          if (c == BN / 32 - 1) {
            // the slot is fully read: let the MMA warp start the job after next in it
            tc_fence_before();
            mbar_arrive(acce0 + 8 * slot);
          }
          // source columns of this 32-column chunk
          const int64_t gc = (int64_t)nt * (BN / 32) + c;
          int LB, nB;
          if (g.b_outer) {
            if (gc < g.n_grp_b) {
              LB = g.grpB_L[gc];
              nB = g.grpB_n[gc];
            } else {
              LB = 1;
              nB = 0;
            }
            if (et < nB) s_csrc[et] = g.srcB[gc * 32 + (int64_t)et * LB];
          } else {
            LB = 1;
            const int64_t rem = g.N - gc * 32;
            nB = rem <= 0 ? 0 : (rem < 32 ? (int)rem : 32);
            if (et < nB) s_csrc[et] = (int32_t)(gc * 32 + et);
          }
          named_bar_sync(1, EPI_THREADS);
          const int total = nA * nB;
          for (int o = et; o < total; o += EPI_THREADS) {
            const int r = o / nB, s = o - r * nB;
            int64_t acc = 0;
            for (int la = 0; la < LA; ++la) {
              const int rr = r * LA + la;
              for (int lb = 0; lb < LB; ++lb) {
                const int cc = s * LB + lb;
                acc += (int64_t)stg[rr * 32 + (cc ^ (rr & 31))] * ((int64_t)1 << ((la + lb) * g.bm1));
              }
            }
            acc *= mul;
            const int64_t i = s_rsrc[r], col = s_csrc[s];
            // the same thread owns output (i, col) in every job of this tile
            if (g.c64) {
              int64_t* cp = static_cast<int64_t*>(g.C) + i * g.ldc + col;
              if (!first) acc += *cp;
              *cp = acc;
            } else if (g.C) {
              int32_t* cp = static_cast<int32_t*>(g.C) + i * g.ldc + col;
              if (!first) acc += *cp;
              *cp = (int32_t)acc;
            }
            if (last && g.Cf) {
              const float sa = g.dA[g.dA_per_row ? i : 0], sb = g.dB[g.dB_per_col ? col : 0];
              g.Cf[i * g.ldcf + col] = __fmul_rn(__ll2float_rn(acc), __fmul_rn(sa, sb));
            }
          }
          named_bar_sync(1, EPI_THREADS);
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
  if (!C && pl->n_jobs > 1) return IMQ_ERR_ARG;  // the jobs of a tile accumulate in C
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
  g.n_jobs = pl->n_jobs;
  for (int j = 0; j < pl->n_jobs; ++j) {
    g.job_kb0[j] = (int32_t)(pl->job_k0[j] / BK);
    g.job_nkb[j] = (int32_t)(pl->job_klen[j] / BK);
    g.job_shift[j] = (int8_t)pl->job_shift[j];
  }
  g.bm1 = I.b - 1;
  g.a_outer = I.dir_a == IMQ_DIR_OUTER;
  g.b_outer = I.dir_b == IMQ_DIR_OUTER;
  g.srcA = pl->srcA;
  g.grpA_L = pl->grpA_L;
  g.grpA_n = pl->grpA_n;
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
  IMQ_CUDA_TRY(cudaFuncSetAttribute(k_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  k_gemm<<<grid, NUM_THREADS, smem, st>>>(tmA, tmB, g);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

static_assert(Smem::kBytes <= 232448, "shared memory budget");

}  // namespace imq
