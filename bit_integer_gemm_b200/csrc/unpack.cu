// unpack.cu -- digit split of the quantised operands into b-bit int8 operands (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Approach": out-of-bound integers become several in-bound b-bit integers by row or column
// unpacking.  Entry p of unpacked line u is digit (line level + inner level of p) of the source entry
// (source line of u, inner index tK[p]); the layout is the one documented in include/imq.h.
//
// Both unpacked operands are K-major (the inner index contiguous) because that is what the tcgen05
// GEMM reads through TMA.  Two kernels cover the two storage orders of a source matrix:
//   k_unpack_rows  the source line is a stored row (A, or B given as B^T): one CTA stages the line in
//                  shared memory and streams out all its unpacked lines with 16-byte stores.
//   k_unpack_cols  the source line is a stored column (B, or A given as A^T): a CTA transposes a
//                  128 (inner) x 32 (lines) tile through shared memory, reading 64-byte row segments
//                  and writing 128-byte segments of unpacked lines.
// HBM traffic: each source entry is read once (the gathered rows are L2-resident), each unpacked byte
// is written once.
#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

// Row gather: a CTA stages a batch of NL source lines in shared memory, then for each 4-byte piece of
// the inner dimension reads the index maps once and writes the digits of every line of the batch (and
// every level of an OUTER line).  Lines too long to stage are gathered from global memory (L2).
template <typename T, bool kStaged>
__global__ void __launch_bounds__(256) k_unpack_rows(const T* __restrict__ X, int64_t nlines, int64_t K,
                                                     int64_t ld, int NL, int outer, const int8_t* __restrict__ lvl,
                                                     const int32_t* __restrict__ pos,
                                                     const int32_t* __restrict__ tK,
                                                     const int8_t* __restrict__ lk, int64_t K_unp,
                                                     int bm1, int8_t* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char dsm[];
  T* lines = reinterpret_cast<T*>(dsm);  // [NL][K]
  __shared__ int s_L[8];
  __shared__ int64_t s_base[8];
  const int tid = threadIdx.x;
  for (int64_t i0 = (int64_t)blockIdx.x * NL; i0 < nlines; i0 += (int64_t)gridDim.x * NL) {
    const int nb = nlines - i0 < NL ? (int)(nlines - i0) : NL;
    if (tid < nb) {
      s_L[tid] = outer ? (int)lvl[i0 + tid] : 1;
      s_base[tid] = outer ? (int64_t)pos[i0 + tid] : i0 + tid;
    }
    if (kStaged) {
      for (int b = 0; b < nb; ++b)
        for (int64_t t = tid; t < K; t += 256) lines[b * K + t] = X[(i0 + b) * ld + t];
    }
    __syncthreads();
    // lane = 4 consecutive inner positions, a warp = 128: index maps read once per batch, 128-byte
    // coalesced stores, shared-memory gathers at most 2-way bank conflicted
    const int lane = tid & 31, warp = tid >> 5;
    for (int64_t p = (int64_t)warp * 128 + lane * 4; p < K_unp; p += 8 * 128) {
      const int4 t4 = *reinterpret_cast<const int4*>(tK + p);
      const uint32_t l4 = *reinterpret_cast<const uint32_t*>(lk + p);
      const int32_t tt[4] = {t4.x, t4.y, t4.z, t4.w};
      int ll[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) ll[r] = (int)(int8_t)(l4 >> (8 * r));
      for (int b = 0; b < nb; ++b) {
        int32_t v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int32_t t = tt[r] >= 0 ? tt[r] : 0;
          v[r] = tt[r] < 0 ? 0 : (kStaged ? (int32_t)lines[b * K + t] : (int32_t)X[(i0 + b) * ld + t]);
        }
        const int L = s_L[b];
        for (int l = 0; l < L; ++l) {
          uint32_t packed = 0;
#pragma unroll
          for (int r = 0; r < 4; ++r)
            packed |= ((uint32_t)(uint8_t)(int8_t)digit_of(v[r], l + ll[r], bm1)) << (8 * r);
          *reinterpret_cast<uint32_t*>(out + (s_base[b] + l) * K_unp + p) = packed;
        }
      }
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_unpack_cols(const T* __restrict__ X, int64_t nlines, int64_t ld,
                                                     int outer, const int8_t* __restrict__ lvl,
                                                     const int32_t* __restrict__ pos,
                                                     const int32_t* __restrict__ tK,
                                                     const int8_t* __restrict__ lk, int64_t K_unp,
                                                     int bm1, int8_t* __restrict__ out) {
  __shared__ int32_t S[32][129];  // [line][inner]
  __shared__ int32_t s_t[128];
  __shared__ int32_t s_l[128];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t j0 = (int64_t)blockIdx.x * 32;
  const int64_t p0 = (int64_t)blockIdx.y * 128;
  if (tid < 128) {
    s_t[tid] = tK[p0 + tid];
    s_l[tid] = lk[p0 + tid];
  }
  __syncthreads();
  const int64_t j = j0 + lane;
#pragma unroll 4
  for (int r = 0; r < 16; ++r) {
    const int pp = warp * 16 + r;
    const int32_t t = s_t[pp];
    S[lane][pp] = (t >= 0 && j < nlines) ? (int32_t)X[(int64_t)t * ld + j] : 0;
  }
  __syncthreads();
  for (int jj = warp; jj < 32; jj += 8) {
    const int64_t jg = j0 + jj;
    if (jg >= nlines) break;
    const int L = outer ? (int)lvl[jg] : 1;
    const int64_t base = outer ? (int64_t)pos[jg] : jg;
    for (int l = 0; l < L; ++l) {
      uint32_t packed = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int pp = lane * 4 + r;
        const int32_t d = s_t[pp] >= 0 ? digit_of(S[jj][pp], l + s_l[pp], bm1) : 0;
        packed |= ((uint32_t)(uint8_t)(int8_t)d) << (8 * r);
      }
      *reinterpret_cast<uint32_t*>(out + (base + l) * K_unp + p0 + lane * 4) = packed;
    }
  }
}

// Zeroes the unused lines of every OUTER group (lines n*L .. G-1 of group g).
__global__ void k_zero_unused(const int32_t* __restrict__ grpL, const int32_t* __restrict__ grpN,
                              int64_t ngrp, int G, int64_t K_unp, int8_t* __restrict__ out) {
  for (int64_t g = blockIdx.x; g < ngrp; g += gridDim.x) {
    const int64_t first = g * G + (int64_t)grpN[g] * grpL[g];
    const int64_t last = (g + 1) * G;
    const int64_t n16 = (last - first) * K_unp / 16;
    int4* o = reinterpret_cast<int4*>(out + first * K_unp);
    for (int64_t k = threadIdx.x; k < n16; k += blockDim.x) o[k] = make_int4(0, 0, 0, 0);
  }
}

template <typename T>
imq_status unpack_one(const T* X, int64_t nlines, int64_t K, int64_t ld, bool line_is_row, int outer,
                      const int8_t* lvl, const int32_t* pos, const int32_t* tK, const int8_t* lk,
                      int64_t K_unp, int bm1, int8_t* out, int num_sms, cudaStream_t st) {
  if (nlines == 0 || K_unp == 0) return IMQ_OK;
  if (line_is_row) {
    // batches of up to 8 lines (64 KB of shared memory per CTA at most); lines longer than that are
    // gathered from global memory
    const size_t line_bytes = (size_t)(K > 0 ? K : 1) * sizeof(T);
    int NL = (int)((64 * 1024) / line_bytes);
    if (NL > 8) NL = 8;
    const bool staged = NL >= 1;
    if (!staged) NL = 8;
    const size_t smem = staged ? (size_t)NL * line_bytes : 0;
    const int per_sm = staged ? (int)((200 * 1024) / (smem + 2048)) : 8;
    const int64_t batches = (nlines + NL - 1) / NL;
    int64_t grid = (int64_t)num_sms * (per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm));
    if (grid > batches) grid = batches;
    if (staged) {
      IMQ_CUDA_TRY(cudaFuncSetAttribute(k_unpack_rows<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      k_unpack_rows<T, true><<<(unsigned)grid, 256, smem, st>>>(X, nlines, K, ld, NL, outer, lvl, pos, tK, lk, K_unp,
                                                                bm1, out);
    } else {
      k_unpack_rows<T, false><<<(unsigned)grid, 256, 0, st>>>(X, nlines, K, ld, NL, outer, lvl, pos, tK, lk, K_unp,
                                                              bm1, out);
    }
  } else {
    const dim3 grid((unsigned)((nlines + 31) / 32), (unsigned)(K_unp / 128));
    if (K_unp / 128 > 65535) return IMQ_ERR_UNSUPPORTED;
    k_unpack_cols<T><<<grid, 256, 0, st>>>(X, nlines, ld, outer, lvl, pos, tK, lk, K_unp, bm1, out);
  }
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

template <typename T>
imq_status unpack_typed(const imq_plan_t* pl, const T* A, const T* B, int8_t* Au, int8_t* Bu, int num_sms,
                        cudaStream_t st) {
  const imq_plan_info& I = pl->info;
  const int bm1 = I.b - 1;
  const int a_outer = I.dir_a == IMQ_DIR_OUTER, b_outer = I.dir_b == IMQ_DIR_OUTER;
  // A' lines are the logical rows of A: stored rows unless A is given transposed
  imq_status s = unpack_one<T>(A, I.M, I.K, pl->lda, !pl->transA, a_outer, pl->lv_a_row, pl->posA, pl->tK,
                               pl->lAk, I.K_unp, bm1, Au, num_sms, st);
  if (s != IMQ_OK) return s;
  // B'^T lines are the logical columns of B: stored rows only when B is given transposed
  s = unpack_one<T>(B, I.N, I.K, pl->ldb, pl->transB != 0, b_outer, pl->lv_b_col, pl->posB, pl->tK, pl->lBk,
                    I.K_unp, bm1, Bu, num_sms, st);
  if (s != IMQ_OK) return s;
  if (I.K_unp > 0) {
    if (a_outer && pl->n_grp_a > 0)
      k_zero_unused<<<(unsigned)(pl->n_grp_a < 4096 ? pl->n_grp_a : 4096), 256, 0, st>>>(
          pl->grpA_L, pl->grpA_n, pl->n_grp_a, IMQ_A_GROUP, I.K_unp, Au);
    if (b_outer && pl->n_grp_b > 0)
      k_zero_unused<<<(unsigned)(pl->n_grp_b < 4096 ? pl->n_grp_b : 4096), 256, 0, st>>>(
          pl->grpB_L, pl->grpB_n, pl->n_grp_b, IMQ_B_GROUP, I.K_unp, Bu);
  }
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

}  // namespace

imq_status launch_unpack(const imq_plan_t* pl, const void* A, const void* B, int8_t* Au, int8_t* Bu,
                         cudaStream_t st) {
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (pl->it == IMQ_I16)
    return unpack_typed<int16_t>(pl, static_cast<const int16_t*>(A), static_cast<const int16_t*>(B), Au, Bu,
                                 ds->num_sms, st);
  return unpack_typed<int32_t>(pl, static_cast<const int32_t*>(A), static_cast<const int32_t*>(B), Au, Bu,
                               ds->num_sms, st);
}

}  // namespace imq
