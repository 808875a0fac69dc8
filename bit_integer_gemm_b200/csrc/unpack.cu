// unpack.cu -- digit split of the quantised operands into b-bit int8 operands (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Approach": out-of-bound integers become several in-bound b-bit integers by row or column
// unpacking.  Entry p of unpacked line u is digit (line level + inner level of p) of the source entry
// (source line of u, inner index tK[p]); the layout is the one documented in include/imq.h.
//
// A line of a source unpacked OUTER with level L > 1 under the hybrid strategy holds all the digits of
// its entries, so it is zero at inner positions of level lk > 0 (the other sources, single lines, hold
// the digits of every inner level); for the pure strategies one of L > 1, lk > 0 never holds.
//
// Both unpacked operands are K-major (the inner index contiguous) because that is what the tcgen05
// GEMM reads through TMA.  A source line is staged in the plan's staging order (index order, or its
// inner indices grouped by level class when the plan chose that), so that most 16-position blocks are
// runs of consecutive staged entries.  The kernels:
//   k_unpack_planes   long stored rows unpacked INNER (one unpacked line per source line): a team of
//                  warps per line writes each entry's digits once into byte planes, then copies every
//                  block out of them; the team's next line is loaded meanwhile.
//   k_unpack_lines16  other stored rows (A, or B given as B^T), int16 or int32: a line per warp (or per
//                  team of warps for long lines); per block of one inner level the magnitudes of its 16
//                  entries are taken once and the digit of every output line emitted; blocks that mix
//                  levels are taken by the whole warp; it also zeroes the unused lines of OUTER groups.
//   k_unpack_lines / k_unpack_rows  fallbacks with per-line digit planes (lines too long for the
//                  kernels above); k_unpack_rows_direct gathers from global memory when planes do not fit.
//   k_unpack_cols  the source line is a stored column (B, or A given as A^T): a CTA transposes a
//                  128 (inner) x 32 (lines) tile through shared memory, reading 64-byte row segments
//                  and writing 128-byte segments of unpacked lines.
// HBM traffic: each source entry is read once (the gathered rows are L2-resident), each unpacked byte
// is written once.
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

// Copies n16 16-byte pieces from global to shared memory over one warp, kBatch loads in flight per lane
// before their stores (a store waits for its load).
template <int kBatch>
__device__ __forceinline__ void warp_copy16_global(const uint4* __restrict__ src, uint4* dst, int n16, int lane) {
  for (int c0 = lane; c0 < n16; c0 += 32 * kBatch) {
    uint4 buf[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int c = c0 + 32 * j;
      if (c < n16) buf[j] = src[c];
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int c = c0 + 32 * j;
      if (c < n16) dst[c] = buf[j];
    }
  }
}

// Staging positions of the 8 entries t .. t+7 (the identity without a staging order; -1 past K).
__device__ __forceinline__ void octet_positions(const int32_t* __restrict__ pinv, int64_t t, int64_t K, int32_t (&pj)[8]) {
#pragma unroll
  for (int r = 0; r < 8; ++r) pj[r] = t + r < K ? (pinv ? pinv[t + r] : (int32_t)(t + r)) : -1;
}
// Stores the 8 digit bytes (lo: entries 0-3, hi: 4-7) of an octet at plane row prow: one 8-byte store in
// index order, or byte by byte at the entries' staging positions.
__device__ __forceinline__ void store_octet(int8_t* prow, int64_t t, uint32_t lo, uint32_t hi, bool permuted,
                                            const int32_t (&pj)[8]) {
  if (!permuted) {
    *reinterpret_cast<uint2*>(prow + t) = make_uint2(lo, hi);
    return;
  }
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (pj[r] >= 0) prow[pj[r]] = (int8_t)(((r < 4 ? lo : hi) >> (8 * (r & 3))) & 0xFFu);
}

// Row gather: a CTA takes a batch of NL source lines and writes their digit planes to shared memory,
// plane[b][l][t] = d_l(line b, entry t) for the P levels the batch needs, one byte each.  Then each
// lane writes 16 consecutive inner positions of an output line: a block the plan marked contiguous
// (t0..t0+15, one level) is a 16-byte copy from a plane; any other block is gathered byte by byte.
template <typename T>
__global__ void __launch_bounds__(256) k_unpack_rows(const T* __restrict__ X, int64_t nlines, int64_t K,
                                                     int64_t ld, int NL, int P, int outer,
                                                     const int8_t* __restrict__ lvl, const int32_t* __restrict__ pos,
                                                     const int32_t* __restrict__ pinv, const int32_t* __restrict__ tJ,
                                                     const int8_t* __restrict__ lk,
                                                     const int32_t* __restrict__ blk16, int64_t K_unp, int bm1,
                                                     int8_t* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char dsm[];
  const int64_t Kp = (K + 15) / 16 * 16;  // plane row length, 16-byte aligned
  int8_t* planes = reinterpret_cast<int8_t*>(dsm);  // [NL][P][Kp]
  __shared__ int s_L[8];
  __shared__ int64_t s_base[8];
  const int tid = threadIdx.x;
  const int64_t nchunk = K_unp / 16;
  constexpr int kU = sizeof(T) == 2 ? 8 : 4;  // octets in flight per thread
  // whole-octet 16-byte loads: every line start and octet 16-byte aligned
  const bool vec8 = (K % 8 == 0) && (ld % 8 == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  for (int64_t i0 = (int64_t)blockIdx.x * NL; i0 < nlines; i0 += (int64_t)gridDim.x * NL) {
    const int nb = nlines - i0 < NL ? (int)(nlines - i0) : NL;
    if (tid < nb) {
      s_L[tid] = outer ? (int)lvl[i0 + tid] : 1;
      s_base[tid] = outer ? (int64_t)pos[i0 + tid] : i0 + tid;
    }
    // digit planes: a thread takes octets (8 consecutive entries of one line) and has kU of them in
    // flight before it computes any digit, so that the line loads overlap
    const int64_t q_line = Kp / 8;  // octets per line (Kp is a multiple of 16)
    const int64_t nq = (int64_t)nb * q_line;
    for (int64_t f0 = 0; f0 < nq; f0 += 256 * kU) {
      int32_t v[kU][8];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t f = f0 + (int64_t)u * 256 + tid;
        const int32_t b = (int32_t)f / (int32_t)q_line;  // nb * q_line < 2^31 (nb <= 8, lines < 2^31 bytes)
        const int64_t t = (f - (int64_t)b * q_line) * 8;
        const T* xr = X + (i0 + b) * ld + t;
        if (f < nq && vec8 && t + 8 <= K) {
          if (sizeof(T) == 2) {
            const uint4 w = *reinterpret_cast<const uint4*>(xr);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              v[u][2 * r] = (int16_t)(ww[r] & 0xFFFFu);
              v[u][2 * r + 1] = (int16_t)(ww[r] >> 16);
            }
          } else {
            const int4 w0 = *reinterpret_cast<const int4*>(xr), w1 = *reinterpret_cast<const int4*>(xr + 4);
            v[u][0] = w0.x; v[u][1] = w0.y; v[u][2] = w0.z; v[u][3] = w0.w;
            v[u][4] = w1.x; v[u][5] = w1.y; v[u][6] = w1.z; v[u][7] = w1.w;
          }
        } else {
#pragma unroll
          for (int r = 0; r < 8; ++r) v[u][r] = (f < nq && t + r < K) ? (int32_t)xr[r] : 0;
        }
      }
      const uint32_t mask = (1u << bm1) - 1u;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t f = f0 + (int64_t)u * 256 + tid;
        if (f >= nq) continue;
        const int32_t b = (int32_t)f / (int32_t)q_line;
        const int64_t t = (f - (int64_t)b * q_line) * 8;
        int8_t* pb = planes + (int64_t)b * P * Kp;
        int32_t pj[8];
        octet_positions(pinv, t, K, pj);
        uint32_t a[8], sg[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          sg[r] = v[u][r] < 0 ? 0xFFFFFFFFu : 0u;
          a[r] = v[u][r] < 0 ? (uint32_t)(-(int64_t)v[u][r]) : (uint32_t)v[u][r];
        }
        for (int l = 0; l < P; ++l) {
          const int sh = l * bm1;
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t d0 = sh < 31 ? ((a[r] >> sh) & mask) : 0u;
            const uint32_t d1 = sh < 31 ? ((a[r + 4] >> sh) & mask) : 0u;
            lo |= (((d0 ^ sg[r]) - sg[r]) & 0xFFu) << (8 * r);
            hi |= (((d1 ^ sg[r + 4]) - sg[r + 4]) & 0xFFu) << (8 * r);
          }
          store_octet(pb + (int64_t)l * Kp, t, lo, hi, pinv != nullptr, pj);
        }
      }
    }
    __syncthreads();
    for (int64_t c = tid; c < nchunk; c += 256) {
      const int32_t t0 = blk16[c];
      const int64_t p = c * 16;
      if (t0 >= 0) {
        const int lk0 = lk[p];
        for (int b = 0; b < nb; ++b) {
          const int L = s_L[b];
          const bool zero = L > 1 && lk0 > 0;
          for (int l = 0; l < L; ++l) {
            const uint4 w = zero ? make_uint4(0u, 0u, 0u, 0u)
                                 : *reinterpret_cast<const uint4*>(planes + ((int64_t)b * P + l + lk0) * Kp + t0);
            *reinterpret_cast<uint4*>(out + (s_base[b] + l) * K_unp + p) = w;
          }
        }
      } else {
        const int4* tq = reinterpret_cast<const int4*>(tJ + p);
        const int4 ta = tq[0], tb = tq[1], tc = tq[2], td = tq[3];
        const int32_t tt[16] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w,
                                tc.x, tc.y, tc.z, tc.w, td.x, td.y, td.z, td.w};
        const int4 lq = *reinterpret_cast<const int4*>(lk + p);
        const int8_t* ll = reinterpret_cast<const int8_t*>(&lq);
        for (int b = 0; b < nb; ++b) {
          const int L = s_L[b];
          for (int l = 0; l < L; ++l) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t packed = 0;
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int k = q * 4 + r;
                const uint32_t byte = (tt[k] >= 0 && (L == 1 || ll[k] == 0))
                                          ? (uint8_t)planes[((int64_t)b * P + l + ll[k]) * Kp + tt[k]]
                                          : 0u;
                packed |= byte << (8 * r);
              }
              w[q] = packed;
            }
            *reinterpret_cast<uint4*>(out + (s_base[b] + l) * K_unp + p) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    __syncthreads();
  }
}

// Digit planes of one int16 line, SIMD within a register: a word holds two entries; their magnitudes
// come from a branch-free absolute value per 16-bit half, a plane's digits from one mask and shift per
// word (masking first keeps the upper half's bits out of the lower half), four digits are gathered into the bytes of one word with a byte permute, and the negative
// entries' digits are negated byte-wise as (0x80808080 - d) ^ 0x80808080 (a digit is at most 127, so
// no byte borrows).  Digits of level l with l * bm1 >= 16 are zero for int16 magnitudes.  The line is
// 16-byte aligned and K a multiple of 8; entries K .. Kp-1 of the planes are written as zeros.
__device__ __forceinline__ void digit_planes_i16(const int16_t* __restrict__ xr, int64_t K, int64_t Kp, int P,
                                                 int bm1, const int32_t* __restrict__ pinv,
                                                 int8_t* __restrict__ planes, int lane) {
  const uint32_t mask = (1u << bm1) - 1u;
  const int64_t nq = Kp / 8;
  constexpr int kU = 8;
  for (int64_t q0 = 0; q0 < nq; q0 += 32 * kU) {
    uint4 w[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t t = (q0 + u * 32 + lane) * 8;
      w[u] = t + 8 <= K ? *reinterpret_cast<const uint4*>(xr + t) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t t = (q0 + u * 32 + lane) * 8;
      if (t >= Kp) continue;
      int32_t pj[8];
      octet_positions(pinv, t, K, pj);
      const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      uint32_t A[4], S[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t sgn = (ww[r] >> 15) & 0x00010001u;  // 1 in each negative half
        S[r] = sgn * 0xFFFFu;                              // 0xFFFF in each negative half
        A[r] = (ww[r] ^ S[r]) + sgn;                       // |entry| per half (no carry between halves)
      }
      const uint32_t Mlo = __byte_perm(S[0], S[1], 0x6420), Mhi = __byte_perm(S[2], S[3], 0x6420);
      for (int l = 0; l < P; ++l) {
        const int sh = l * bm1;
        uint32_t lo = 0, hi = 0;
        if (sh < 16) {
          // the digit's bits of both halves (clipped to 16 bits), then shifted down within each half
          const uint32_t m2 = ((mask << sh) & 0xFFFFu) * 0x00010001u;
          const uint32_t d0 = (A[0] & m2) >> sh, d1 = (A[1] & m2) >> sh;
          const uint32_t d2 = (A[2] & m2) >> sh, d3 = (A[3] & m2) >> sh;
          const uint32_t plo = __byte_perm(d0, d1, 0x6420), phi = __byte_perm(d2, d3, 0x6420);
          const uint32_t nlo = (0x80808080u - plo) ^ 0x80808080u, nhi = (0x80808080u - phi) ^ 0x80808080u;
          lo = (plo & ~Mlo) | (nlo & Mlo);
          hi = (phi & ~Mhi) | (nhi & Mhi);
        }
        store_octet(planes + (int64_t)l * Kp, t, lo, hi, pinv != nullptr, pj);
      }
    }
  }
}

// Row gather, one warp per source line: the warp loads its line (every load of a lane in flight before
// any digit is computed), writes the line's P digit planes to its own shared memory,
// plane[l][t] = d_l(entry t), and streams out the line's unpacked lines: a 16-byte block the plan marked
// contiguous (t0..t0+15, one level) is one 16-byte copy from a plane, any other block is gathered byte by
// byte.  Warps work independently (no CTA barrier), so one warp's loads overlap another's stores.
// The per-chunk plan metadata (block start and first inner level), the same for every line, is copied
// to shared memory once per CTA when it fits (meta_smem), so that the output loop reads it at shared-
// memory latency.
constexpr int64_t kMetaMaxChunks = 4096;

// What differs between the problems of a batched unpack launch (blockIdx.y = problem): the source, the
// plan's maps and the destination.  A single-problem launch passes no table and its own arguments.
struct LineJob {
  const void* X;
  int outer;
  const int8_t* lvl;
  const int32_t* pos;
  const int32_t* pinv;  // staging position of each inner index (null: the identity)
  const int32_t* tJ;    // staging position of the index at each inner position
  const int8_t* lk;
  const int32_t* blk16;
  int64_t K_unp;
  int8_t* out;
  const int32_t* grpL;
  const int32_t* grpN;
  int64_t ngrp;
};
// The same bound for the int16 staged-line kernel below (its chunk index is an int).
constexpr int64_t kMetaMaxChunks16 = 32768;

template <typename T>
__global__ void __launch_bounds__(256) k_unpack_lines(const T* X, int64_t nlines, int64_t K,
                                                      int64_t ld, int P, int nwarps, int outer,
                                                      const int8_t* lvl, const int32_t* pos,
                                                      const int32_t* pinv, const int32_t* tJ, const int8_t* lk,
                                                      const int32_t* blk16, int64_t K_unp, int bm1,
                                                      int meta_smem, int8_t* out, const int32_t* grpL,
                                                      const int32_t* grpN, int64_t ngrp, int G,
                                                      const LineJob* __restrict__ jobs) {
  extern __shared__ __align__(16) unsigned char dsm[];
  if (jobs) {
    const LineJob& jb = jobs[blockIdx.y];
    X = static_cast<const T*>(jb.X);
    outer = jb.outer;
    lvl = jb.lvl;
    pos = jb.pos;
    pinv = jb.pinv;
    tJ = jb.tJ;
    lk = jb.lk;
    blk16 = jb.blk16;
    K_unp = jb.K_unp;
    out = jb.out;
    grpL = jb.grpL;
    grpN = jb.grpN;
    ngrp = jb.ngrp;
  }
  // unused lines of the OUTER groups dealt to this CTA (lines n*L .. G-1 of a group of n sources of level
  // L, which no source line writes), before the lines themselves
  for (int64_t g = blockIdx.x; g < ngrp; g += gridDim.x) {
    const int64_t first = g * G + (int64_t)grpN[g] * grpL[g];
    const int64_t n16 = ((g + 1) * G - first) * K_unp / 16;
    uint4* o = reinterpret_cast<uint4*>(out + first * K_unp);
    for (int64_t k = threadIdx.x; k < n16; k += blockDim.x) o[k] = make_uint4(0u, 0u, 0u, 0u);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t Kp = (K + 15) / 16 * 16;  // plane row length, 16-byte aligned
  const int64_t nchunk = K_unp / 16;
  // [planes of nwarps lines][block starts, int32 x nchunk][first inner levels, int8 x nchunk]
  int32_t* s_blk = reinterpret_cast<int32_t*>(dsm + (int64_t)nwarps * P * Kp);
  int8_t* s_lk0 = reinterpret_cast<int8_t*>(s_blk + nchunk);
  if (meta_smem) {
    for (int64_t c = threadIdx.x; c < nchunk; c += blockDim.x) {
      s_blk[c] = blk16[c];
      s_lk0[c] = lk[c * 16];
    }
    __syncthreads();
  }
  if (warp >= nwarps) return;
  int8_t* planes = reinterpret_cast<int8_t*>(dsm) + (int64_t)warp * P * Kp;  // [P][Kp]
  constexpr int kU = sizeof(T) == 2 ? 8 : 4;  // octets in flight per lane
  const bool vec8 = (K % 8 == 0) && (ld % 8 == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  const int64_t nq = Kp / 8;  // octets per line
  const uint32_t mask = (1u << bm1) - 1u;
  for (int64_t line = (int64_t)blockIdx.x * nwarps + warp; line < nlines; line += (int64_t)gridDim.x * nwarps) {
    const T* xr = X + line * ld;
    const int L = outer ? (int)lvl[line] : 1;
    const int64_t base = outer ? (int64_t)pos[line] : line;
    // 1. digit planes of the line
    bool planes_done = false;
    if constexpr (sizeof(T) == 2) {
      if (vec8) {
        digit_planes_i16(reinterpret_cast<const int16_t*>(xr), K, Kp, P, bm1, pinv, planes, lane);
        planes_done = true;
      }
    }
    for (int64_t q0 = 0; q0 < (planes_done ? 0 : nq); q0 += 32 * kU) {
      int32_t v[kU][8];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t t = (q0 + u * 32 + lane) * 8;
        if (t + 8 <= K && vec8) {
          if (sizeof(T) == 2) {
            const uint4 w = *reinterpret_cast<const uint4*>(xr + t);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              v[u][2 * r] = (int16_t)(ww[r] & 0xFFFFu);
              v[u][2 * r + 1] = (int16_t)(ww[r] >> 16);
            }
          } else {
            const int4 w0 = *reinterpret_cast<const int4*>(xr + t), w1 = *reinterpret_cast<const int4*>(xr + t + 4);
            v[u][0] = w0.x; v[u][1] = w0.y; v[u][2] = w0.z; v[u][3] = w0.w;
            v[u][4] = w1.x; v[u][5] = w1.y; v[u][6] = w1.z; v[u][7] = w1.w;
          }
        } else {
#pragma unroll
          for (int r = 0; r < 8; ++r) v[u][r] = (t < Kp && t + r < K) ? (int32_t)xr[t + r] : 0;
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t t = (q0 + u * 32 + lane) * 8;
        if (t >= Kp) continue;
        int32_t pj[8];
        octet_positions(pinv, t, K, pj);
        uint32_t a[8], sg[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          sg[r] = v[u][r] < 0 ? 0xFFFFFFFFu : 0u;
          a[r] = v[u][r] < 0 ? (uint32_t)(-(int64_t)v[u][r]) : (uint32_t)v[u][r];
        }
        for (int l = 0; l < P; ++l) {
          const int sh = l * bm1;
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t d0 = sh < 31 ? ((a[r] >> sh) & mask) : 0u;
            const uint32_t d1 = sh < 31 ? ((a[r + 4] >> sh) & mask) : 0u;
            lo |= (((d0 ^ sg[r]) - sg[r]) & 0xFFu) << (8 * r);
            hi |= (((d1 ^ sg[r + 4]) - sg[r + 4]) & 0xFFu) << (8 * r);
          }
          store_octet(planes + (int64_t)l * Kp, t, lo, hi, pinv != nullptr, pj);
        }
      }
    }
    __syncwarp();
    // 2. the L unpacked lines, 16 inner positions per lane and step (512 contiguous bytes per warp)
    for (int64_t c = lane; c < nchunk; c += 32) {
      const int32_t t0 = meta_smem ? s_blk[c] : blk16[c];
      const int64_t p = c * 16;
      if (t0 >= 0) {
        const int lk0 = meta_smem ? s_lk0[c] : lk[p];
        const bool zero = L > 1 && lk0 > 0;
        for (int l = 0; l < L; ++l) {
          const uint4 w = zero ? make_uint4(0u, 0u, 0u, 0u)
                               : *reinterpret_cast<const uint4*>(planes + (int64_t)(l + lk0) * Kp + t0);
          *reinterpret_cast<uint4*>(out + (base + l) * K_unp + p) = w;
        }
      } else {
        const int4* tq = reinterpret_cast<const int4*>(tJ + p);
        const int4 ta = tq[0], tb = tq[1], tc = tq[2], td = tq[3];
        const int32_t tt[16] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w,
                                tc.x, tc.y, tc.z, tc.w, td.x, td.y, td.z, td.w};
        const int4 lq = *reinterpret_cast<const int4*>(lk + p);
        const int8_t* ll = reinterpret_cast<const int8_t*>(&lq);
        for (int l = 0; l < L; ++l) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t packed = 0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int k = q * 4 + r;
              const uint32_t byte = (tt[k] >= 0 && (L == 1 || ll[k] == 0))
                                        ? (uint8_t)planes[(int64_t)(l + ll[k]) * Kp + tt[k]]
                                        : 0u;
              packed |= byte << (8 * r);
            }
            w[q] = packed;
          }
          *reinterpret_cast<uint4*>(out + (base + l) * K_unp + p) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    __syncwarp();
  }
}

// Digit kL (base 2^kBm1, sign-magnitude) of the 16 entries of m as 16 bytes in entry order, with the
// level and base fixed at compile time (digits16_from with its masks and shifts folded).
template <int kBm1, int kL>
__device__ __forceinline__ uint4 digits16_fixed(const Mag16& m) {
  constexpr int sh = kL * kBm1;
  if constexpr (sh >= 16) {
    return make_uint4(0u, 0u, 0u, 0u);
  } else {
    constexpr uint32_t m2 = ((((1u << kBm1) - 1u) << sh) & 0xFFFFu) * 0x00010001u;
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t pd = __byte_perm((m.a[2 * q] & m2) >> sh, (m.a[2 * q + 1] & m2) >> sh, 0x6420);
      const uint32_t nd = (0x80808080u - pd) ^ 0x80808080u;
      o[q] = (pd & ~m.neg[q]) | (nd & m.neg[q]);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Magnitudes and signs of 16 int32 entries, for their digits of any level: per 4 entries a byte mask
// (0xFF where the entry is negative) in entry order.
struct Mag16w {
  uint32_t m[16];
  uint32_t neg[4];
};
__device__ __forceinline__ Mag16w mag16_i32(const int32_t (&e)[16]) {
  Mag16w r;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t nm = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int32_t v = e[4 * q + k];
      r.m[4 * q + k] = v < 0 ? 0u - (uint32_t)v : (uint32_t)v;
      nm |= ((uint32_t)(v >> 31) & 0xFFu) << (8 * k);
    }
    r.neg[q] = nm;
  }
  return r;
}
// Lines staged one per team of warps (long lines) keep a 4-byte pad word after every 16 entries (pad = 4 /
// sizeof(T) entries, else 0): a lane's 16-position block starts 32 (int16) or 64 (int32) bytes after its
// neighbour's, which without the pad puts a warp's loads on 4 or 2 of the 32 banks; with it neighbouring
// lanes are 9 or 17 words apart and every bank is used once.
__device__ __forceinline__ int slot(int j, int pad) { return j + (j >> 4) * pad; }
// Entries a staged line of K entries occupies (a padded line with 8 spare entries; the ninth word of a
// block's loads may reach one word past a line, which stays inside the shared memory of the launch: the
// next line or the block metadata).
__host__ __device__ constexpr int64_t staged_len(int64_t K, int pad) {
  return (K + 15) / 16 * (16 + pad) + (pad ? 8 : 0);
}

// The 16 int32 entries at staging positions t0 .. t0 + 15 of a staged line (16-byte loads for an unpadded
// line and t0 % 4 == 0).
__device__ __forceinline__ void load16_i32(const int32_t* row, int t0, int pad, int32_t (&e)[16]) {
  if (pad == 0 && (t0 & 3) == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int4 w = reinterpret_cast<const int4*>(row + t0)[q];
      e[4 * q] = w.x; e[4 * q + 1] = w.y; e[4 * q + 2] = w.z; e[4 * q + 3] = w.w;
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) e[k] = row[slot(t0 + k, pad)];
}
// The 16 entries at staging positions j[0..15] of a staged line (0 where j < 0: padding).
__device__ __forceinline__ void gather16_i32(const int32_t* row, const int32_t* __restrict__ j, int pad,
                                             int32_t (&e)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int4 v = reinterpret_cast<const int4*>(j)[q];
    e[4 * q] = v.x >= 0 ? row[slot(v.x, pad)] : 0;
    e[4 * q + 1] = v.y >= 0 ? row[slot(v.y, pad)] : 0;
    e[4 * q + 2] = v.z >= 0 ? row[slot(v.z, pad)] : 0;
    e[4 * q + 3] = v.w >= 0 ? row[slot(v.w, pad)] : 0;
  }
}
__device__ __forceinline__ void gather16_i16(const int16_t* row, const int32_t* __restrict__ j, int pad,
                                             uint32_t (&w)[8]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int4 v = reinterpret_cast<const int4*>(j)[q];
    const uint32_t e0 = v.x >= 0 ? (uint32_t)(uint16_t)row[slot(v.x, pad)] : 0u;
    const uint32_t e1 = v.y >= 0 ? (uint32_t)(uint16_t)row[slot(v.y, pad)] : 0u;
    const uint32_t e2 = v.z >= 0 ? (uint32_t)(uint16_t)row[slot(v.z, pad)] : 0u;
    const uint32_t e3 = v.w >= 0 ? (uint32_t)(uint16_t)row[slot(v.w, pad)] : 0u;
    w[2 * q] = e0 | (e1 << 16);
    w[2 * q + 1] = e2 | (e3 << 16);
  }
}
// Digit l (base 2^bm1, sign-magnitude) of the 16 entries as 16 bytes in entry order: four digits
// gathered into one word by byte permutes, the negative entries' digits negated byte-wise as
// (0x80808080 - d) ^ 0x80808080 (a digit is at most 127, so no byte borrows).
__device__ __forceinline__ uint4 digits16_i32(const Mag16w& m, int l, int bm1) {
  const int sh = l * bm1;
  if (sh >= 31) return make_uint4(0u, 0u, 0u, 0u);
  const uint32_t mask = (1u << bm1) - 1u;
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t d0 = (m.m[4 * q] >> sh) & mask, d1 = (m.m[4 * q + 1] >> sh) & mask;
    const uint32_t d2 = (m.m[4 * q + 2] >> sh) & mask, d3 = (m.m[4 * q + 3] >> sh) & mask;
    const uint32_t pd = __byte_perm(__byte_perm(d0, d1, 0x0040), __byte_perm(d2, d3, 0x0040), 0x5410);
    const uint32_t nd = (0x80808080u - pd) ^ 0x80808080u;
    o[q] = (pd & ~m.neg[q]) | (nd & m.neg[q]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The 16 int16 entries at staging positions t0 .. t0 + 15 of a staged line at any t0, as 8 words of two
// entries (low half first): two 16-byte loads for an unpadded line and t0 % 8 == 0, else nine 32-bit loads
// of entry pairs (a pair never straddles a pad word) and a funnel shift for odd t0.
__device__ __forceinline__ void load16_i16(const int16_t* row, int t0, int pad, uint32_t (&w)[8]) {
  if (pad == 0 && (t0 & 7) == 0) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + t0), b = *reinterpret_cast<const uint4*>(row + t0 + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    return;
  }
  const int e0 = t0 & ~1;
  uint32_t v[9];
#pragma unroll
  for (int i = 0; i < 9; ++i) v[i] = *reinterpret_cast<const uint32_t*>(row + slot(e0 + 2 * i, pad));
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = (t0 & 1) ? __funnelshift_r(v[i], v[i + 1], 16) : v[i];
}

constexpr int kFastLevels = 4;  // OUTER lines of up to this many levels take the unrolled path

// Stages source line xr (K entries) in the padded staged layout: entry t at row[slot(t)], or with a
// staging order at row[slot(pinv[t])].  Threads i0, i0 + step, ... take 16-byte pieces (vec: K, the row
// start and the line stride allow them), two in flight before their shared-memory stores.
template <typename T>
__device__ __forceinline__ void stage_line(const T* __restrict__ xr, int64_t K, bool vec,
                                           const int32_t* __restrict__ pinv, int pad, T* row, int i0, int step) {
  constexpr int V = 16 / (int)sizeof(T);
  constexpr int kBatch = 2;
  if (vec) {
    const int64_t nq = K / V;
    for (int64_t q0 = i0; q0 < nq; q0 += (int64_t)step * kBatch) {
      uint4 w[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t q = q0 + (int64_t)u * step;
        if (q < nq) w[u] = reinterpret_cast<const uint4*>(xr)[q];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t q = q0 + (int64_t)u * step;
        if (q >= nq) continue;
        const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        if (!pinv) {
          // a piece lies inside one group of 16 entries: four word stores from its first slot
          uint32_t* d = reinterpret_cast<uint32_t*>(row + slot((int)(q * V), pad));
#pragma unroll
          for (int k = 0; k < 4; ++k) d[k] = ww[k];
        } else if constexpr (sizeof(T) == 2) {
          const int4* pj = reinterpret_cast<const int4*>(pinv + q * V);
          const int4 a = pj[0], b = pj[1];
          row[slot(a.x, pad)] = (T)(ww[0] & 0xFFFFu); row[slot(a.y, pad)] = (T)(ww[0] >> 16);
          row[slot(a.z, pad)] = (T)(ww[1] & 0xFFFFu); row[slot(a.w, pad)] = (T)(ww[1] >> 16);
          row[slot(b.x, pad)] = (T)(ww[2] & 0xFFFFu); row[slot(b.y, pad)] = (T)(ww[2] >> 16);
          row[slot(b.z, pad)] = (T)(ww[3] & 0xFFFFu); row[slot(b.w, pad)] = (T)(ww[3] >> 16);
        } else {
          const int4 a = *reinterpret_cast<const int4*>(pinv + q * V);
          row[slot(a.x, pad)] = (T)ww[0]; row[slot(a.y, pad)] = (T)ww[1];
          row[slot(a.z, pad)] = (T)ww[2]; row[slot(a.w, pad)] = (T)ww[3];
        }
      }
    }
  } else {
    for (int64_t t = i0; t < K; t += step) row[slot(pinv ? pinv[t] : (int)t, pad)] = xr[t];
  }
}

// Named barrier 1 (id 1) or 2 (any other id) over `n` threads (a team of the CTA).  The ids are immediates,
// so that a CTA reserves three barriers rather than all sixteen (which would cap the CTAs per SM).
__device__ __forceinline__ void team_sync(int id, int n) {
  if (id == 1)
    asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory");
  else
    asm volatile("bar.sync 2, %0;" ::"r"(n) : "memory");
}

// Row gather for int16 and int32 sources, the base 2^kBm1 fixed at compile time.  Each source line is
// staged in shared memory in the plan's staging order (one line per warp, or per CTA for long lines) and
// the line's L unpacked lines are written 16 inner positions per lane and step.  A block the plan marked
// a run (the indices at staging positions j0..j0+15, one inner level lk0) takes the magnitudes and signs
// of its 16 staged entries once and emits digit (l + lk0) for every output line l from them.  The few
// other blocks (those across a segment or range boundary, and padding) are taken by the whole warp after
// the runs of its step: a half-warp per block, one position per lane, read through the plan's staging
// positions tJ.  The per-block plan metadata is staged in shared memory once per CTA.  Lines are dealt to
// the CTAs in turn (line i to CTA i mod gridDim.x).  After its lines, each CTA zeroes the unused lines of
// the OUTER groups dealt to it (group g to CTA g mod gridDim.x), lines n*L .. G-1 of a group of n sources
// of level L, which no source line writes.  teams > 0: lines too long for a line per warp are taken one
// at a time by each of `teams` teams of warps of the CTA (each with its own staged line, padded against
// bank conflicts, and its own named barrier), whose threads stage the line and write its blocks; one
// team's staging overlaps another's writes.
template <typename T, int kBm1>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 3 : 2) k_unpack_lines16(const T* X, int64_t nlines, int64_t K,
                                                           int64_t ld, int nwarps, int outer, const int8_t* lvl,
                                                           const int32_t* pos, const int32_t* pinv, const int32_t* tJ,
                                                           const int8_t* lk, const int32_t* blk16, int64_t K_unp,
                                                           int8_t* out, const int32_t* grpL, const int32_t* grpN,
                                                           int64_t ngrp, int G, int teams,
                                                           const LineJob* __restrict__ jobs) {
  extern __shared__ __align__(16) unsigned char dsm[];
  if (jobs) {
    const LineJob& jb = jobs[blockIdx.y];
    X = static_cast<const T*>(jb.X);
    outer = jb.outer;
    lvl = jb.lvl;
    pos = jb.pos;
    pinv = jb.pinv;
    tJ = jb.tJ;
    lk = jb.lk;
    blk16 = jb.blk16;
    K_unp = jb.K_unp;
    out = jb.out;
    grpL = jb.grpL;
    grpN = jb.grpN;
    ngrp = jb.ngrp;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pad = teams ? 4 / (int)sizeof(T) : 0;
  const int64_t SL = staged_len(K, pad);  // staged line length in entries
  const int nchunk = (int)(K_unp / 16);
  // [staged lines of nwarps warps or of the teams, T x SL][block starts, int32 x nchunk]
  // [first inner levels, int8 x nchunk]
  int32_t* s_blk = reinterpret_cast<int32_t*>(dsm + (int64_t)(teams ? teams : nwarps) * SL * (int64_t)sizeof(T));
  int8_t* s_lk0 = reinterpret_cast<int8_t*>(s_blk + nchunk);  // inner level of each block, -1 mixed
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    s_blk[c] = blk16[c];
    // the block's inner level, or -1 when its 16 positions do not share one
    const uint4 q = *reinterpret_cast<const uint4*>(lk + (int64_t)c * 16);
    const uint32_t b0 = (q.x & 0xFFu) * 0x01010101u;
    s_lk0[c] = (q.x == b0 && q.y == b0 && q.z == b0 && q.w == b0) ? (int8_t)(q.x & 0xFFu) : (int8_t)-1;
  }
  __syncthreads();
  constexpr int kPer16 = 16 / (int)sizeof(T);  // entries per 16-byte load
  const bool vec8 = (K % kPer16 == 0) && (ld % kPer16 == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  // Warp-cooperative write of the irregular blocks flagged in `irr` (bit k: block cb + k): lanes 0-15 take
  // one block, lanes 16-31 the next, one position per lane and a byte store per output line.
  auto irregular = [&](const T* row, int8_t* o0, int L, int cb, unsigned irr) {
    while (irr) {
      const int k0 = __ffs(irr) - 1;
      irr &= irr - 1;
      int k1 = -1;
      if (irr) {
        k1 = __ffs(irr) - 1;
        irr &= irr - 1;
      }
      const int kk = lane < 16 ? k0 : k1;
      if (kk < 0) continue;
      const int64_t pp = (int64_t)(cb + kk) * 16 + (lane & 15);
      const int32_t j = tJ[pp];
      const int lr = lk[pp];
      const int32_t v = j >= 0 ? (int32_t)row[slot(j, pad)] : 0;
      const bool use = j >= 0 && (L == 1 || lr == 0);
      for (int l = 0; l < L; ++l) o0[(int64_t)l * K_unp + pp] = (int8_t)(use ? digit_of(v, l + lr, kBm1) : 0);
    }
  };
  // The unpacked lines of source line `line`, staged in `row`: the warp's blocks cb0 + lane, cb0 + lane +
  // c_step, ... (cb0 and c_step the same for all its lanes).
  auto emit = [&](int64_t line, const T* row, int cb0, int c_step) {
      const int L = outer ? (int)lvl[line] : 1;
      int8_t* o0 = out + (outer ? (int64_t)pos[line] : line) * K_unp;
      for (int cb = cb0; cb < nchunk; cb += c_step) {
        const int c = cb + lane;
        const int tb = c < nchunk ? s_blk[c] : -1;
        const int lk0 = c < nchunk ? s_lk0[c] : -1;
        // a run, or a block of one inner level gathered through tJ: the lane's own block, the digits
        // computed the same way for both; any other block is taken by the whole warp below
        const bool uni = c < nchunk && (tb != -1 || lk0 >= 0);
        if (uni) {
          const int64_t p = (int64_t)c * 16;
          const int t0 = tb >= 0 ? tb : -tb - 2;  // first staging position of a run (aligned or not)
          if (L > 1 && lk0 > 0) {
            for (int l = 0; l < L; ++l) *reinterpret_cast<uint4*>(o0 + (int64_t)l * K_unp + p) = make_uint4(0u, 0u, 0u, 0u);
          } else if constexpr (sizeof(T) == 2) {
            uint32_t w[8];
            if (tb != -1) load16_i16(reinterpret_cast<const int16_t*>(row), t0, pad, w);
            else gather16_i16(reinterpret_cast<const int16_t*>(row), tJ + p, pad, w);
            const Mag16 m = mag16_i16(w);
            if (L == 1) {
              *reinterpret_cast<uint4*>(o0 + p) = digits16_from(m, lk0, kBm1);
            } else if (L <= kFastLevels) {
              *reinterpret_cast<uint4*>(o0 + p) = digits16_fixed<kBm1, 0>(m);
              *reinterpret_cast<uint4*>(o0 + K_unp + p) = digits16_fixed<kBm1, 1>(m);
              if (L > 2) *reinterpret_cast<uint4*>(o0 + 2 * K_unp + p) = digits16_fixed<kBm1, 2>(m);
              if (L > 3) *reinterpret_cast<uint4*>(o0 + 3 * K_unp + p) = digits16_fixed<kBm1, 3>(m);
            } else {
              for (int l = 0; l < L; ++l) *reinterpret_cast<uint4*>(o0 + (int64_t)l * K_unp + p) = digits16_from(m, l, kBm1);
            }
          } else {
            int32_t e[16];
            if (tb != -1) load16_i32(reinterpret_cast<const int32_t*>(row), t0, pad, e);
            else gather16_i32(reinterpret_cast<const int32_t*>(row), tJ + p, pad, e);
            const Mag16w m = mag16_i32(e);
            if (L == 1) {
              *reinterpret_cast<uint4*>(o0 + p) = digits16_i32(m, lk0, kBm1);
            } else {
              for (int l = 0; l < L; ++l) *reinterpret_cast<uint4*>(o0 + (int64_t)l * K_unp + p) = digits16_i32(m, l, kBm1);
            }
          }
        }
        irregular(row, o0, L, cb, __ballot_sync(0xffffffffu, c < nchunk && !uni));
      }
  };
  if (teams) {
    // long lines: one at a time per team, staged by the team's threads, its blocks spread over them
    const int tpt = (int)blockDim.x / teams;  // threads per team (a multiple of 32)
    const int team = (int)threadIdx.x / tpt, ti = (int)threadIdx.x % tpt;
    T* row = reinterpret_cast<T*>(dsm) + (int64_t)team * SL;
    for (int64_t line = (int64_t)blockIdx.x * teams + team; line < nlines; line += (int64_t)gridDim.x * teams) {
      team_sync(1 + team, tpt);  // the team's previous line has been read
      stage_line<T>(X + line * ld, K, vec8, pinv, pad, row, ti, tpt);
      team_sync(1 + team, tpt);
      emit(line, row, (ti >> 5) * 32, tpt);
    }
  } else if (warp < nwarps) {
    T* row = reinterpret_cast<T*>(dsm) + (int64_t)warp * SL;
    for (int64_t line = (int64_t)warp * gridDim.x + blockIdx.x; line < nlines;
         line += (int64_t)gridDim.x * nwarps) {
      const T* xr = X + line * ld;
      if (pinv) {
        stage_line<T>(xr, K, vec8, pinv, 0, row, lane, 32);
      } else if (vec8) {
        warp_copy16_global<4>(reinterpret_cast<const uint4*>(xr), reinterpret_cast<uint4*>(row), (int)(K / kPer16),
                              lane);
      } else {
        for (int64_t t = lane; t < K; t += 32) row[t] = xr[t];
      }
      __syncwarp();
      emit(line, row, 0, 32);
      __syncwarp();
    }
  }
  // unused lines of the OUTER groups dealt to this CTA
  for (int64_t g = blockIdx.x; g < ngrp; g += gridDim.x) {
    const int64_t first = g * G + (int64_t)grpN[g] * grpL[g];
    const int64_t n16 = ((g + 1) * G - first) * K_unp / 16;
    uint4* o = reinterpret_cast<uint4*>(out + first * K_unp);
    for (int64_t k = threadIdx.x; k < n16; k += blockDim.x) o[k] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// ------------------------------------------------------------------------------------------------
// Digit planes for lines unpacked INNER (one unpacked line per source line, the digit level set by the
// inner position).  An entry appears at several inner positions, once per (lA, lB) segment it belongs
// to, so its digits are computed once per line into byte planes -- plane[l][j] = digit l of the staged
// entry at staging position j -- and every 16-position block of one inner level is then a copy of 16
// plane bytes: a run from consecutive staging positions, or a gather through tJ.
// ------------------------------------------------------------------------------------------------
// Byte offset of staging position j in a plane: 4 pad bytes after every 16, so that lanes copying runs
// 16 bytes apart read words 5 apart and every bank once.
__device__ __forceinline__ int pslot(int j) { return j + ((j >> 4) << 2); }
// Bytes of one plane of K positions: 20 per group of 16 and one spare group, rounded up to 16.
__host__ __device__ constexpr int64_t plane_bytes(int64_t K) { return (((K + 15) / 16 + 1) * 20 + 15) / 16 * 16; }
// Entries of the staged line (a 16-byte multiple).
template <typename T>
__host__ __device__ constexpr int64_t plane_row_len(int64_t K) {
  return (K + 15) / 16 * 16;
}

// Digit l of 8 entries as two words (bytes in entry order): magnitudes in `a` (int16: two per word, four
// words; int32: one per word, eight words) and byte masks of the negative entries in `neg`.
template <typename T>
__device__ __forceinline__ void digits8(const uint32_t* a, const uint32_t (&neg)[2], int l, int bm1,
                                        uint32_t& lo, uint32_t& hi) {
  const int sh = l * bm1;
  uint32_t pd[2];
  if constexpr (sizeof(T) == 2) {
    if (sh >= 16) {
      lo = hi = 0u;
      return;
    }
    const uint32_t m2 = ((((1u << bm1) - 1u) << sh) & 0xFFFFu) * 0x00010001u;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      pd[h] = __byte_perm((a[2 * h] & m2) >> sh, (a[2 * h + 1] & m2) >> sh, 0x6420);
  } else {
    if (sh >= 31) {
      lo = hi = 0u;
      return;
    }
    const uint32_t mask = (1u << bm1) - 1u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t d0 = (a[4 * h] >> sh) & mask, d1 = (a[4 * h + 1] >> sh) & mask;
      const uint32_t d2 = (a[4 * h + 2] >> sh) & mask, d3 = (a[4 * h + 3] >> sh) & mask;
      pd[h] = __byte_perm(__byte_perm(d0, d1, 0x0040), __byte_perm(d2, d3, 0x0040), 0x5410);
    }
  }
  const uint32_t n0 = (0x80808080u - pd[0]) ^ 0x80808080u, n1 = (0x80808080u - pd[1]) ^ 0x80808080u;
  lo = (pd[0] & ~neg[0]) | (n0 & neg[0]);
  hi = (pd[1] & ~neg[1]) | (n1 & neg[1]);
}

// Teams of warps (`teams` per CTA, named barriers 1 .. teams) take one source line at a time: stage it in
// staging order, write its P digit planes, then write its unpacked line.  Lines are dealt to the teams in
// turn.  Blocks of one inner level copy plane bytes; blocks that mix levels (segment boundaries, padding)
// are taken by the whole warp, one position per lane.
template <typename T, int kBm1>
__global__ void __launch_bounds__(256, 2) k_unpack_planes(const T* X, int64_t nlines, int64_t K, int64_t ld, int P,
                                                          int teams, const int32_t* pinv, const int32_t* tJ,
                                                          const int8_t* lk, const int32_t* blk16, int64_t K_unp,
                                                          int8_t* out, const LineJob* __restrict__ jobs) {
  extern __shared__ __align__(16) unsigned char dsm[];
  if (jobs) {
    const LineJob& jb = jobs[blockIdx.y];
    X = static_cast<const T*>(jb.X);
    pinv = jb.pinv;
    tJ = jb.tJ;
    lk = jb.lk;
    blk16 = jb.blk16;
    K_unp = jb.K_unp;
    out = jb.out;
  }
  const int lane = threadIdx.x & 31;
  const int64_t RL = plane_row_len<T>(K), PB = plane_bytes(K);
  const int64_t team_bytes = RL * (int64_t)sizeof(T) + (int64_t)P * PB;
  const int nchunk = (int)(K_unp / 16);
  // [teams x (staged line, T x RL | P planes of PB bytes)][block starts, int32 x nchunk][levels, int8 x nchunk]
  int32_t* s_blk = reinterpret_cast<int32_t*>(dsm + (int64_t)teams * team_bytes);
  int8_t* s_lk0 = reinterpret_cast<int8_t*>(s_blk + nchunk);  // inner level of each block, -1 mixed
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    s_blk[c] = blk16[c];
    const uint4 q = *reinterpret_cast<const uint4*>(lk + (int64_t)c * 16);
    const uint32_t b0 = (q.x & 0xFFu) * 0x01010101u;
    s_lk0[c] = (q.x == b0 && q.y == b0 && q.z == b0 && q.w == b0) ? (int8_t)(q.x & 0xFFu) : (int8_t)-1;
  }
  __syncthreads();
  const int tpt = (int)blockDim.x / teams;  // threads per team (a multiple of 32)
  const int team = (int)threadIdx.x / tpt, ti = (int)threadIdx.x % tpt;
  T* row = reinterpret_cast<T*>(dsm + (int64_t)team * team_bytes);
  uint8_t* planes = reinterpret_cast<uint8_t*>(row + RL);
  constexpr int kPer16 = 16 / (int)sizeof(T);
  const bool vec = (K % kPer16 == 0) && (ld % kPer16 == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  // The team's next line is loaded into registers (up to kPF 16-byte pieces per thread) while the current
  // one is split and written, so that its load latency is hidden; pieces beyond that are loaded when the
  // line is staged.
  constexpr int kPF = 8;
  const int64_t nq = vec ? K / kPer16 : 0;
  uint4 pf[kPF];
  auto prefetch = [&](int64_t ln) {
    const uint4* src = reinterpret_cast<const uint4*>(X + ln * ld);
#pragma unroll
    for (int k = 0; k < kPF; ++k) {
      const int64_t q = ti + (int64_t)k * tpt;
      if (q < nq) pf[k] = __ldcs(src + q);
    }
  };
  // piece q (entries q * kPer16 ...) into the staged line, in staging order when there is one
  auto put = [&](int64_t q, const uint4& w) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    if (!pinv) {
      *reinterpret_cast<uint4*>(row + q * kPer16) = w;
    } else if constexpr (sizeof(T) == 2) {
      const int4* pj = reinterpret_cast<const int4*>(pinv + q * kPer16);
      const int4 a = pj[0], b = pj[1];
      row[a.x] = (T)(ww[0] & 0xFFFFu); row[a.y] = (T)(ww[0] >> 16);
      row[a.z] = (T)(ww[1] & 0xFFFFu); row[a.w] = (T)(ww[1] >> 16);
      row[b.x] = (T)(ww[2] & 0xFFFFu); row[b.y] = (T)(ww[2] >> 16);
      row[b.z] = (T)(ww[3] & 0xFFFFu); row[b.w] = (T)(ww[3] >> 16);
    } else {
      const int4 a = *reinterpret_cast<const int4*>(pinv + q * kPer16);
      row[a.x] = (T)ww[0]; row[a.y] = (T)ww[1]; row[a.z] = (T)ww[2]; row[a.w] = (T)ww[3];
    }
  };
  const int64_t first = (int64_t)blockIdx.x * teams + team, stride = (int64_t)gridDim.x * teams;
  if (vec && first < nlines) prefetch(first);
  for (int64_t line = first; line < nlines; line += stride) {
    team_sync(1 + team, tpt);  // the team's previous line and planes have been read
    if (vec) {
#pragma unroll
      for (int k = 0; k < kPF; ++k) {
        const int64_t q = ti + (int64_t)k * tpt;
        if (q < nq) put(q, pf[k]);
      }
      const uint4* src = reinterpret_cast<const uint4*>(X + line * ld);
      for (int64_t q = ti + (int64_t)kPF * tpt; q < nq; q += tpt) put(q, src[q]);
      if (line + stride < nlines) prefetch(line + stride);
    } else {
      stage_line<T>(X + line * ld, K, false, pinv, 0, row, ti, tpt);
    }
    team_sync(1 + team, tpt);
    // planes: 8 staging positions per thread and step
    for (int m = ti; m < (int)(RL / 8); m += tpt) {
      uint32_t a[sizeof(T) == 2 ? 4 : 8];
      uint32_t neg[2];
      if constexpr (sizeof(T) == 2) {
        const uint4 w = reinterpret_cast<const uint4*>(row)[m];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t S[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t sgn = (ww[h] >> 15) & 0x00010001u;
          S[h] = sgn * 0xFFFFu;
          a[h] = (ww[h] ^ S[h]) + sgn;
        }
        neg[0] = __byte_perm(S[0], S[1], 0x6420);
        neg[1] = __byte_perm(S[2], S[3], 0x6420);
      } else {
        const int4 w0 = reinterpret_cast<const int4*>(row)[2 * m], w1 = reinterpret_cast<const int4*>(row)[2 * m + 1];
        const int32_t e[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t nm = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int32_t v = e[4 * h + k];
            a[4 * h + k] = v < 0 ? 0u - (uint32_t)v : (uint32_t)v;
            nm |= ((uint32_t)(v >> 31) & 0xFFu) << (8 * k);
          }
          neg[h] = nm;
        }
      }
      uint32_t* dst = reinterpret_cast<uint32_t*>(planes + pslot(8 * m));
      for (int l = 0; l < P; ++l) {
        uint32_t lo, hi;
        digits8<T>(a, neg, l, kBm1, lo, hi);
        dst[0] = lo;
        dst[1] = hi;
        dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(dst) + PB);
      }
    }
    team_sync(1 + team, tpt);
    int8_t* o0 = out + line * K_unp;
    for (int cb = (ti >> 5) * 32; cb < nchunk; cb += tpt) {
      const int c = cb + lane;
      const int tb = c < nchunk ? s_blk[c] : -1;
      const int lk0 = c < nchunk ? s_lk0[c] : -1;
      const bool uni = c < nchunk && (tb != -1 || lk0 >= 0);
      if (uni) {
        const uint8_t* pl = planes + (int64_t)lk0 * PB;
        uint4 o;
        if (tb != -1) {
          // a run: staging positions j0 .. j0 + 15 -- five words of the padded plane, shifted by j0 % 4 bytes
          const int j0 = tb >= 0 ? tb : -tb - 2;
          const int v0 = j0 >> 2, sh = (j0 & 3) * 8;
          uint32_t wv[5];
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            const int vw = v0 + i;
            wv[i] = reinterpret_cast<const uint32_t*>(pl)[vw + (vw >> 2)];
          }
          o.x = __funnelshift_r(wv[0], wv[1], sh);
          o.y = __funnelshift_r(wv[1], wv[2], sh);
          o.z = __funnelshift_r(wv[2], wv[3], sh);
          o.w = __funnelshift_r(wv[3], wv[4], sh);
        } else {
          // one inner level at scattered staging positions
          uint32_t wv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int4 jj = reinterpret_cast<const int4*>(tJ + (int64_t)c * 16)[q];
            const uint32_t b0 = jj.x >= 0 ? pl[pslot(jj.x)] : 0u, b1 = jj.y >= 0 ? pl[pslot(jj.y)] : 0u;
            const uint32_t b2 = jj.z >= 0 ? pl[pslot(jj.z)] : 0u, b3 = jj.w >= 0 ? pl[pslot(jj.w)] : 0u;
            wv[q] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
          }
          o = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        *reinterpret_cast<uint4*>(o0 + (int64_t)c * 16) = o;
      }
      unsigned irr = __ballot_sync(0xffffffffu, c < nchunk && !uni);
      while (irr) {
        // two mixed blocks per pass: lanes 0-15 the first, 16-31 the second, one position per lane
        const int k0 = __ffs(irr) - 1;
        irr &= irr - 1;
        int k1 = -1;
        if (irr) {
          k1 = __ffs(irr) - 1;
          irr &= irr - 1;
        }
        const int kk = lane < 16 ? k0 : k1;
        if (kk < 0) continue;
        const int64_t pp = (int64_t)(cb + kk) * 16 + (lane & 15);
        const int32_t j = tJ[pp];
        const int lr = lk[pp];
        o0[pp] = (int8_t)(j >= 0 ? planes[(int64_t)lr * PB + pslot(j)] : 0u);
      }
    }
  }
}

// Whether INNER lines of K entries, P digit planes and K_unp unpacked positions take the plane kernel:
// the lines are long (a team per line spends its barriers on enough output) and an entry appears at
// enough positions (K_unp / K) to repay writing its P plane bytes once.
__host__ __device__ constexpr bool planes_pay(int64_t K, int P, int64_t K_unp) {
  return K >= 1024 && 2 * K_unp >= (int64_t)(P + 1) * K;
}

// Launch shape of the plane kernel for lines of K entries of T, P planes and nchunk blocks: two teams of
// four warps when both teams' lines and planes and the metadata fit about half an SM (two CTAs per SM),
// else one team of eight within the budget.  False when neither fits.
bool planes_shape(int64_t K, size_t elem, int P, int64_t nchunk, int* teams, size_t* smem) {
  const size_t team = (size_t)plane_row_len<int16_t>(K) * elem + (size_t)P * (size_t)plane_bytes(K);
  const size_t meta = (size_t)nchunk * 5;
  if (2 * team + meta <= 110 * 1024) {
    *teams = 2;
  } else if (team + meta <= 200 * 1024) {
    *teams = 1;
  } else {
    return false;
  }
  *smem = (size_t)*teams * team + meta;
  return nchunk <= kMetaMaxChunks16;
}

template <typename T, int kBm1>
imq_status launch_planes_b(const T* X, int64_t nlines, int64_t K, int64_t ld, int P, int teams, const int32_t* pinv,
                           const int32_t* tJ, const int8_t* lk, const int32_t* blk16, int64_t K_unp, int8_t* out,
                           size_t smem, int num_sms, cudaStream_t st, const LineJob* jobs, int nprob) {
  auto kern = k_unpack_planes<T, kBm1>;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  int per_sm = 0;
  IMQ_CUDA_TRY(blocks_per_sm(reinterpret_cast<const void*>(kern), 256, smem, &per_sm));
  if (per_sm < 1) per_sm = 1;
  int64_t grid = ((int64_t)num_sms * per_sm + nprob - 1) / nprob;
  const int64_t need = (nlines + teams - 1) / teams;
  if (grid > need) grid = need;
  kern<<<dim3((unsigned)grid, (unsigned)nprob), 256, smem, st>>>(X, nlines, K, ld, P, teams, pinv, tJ, lk, blk16,
                                                                 K_unp, out, jobs);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

template <typename T>
imq_status launch_planes(int bm1, const T* X, int64_t nlines, int64_t K, int64_t ld, int P, int teams,
                         const int32_t* pinv, const int32_t* tJ, const int8_t* lk, const int32_t* blk16, int64_t K_unp,
                         int8_t* out, size_t smem, int num_sms, cudaStream_t st, const LineJob* jobs, int nprob) {
#define IMQ_PLANES(B) \
  launch_planes_b<T, B>(X, nlines, K, ld, P, teams, pinv, tJ, lk, blk16, K_unp, out, smem, num_sms, st, jobs, nprob)
  switch (bm1) {
    case 1: return IMQ_PLANES(1);
    case 2: return IMQ_PLANES(2);
    case 3: return IMQ_PLANES(3);
    case 4: return IMQ_PLANES(4);
    case 5: return IMQ_PLANES(5);
    case 6: return IMQ_PLANES(6);
    default: return IMQ_PLANES(7);
  }
#undef IMQ_PLANES
}

// nprob > 1: `jobs` (device) holds the per-problem arguments and the ones given here are ignored.
template <typename T, int kBm1>
imq_status launch_lines16(const T* X, int64_t nlines, int64_t K, int64_t ld, int nw, int outer,
                          const int8_t* lvl, const int32_t* pos, const int32_t* pinv, const int32_t* tJ,
                          const int8_t* lk, const int32_t* blk16, int64_t K_unp, int8_t* out, const int32_t* grpL,
                          const int32_t* grpN, int64_t ngrp, int G, size_t smem, int num_sms, cudaStream_t st,
                          const LineJob* jobs = nullptr, int nprob = 1) {
  auto kern = k_unpack_lines16<T, kBm1>;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  int per_sm = 0;
  IMQ_CUDA_TRY(blocks_per_sm(reinterpret_cast<const void*>(kern), 256, smem, &per_sm));
  if (per_sm < 1) per_sm = 1;
  // every resident slot once over the whole batch; a CTA takes a line per warp or per team at a time
  const int teams = nw < 0 ? -nw : 0;
  int64_t grid = ((int64_t)num_sms * per_sm + nprob - 1) / nprob;
  const int64_t need = teams ? (nlines + teams - 1) / teams : nlines;
  if (grid > need) grid = need;
  kern<<<dim3((unsigned)grid, (unsigned)nprob), 256, smem, st>>>(X, nlines, K, ld, nw > 0 ? nw : 0, outer, lvl, pos,
                                                                 pinv, tJ, lk, blk16, K_unp, out, grpL, grpN, ngrp,
                                                                 G, teams, jobs);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

// The staged-line kernel for base 2^bm1 (bm1 in 1..7), the base fixed at compile time.
template <typename T>
imq_status launch_staged(int bm1, const T* X, int64_t nlines, int64_t K, int64_t ld, int nw, int outer,
                         const int8_t* lvl, const int32_t* pos, const int32_t* pinv, const int32_t* tJ,
                         const int8_t* lk, const int32_t* blk16, int64_t K_unp, int8_t* out, const int32_t* grpL,
                         const int32_t* grpN, int64_t ngrp, int G, size_t smem, int num_sms, cudaStream_t st,
                         const LineJob* jobs, int nprob) {
#define IMQ_STAGED(B) \
  launch_lines16<T, B>(X, nlines, K, ld, nw, outer, lvl, pos, pinv, tJ, lk, blk16, K_unp, out, grpL, grpN, ngrp, G, smem, \
                       num_sms, st, jobs, nprob)
  switch (bm1) {
    case 1: return IMQ_STAGED(1);
    case 2: return IMQ_STAGED(2);
    case 3: return IMQ_STAGED(3);
    case 4: return IMQ_STAGED(4);
    case 5: return IMQ_STAGED(5);
    case 6: return IMQ_STAGED(6);
    default: return IMQ_STAGED(7);
  }
#undef IMQ_STAGED
}

// Launch shape of the staged-line kernel for lines of K entries of T and nchunk 16-position blocks: a
// line per warp (*nw_out > 0 warps, 8 while their lines fit in 64 KB, so that three CTAs share an SM),
// or for lines above 16 KB a line per team (*nw_out = -teams: two teams of four warps when two padded
// lines and the metadata fit the budget, else one of eight).  False when nothing fits the shared-memory
// budget or the block metadata (5 bytes per block, staged whole) is too long.
bool staged_shape(int64_t K, size_t elem, int64_t nchunk, int* nw_out, size_t* smem_out) {
  constexpr size_t kBudget = 200 * 1024;
  const size_t meta = (size_t)nchunk * 5;
  const int64_t plain = staged_len(K, 0) * (int64_t)elem;
  size_t smem;
  if (plain <= 16 * 1024) {
    int nw = (int)((64 * 1024) / plain);
    if (nw > 8) nw = 8;
    *nw_out = nw;
    smem = (size_t)nw * plain + meta;
  } else {
    const size_t padded = (size_t)staged_len(K, 4 / (int)elem) * elem;
    const int teams = 2 * padded + meta <= kBudget ? 2 : 1;
    *nw_out = -teams;
    smem = (size_t)teams * padded + meta;
  }
  *smem_out = smem;
  return nchunk <= kMetaMaxChunks16 && smem <= kBudget;
}

// Row gather for lines too long for shared-memory planes: digits are computed from the source line in
// global memory (L2); lane = 4 consecutive inner positions, 128-byte coalesced stores per warp.
template <typename T>
__global__ void __launch_bounds__(256) k_unpack_rows_direct(const T* __restrict__ X, int64_t nlines, int64_t ld,
                                                            int outer, const int8_t* __restrict__ lvl,
                                                            const int32_t* __restrict__ pos,
                                                            const int32_t* __restrict__ tK,
                                                            const int8_t* __restrict__ lk, int64_t K_unp, int bm1,
                                                            int8_t* __restrict__ out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t i = blockIdx.x; i < nlines; i += gridDim.x) {
    const T* xr = X + i * ld;
    const int L = outer ? (int)lvl[i] : 1;
    const int64_t base = outer ? (int64_t)pos[i] : i;
    for (int64_t p = (int64_t)warp * 128 + lane * 4; p < K_unp; p += 8 * 128) {
      const int4 t4 = *reinterpret_cast<const int4*>(tK + p);
      const uint32_t l4 = *reinterpret_cast<const uint32_t*>(lk + p);
      const int32_t tt[4] = {t4.x, t4.y, t4.z, t4.w};
      int32_t v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) v[r] = tt[r] >= 0 ? (int32_t)xr[tt[r]] : 0;
      for (int l = 0; l < L; ++l) {
        uint32_t packed = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int lkr = (int)(int8_t)(l4 >> (8 * r));
          const int32_t d = (L > 1 && lkr > 0) ? 0 : digit_of(v[r], l + lkr, bm1);
          packed |= ((uint32_t)(uint8_t)(int8_t)d) << (8 * r);
        }
        *reinterpret_cast<uint32_t*>(out + (base + l) * K_unp + p) = packed;
      }
    }
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
        const int32_t d = (s_t[pp] >= 0 && (L == 1 || s_l[pp] == 0)) ? digit_of(S[jj][pp], l + s_l[pp], bm1) : 0;
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

// The unused lines of an operand's OUTER groups (zeroed by the int16 row kernel itself, else by
// k_zero_unused after the operand's unpack).
struct ZeroJob {
  const int32_t* grpL = nullptr;
  const int32_t* grpN = nullptr;
  int64_t ngrp = 0;
  int G = 0;
};

// One operand.  *zeroed is set when the launch also zeroed the operand's unused OUTER lines.
template <typename T>
imq_status unpack_one(const T* X, int64_t nlines, int64_t K, int64_t ld, bool line_is_row, int outer, int P,
                      const int8_t* lvl, const int32_t* pos, const int32_t* tK, const int32_t* pinv,
                      const int32_t* tJ, const int8_t* lk, const int32_t* blk16, int64_t K_unp, int bm1, int8_t* out,
                      int num_sms, cudaStream_t st,
                      const ZeroJob& zj, bool* zeroed) {
  *zeroed = false;
  if (nlines == 0 || K_unp == 0) return IMQ_OK;
  // long rows unpacked INNER: the digit-plane kernel
  if (line_is_row && !outer && bm1 >= 1 && bm1 <= 7 && planes_pay(K, P, K_unp)) {
    int teams = 0;
    size_t smem = 0;
    if (planes_shape(K, sizeof(T), P, K_unp / 16, &teams, &smem))
      return launch_planes<T>(bm1, X, nlines, K, ld, P, teams, pinv, tJ, lk, blk16, K_unp, out, smem, num_sms, st,
                              nullptr, 1);
  }
  // rows (int16 or int32): the staged-line kernel, which also zeroes the unused OUTER lines
  {
    const int64_t nchunk = K_unp / 16;
    int nw = 0;
    size_t smem = 0;
    if (line_is_row && bm1 >= 1 && bm1 <= 7 && staged_shape(K, sizeof(T), nchunk, &nw, &smem)) {
      const int64_t ng = outer ? zj.ngrp : 0;
      const imq_status s = launch_staged<T>(bm1, X, nlines, K, ld, nw, outer, lvl, pos, pinv, tJ, lk, blk16, K_unp, out,
                                            zj.grpL, zj.grpN, ng, zj.G, smem, num_sms, st, nullptr, 1);
      *zeroed = s == IMQ_OK;
      return s;
    }
  }
  if (line_is_row) {
    // P planes per line: the levels an output line can ask for (line level + inner level)
    const int64_t Kp = (K + 15) / 16 * 16;
    // one warp per line, each with its own planes, while 8 warps' planes fit in 96 KB (two CTAs per
    // SM), else fewer warps per CTA down to one
    {
      const int64_t per_warp = (int64_t)P * Kp;
      int nw = (int)((96 * 1024) / per_warp);
      if (nw > 8) nw = 8;
      if (nw >= 1) {
        const int64_t nchunk = K_unp / 16;
        const int meta_smem = nchunk <= kMetaMaxChunks ? 1 : 0;
        const size_t smem = (size_t)nw * per_warp + (meta_smem ? (size_t)nchunk * 5 : 0);
        const int per_sm = (int)((200 * 1024) / (smem + 1024)) < 1 ? 1 : (int)((200 * 1024) / (smem + 1024));
        const int64_t ctas = (nlines + nw - 1) / nw;
        int64_t grid = (int64_t)num_sms * (per_sm > 8 ? 8 : per_sm);
        if (grid > ctas) grid = ctas;
        IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_unpack_lines<T>), smem));
        k_unpack_lines<T><<<(unsigned)grid, 256, smem, st>>>(X, nlines, K, ld, P, nw, outer, lvl, pos, pinv, tJ, lk, blk16,
                                                             K_unp, bm1, meta_smem, out, zj.grpL, zj.grpN,
                                                             outer ? zj.ngrp : 0, zj.G, nullptr);
        *zeroed = true;
        return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
      }
    }
    int NL = (int)((96 * 1024) / ((int64_t)P * Kp));
    if (NL > 8) NL = 8;
    if (NL < 1) {
      if ((int64_t)P * Kp > 200 * 1024) {
        // planes do not fit: compute the digits straight from global memory
        const int64_t grid = nlines < (int64_t)num_sms * 8 ? nlines : (int64_t)num_sms * 8;
        k_unpack_rows_direct<T><<<(unsigned)grid, 256, 0, st>>>(X, nlines, ld, outer, lvl, pos, tK, lk, K_unp, bm1,
                                                                 out);
        return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
      }
      NL = 1;
    }
    const size_t smem = (size_t)NL * P * Kp;
    const int per_sm = (int)((200 * 1024) / (smem + 2048)) < 1 ? 1 : (int)((200 * 1024) / (smem + 2048));
    const int64_t batches = (nlines + NL - 1) / NL;
    int64_t grid = (int64_t)num_sms * (per_sm > 8 ? 8 : per_sm);
    if (grid > batches) grid = batches;
    IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_unpack_rows<T>), smem));
    k_unpack_rows<T><<<(unsigned)grid, 256, smem, st>>>(X, nlines, K, ld, NL, P, outer, lvl, pos, pinv, tJ, lk, blk16,
                                                        K_unp, bm1, out);
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
  const int a_outer = (I.dir_a & IMQ_DIR_OUTER) != 0, b_outer = (I.dir_b & IMQ_DIR_OUTER) != 0;
  const int a_inner = (I.dir_a & IMQ_DIR_INNER) != 0, b_inner = (I.dir_b & IMQ_DIR_INNER) != 0;
  // A' lines are the logical rows of A: stored rows unless A is given transposed
  // planes an output line may read: OUTER lines their own levels, INNER ones the inner levels (the
  // hybrid's OUTER lines read only inner level 0, its single lines only the inner levels)
  const int pa_o = a_outer ? I.lmax_a_row : 1, pa_i = a_inner ? I.lmax_a_col : 1;
  const int pb_o = b_outer ? I.lmax_b_col : 1, pb_i = b_inner ? I.lmax_b_row : 1;
  const int pa = pa_o > pa_i ? pa_o : pa_i;
  const int pb = pb_o > pb_i ? pb_o : pb_i;
  ZeroJob za, zb;
  if (a_outer) za = ZeroJob{pl->grpA_L, pl->grpA_n, pl->n_grp_a, IMQ_A_GROUP};
  if (b_outer) zb = ZeroJob{pl->grpB_L, pl->grpB_n, pl->n_grp_b, IMQ_B_GROUP};
  bool za_done = false, zb_done = false;
  imq_status s = unpack_one<T>(A, I.M, I.K, pl->lda, !pl->transA, a_outer, pa, pl->lv_a_row, pl->posA, pl->tK,
                               pl->pinv, pl->tJ, pl->lAk, pl->blk16, I.K_unp, bm1, Au, num_sms, st, za, &za_done);
  if (s != IMQ_OK) return s;
  // B'^T lines are the logical columns of B: stored rows only when B is given transposed
  s = unpack_one<T>(B, I.N, I.K, pl->ldb, pl->transB != 0, b_outer, pb, pl->lv_b_col, pl->posB, pl->tK, pl->pinv,
                    pl->tJ, pl->lBk, pl->blk16, I.K_unp, bm1, Bu, num_sms, st, zb, &zb_done);
  if (s != IMQ_OK) return s;
  if (I.K_unp > 0) {
    if (a_outer && pl->n_grp_a > 0 && !za_done)
      k_zero_unused<<<(unsigned)(pl->n_grp_a < 4096 ? pl->n_grp_a : 4096), 256, 0, st>>>(
          pl->grpA_L, pl->grpA_n, pl->n_grp_a, IMQ_A_GROUP, I.K_unp, Au);
    if (b_outer && pl->n_grp_b > 0 && !zb_done)
      k_zero_unused<<<(unsigned)(pl->n_grp_b < 4096 ? pl->n_grp_b : 4096), 256, 0, st>>>(
          pl->grpB_L, pl->grpB_n, pl->n_grp_b, IMQ_B_GROUP, I.K_unp, Bu);
  }
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}


// One operand side (A when side == 0, else B) of a batch of plans made together (equal shapes, layouts
// and b): one launch for the whole batch when every problem takes the staged int16 kernel or the digit-
// plane kernel, else one unpack per problem.
template <typename T>
imq_status unpack_side_batch(const imq_plan_t* const* pls, int n, const void* const* src, int8_t* const* dst,
                             int side, int num_sms, cudaStream_t st) {
  const imq_plan_t* p0 = pls[0];
  const imq_plan_info& I0 = p0->info;
  const int bm1 = I0.b - 1;
  const int64_t K = I0.K;
  const int64_t nlines = side == 0 ? I0.M : I0.N;
  const int64_t ld = side == 0 ? p0->lda : p0->ldb;
  const bool line_is_row = side == 0 ? !p0->transA : p0->transB != 0;
  int64_t nchunk = 0;
  int P = 1;
  std::vector<LineJob> jobs((size_t)n);
  for (int h = 0; h < n; ++h) {
    const imq_plan_t* pl = pls[h];
    const imq_plan_info& I = pl->info;
    const int dir = side == 0 ? I.dir_a : I.dir_b;
    const int outer = (dir & IMQ_DIR_OUTER) != 0, inner = (dir & IMQ_DIR_INNER) != 0;
    const int po = outer ? (side == 0 ? I.lmax_a_row : I.lmax_b_col) : 1;
    const int pi = inner ? (side == 0 ? I.lmax_a_col : I.lmax_b_row) : 1;
    P = P > po ? P : po;
    P = P > pi ? P : pi;
    nchunk = nchunk > I.K_unp / 16 ? nchunk : I.K_unp / 16;
    LineJob& j = jobs[h];
    j.X = src[h];
    j.outer = outer;
    j.lvl = side == 0 ? pl->lv_a_row : pl->lv_b_col;
    j.pos = side == 0 ? pl->posA : pl->posB;
    j.pinv = pl->pinv;
    j.tJ = pl->tJ;
    j.lk = side == 0 ? pl->lAk : pl->lBk;
    j.blk16 = pl->blk16;
    j.K_unp = I.K_unp;
    j.out = dst[h];
    j.grpL = outer ? (side == 0 ? pl->grpA_L : pl->grpB_L) : nullptr;
    j.grpN = outer ? (side == 0 ? pl->grpA_n : pl->grpB_n) : nullptr;
    j.ngrp = outer ? (side == 0 ? pl->n_grp_a : pl->n_grp_b) : 0;
    if (I.b != I0.b || I.K != K || I.M != I0.M || I.N != I0.N) return IMQ_ERR_ARG;
  }
  if (nlines == 0 || nchunk == 0) return IMQ_OK;
  void* dj = nullptr;
  imq_status s = IMQ_OK;
  if (line_is_row && bm1 >= 1 && bm1 <= 7 && K >= 1024) {
    // the problems whose lines are unpacked INNER take the digit-plane kernel in one launch; the others
    // (OUTER lines) follow as a batch of their own
    std::vector<LineJob> in_jobs;
    std::vector<const imq_plan_t*> o_pls;
    std::vector<const void*> o_src;
    std::vector<int8_t*> o_dst;
    int P_in = 1;
    int64_t nchunk_in = 0;
    for (int h = 0; h < n; ++h) {
      const imq_plan_info& Ih = pls[h]->info;
      const int pih = ((side == 0 ? Ih.dir_a : Ih.dir_b) & IMQ_DIR_INNER) ? (side == 0 ? Ih.lmax_a_col : Ih.lmax_b_row) : 1;
      if (jobs[h].outer || !planes_pay(K, pih, Ih.K_unp)) {
        o_pls.push_back(pls[h]);
        o_src.push_back(src[h]);
        o_dst.push_back(dst[h]);
        continue;
      }
      const imq_plan_info& I = pls[h]->info;
      const int dir = side == 0 ? I.dir_a : I.dir_b;
      const int pi = (dir & IMQ_DIR_INNER) ? (side == 0 ? I.lmax_a_col : I.lmax_b_row) : 1;
      P_in = P_in > pi ? P_in : pi;
      nchunk_in = nchunk_in > I.K_unp / 16 ? nchunk_in : I.K_unp / 16;
      in_jobs.push_back(jobs[h]);
    }
    int teams = 0;
    size_t smem = 0;
    if (!in_jobs.empty() && planes_shape(K, sizeof(T), P_in, nchunk_in, &teams, &smem)) {
      s = upload_table(in_jobs.data(), sizeof(LineJob) * in_jobs.size(), &dj, st);
      if (s != IMQ_OK) return s;
      s = launch_planes<T>(bm1, static_cast<const T*>(src[0]), nlines, K, ld, P_in, teams, nullptr, nullptr, nullptr,
                           nullptr, 0, nullptr, smem, num_sms, st, static_cast<const LineJob*>(dj),
                           (int)in_jobs.size());
      cudaFreeAsync(dj, st);
      if (s != IMQ_OK || o_pls.empty()) return s;
      return unpack_side_batch<T>(o_pls.data(), (int)o_pls.size(), o_src.data(), o_dst.data(), side, num_sms, st);
    }
  }
  {
    int nw = 0;
    size_t smem = 0;
    if (line_is_row && bm1 >= 1 && bm1 <= 7 && staged_shape(K, sizeof(T), nchunk, &nw, &smem)) {
      s = upload_table(jobs.data(), sizeof(LineJob) * (size_t)n, &dj, st);
      if (s != IMQ_OK) return s;
      s = launch_staged<T>(bm1, static_cast<const T*>(src[0]), nlines, K, ld, nw, 0, nullptr, nullptr, nullptr,
                           nullptr, nullptr, nullptr, 0, nullptr, nullptr, nullptr, 0,
                           side == 0 ? IMQ_A_GROUP : IMQ_B_GROUP,
                           smem, num_sms, st, static_cast<const LineJob*>(dj), n);
      cudaFreeAsync(dj, st);
      return s;
    }
  }
  if (line_is_row) {
    const int64_t Kp = (K + 15) / 16 * 16;
    const int64_t per_warp = (int64_t)P * Kp;
    int nw = (int)((96 * 1024) / per_warp);
    if (nw > 8) nw = 8;
    if (nw >= 1) {
      const int meta_smem = nchunk <= kMetaMaxChunks ? 1 : 0;
      const size_t smem = (size_t)nw * per_warp + (meta_smem ? (size_t)nchunk * 5 : 0);
      const int per_sm = (int)((200 * 1024) / (smem + 1024)) < 1 ? 1 : (int)((200 * 1024) / (smem + 1024));
      const int64_t ctas = (nlines + nw - 1) / nw;
      int64_t grid = ((int64_t)num_sms * (per_sm > 8 ? 8 : per_sm) + n - 1) / n;
      if (grid > ctas) grid = ctas;
      s = upload_table(jobs.data(), sizeof(LineJob) * (size_t)n, &dj, st);
      if (s != IMQ_OK) return s;
      IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_unpack_lines<T>), smem));
      k_unpack_lines<T><<<dim3((unsigned)grid, (unsigned)n), 256, smem, st>>>(
          static_cast<const T*>(src[0]), nlines, K, ld, P, nw, 0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
          0, bm1,
          meta_smem, nullptr, nullptr, nullptr, 0, side == 0 ? IMQ_A_GROUP : IMQ_B_GROUP,
          static_cast<const LineJob*>(dj));
      s = cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
      cudaFreeAsync(dj, st);
      return s;
    }
  }
  // anything else: problem by problem
  for (int h = 0; h < n; ++h) {
    const imq_plan_t* pl = pls[h];
    const LineJob& j = jobs[h];
    ZeroJob zj;
    if (j.outer) zj = ZeroJob{j.grpL, j.grpN, j.ngrp, side == 0 ? IMQ_A_GROUP : IMQ_B_GROUP};
    bool zeroed = false;
    s = unpack_one<T>(static_cast<const T*>(j.X), nlines, K, ld, line_is_row, j.outer, P, j.lvl, j.pos, pl->tK,
                      pl->pinv, pl->tJ, j.lk, pl->blk16, j.K_unp, bm1, j.out, num_sms, st, zj, &zeroed);
    if (s != IMQ_OK) return s;
    if (j.outer && j.ngrp > 0 && !zeroed && j.K_unp > 0)
      k_zero_unused<<<(unsigned)(j.ngrp < 4096 ? j.ngrp : 4096), 256, 0, st>>>(j.grpL, j.grpN, j.ngrp, zj.G, j.K_unp,
                                                                               j.out);
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

namespace imq {
imq_status launch_unpack_batch(const imq_plan_t* const* pls, int n, const void* const* A, const void* const* B,
                               int8_t* const* Au, int8_t* const* Bu, cudaStream_t st) {
  if (n <= 0) return IMQ_OK;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (pls[0]->it == IMQ_I16) {
    s = unpack_side_batch<int16_t>(pls, n, A, Au, 0, ds->num_sms, st);
    if (s == IMQ_OK) s = unpack_side_batch<int16_t>(pls, n, B, Bu, 1, ds->num_sms, st);
  } else {
    s = unpack_side_batch<int32_t>(pls, n, A, Au, 0, ds->num_sms, st);
    if (s == IMQ_OK) s = unpack_side_batch<int32_t>(pls, n, B, Bu, 1, ds->num_sms, st);
  }
  return s;
}
}  // namespace imq
