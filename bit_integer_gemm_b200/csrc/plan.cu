// plan.cu -- the unpack plan: line levels, outlier counts, per-matrix direction and layout maps.
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Approach": rows or columns holding out-of-bound entries are unpacked, the choice made per
// matrix from outlier counts; measured-effects table: Mix against fixed row/col strategies, compared by
// unpack ratio.  The rules (levels, expansion factors, Mix tie-breaks, ratio, layout) are documented in
// include/imq.h.
//
// Device work, in stream order:
//   k_line_max     max |v| of every logical line, unless the caller passes the quantiser's side outputs
//   k_hyb_*        (hybrid strategy only) the carried level of every line, decided on the device
//   k_levels       int8 level of every line plus a summary: level sums, lines with level > 1, level
//                  histograms, the joint histogram of (level of A column t, level of B row t), and the
//                  exact 128-bit bound sum_t max|A[:,t]| * max|B[t,:]|
//   -- the summary (a few KB) is read back; the host fixes directions, groups and sizes --
//   k_plan_order   (plans that use a staging order) one CTA per (A column, B row) level class: the
//                  class's inner indices at their staging positions
//   k_plan_maps    one launch: one CTA per exponent group of the inner dimension (each of its (lA, lB)
//                  segments as ranges of the staging order, padding, 16-position blocks) and one CTA per
//                  OUTER level class (stable compaction of the lines of that level into groups)
#include <math.h>
#include <stddef.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

constexpr int kLv = 33;  // levels 1..32

struct Summary {
  unsigned long long sum[4];
  unsigned long long oor[4];
  unsigned int lmax[4];
  unsigned int hist[4][kLv];
  unsigned int joint[kLv][kLv];
  unsigned long long bound_lo, bound_hi;  // sums of the bound's products' low / high 32-bit halves
  int32_t status;  // copy of the device status word taken in stream order
  uint32_t done;   // blocks of k_levels that have added their part
};

// The summary as the host receives it: pinned host memory that k_levels' last block writes directly (a
// mapped pointer), then `seq`, which the host waits for.  No copy is enqueued and the stream is not
// synchronised: the host sees the summary as soon as it exists.
struct HostSummary {
  Summary s;
  uint32_t seq;
};

// Copies a summary to the mapped host copy with the threads of one block: everything but the rows of
// the joint histogram above max(1, largest A column level), which are zero and which the host never
// reads, so that few words cross to host memory.
__device__ void summary_to_host(const Summary* src, Summary* dst, unsigned lmax_a_col) {
  const unsigned rows = (lmax_a_col > 1 ? lmax_a_col : 1) + 1;
  const int head = (int)((offsetof(Summary, joint) + sizeof(unsigned int) * kLv * rows) / 4);
  const int tail0 = (int)(offsetof(Summary, bound_lo) / 4), n = (int)(sizeof(Summary) / 4);
  const volatile uint32_t* s = reinterpret_cast<const volatile uint32_t*>(src);
  uint32_t* d = reinterpret_cast<uint32_t*>(dst);
  for (int i = threadIdx.x; i < head; i += blockDim.x) d[i] = s[i];
  for (int i = tail0 + threadIdx.x; i < n; i += blockDim.x) d[i] = s[i];
}

// ------------------------------------------------------------------------------------------------
// line maxima of a stored integer matrix
// ------------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_line_max(const T* __restrict__ X, int64_t rows, int64_t cols,
                                                  int64_t ld, int32_t* __restrict__ rowmax,
                                                  int32_t* __restrict__ colmax, int smem_cols) {
  extern __shared__ uint32_t cmax[];
  __shared__ uint32_t red[8];
  const int tid = threadIdx.x;
  if (smem_cols)
    for (int64_t c = tid; c < cols; c += 256) cmax[c] = 0;
  __syncthreads();
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    uint32_t m = 0;
    for (int64_t c = tid; c < cols; c += 256) {
      const int64_t v = X[r * ld + c];
      const uint32_t a = (uint32_t)(v < 0 ? -v : v);
      m = max(m, a);
      if (colmax) {
        if (smem_cols) cmax[c] = max(cmax[c], a);
        else if (a) atomicMax(colmax + c, (int32_t)a);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0 && rowmax) {
      uint32_t r2 = 0;
      for (int w = 0; w < 8; ++w) r2 = max(r2, red[w]);
      rowmax[r] = (int32_t)r2;
    }
    __syncthreads();
  }
  if (colmax && smem_cols)
    for (int64_t c = tid; c < cols; c += 256)
      if (cmax[c]) atomicMax(colmax + c, (int32_t)cmax[c]);
}

// The line maxima of the matrices of a batch of plans in one launch (blockIdx.y = matrix): a block per
// stored row at a time, 16-byte loads where the matrix allows; column maxima through shared memory, then
// atomicMax into colmax, which k_zero_batch has cleared.  Rows are written whole (0 for empty rows).
struct LineMaxJob {
  const void* X;
  int64_t rows, cols, ld;
  int32_t* rowmax;
  int32_t* colmax;
};
template <typename T>
__global__ void __launch_bounds__(256) k_line_max_batch(const LineMaxJob* __restrict__ jobs) {
  extern __shared__ uint32_t cmax_s[];
  __shared__ uint32_t red[8];
  const LineMaxJob J = jobs[blockIdx.y];
  const T* X = static_cast<const T*>(J.X);
  const int tid = threadIdx.x;
  constexpr int V = 16 / (int)sizeof(T);
  const bool vec = J.cols % V == 0 && J.ld % V == 0 && (reinterpret_cast<uintptr_t>(X) & 15) == 0;
  for (int64_t c = tid; c < J.cols; c += 256) cmax_s[c] = 0;
  __syncthreads();
  for (int64_t r = blockIdx.x; r < J.rows; r += gridDim.x) {
    uint32_t m = 0;
    if (vec) {
      const uint4* xr = reinterpret_cast<const uint4*>(X + r * J.ld);
      for (int64_t q = tid; q < J.cols / V; q += 256) {
        const uint4 w = __ldcs(xr + q);
        const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
        for (int k = 0; k < V; ++k) {
          const int64_t v = e[k];
          const uint32_t a = (uint32_t)(v < 0 ? -v : v);
          m = max(m, a);
          cmax_s[q * V + k] = max(cmax_s[q * V + k], a);
        }
      }
    } else {
      for (int64_t c = tid; c < J.cols; c += 256) {
        const int64_t v = X[r * J.ld + c];
        const uint32_t a = (uint32_t)(v < 0 ? -v : v);
        m = max(m, a);
        cmax_s[c] = max(cmax_s[c], a);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
      uint32_t r2 = 0;
      for (int w = 0; w < 8; ++w) r2 = max(r2, red[w]);
      J.rowmax[r] = (int32_t)r2;
    }
    __syncthreads();
  }
  for (int64_t c = tid; c < J.cols; c += 256)
    if (cmax_s[c]) atomicMax(J.colmax + c, (int32_t)cmax_s[c]);
}

// Clears the byte ranges of a batch (blockIdx.y = range; every range 16-byte aligned, a 4-byte multiple).
struct ZeroSpan {
  void* p;
  int64_t bytes;
};
__global__ void __launch_bounds__(256) k_zero_batch(const ZeroSpan* __restrict__ spans) {
  const ZeroSpan z = spans[blockIdx.y];
  uint4* q = static_cast<uint4*>(z.p);
  const int64_t n16 = z.bytes / 16;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
    q[i] = make_uint4(0u, 0u, 0u, 0u);
  uint32_t* w = static_cast<uint32_t*>(z.p);
  for (int64_t i = n16 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < z.bytes / 4;
       i += (int64_t)gridDim.x * blockDim.x)
    w[i] = 0u;
}

// ------------------------------------------------------------------------------------------------
// levels and summary.  Vectors: 0 = A rows (M), 1 = A cols (K), 2 = B rows (K), 3 = B cols (N).
// ------------------------------------------------------------------------------------------------
struct LevelArgs {
  const int32_t* mx[4];
  const int8_t* lvin[4];  // when not null, the levels themselves (the hybrid's carried levels)
  int8_t* lv[4];
  int64_t n[4];
  int32_t bm1;
  int32_t* keep_a_col;     // when set, A's column maxima mx[1] are copied here (kept in the plan)
  Summary* sum;
  const int32_t* status;  // the device status word, copied into the summary by block 0
  HostSummary* hsum;      // device address of the mapped host copy
  uint32_t seq;           // written to hsum->seq once hsum->s is complete
  uint32_t nblk;          // blocks of this plan's level kernel (the last one publishes the summary)
};

__device__ __forceinline__ void levels_body(const LevelArgs& a) {
  __shared__ unsigned int hist[4][kLv];
  __shared__ unsigned int joint[kLv][kLv];
  __shared__ unsigned long long ssum[4], soor[4];
  __shared__ unsigned int slmax[4];
  const int tid = threadIdx.x;
  // every kernel before this one in stream order has finished: its errors are in the status word
  if (blockIdx.x == 0 && tid == 0) a.sum->status = *a.status;
  for (int i = tid; i < 4 * kLv; i += 256) (&hist[0][0])[i] = 0;
  for (int i = tid; i < kLv * kLv; i += 256) (&joint[0][0])[i] = 0;
  if (tid < 4) {
    ssum[tid] = 0;
    soor[tid] = 0;
    slmax[tid] = 0;
  }
  __syncthreads();
  const int64_t stride = (int64_t)a.nblk * blockDim.x;
  unsigned long long bsum[4] = {0, 0, 0, 0}, boor[4] = {0, 0, 0, 0};
  unsigned int blmax[4] = {0, 0, 0, 0};
  // the bound sum_t max|A[:,t]| * max|B[t,:]| as two 64-bit sums, of the products' low 32-bit halves and
  // of their high halves (products < 2^62 and at most 2^31 lines: neither sum can overflow, so blocks add
  // them without carries and the host joins them as hi * 2^32 + lo)
  unsigned long long blo = 0, bhi = 0;
  const int64_t nmax = max(max(a.n[0], a.n[1]), max(a.n[2], a.n[3]));
  // whole warps iterate together so the aggregated counters see every lane; the entries of all four
  // vectors are loaded before any is used, so that their loads are in flight together
  for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x; i0 < nmax; i0 += stride) {
    const int64_t i = i0 + tid;
    bool in[4];
    uint32_t m[4];
    int lvi[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      in[v] = i < a.n[v];
      m[v] = in[v] ? (uint32_t)a.mx[v][i] : 0u;
      lvi[v] = (in[v] && a.lvin[v]) ? (int)a.lvin[v][i] : -1;
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      int L = 1;
      if (in[v]) {
        if (v == 1 && a.keep_a_col) a.keep_a_col[i] = (int32_t)m[v];
        L = lvi[v] >= 0 ? lvi[v] : level_of(m[v], a.bm1);
        a.lv[v][i] = (int8_t)L;
        bsum[v] += (unsigned)L;
        boor[v] += (L > 1);
        blmax[v] = max(blmax[v], (unsigned)L);
        if (v == 1) {
          const unsigned long long prod = (unsigned long long)m[1] * (unsigned long long)m[2];
          blo += prod & 0xFFFFFFFFull;
          bhi += prod >> 32;
        }
      }
      warp_count(&hist[v][0], (uint32_t)L, in[v]);
      if (v == 1) {
        const int Lb = !in[1] ? 1 : (lvi[2] >= 0 ? lvi[2] : level_of(m[2], a.bm1));
        warp_count(&joint[0][0], (uint32_t)(L * kLv + Lb), in[1]);
      }
    }
  }
  // warp reductions first, then one shared atomic per warp, then one global atomic per block
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    for (int v = 0; v < 4; ++v) {
      bsum[v] += __shfl_xor_sync(0xffffffffu, bsum[v], o);
      boor[v] += __shfl_xor_sync(0xffffffffu, boor[v], o);
      blmax[v] = max(blmax[v], __shfl_xor_sync(0xffffffffu, blmax[v], o));
    }
    blo += __shfl_xor_sync(0xffffffffu, blo, o);
    bhi += __shfl_xor_sync(0xffffffffu, bhi, o);
  }
  __shared__ unsigned long long sblo, sbhi;
  if (tid == 0) {
    sblo = 0;
    sbhi = 0;
  }
  __syncthreads();
  if ((tid & 31) == 0) {
    for (int v = 0; v < 4; ++v) {
      if (bsum[v]) atomicAdd(&ssum[v], bsum[v]);
      if (boor[v]) atomicAdd(&soor[v], boor[v]);
      if (blmax[v]) atomicMax(&slmax[v], blmax[v]);
    }
    if (blo) atomicAdd(&sblo, blo);
    if (bhi) atomicAdd(&sbhi, bhi);
  }
  __syncthreads();
  if (tid == 0) {
    if (sblo) atomicAdd(&a.sum->bound_lo, sblo);
    if (sbhi) atomicAdd(&a.sum->bound_hi, sbhi);
  }
  __syncthreads();
  if (tid < 4) {
    if (ssum[tid]) atomicAdd(&a.sum->sum[tid], ssum[tid]);
    if (soor[tid]) atomicAdd(&a.sum->oor[tid], soor[tid]);
    if (slmax[tid]) atomicMax(&a.sum->lmax[tid], slmax[tid]);
  }
  for (int i = tid; i < 4 * kLv; i += 256)
    if ((&hist[0][0])[i]) atomicAdd(&a.sum->hist[0][0] + i, (&hist[0][0])[i]);
  for (int i = tid; i < kLv * kLv; i += 256)
    if ((&joint[0][0])[i]) atomicAdd(&a.sum->joint[0][0] + i, (&joint[0][0])[i]);
  // the last block to finish copies the completed summary to the host, then publishes `seq`
  __shared__ bool last;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&a.sum->done, 1u) == a.nblk - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  summary_to_host(a.sum, &a.hsum->s, *reinterpret_cast<volatile unsigned int*>(&a.sum->lmax[1]));
  __threadfence_system();
  __syncthreads();
  // the fence above orders the summary before `seq`; nothing after it needs to wait for the write
  if (tid == 0) *reinterpret_cast<volatile uint32_t*>(&a.hsum->seq) = a.seq;
}

__global__ void __launch_bounds__(256) k_levels(LevelArgs a) { levels_body(a); }

// The level kernels of a batch of plans in one launch: blockIdx.y = plan, its blocks blockIdx.x <
// nblk[plan] (the others return at once).
__global__ void __launch_bounds__(256) k_levels_batch(const LevelArgs* __restrict__ args, const int* __restrict__ nblk) {
  if ((int)blockIdx.x >= nblk[blockIdx.y]) return;
  const LevelArgs a = args[blockIdx.y];
  levels_body(a);
}

// ------------------------------------------------------------------------------------------------
// hybrid choice ("unpack both"): per matrix, the outer lines holding at least tau out-of-range entries
// are unpacked OUTER, the others INNER, tau of least unpacked size (smallest on a tie).
//   k_hyb_rows    outer lines stored as rows: a CTA per row counts its out-of-range entries, cnt[o], and
//                 takes the count into mex[t][l] = least cnt[o] over the lines o whose entry t has level l
//   k_hyb_count   outer lines stored as columns: cnt[o] ...
//   k_hyb_minc    ... then mex, two passes
//   k_hyb_hist    suffix minima over l (then mex[t][l] = least count of a line reaching level >= l at t),
//                 H[c] = #(t, l >= 2) with mex[t][l] = c, G[c] = sum of (level - 1) over lines of count c
//   k_hyb_choose  one CTA per matrix: with S(tau) = {o : cnt[o] >= tau},
//                 size(tau) = (n_out + sum_{c >= tau} G[c]) * (n_in + sum_{c < tau} H[c]),
//                 since the inner level of t over the lines outside S(tau) is 1 + #{l >= 2 : mex[t][l] < tau}
//   k_hyb_apply   the carried levels: lo[o] = level of o if cnt[o] >= tau else 1;
//                 li[t] = largest l with mex[t][l] < tau, else 1
// ------------------------------------------------------------------------------------------------
constexpr int kHybL = 33;                 // levels 0..32 (level_of of a 32-bit magnitude is at most 32)
constexpr int32_t kHybInf = 0x7F7F7F7F;   // mex before any entry (a memset byte pattern above any count)

struct HybMat {
  const void* X;        // the stored matrix, int16 or int32
  int64_t rows, cols, ld;
  int outer_is_row;     // outer lines are the stored rows (else the stored columns)
  int64_t n_out, n_in;
  const int32_t* omax;  // max |v| of every outer line
  int32_t* cnt;         // [n_out]
  int32_t* mex;         // [kHybL][n_in], level-major so that a warp's inner indices are adjacent
  unsigned long long* H;  // [n_in + 2]
  unsigned long long* G;  // [n_in + 2]
  int32_t* tau;         // [1]
  int32_t* cmax;        // [1] largest cnt[o] (zeroed with the counts)
  int8_t* lo;           // [n_out] carried levels of the outer lines
  int8_t* li;           // [n_in] carried levels of the inner indices
};

struct HybArgs {
  HybMat m[2];
  int32_t bm1;
};

// The matrices whose outer lines are stored columns: tiles of 8 stored rows x (256 kC) stored columns,
// kC consecutive columns per thread (one 16-byte load per row when the rows are 16-byte aligned, else
// one column per thread; blockIdx.z = matrix).  k_hyb_count adds each column's out-of-range entries of
// the tile into cnt; k_hyb_minc then takes the column's count into mex for each of them.
template <typename T, bool kMin>
__device__ __forceinline__ void hyb_cols_tile(const HybMat& m, uint32_t lim, int bm1) {
  constexpr int kV = 16 / sizeof(T);
  const T* X = static_cast<const T*>(m.X);
  const bool vec = (m.cols % kV == 0) && (m.ld % kV == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  const int kC = vec ? kV : 1;
  const int64_t c0 = ((int64_t)blockIdx.x * 256 + threadIdx.x) * kC;
  if (c0 >= m.cols) return;
  int32_t cnt[kV];
#pragma unroll
  for (int k = 0; k < kV; ++k) cnt[k] = 0;
  if (kMin) {
#pragma unroll
    for (int k = 0; k < kV; ++k) cnt[k] = k < kC ? m.cnt[c0 + k] : 0;
  }
  for (int64_t r0 = (int64_t)blockIdx.y * 8; r0 < m.rows; r0 += (int64_t)gridDim.y * 8) {
    const int64_t r1 = r0 + 8 < m.rows ? r0 + 8 : m.rows;
    int32_t add[kV];
#pragma unroll
    for (int k = 0; k < kV; ++k) add[k] = 0;
#pragma unroll 8
    for (int64_t r = r0; r < r1; ++r) {
      T v[kV];
      if (vec) {
        const uint4 w = *reinterpret_cast<const uint4*>(X + r * m.ld + c0);
        const T* p = reinterpret_cast<const T*>(&w);
#pragma unroll
        for (int k = 0; k < kV; ++k) v[k] = p[k];
      } else {
        v[0] = X[r * m.ld + c0];
#pragma unroll
        for (int k = 1; k < kV; ++k) v[k] = 0;
      }
#pragma unroll
      for (int k = 0; k < kV; ++k) {
        const int64_t x = v[k];
        const uint32_t mag = (uint32_t)(x < 0 ? -x : x);
        if (mag > lim) {
          if (kMin)
            atomicMin(m.mex + (int64_t)level_of(mag, bm1) * m.n_in + r, cnt[k]);
          else
            add[k] += 1;
        }
      }
    }
    if (!kMin) {
#pragma unroll
      for (int k = 0; k < kV; ++k)
        if (add[k]) atomicAdd(m.cnt + c0 + k, add[k]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_hyb_count(HybArgs a) {
  const HybMat& m = a.m[blockIdx.z];
  if (m.outer_is_row) return;
  hyb_cols_tile<T, false>(m, (1u << a.bm1) - 1u, a.bm1);
}

template <typename T>
__global__ void __launch_bounds__(256) k_hyb_minc(HybArgs a) {
  const HybMat& m = a.m[blockIdx.z];
  if (m.outer_is_row) return;
  hyb_cols_tile<T, true>(m, (1u << a.bm1) - 1u, a.bm1);
}

// Count and least counts in one pass when the outer lines are the stored rows: one warp per row counts
// the row's out-of-range entries (16-byte loads when the rows are 16-byte aligned), then sweeps the
// row again (now in L1 / L2) to take the count into mex for each of them.  blockIdx.y = matrix; a
// matrix whose outer lines are stored columns is skipped here (k_hyb_count / k_hyb_minc serve it).
// Out-of-range halves of a word of two int16 entries: bit 15 / bit 31 set where |entry| > lim (lim <=
// 127).  |entry| per half without a carry between halves (as in the unpack kernel), then lim is
// subtracted by adding 0x7FFF - lim: a half reaches 0x8000 exactly when it exceeds lim, and no half
// carries out (|entry| <= 0x8000).
__device__ __forceinline__ uint32_t oor_halves(uint32_t w, uint32_t lim) {
  const uint32_t sgn = (w >> 15) & 0x00010001u;
  const uint32_t mag = (w ^ (sgn * 0xFFFFu)) + sgn;
  return (mag + (0x7FFFu - lim) * 0x00010001u) & 0x80008000u;
}

// One stored row (an outer line) per CTA of kRowThreads threads: the row's out-of-range entries are
// counted (16-byte loads, two int16 entries per word at a time) and summed over the CTA, then the row is
// swept again (now in L1 / L2) to take the count into mex for each of them.
constexpr int kRowThreads = 128;

template <typename T>
__device__ __forceinline__ void hyb_row(const HybMat& m, int64_t r, uint32_t lim, int bm1, int* red) {
  const T* xr = static_cast<const T*>(m.X) + r * m.ld;
  constexpr int kV = 16 / sizeof(T);  // entries per 16-byte load
  constexpr int kU = 4;               // 16-byte loads of a thread in flight
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool vec = (m.cols % kV == 0) && (m.ld % kV == 0) && ((reinterpret_cast<uintptr_t>(m.X) & 15) == 0);
  int c = 0;
  if (vec) {
    for (int64_t t0 = (int64_t)tid * kV; t0 < m.cols; t0 += (int64_t)kRowThreads * kV * kU) {
      uint4 w[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t t = t0 + (int64_t)u * kRowThreads * kV;
        w[u] = t < m.cols ? *reinterpret_cast<const uint4*>(xr + t) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if constexpr (sizeof(T) == 2) {
          c += __popc(oor_halves(w[u].x, lim) | (oor_halves(w[u].y, lim) >> 1)) +
               __popc(oor_halves(w[u].z, lim) | (oor_halves(w[u].w, lim) >> 1));
        } else {
          const int32_t v[4] = {(int32_t)w[u].x, (int32_t)w[u].y, (int32_t)w[u].z, (int32_t)w[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) c += (uint32_t)(v[k] < 0 ? -(int64_t)v[k] : v[k]) > lim;
        }
      }
    }
  } else {
    for (int64_t t = tid; t < m.cols; t += kRowThreads) {
      const int64_t x = xr[t];
      c += (uint64_t)(x < 0 ? -x : x) > lim;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) red[warp] = c;
  __syncthreads();
  c = 0;
#pragma unroll
  for (int w = 0; w < kRowThreads / 32; ++w) c += red[w];
  __syncthreads();  // red is reused by the next row
  if (tid == 0) m.cnt[r] = c;
  if (c == 0) return;
  if (vec && sizeof(T) == 2) {
    for (int64_t t0 = (int64_t)tid * kV; t0 < m.cols; t0 += (int64_t)kRowThreads * kV * kU) {
      uint4 w[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t t = t0 + (int64_t)u * kRowThreads * kV;
        w[u] = t < m.cols ? *reinterpret_cast<const uint4*>(xr + t) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        const int64_t t = t0 + (int64_t)u * kRowThreads * kV;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t hit = oor_halves(ww[q], lim);
          if (hit == 0) continue;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (!(hit & (0x8000u << (16 * hf)))) continue;
            const int32_t x = (int16_t)(ww[q] >> (16 * hf));
            const uint32_t mag = (uint32_t)(x < 0 ? -x : x);
            atomicMin(m.mex + (int64_t)level_of(mag, bm1) * m.n_in + t + 2 * q + hf, c);
          }
        }
      }
    }
  } else {
    for (int64_t t = tid; t < m.cols; t += kRowThreads) {
      const int64_t x = xr[t];
      const uint32_t mag = (uint32_t)(x < 0 ? -x : x);
      if (mag > lim) atomicMin(m.mex + (int64_t)level_of(mag, bm1) * m.n_in + t, c);
    }
  }
}

// The matrices whose outer lines are stored rows: CTAs run over the rows of matrix 0 then matrix 1 (a
// matrix whose outer lines are stored columns has none here; the column kernels serve it).
template <typename T>
__global__ void __launch_bounds__(kRowThreads) k_hyb_rows(HybArgs a) {
  __shared__ int red[kRowThreads / 32];
  const uint32_t lim = (1u << a.bm1) - 1u;
  const int64_t n0 = a.m[0].outer_is_row ? a.m[0].rows : 0;
  const int64_t n1 = a.m[1].outer_is_row ? a.m[1].rows : 0;
  for (int64_t w = blockIdx.x; w < n0 + n1; w += gridDim.x) {
    if (w < n0)
      hyb_row<T>(a.m[0], w, lim, a.bm1, red);
    else
      hyb_row<T>(a.m[1], w - n0, lim, a.bm1, red);
  }
}

// blockIdx.y = matrix; grid-stride over the inner indices, then over the outer lines.  The levels 2..32
// of one inner index are loaded together (independent loads), turned into suffix minima in registers and
// written back (level-major: the loads of a warp are coalesced).
__global__ void __launch_bounds__(256) k_hyb_hist(HybArgs a) {
  const HybMat& m = a.m[blockIdx.y];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < m.n_in; t += stride) {
    int32_t v[kHybL];
#pragma unroll
    for (int l = 2; l < kHybL; ++l) v[l] = m.mex[(int64_t)l * m.n_in + t];
    int32_t run = kHybInf;
#pragma unroll
    for (int l = kHybL - 1; l >= 2; --l) {
      run = min(run, v[l]);
      v[l] = run;
    }
#pragma unroll
    for (int l = 2; l < kHybL; ++l) {
      m.mex[(int64_t)l * m.n_in + t] = v[l];
      if (v[l] != kHybInf) atomicAdd(m.H + v[l], 1ull);
    }
  }
  int32_t cm = 0;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < m.n_out; o += stride) {
    const int32_t c = m.cnt[o];
    if (c > 0) {
      atomicAdd(m.G + c, (unsigned long long)(level_of((uint32_t)m.omax[o], a.bm1) - 1));
      cm = max(cm, c);
    }
  }
  // the largest count, one atomic per warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, o));
  if ((threadIdx.x & 31) == 0 && cm > 0) atomicMax(m.cmax, cm);
}

// Inclusive block scan (1024 threads) of v; *total gets the block sum.
__device__ __forceinline__ unsigned long long block_scan_ull(unsigned long long v, unsigned long long* warp_tot,
                                                             unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    warp_tot[lane] = w;
    if (lane == 31) *total = w;
  }
  __syncthreads();
  const unsigned long long r = v + (warp > 0 ? warp_tot[warp - 1] : 0ull);
  __syncthreads();
  return r;
}

// One CTA of 1024 threads per matrix (blockIdx.x): tau from 1 to the largest count + 1, a contiguous
// run of thresholds per thread.  One block scan of the per-thread sums of H and G gives each thread the
// sums below its first threshold; the thread then walks its run.
__global__ void __launch_bounds__(1024) k_hyb_choose(HybArgs a) {
  const HybMat& m = a.m[blockIdx.x];
  __shared__ unsigned long long warp_tot[32];
  __shared__ unsigned long long tot;
  __shared__ unsigned long long best_hi[32], best_lo[32];
  __shared__ int64_t best_tau[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // thresholds 1 .. cmax + 1: above the largest count every threshold leaves S empty, and H and G are 0
  // beyond it (H and G are indexed 0 .. n_in + 1, cmax <= n_in)
  const int64_t nt = (int64_t)*m.cmax + 1;
  const int64_t per = (nt + blockDim.x - 1) / blockDim.x;
  const int64_t tau0 = 1 + (int64_t)threadIdx.x * per;
  const int64_t tau1 = tau0 + per - 1 < nt ? tau0 + per - 1 : nt;  // this thread's run tau0 .. tau1
  // element c = tau - 1 joins the sums below tau + 1
  unsigned long long hs = 0, gs = 0;
  for (int64_t tau = tau0; tau <= tau1; ++tau) {
    hs += m.H[tau - 1];
    gs += m.G[tau - 1];
  }
  const unsigned long long hin = block_scan_ull(hs, warp_tot, &tot);
  const unsigned long long gin = block_scan_ull(gs, warp_tot, &tot);
  const unsigned long long gtot = tot;
  unsigned long long hbelow = hin - hs, gbelow = gin - gs;  // sums over c < tau0 - 1
  unsigned __int128 best = ~(unsigned __int128)0;
  int64_t btau = 1;
  for (int64_t tau = tau0; tau <= tau1; ++tau) {
    hbelow += m.H[tau - 1];
    gbelow += m.G[tau - 1];
    const unsigned __int128 mo = (unsigned __int128)m.n_out + (gtot - gbelow);
    const unsigned __int128 ki = (unsigned __int128)m.n_in + hbelow;
    const unsigned __int128 cost = mo * ki;
    if (cost < best) {  // thresholds ascend: the first strict minimum is the smallest tau
      best = cost;
      btau = tau;
    }
  }
  // (cost, tau) lexicographic minimum over the block
  unsigned long long bh = (unsigned long long)(best >> 64), bl = (unsigned long long)best;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long oh = __shfl_xor_sync(0xffffffffu, bh, o), ol = __shfl_xor_sync(0xffffffffu, bl, o);
    const int64_t ot = __shfl_xor_sync(0xffffffffu, btau, o);
    if (oh < bh || (oh == bh && (ol < bl || (ol == bl && ot < btau)))) {
      bh = oh;
      bl = ol;
      btau = ot;
    }
  }
  if (lane == 0) {
    best_hi[warp] = bh;
    best_lo[warp] = bl;
    best_tau[warp] = btau;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (best_hi[w] < bh || (best_hi[w] == bh && (best_lo[w] < bl || (best_lo[w] == bl && best_tau[w] < btau)))) {
        bh = best_hi[w];
        bl = best_lo[w];
        btau = best_tau[w];
      }
    *m.tau = (int32_t)btau;
  }
}

// blockIdx.y = matrix.
__global__ void __launch_bounds__(256) k_hyb_apply(HybArgs a) {
  const HybMat& m = a.m[blockIdx.y];
  const int32_t tau = *m.tau;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < m.n_out; o += stride)
    m.lo[o] = (int8_t)(m.cnt[o] >= tau ? level_of((uint32_t)m.omax[o], a.bm1) : 1);
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < m.n_in; t += stride) {
    // suffix minima are non-decreasing in l: the levels below tau are 2 .. L
    int l = 1;
#pragma unroll
    for (int k = 2; k < kHybL; ++k) l += m.mex[(int64_t)k * m.n_in + t] < tau;
    m.li[t] = (int8_t)l;
  }
}

// ------------------------------------------------------------------------------------------------
// maps
// ------------------------------------------------------------------------------------------------
// Block-wide exclusive scan of a 0/1 predicate (1024 threads); returns the rank and the block total.
__device__ __forceinline__ int block_rank(int pred, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned ball = __ballot_sync(0xffffffffu, pred);
  const int in_warp = __popc(ball & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(ball);
  __syncthreads();
  if (warp == 0) {
    const int v = warp_tot[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    warp_tot[lane] = incl - v;
    if (lane == 31) *total = incl;
  }
  __syncthreads();
  const int r = warp_tot[warp] + in_warp;
  return r;
}

struct InnerSeg {
  int32_t la, lb;
  int64_t off;
};

// One exponent group of the unpacked inner dimension: positions [k0, k0 + kpad), filled by segments
// seg0 .. seg0 + nseg - 1 in order and padded (source -1) up to kpad, a multiple of IMQ_INNER_PAD.
struct InnerGroup {
  int64_t k0, kpad;
  int32_t seg0, nseg;
};

// The staging order of the inner indices.  Index t belongs to class (ea, eb): ea = level of A column t
// when A is unpacked INNER (else 1), eb = level of B row t when B is (else 1).  The staging order lists
// the classes in descending (ea, eb), each class's indices ascending, so that the indices a segment
// (lA, lB) holds -- every class with ea > lA and eb > lB -- are, for each ea, one contiguous range of
// staging positions.  E[ea * ew + s] (ew = maxlb + 1) is the first staging position past the classes
// (ea, eb) with eb > s: class (ea, eb) occupies [E[ea*ew + eb], E[ea*ew + eb - 1]).  perm[j] is the index at
// staging position j and pinv its inverse; both are null when the order is the identity (one class, or
// a plan whose segments keep most 16-position blocks runs in index order).
struct StageOrder {
  const int32_t* E;
  int ew;
  int maxla, maxlb;
  int32_t* perm;
  int32_t* pinv;
};

// The staging order of one class (one CTA of 1024 threads): its indices, ascending, at its positions.
__device__ void stage_class(int ea, int eb, const StageOrder& so, const int8_t* __restrict__ lva,
                            const int8_t* __restrict__ lvb, int a_inner, int b_inner, int64_t K) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int64_t j0 = so.E[ea * so.ew + eb];
  if (so.E[ea * so.ew + eb - 1] == j0) return;  // empty class
  int64_t rank0 = 0;
  for (int64_t t0 = 0; t0 < K; t0 += 1024) {
    const int64_t t = t0 + threadIdx.x;
    int pred = 0;
    if (t < K) pred = (a_inner ? lva[t] : 1) == ea && (b_inner ? lvb[t] : 1) == eb;
    const int r = block_rank(pred, warp_tot, &total);
    if (pred) {
      const int64_t j = j0 + rank0 + r;
      so.perm[j] = (int32_t)t;
      so.pinv[t] = (int32_t)j;
    }
    __syncthreads();
    rank0 += total;
    __syncthreads();
  }
}

// The inner map of one exponent group (one CTA of 1024 threads): each segment (lA, lB) holds the inner
// indices of the classes ea > lA, eb > lB -- with a staging order, in that order (for each ea, from the
// largest, one range of staging positions), else ascending -- then the padding, then blk16 for the
// group's 16-position blocks: blk16[c] = j0
// when block c holds the indices at staging positions j0..j0+15 with one (lA, lB) pair (j0 % 16 == 0),
// -(j0 + 2) for such a run at any other j0, else -1.  tJ[p] = staging position of position p's index.
__device__ void inner_map_group(const InnerGroup grp, const InnerSeg* __restrict__ segs, const StageOrder& so,
                                const int8_t* __restrict__ lva, const int8_t* __restrict__ lvb, int a_inner,
                                int b_inner, int64_t K, int32_t* tK, int32_t* tJ, int8_t* __restrict__ lAk,
                                int8_t* __restrict__ lBk, int32_t* __restrict__ blk16) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  int64_t base = grp.k0;
  for (int si = 0; si < grp.nseg; ++si) {
    const InnerSeg sg = segs[grp.seg0 + si];
    if (so.perm) {
      // the segment's ranges of the staging order, one per A level ea > lA
      for (int ea = so.maxla; ea > sg.la; --ea) {
        const int64_t jb = so.E[ea * so.ew + so.maxlb], je = so.E[ea * so.ew + sg.lb];
        for (int64_t i = threadIdx.x; i < je - jb; i += blockDim.x) {
          const int64_t j = jb + i, q = base + i;
          tK[q] = so.perm[j];
          tJ[q] = (int32_t)j;
          lAk[q] = (int8_t)sg.la;
          lBk[q] = (int8_t)sg.lb;
        }
        base += je - jb;
      }
    } else {
      // index order: the segment's indices by stream compaction
      for (int64_t t0 = 0; t0 < K; t0 += 1024) {
        const int64_t t = t0 + threadIdx.x;
        int pred = 0;
        if (t < K) pred = ((a_inner ? lva[t] : 1) > sg.la) && ((b_inner ? lvb[t] : 1) > sg.lb);
        const int r = block_rank(pred, warp_tot, &total);
        if (pred) {
          tK[base + r] = (int32_t)t;
          tJ[base + r] = (int32_t)t;
          lAk[base + r] = (int8_t)sg.la;
          lBk[base + r] = (int8_t)sg.lb;
        }
        __syncthreads();
        base += total;
        __syncthreads();
      }
    }
  }
  for (int64_t q = base + threadIdx.x; q < grp.k0 + grp.kpad; q += blockDim.x) {
    tK[q] = -1;
    tJ[q] = -1;
    lAk[q] = 0;
    lBk[q] = 0;
  }
  __syncthreads();  // the block's writes above are visible to all its threads after this
  for (int64_t c = grp.k0 / 16 + threadIdx.x; c < (grp.k0 + grp.kpad) / 16; c += blockDim.x) {
    const int32_t* j = tJ + c * 16;
    const int32_t j0 = j[0];
    bool run = j0 >= 0;
    for (int k = 1; k < 16 && run; ++k)
      run = j[k] == j0 + k && lAk[c * 16 + k] == lAk[c * 16] && lBk[c * 16 + k] == lBk[c * 16];
    // the staged unpackers read an unaligned run with unaligned loads; every other reader treats a
    // negative entry as a gathered block
    blk16[c] = !run ? -1 : ((j0 & 15) == 0 ? j0 : -(j0 + 2));
  }
}

struct OuterClass {
  int32_t L;
  int32_t per;      // source lines per group
  int64_t grp0;     // first group of this class
  int64_t count;    // lines of this level
};

// The OUTER layout of one matrix: classes of lines of equal level, each a run of groups of G unpacked
// lines.  One CTA per class.
struct OuterJob {
  int cls0;  // first class of this matrix in the class table
  int ncls;
  const int8_t* lv;
  int64_t n;
  int G;
  int32_t* pos;
  int32_t* src;
  int32_t* grpL;
  int32_t* grpN;
};

__device__ void outer_map_class(const OuterClass c, const int8_t* __restrict__ lv, int64_t n, int G,
                                int32_t* __restrict__ pos, int32_t* __restrict__ src, int32_t* __restrict__ grpL,
                                int32_t* __restrict__ grpN) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int64_t ngrp = (c.count + c.per - 1) / c.per;
  for (int64_t g = threadIdx.x; g < ngrp; g += blockDim.x) {
    const int32_t ng = (int32_t)(g < ngrp - 1 ? c.per : c.count - (ngrp - 1) * c.per);
    grpL[c.grp0 + g] = c.L;
    grpN[c.grp0 + g] = ng;
    for (int u = ng * c.L; u < G; ++u) src[(c.grp0 + g) * G + u] = -1;  // unused unpacked lines
  }
  int64_t rank0 = 0;
  for (int64_t i0 = 0; i0 < n; i0 += 1024) {
    const int64_t i = i0 + threadIdx.x;
    const int pred = (i < n) && (lv[i] == c.L);
    const int r = block_rank(pred, warp_tot, &total);
    if (pred) {
      const int64_t rank = rank0 + r;
      const int64_t p = (c.grp0 + rank / c.per) * G + (rank % c.per) * c.L;
      pos[i] = (int32_t)p;
      for (int l = 0; l < c.L; ++l) src[p + l] = (int32_t)i;
    }
    __syncthreads();
    rank0 += total;
    __syncthreads();
  }
}

// The segment, class and group tables of a plan.  They travel inside the launch's parameters when the
// segments fit (the usual case: a separate upload would cost a copy and an event on the host); the
// parameter block is read in place (__grid_constant__).
// Tables passed inline in the maps kernel's parameters when they fit (about 1.3 KB, so the launch stays
// within the classic 4 KB parameter space); larger plans upload them to device memory instead.
constexpr int kParamSegs = 24;
constexpr int kParamCls = 24;
constexpr int kParamGrps = 16;
constexpr int kParamE = 100;
struct MapsTables {
  InnerSeg segs[kParamSegs];
  OuterClass cls[kParamCls];
  InnerGroup grps[kParamGrps];
  int32_t E[kParamE];
};

// Stage 2 of a plan.  k_plan_order (only when the staging order is not the identity): one CTA per class
// (ea, eb), blockIdx.x = (maxla - ea) * maxlb + (maxlb - eb).  Then k_plan_maps: blocks [0, ngrp) build the
// inner map of one exponent group each, the next a.ncls blocks one OUTER class of A each, the rest one
// OUTER class of B each.
struct MapsArgs {
  int inline_tables;       // 1: the tables are `t` below, 0: the device copies at grps / segs / cls / E
  const InnerGroup* grps;
  int ngrp;
  const InnerSeg* segs;
  const OuterClass* cls;
  const int32_t* E;
  int ew, maxla, maxlb;
  const int8_t* lva;
  const int8_t* lvb;
  int a_inner, b_inner;
  int64_t K;
  int32_t* perm;
  int32_t* pinv;
  int32_t* tK;
  int32_t* tJ;
  int8_t* lAk;
  int8_t* lBk;
  int32_t* blk16;
  OuterJob a, b;
  MapsTables t;
};
// kernel parameters above 4 KB need CUDA 12.1 or later; the limit there is 32 764 bytes
static_assert(sizeof(MapsArgs) <= 32764, "plan tables exceed the kernel parameter limit");
// a batch's maps launch uploads the arguments of up to 64 plans through one 256 KB staging buffer
static_assert(sizeof(MapsArgs) * 64 <= 256 * 1024, "64 plans' maps arguments exceed a staging buffer");

__device__ __forceinline__ StageOrder stage_order(const MapsArgs& m) {
  return StageOrder{m.inline_tables ? m.t.E : m.E, m.ew, m.maxla, m.maxlb, m.perm, m.pinv};
}

__global__ void __launch_bounds__(1024) k_plan_order(const __grid_constant__ MapsArgs m) {
  const int bx = (int)blockIdx.x;
  const int ea = m.maxla - bx / m.maxlb, eb = m.maxlb - bx % m.maxlb;
  stage_class(ea, eb, stage_order(m), m.lva, m.lvb, m.a_inner, m.b_inner, m.K);
}

__device__ __forceinline__ void maps_body(const MapsArgs& m, int bx);

__global__ void __launch_bounds__(1024) k_plan_maps(const __grid_constant__ MapsArgs m) { maps_body(m, (int)blockIdx.x); }

// The order and maps kernels of a batch of plans in one launch each: blockIdx.y = plan, reading its
// arguments from a device table; blocks past the plan's own count return at once.
__global__ void __launch_bounds__(1024) k_plan_order_batch(const MapsArgs* __restrict__ tab) {
  const MapsArgs& m = tab[blockIdx.y];
  if (!m.perm || (int)blockIdx.x >= m.maxla * m.maxlb) return;
  const int bx = (int)blockIdx.x;
  const int ea = m.maxla - bx / m.maxlb, eb = m.maxlb - bx % m.maxlb;
  stage_class(ea, eb, stage_order(m), m.lva, m.lvb, m.a_inner, m.b_inner, m.K);
}
__global__ void __launch_bounds__(1024) k_plan_maps_batch(const MapsArgs* __restrict__ tab) {
  const MapsArgs& m = tab[blockIdx.y];
  if ((int)blockIdx.x >= m.ngrp + m.a.ncls + m.b.ncls) return;
  maps_body(m, (int)blockIdx.x);
}

__device__ __forceinline__ void maps_body(const MapsArgs& m, int bx) {
  const InnerSeg* segs = m.inline_tables ? m.t.segs : m.segs;
  const OuterClass* cls = m.inline_tables ? m.t.cls : m.cls;
  const InnerGroup* grps = m.inline_tables ? m.t.grps : m.grps;
  if (bx < m.ngrp) {
    inner_map_group(grps[bx], segs, stage_order(m), m.lva, m.lvb, m.a_inner, m.b_inner, m.K, m.tK, m.tJ, m.lAk,
                    m.lBk, m.blk16);
    return;
  }
  const int ob = bx - m.ngrp;
  const bool is_a = ob < m.a.ncls;
  const OuterJob& j = is_a ? m.a : m.b;
  const int ci = is_a ? ob : ob - m.a.ncls;
  outer_map_class(cls[j.cls0 + ci], j.lv, j.n, j.G, j.pos, j.src, j.grpL, j.grpN);
}

#ifdef IMQ_DEBUG
// ------------------------------------------------------------------------------------------------
// Debug build only: every index of a finished plan that the unpack and GEMM kernels read, checked
// against the plan's sizes.  A violation records IMQ_ERR_BOUNDS in the status word (nothing traps and
// nothing else changes); the checks run right after the maps kernel, in stream order.
// ------------------------------------------------------------------------------------------------
struct CheckGroup {
  int64_t off, len, padded;
  int32_t e;
};
struct CheckOuter {
  int on;                 // the operand is unpacked OUTER
  int64_t n, n_unp, ngrp;  // source lines, unpacked lines, groups of IMQ_*_GROUP lines
  const int8_t* lv;        // levels of the source lines
  const int32_t* pos;
  const int32_t* src;
  const int32_t* grpL;
  const int32_t* grpN;
};
struct CheckArgs {
  int64_t K, K_unp;
  int a_inner, b_inner;
  const int8_t* lva;  // levels of A's columns
  const int8_t* lvb;  // levels of B's rows
  const int32_t* tK;
  const int32_t* tJ;    // staging position of each inner position's index (tK itself when perm is null)
  const int32_t* perm;  // staging order (null: the identity)
  const int32_t* pinv;
  const int8_t* lAk;
  const int8_t* lBk;
  const int32_t* blk16;
  int ng;
  CheckGroup grp[IMQ_MAX_GROUPS];
  CheckOuter o[2];
  int32_t* status;
};

__device__ __forceinline__ void check(bool ok, int32_t* status) {
  if (!ok) set_status(status, IMQ_ERR_BOUNDS);
}

__global__ void __launch_bounds__(256) k_plan_check(const __grid_constant__ CheckArgs c) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  // inner positions: source index, levels, exponent and padding of their group
  for (int64_t p = i0; p < c.K_unp; p += stride) {
    int g = -1;
    for (int k = 0; k < c.ng; ++k)
      if (p >= c.grp[k].off && p < c.grp[k].off + c.grp[k].padded) g = k;
    check(g >= 0, c.status);
    if (g < 0) continue;
    const int32_t t = c.tK[p];
    const bool real = p < c.grp[g].off + c.grp[g].len;
    check(real ? (t >= 0 && t < c.K) : t == -1, c.status);
    check(c.tJ[p] == (t >= 0 && t < c.K && c.pinv ? c.pinv[t] : t), c.status);
    if (t < 0 || t >= c.K) continue;
    const int la = c.a_inner ? c.lva[t] : 1, lb = c.b_inner ? c.lvb[t] : 1;
    const int lA = c.lAk[p], lB = c.lBk[p];
    check(lA >= 0 && lA < la && lB >= 0 && lB < lb && lA + lB == c.grp[g].e, c.status);
  }
  // the staging order: a permutation of the inner indices
  if (c.perm) {
    for (int64_t j = i0; j < c.K; j += stride) {
      const int32_t t = c.perm[j];
      check(t >= 0 && t < c.K, c.status);
      if (t >= 0 && t < c.K) check(c.pinv[t] == (int32_t)j, c.status);
    }
  }
  // 16-position blocks: a run entry must describe the positions exactly (staging positions j0..j0+15)
  for (int64_t b = i0; b < c.K_unp / 16; b += stride) {
    const int32_t v = c.blk16[b];
    if (v == -1) continue;
    const int32_t j0 = v >= 0 ? v : -v - 2;
    check(v < 0 || (j0 & 15) == 0, c.status);
    check(j0 >= 0 && j0 + 16 <= c.K, c.status);
    if (!(j0 >= 0 && j0 + 16 <= c.K)) continue;
    for (int k = 0; k < 16; ++k)
      check(c.tK[b * 16 + k] == (c.perm ? c.perm[j0 + k] : j0 + k) && c.tJ[b * 16 + k] == j0 + k &&
                c.lAk[b * 16 + k] == c.lAk[b * 16] && c.lBk[b * 16 + k] == c.lBk[b * 16],
            c.status);
  }
  // OUTER lines: every source line's L lines inside the unpacked operand and inside one group of its level,
  // every used unpacked line pointing back at its source, every group's level and count in range
  for (int o = 0; o < 2; ++o) {
    const CheckOuter& q = c.o[o];
    if (!q.on) continue;
    check(q.ngrp * 32 == q.n_unp, c.status);
    for (int64_t i = i0; i < q.n; i += stride) {
      const int L = q.lv[i];
      const int64_t u = q.pos[i];
      check(L >= 1 && L <= 31 && u >= 0 && u + L <= q.n_unp, c.status);
      if (!(L >= 1 && L <= 31 && u >= 0 && u + L <= q.n_unp)) continue;
      check(u / 32 == (u + L - 1) / 32 && q.grpL[u / 32] == L && (u % 32) % L == 0 && (u % 32) / L < q.grpN[u / 32],
            c.status);
      for (int l = 0; l < L; ++l) check(q.src[u + l] == (int32_t)i, c.status);
    }
    for (int64_t u = i0; u < q.n_unp; u += stride) {
      const int32_t s = q.src[u];
      check(s >= -1 && s < q.n, c.status);
      if (s >= 0 && s < q.n) check(q.pos[s] <= u && u < q.pos[s] + q.lv[s], c.status);
    }
    for (int64_t g = i0; g < q.ngrp; g += stride) {
      const int L = q.grpL[g], nn = q.grpN[g];
      check(L >= 1 && L <= 31 && nn >= 0 && nn * L <= 32, c.status);
    }
  }
}
#endif

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
struct Pinned {
  HostSummary* sum = nullptr;   // mapped pinned memory: `cap` summary slots, one per plan of a batch
  HostSummary* sum_dev = nullptr;  // their device address
  int cap = 0;
  uint32_t seq = 0;
  void* tables = nullptr;          // staging of the segment and class tables for their upload
  cudaEvent_t tables_done = nullptr;  // recorded after the last upload from `tables`
  std::mutex mu;
};
Pinned g_pinned[64];

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

namespace {
// out[i] = min(R^L - 1, cap) with L the level of m[i] (R = 2^bm1): the largest magnitude with as many
// base-R digits as m[i].
__global__ void __launch_bounds__(256) k_level_cover(const int32_t* __restrict__ m, int64_t n, int32_t bm1,
                                                     int32_t cap, int32_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int L = level_of((uint32_t)m[i], bm1);
    const int64_t top = (int64_t)L * bm1 >= 31 ? (int64_t)INT32_MAX : ((int64_t)1 << (L * bm1)) - 1;
    out[i] = (int32_t)(top < cap ? top : cap);
  }
}
}  // namespace

imq_status launch_level_cover(const int32_t* maxima, int64_t n, int32_t b, int32_t cap, int32_t* out,
                              cudaStream_t st) {
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (n == 0) return IMQ_OK;
  int64_t grid = (n + 255) / 256;
  if (grid > (int64_t)ds->num_sms * 4) grid = (int64_t)ds->num_sms * 4;
  k_level_cover<<<(unsigned)grid, 256, 0, st>>>(maxima, n, b - 1, cap, out);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

imq_status launch_line_max(const void* X, imq_dtype it, int64_t rows, int64_t cols, int64_t ld,
                           int32_t* rowmax, int32_t* colmax, cudaStream_t st) {
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (rows == 0 || cols == 0) return IMQ_OK;
  if (rowmax) IMQ_CUDA_TRY(cudaMemsetAsync(rowmax, 0, (size_t)rows * 4, st));
  if (colmax) IMQ_CUDA_TRY(cudaMemsetAsync(colmax, 0, (size_t)cols * 4, st));
  const int smem_cols = (colmax && cols <= 32768) ? 1 : 0;
  const size_t smem = smem_cols ? (size_t)cols * 4 : 0;
  const int64_t grid = rows < (int64_t)ds->num_sms * 4 ? rows : (int64_t)ds->num_sms * 4;
  if (it == IMQ_I16) {
    IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_line_max<int16_t>), smem));
    k_line_max<int16_t><<<(unsigned)grid, 256, smem, st>>>(static_cast<const int16_t*>(X), rows, cols, ld,
                                                           rowmax, colmax, smem_cols);
  } else {
    IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_line_max<int32_t>), smem));
    k_line_max<int32_t><<<(unsigned)grid, 256, smem, st>>>(static_cast<const int32_t*>(X), rows, cols, ld,
                                                           rowmax, colmax, smem_cols);
  }
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

// The maps kernels of a batch run as one launch, except in the debug build, whose index checks follow each
// plan's own maps.
#ifdef IMQ_DEBUG
constexpr bool kBatchMaps = false;
#else
constexpr bool kBatchMaps = true;
#endif

// One plan in the making: its arguments and what its first stage leaves for the second.
struct PlanJob {
  const void* A;
  const void* B;
  imq_dtype it;
  int64_t M, K, N;
  int32_t transA;
  int64_t lda;
  int32_t transB;
  int64_t ldb;
  int32_t b;
  imq_strategy strategy;
  const int32_t* a_rowmax;
  const int32_t* a_colmax;
  const int32_t* b_rowmax;
  const int32_t* b_colmax;
  int slot;  // summary slot of the batch
  // batched: this plan's kernels are queued by build_plans together with the other plans' of its batch
  // (one launch per kind); plan_begin and plan_finish only record their arguments
  bool batched = false;
  // state after plan_begin
  imq_plan_t* pl = nullptr;
  char* blk1 = nullptr;
  Summary* dsum = nullptr;
  size_t o_segs = 0, o_cls = 0, o_grps = 0, o_E = 0;
  uint32_t seq = 0;
  LevelArgs la{};
  int nlm = 0;  // line maxima to compute (batched)
  LineMaxJob lm[2]{};
  int nzero = 0;
  ZeroSpan zero[3]{};
  // state after plan_finish (batched)
  bool has_maps = false;
  int order_blocks = 0, maps_blocks = 0;
  MapsArgs maps{};
};

// Frees a plan that failed before it was returned.
imq_status plan_fail(imq_plan_t* pl, imq_status e, cudaStream_t st) {
  if (!pl) return e;
  if (pl->dev_block) cudaFreeAsync(pl->dev_block, st);
  if (pl->dev_block2) cudaFreeAsync(pl->dev_block2, st);
  free(pl->host_tables);
  delete pl;
  return e;
}

// Makes sure the pinned summary slots and table staging of this device exist (nslots slots).
imq_status pinned_ready(Pinned& pin, int nslots) {
  const size_t staging_bytes = align_up(sizeof(InnerSeg) * kLv * kLv, 256) +
                               align_up(sizeof(OuterClass) * 2 * kLv, 256) +
                               align_up(sizeof(InnerGroup) * IMQ_MAX_GROUPS, 256) + sizeof(int32_t) * kLv * kLv;
  if (pin.cap < nslots) {
    // every earlier plan has read its summary before returning, so the old slots are idle
    if (pin.sum) cudaFreeHost(pin.sum);
    pin.sum = nullptr;
    pin.cap = 0;
    const int cap = nslots < 16 ? 16 : nslots;
    IMQ_CUDA_TRY(cudaHostAlloc(reinterpret_cast<void**>(&pin.sum), sizeof(HostSummary) * (size_t)cap,
                               cudaHostAllocMapped));
    IMQ_CUDA_TRY(cudaHostGetDevicePointer(reinterpret_cast<void**>(&pin.sum_dev), pin.sum, 0));
    for (int i = 0; i < cap; ++i) pin.sum[i].seq = 0;
    pin.cap = cap;
  }
  if (!pin.tables) IMQ_CUDA_TRY(cudaMallocHost(&pin.tables, staging_bytes));
  if (!pin.tables_done) IMQ_CUDA_TRY(cudaEventCreateWithFlags(&pin.tables_done, cudaEventDisableTiming));
  return IMQ_OK;
}

// Stage 1 of a plan: line maxima (unless given), the hybrid's choice, the level kernel, which writes the
// plan's summary into summary slot j.slot.  Nothing is waited for.
imq_status plan_begin(PlanJob& job, Pinned& pin, DeviceState* ds, int dev, cudaStream_t st) {
  const void* A = job.A;
  const void* B = job.B;
  const imq_dtype it = job.it;
  const int64_t M = job.M, K = job.K, N = job.N;
  const int32_t transA = job.transA, transB = job.transB;
  const int64_t lda = job.lda, ldb = job.ldb;
  const int32_t b = job.b;
  const imq_strategy strategy = job.strategy;
  const int32_t *a_rowmax = job.a_rowmax, *a_colmax = job.a_colmax, *b_rowmax = job.b_rowmax,
                *b_colmax = job.b_colmax;
  const size_t tables_bytes = sizeof(InnerSeg) * kLv * kLv + sizeof(OuterClass) * 2 * kLv +
                              sizeof(InnerGroup) * IMQ_MAX_GROUPS + sizeof(int32_t) * kLv * kLv;
  imq_plan_t* pl = new imq_plan_t;
  memset(pl, 0, sizeof(*pl));
  pl->host_tables = malloc(tables_bytes);
  if (!pl->host_tables) {
    delete pl;
    return IMQ_ERR_CUDA;
  }
  pl->device = dev;
  pl->A = A;
  pl->B = B;
  pl->it = it;
  pl->transA = transA;
  pl->transB = transB;
  pl->lda = lda;
  pl->ldb = ldb;
  imq_plan_info& I = pl->info;
  I.b = b;
  I.strategy = strategy;
  I.M = M;
  I.K = K;
  I.N = N;

  // ---- stage 1: maxima, levels, summary ----
  const int64_t nvec[4] = {M, K, K, N};
  size_t off = 0;
  size_t o_max[4], o_lv[4];
  for (int v = 0; v < 4; ++v) { o_max[v] = off; off = align_up(off + (size_t)nvec[v] * 4, 256); }
  for (int v = 0; v < 4; ++v) { o_lv[v] = off; off = align_up(off + (size_t)nvec[v], 256); }
  const size_t o_sum = off;
  off = align_up(off + sizeof(Summary), 256);
  const size_t o_segs = off;
  off = align_up(off + sizeof(InnerSeg) * kLv * kLv, 256);
  const size_t o_cls = off;
  off = align_up(off + sizeof(OuterClass) * 2 * kLv, 256);
  const size_t o_grps = off;
  off = align_up(off + sizeof(InnerGroup) * IMQ_MAX_GROUPS, 256);
  const size_t o_E = off;
  off = align_up(off + sizeof(int32_t) * kLv * kLv, 256);
  // hybrid scratch: per matrix (A: M outer lines, B: N outer lines; K inner indices each) the counts and
  // the two histograms (zeroed together), then the least-count tables (filled with kHybInf), then the
  // threshold and the carried levels
  const bool hybrid = strategy == IMQ_HYBRID;
  const int64_t hyb_out[2] = {M, N};
  size_t o_hcnt[2] = {0, 0}, o_hH[2] = {0, 0}, o_hG[2] = {0, 0}, o_hmex[2] = {0, 0}, o_htau[2] = {0, 0};
  size_t o_hlo[2] = {0, 0}, o_hli[2] = {0, 0}, o_hcmax[2] = {0, 0}, o_hzero = 0, o_hinf = 0, o_hend = 0;
  if (hybrid) {
    o_hzero = off;
    for (int h = 0; h < 2; ++h) {
      o_hcnt[h] = off; off = align_up(off + (size_t)hyb_out[h] * 4, 256);
      o_hH[h] = off; off = align_up(off + (size_t)(K + 2) * 8, 256);
      o_hG[h] = off; off = align_up(off + (size_t)(K + 2) * 8, 256);
    }
    for (int h = 0; h < 2; ++h) { o_hcmax[h] = off; off = align_up(off + 4, 256); }
    o_hinf = off;
    for (int h = 0; h < 2; ++h) { o_hmex[h] = off; off = align_up(off + (size_t)K * kHybL * 4, 256); }
    o_hend = off;
    for (int h = 0; h < 2; ++h) {
      o_htau[h] = off; off = align_up(off + 4, 256);
      o_hlo[h] = off; off = align_up(off + (size_t)hyb_out[h], 256);
      o_hli[h] = off; off = align_up(off + (size_t)K, 256);
    }
  }
  const size_t stage1 = off;
  char* blk1 = nullptr;
  if (cudaMallocFromPoolAsync((void**)&blk1, stage1, ds->pool, st) != cudaSuccess) {
    free(pl->host_tables);
    delete pl;
    return IMQ_ERR_CUDA;
  }
  pl->dev_block = blk1;
  pl->dev_bytes = stage1;
  int32_t* mx[4];
  for (int v = 0; v < 4; ++v) mx[v] = reinterpret_cast<int32_t*>(blk1 + o_max[v]);
  pl->max_a_row = mx[0];
  pl->max_a_col = mx[1];
  pl->max_b_row = mx[2];
  pl->max_b_col = mx[3];
  pl->lv_a_row = reinterpret_cast<int8_t*>(blk1 + o_lv[0]);
  pl->lv_a_col = reinterpret_cast<int8_t*>(blk1 + o_lv[1]);
  pl->lv_b_row = reinterpret_cast<int8_t*>(blk1 + o_lv[2]);
  pl->lv_b_col = reinterpret_cast<int8_t*>(blk1 + o_lv[3]);
  Summary* dsum = reinterpret_cast<Summary*>(blk1 + o_sum);

  auto fail = [&](imq_status e) { return plan_fail(pl, e, st); };

  const bool have_max = a_rowmax && a_colmax && b_rowmax && b_colmax;
  const int32_t* lmx[4] = {mx[0], mx[1], mx[2], mx[3]};  // the maxima the levels are computed from
  if (have_max) {
    // the caller's maxima are read in place by the kernels below; A's column maxima are also kept in
    // the plan (the fused quantise-and-unpack path checks new activations against them)
    lmx[0] = a_rowmax;
    lmx[1] = a_colmax;
    lmx[2] = b_rowmax;
    lmx[3] = b_colmax;
  } else if (job.batched) {
    // recorded for the batch's line-maxima launch; the column maxima are cleared first
    job.lm[0] = transA ? LineMaxJob{A, K, M, lda, mx[1], mx[0]} : LineMaxJob{A, M, K, lda, mx[0], mx[1]};
    job.lm[1] = transB ? LineMaxJob{B, N, K, ldb, mx[3], mx[2]} : LineMaxJob{B, K, N, ldb, mx[2], mx[3]};
    job.nlm = 2;
    for (int q = 0; q < 2; ++q) job.zero[job.nzero++] = ZeroSpan{job.lm[q].colmax, job.lm[q].cols * 4};
  } else {
    // A stored M x K (or K x M when transposed); B stored K x N (or N x K)
    imq_status e = transA ? launch_line_max(A, it, K, M, lda, mx[1], mx[0], st)
                          : launch_line_max(A, it, M, K, lda, mx[0], mx[1], st);
    if (e != IMQ_OK) return fail(e);
    e = transB ? launch_line_max(B, it, N, K, ldb, mx[3], mx[2], st)
               : launch_line_max(B, it, K, N, ldb, mx[2], mx[3], st);
    if (e != IMQ_OK) return fail(e);
    if (M == 0 && K > 0 && cudaMemsetAsync(mx[1], 0, (size_t)K * 4, st) != cudaSuccess) return fail(IMQ_ERR_CUDA);
    if (N == 0 && K > 0 && cudaMemsetAsync(mx[2], 0, (size_t)K * 4, st) != cudaSuccess) return fail(IMQ_ERR_CUDA);
    if (K == 0) {
      if (M && cudaMemsetAsync(mx[0], 0, (size_t)M * 4, st) != cudaSuccess) return fail(IMQ_ERR_CUDA);
      if (N && cudaMemsetAsync(mx[3], 0, (size_t)N * 4, st) != cudaSuccess) return fail(IMQ_ERR_CUDA);
    }
  }
  if (job.batched) {
    job.zero[job.nzero++] = ZeroSpan{dsum, (int64_t)sizeof(Summary)};
  } else if (cudaMemsetAsync(dsum, 0, sizeof(Summary), st) != cudaSuccess) {
    return fail(IMQ_ERR_CUDA);
  }
  LevelArgs la;
  la.keep_a_col = have_max ? mx[1] : nullptr;  // k_levels copies the caller's A column maxima there
  for (int v = 0; v < 4; ++v) {
    la.mx[v] = lmx[v];
    la.lvin[v] = nullptr;
    la.n[v] = nvec[v];
  }
  if (hybrid) {
    // A: outer lines = its rows (stored rows unless transposed); B: outer lines = its columns (stored
    // columns unless transposed); the inner indices are the other stored axis
    HybArgs ha;
    ha.bm1 = b - 1;
    for (int h = 0; h < 2; ++h) {
      HybMat& m = ha.m[h];
      const int32_t tr = h == 0 ? transA : transB;
      m.X = h == 0 ? A : B;
      m.ld = h == 0 ? lda : ldb;
      m.n_out = hyb_out[h];
      m.n_in = K;
      m.outer_is_row = h == 0 ? !tr : tr;
      m.rows = m.outer_is_row ? m.n_out : K;
      m.cols = m.outer_is_row ? K : m.n_out;
      m.omax = h == 0 ? lmx[0] : lmx[3];
      m.cnt = reinterpret_cast<int32_t*>(blk1 + o_hcnt[h]);
      m.mex = reinterpret_cast<int32_t*>(blk1 + o_hmex[h]);
      m.H = reinterpret_cast<unsigned long long*>(blk1 + o_hH[h]);
      m.G = reinterpret_cast<unsigned long long*>(blk1 + o_hG[h]);
      m.tau = reinterpret_cast<int32_t*>(blk1 + o_htau[h]);
      m.cmax = reinterpret_cast<int32_t*>(blk1 + o_hcmax[h]);
      m.lo = reinterpret_cast<int8_t*>(blk1 + o_hlo[h]);
      m.li = reinterpret_cast<int8_t*>(blk1 + o_hli[h]);
    }
    if (cudaMemsetAsync(blk1 + o_hzero, 0, o_hinf - o_hzero, st) != cudaSuccess ||
        cudaMemsetAsync(blk1 + o_hinf, 0x7F, o_hend - o_hinf, st) != cudaSuccess)
      return fail(IMQ_ERR_CUDA);
    int64_t maxc = 1, maxr = 1, maxn = 1;
    for (int h = 0; h < 2; ++h) {
      maxc = ha.m[h].cols > maxc ? ha.m[h].cols : maxc;
      maxr = ha.m[h].rows > maxr ? ha.m[h].rows : maxr;
      maxn = ha.m[h].n_out > maxn ? ha.m[h].n_out : maxn;
    }
    maxn = K > maxn ? K : maxn;
    // column kernels: 256 threads x up to 16 / sizeof(entry) columns, 8 rows per tile; the grid covers
    // the wider of the two matrices at one column per thread (threads past the end return)
    const dim3 gscan((unsigned)((maxc + 255) / 256), (unsigned)((maxr + 7) / 8 < 4096 ? (maxr + 7) / 8 : 4096), 2);
    const int64_t gl = (maxn + 255) / 256 < (int64_t)ds->num_sms * 8 ? (maxn + 255) / 256 : (int64_t)ds->num_sms * 8;
    const dim3 glines((unsigned)gl, 2);
    const bool any_rows = ha.m[0].outer_is_row || ha.m[1].outer_is_row;
    const bool any_cols = !ha.m[0].outer_is_row || !ha.m[1].outer_is_row;
    int64_t nrows = 0;
    for (int h = 0; h < 2; ++h)
      if (ha.m[h].outer_is_row) nrows += ha.m[h].rows;
    // one CTA per row, up to 16 resident per SM
    int64_t gr = nrows < (int64_t)ds->num_sms * 16 ? nrows : (int64_t)ds->num_sms * 16;
    if (gr < 1) gr = 1;
    const dim3 growsg((unsigned)gr);
    if (it == IMQ_I16) {
      if (any_rows) k_hyb_rows<int16_t><<<growsg, kRowThreads, 0, st>>>(ha);
      if (any_cols) {
        k_hyb_count<int16_t><<<gscan, 256, 0, st>>>(ha);
        k_hyb_minc<int16_t><<<gscan, 256, 0, st>>>(ha);
      }
    } else {
      if (any_rows) k_hyb_rows<int32_t><<<growsg, kRowThreads, 0, st>>>(ha);
      if (any_cols) {
        k_hyb_count<int32_t><<<gscan, 256, 0, st>>>(ha);
        k_hyb_minc<int32_t><<<gscan, 256, 0, st>>>(ha);
      }
    }
    k_hyb_hist<<<glines, 256, 0, st>>>(ha);
    k_hyb_choose<<<2, 1024, 0, st>>>(ha);
    k_hyb_apply<<<glines, 256, 0, st>>>(ha);
    if (cudaGetLastError() != cudaSuccess) return fail(IMQ_ERR_CUDA);
    la.lvin[0] = ha.m[0].lo;
    la.lvin[1] = ha.m[0].li;
    la.lvin[2] = ha.m[1].li;
    la.lvin[3] = ha.m[1].lo;
  }
  la.status = ds->status;
  la.lv[0] = pl->lv_a_row;
  la.lv[1] = pl->lv_a_col;
  la.lv[2] = pl->lv_b_row;
  la.lv[3] = pl->lv_b_col;
  la.bm1 = b - 1;
  la.sum = dsum;
  la.hsum = pin.sum_dev + job.slot;
  la.seq = ++pin.seq;
  {
    const int64_t nmax = (M > K ? M : K) > N ? (M > K ? M : K) : N;
    int64_t grid = (nmax + 255) / 256;
    if (grid > ds->num_sms * 2) grid = ds->num_sms * 2;
    if (grid < 1) grid = 1;
    la.nblk = (uint32_t)grid;
    if (job.batched)
      job.la = la;
    else
      k_levels<<<(unsigned)grid, 256, 0, st>>>(la);
  }
  if (cudaGetLastError() != cudaSuccess) return fail(IMQ_ERR_CUDA);
  job.pl = pl;
  job.blk1 = blk1;
  job.dsum = dsum;
  job.o_segs = o_segs;
  job.o_cls = o_cls;
  job.o_grps = o_grps;
  job.o_E = o_E;
  job.seq = la.seq;
  return IMQ_OK;
}

// Waits for the summary of a plan whose stage 1 is queued on `st`, and copies it to *out.
imq_status plan_wait(PlanJob& job, Pinned& pin, cudaStream_t st, Summary* out) {
  imq_plan_t* pl = job.pl;
  auto fail = [&](imq_status e) {
    job.pl = nullptr;
    return plan_fail(pl, e, st);
  };
  HostSummary* hs = pin.sum + job.slot;
  const Summary* dsum = job.dsum;
  // wait for the summary: spin on its sequence number, asking the stream every few thousand polls
  // whether it is still running (an error there is returned; a finished stream without the number, which
  // a launch failure could leave, falls back to a plain copy of the device summary)
  {
    const volatile uint32_t* seqp = &hs->seq;
    bool have = false;
    for (uint64_t it = 1;; ++it) {
      if (*seqp == job.seq) {
        have = true;
        break;
      }
      if ((it & 4095) == 0) {
        const cudaError_t q = cudaStreamQuery(st);
        if (q == cudaSuccess) {
          have = *seqp == job.seq;
          break;
        }
        if (q != cudaErrorNotReady) return fail(IMQ_ERR_CUDA);
      }
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    if (!have && (cudaMemcpy(&hs->s, dsum, sizeof(Summary), cudaMemcpyDeviceToHost) != cudaSuccess))
      return fail(IMQ_ERR_CUDA);
  }
  *out = hs->s;
  return IMQ_OK;
}

// Stage 2 of a plan: the host decisions from its summary, then the maps kernel.  *out gets the plan.
imq_status plan_finish(PlanJob& job, const Summary& S, Pinned& pin, DeviceState* ds, cudaStream_t st,
                       imq_plan_t** out) {
  imq_plan_t* pl = job.pl;
  job.pl = nullptr;
  auto fail = [&](imq_status e) { return plan_fail(pl, e, st); };
  const int64_t M = job.M, K = job.K, N = job.N;
  const int32_t b = job.b;
  const imq_strategy strategy = job.strategy;
  const int64_t nvec[4] = {M, K, K, N};
  imq_plan_info& I = pl->info;
  InnerSeg* hsegs = static_cast<InnerSeg*>(pl->host_tables);
  OuterClass* hcls = reinterpret_cast<OuterClass*>(hsegs + kLv * kLv);
  InnerGroup* hgrps = reinterpret_cast<InnerGroup*>(hcls + 2 * kLv);
  int32_t* hE = reinterpret_cast<int32_t*>(hgrps + IMQ_MAX_GROUPS);
  char* blk1 = job.blk1;
  const size_t o_segs = job.o_segs, o_cls = job.o_cls, o_grps = job.o_grps, o_E = job.o_E;
  // a pending kernel error (e.g. a non-finite quantiser input) is reported before planning
  if (S.status != IMQ_OK) return fail((imq_status)S.status);

  // ---- host decisions ----
  for (int v = 0; v < 4; ++v) if (S.lmax[v] > 31) return fail(IMQ_ERR_UNSUPPORTED);
  const int64_t lmax[4] = {nvec[0] ? S.lmax[0] : 1, nvec[1] ? S.lmax[1] : 1, nvec[2] ? S.lmax[2] : 1,
                           nvec[3] ? S.lmax[3] : 1};
  I.lmax_a_row = (int32_t)lmax[0];
  I.lmax_a_col = (int32_t)lmax[1];
  I.lmax_b_row = (int32_t)lmax[2];
  I.lmax_b_col = (int32_t)lmax[3];
  I.sum_l_a_row = (int64_t)S.sum[0];
  I.sum_l_a_col = (int64_t)S.sum[1];
  I.sum_l_b_row = (int64_t)S.sum[2];
  I.sum_l_b_col = (int64_t)S.sum[3];
  I.oor_lines_a_row = (int64_t)S.oor[0];
  I.oor_lines_a_col = (int64_t)S.oor[1];
  I.oor_lines_b_row = (int64_t)S.oor[2];
  I.oor_lines_b_col = (int64_t)S.oor[3];

  int da, db;
  if (strategy == IMQ_MIX || strategy == IMQ_MIX_JOINT) {
    if (S.oor[0] == 0 && S.oor[1] == 0) {
      da = IMQ_DIR_NONE;
    } else {
      const __int128 row_side = (__int128)S.sum[0] * K, col_side = (__int128)S.sum[1] * M;
      if (row_side != col_side) da = row_side < col_side ? IMQ_DIR_OUTER : IMQ_DIR_INNER;
      else if (S.oor[0] != S.oor[1]) da = S.oor[0] < S.oor[1] ? IMQ_DIR_OUTER : IMQ_DIR_INNER;
      else da = IMQ_DIR_OUTER;
    }
    if (S.oor[2] == 0 && S.oor[3] == 0) {
      db = IMQ_DIR_NONE;
    } else {
      const __int128 row_side = (__int128)S.sum[2] * N, col_side = (__int128)S.sum[3] * K;
      if (row_side != col_side) db = row_side < col_side ? IMQ_DIR_INNER : IMQ_DIR_OUTER;
      else if (S.oor[2] != S.oor[3]) db = S.oor[2] < S.oor[3] ? IMQ_DIR_INNER : IMQ_DIR_OUTER;
      else db = IMQ_DIR_INNER;
    }
  } else if (strategy == IMQ_HYBRID) {
    // the summary already holds the carried levels of the hybrid choice
    da = (S.oor[0] ? IMQ_DIR_OUTER : 0) | (S.oor[1] ? IMQ_DIR_INNER : 0);
    db = (S.oor[3] ? IMQ_DIR_OUTER : 0) | (S.oor[2] ? IMQ_DIR_INNER : 0);
  } else {
    da = (strategy == IMQ_ROW_ROW || strategy == IMQ_ROW_COL) ? IMQ_DIR_OUTER : IMQ_DIR_INNER;
    db = (strategy == IMQ_ROW_ROW || strategy == IMQ_COL_ROW) ? IMQ_DIR_INNER : IMQ_DIR_OUTER;
  }
  if (strategy == IMQ_MIX_JOINT) {
    // the exact unpacked size M_eff * N_eff * K_eff of a direction pair, from the summary: level sums
    // for the outer dimensions, the joint histogram of (A column level, B row level) for K_eff
    // joint[x][y] is zero above the largest levels, so the sums stop there
    unsigned __int128 kk_both = 0;
    for (int x = 1; x <= (int)lmax[1]; ++x)
      for (int y = 1; y <= (int)lmax[2]; ++y) kk_both += (unsigned __int128)((unsigned)(x * y)) * S.joint[x][y];
    auto size_of = [&](int ca, int cb) {
      const unsigned __int128 me = ca == IMQ_DIR_OUTER ? (unsigned __int128)S.sum[0] : (unsigned __int128)M;
      const unsigned __int128 ne = cb == IMQ_DIR_OUTER ? (unsigned __int128)S.sum[3] : (unsigned __int128)N;
      unsigned __int128 ke = (unsigned __int128)K;
      if (ca == IMQ_DIR_INNER && cb == IMQ_DIR_INNER) ke = kk_both;
      else if (ca == IMQ_DIR_INNER) ke = S.sum[1];
      else if (cb == IMQ_DIR_INNER) ke = S.sum[2];
      return me * ne * ke;
    };
    const int pa[4] = {IMQ_DIR_OUTER, IMQ_DIR_OUTER, IMQ_DIR_INNER, IMQ_DIR_INNER};
    const int pb[4] = {IMQ_DIR_INNER, IMQ_DIR_OUTER, IMQ_DIR_INNER, IMQ_DIR_OUTER};
    unsigned __int128 best = size_of(da, db);
    const bool a_none = da == IMQ_DIR_NONE, b_none = db == IMQ_DIR_NONE;
    for (int c = 0; c < 4; ++c) {
      const int ca = a_none ? IMQ_DIR_NONE : pa[c], cb = b_none ? IMQ_DIR_NONE : pb[c];
      const unsigned __int128 cost = size_of(ca, cb);
      if (cost < best) {
        best = cost;
        da = ca;
        db = cb;
      }
    }
  }
  I.dir_a = da;
  I.dir_b = db;
  const bool a_outer = (da & IMQ_DIR_OUTER) != 0, a_inner = (da & IMQ_DIR_INNER) != 0;
  const bool b_outer = (db & IMQ_DIR_OUTER) != 0, b_inner = (db & IMQ_DIR_INNER) != 0;

  // inner segments from the joint level histogram
  const int maxla = a_inner ? (int)lmax[1] : 1;
  const int maxlb = b_inner ? (int)lmax[2] : 1;
  // inner indices whose (A column, B row) levels exceed (sa, sb); joint[x][y] is zero above the largest
  // levels, so the sum stops there
  auto seg_len = [&](int sa, int sb) {
    int64_t n = 0;
    for (int x = 1; x <= (int)lmax[1]; ++x)
      for (int y = 1; y <= (int)lmax[2]; ++y) {
        const int ea = a_inner ? x : 1, eb = b_inner ? y : 1;
        if (ea > sa && eb > sb) n += S.joint[x][y];
      }
    return n;
  };
  int nseg = 0;
  int64_t koff = 0, keff = 0;
  double scattered = 0.0;
  int ng = 0;
  for (int e = 0; e <= maxla + maxlb - 2; ++e) {
    int64_t glen = 0;
    const int seg_first = nseg;
    for (int sa = 0; sa < maxla; ++sa) {
      const int sb = e - sa;
      if (sb < 0 || sb >= maxlb) continue;
      const int64_t n = seg_len(sa, sb);
      if (n == 0) continue;
      // positions of this segment expected outside 16-long runs of consecutive indices, were its indices
      // placed at random among the K (a segment of density d keeps a block a run with probability d^15)
      scattered += (double)n * (1.0 - pow((double)n / (double)K, 15.0));
      hsegs[nseg].la = sa;
      hsegs[nseg].lb = sb;
      hsegs[nseg].off = koff + glen;
      ++nseg;
      glen += n;
    }
    if (glen == 0) continue;
    if (ng >= IMQ_MAX_GROUPS) return fail(IMQ_ERR_UNSUPPORTED);
    pl->groups[ng].e = e;
    pl->groups[ng].k_offset = koff;
    pl->groups[ng].k_len = glen;
    pl->groups[ng].k_len_padded = (glen + IMQ_INNER_PAD - 1) / IMQ_INNER_PAD * IMQ_INNER_PAD;
    hgrps[ng].k0 = koff;
    hgrps[ng].kpad = pl->groups[ng].k_len_padded;
    hgrps[ng].seg0 = seg_first;
    hgrps[ng].nseg = nseg - seg_first;
    koff += pl->groups[ng].k_len_padded;
    keff += glen;
    ++ng;
  }
  I.n_groups = ng;
  I.K_unp = koff;
  I.K_eff = keff;

  // The staging order of the inner indices (StageOrder): classes (ea, eb) in descending order, their sizes
  // from the joint level histogram.  With one non-empty class the order is the identity.
  const int ew = maxlb + 1;
  int nonempty = 0;
  {
    std::vector<int64_t> ccount((size_t)(maxla + 1) * ew, 0);
    for (int x = 1; x <= (int)lmax[1]; ++x)
      for (int y = 1; y <= (int)lmax[2]; ++y) {
        const int ea = a_inner ? x : 1, eb = b_inner ? y : 1;
        ccount[(size_t)ea * ew + eb] += S.joint[x][y];
      }
    int64_t j = 0;
    for (int ea = maxla; ea >= 1; --ea) {
      hE[ea * ew + maxlb] = (int32_t)j;
      for (int eb = maxlb; eb >= 1; --eb) {
        const int64_t c = ccount[(size_t)ea * ew + eb];
        nonempty += c > 0;
        j += c;
        hE[ea * ew + eb - 1] = (int32_t)j;
      }
    }
    for (int e2 = 0; e2 < ew; ++e2) hE[e2] = (int32_t)j;  // row 0: past every class
    if (j != K) return fail(IMQ_ERR_CUDA);                // the histogram counts every inner index once
  }
  // The staging order costs a scattered staging of every source line; it pays when index order would leave
  // many blocks gathered (segments of middling density: both operands unpacked INNER, typically).
  const bool permuted = nonempty > 1 && koff > 0 && scattered > 0.25 * (double)keff;

  // outer sizes
  int ncls = 0;
  auto outer_classes = [&](int v, int G, int64_t* groups_out) {
    int64_t grp = 0;
    for (int L = 1; L <= (int)lmax[v]; ++L) {
      const int64_t cnt = S.hist[v][L];
      if (cnt == 0) continue;
      const int per = G / L;
      hcls[ncls].L = L;
      hcls[ncls].per = per;
      hcls[ncls].grp0 = grp;
      hcls[ncls].count = cnt;
      ++ncls;
      grp += (cnt + per - 1) / per;
    }
    *groups_out = grp;
  };
  int cls_a0 = 0, cls_a1 = 0, cls_b0 = 0, cls_b1 = 0;
  if (a_outer) {
    cls_a0 = ncls;
    outer_classes(0, IMQ_A_GROUP, &pl->n_grp_a);
    cls_a1 = ncls;
    I.M_unp = pl->n_grp_a * IMQ_A_GROUP;
    I.M_eff = (int64_t)S.sum[0];
  } else {
    I.M_unp = M;
    I.M_eff = M;
  }
  if (b_outer) {
    cls_b0 = ncls;
    outer_classes(3, IMQ_B_GROUP, &pl->n_grp_b);
    cls_b1 = ncls;
    pl->cls_b0 = cls_b0;
    pl->cls_b1 = cls_b1;
    I.N_unp = pl->n_grp_b * IMQ_B_GROUP;
    I.N_eff = (int64_t)S.sum[3];
  } else {
    I.N_unp = N;
    I.N_eff = N;
  }
  I.ratio = (M > 0 && N > 0 && K > 0)
                ? ((double)I.M_eff / (double)M) * ((double)I.N_eff / (double)N) * ((double)I.K_eff / (double)K)
                : 1.0;

  // bound and accumulator schedule
  // k_levels sums the products' low and high 32-bit halves separately
  const unsigned __int128 bound = ((unsigned __int128)S.bound_hi << 32) + S.bound_lo;
  I.bound = (double)bound;
  const unsigned __int128 two31 = (unsigned __int128)1 << 31;
  if (bound >= ((unsigned __int128)1 << 63)) return fail(IMQ_ERR_UNSUPPORTED);  // C itself may leave int64
  I.acc_bits = bound < two31 ? 32 : 64;
  const int bm1 = b - 1;
  const unsigned __int128 R1 = ((unsigned __int128)1 << bm1) - 1;
  // Steps of one output tile, groups in descending exponent e.  A chunk accumulates consecutive groups
  // by Horner's rule in one int32 TMEM slot; after its group of exponent e the slot holds
  // sum_{e' >= e in chunk} R^(e'-e) C_e', which R^e times is a partial sum of the product, so it stays
  // below bound / R^e: a group joins the current chunk only when bound / R^e < 2^31.  A group that opens
  // a chunk needs its raw accumulator below 2^31: by its length (k_len (R-1)^2) or by the bound; when
  // neither holds it is split along K into slices of (2^31 - 1) / (R-1)^2 indices, each its own chunk.
  pl->n_steps = 0;
  pl->n_chunks = 0;
  auto below = [&](unsigned __int128 x, int sh) { return sh >= 127 ? true : (x >> sh) < two31; };
  bool open_chunk = false;
  for (int g = ng - 1; g >= 0; --g) {
    const imq_group& gr = pl->groups[g];
    const int sh = gr.e * bm1;
    const bool fits_horner = below(bound, sh);
    if (open_chunk && fits_horner) {
      // Horner step: the previous step's slot is multiplied by R^(e_prev - e)
      if (pl->n_steps >= kMaxJobs) return fail(IMQ_ERR_UNSUPPORTED);
      const int i = pl->n_steps++;
      pl->step_after[i - 1] = (pl->groups[g + 1].e - gr.e) * bm1;
      pl->step_k0[i] = gr.k_offset;
      pl->step_klen[i] = gr.k_len_padded;
      pl->step_first[i] = 0;
      pl->step_after[i] = -1;
      pl->step_drain_shift[i] = sh;
      // the drain of the chunk now happens after this step
      continue;
    }
    // a new chunk (or several K-slice chunks)
    const unsigned __int128 by_len = (unsigned __int128)gr.k_len * R1 * R1;
    int64_t slice = gr.k_len_padded;
    if (by_len >= two31 && !fits_horner) {
      slice = (int64_t)((two31 - 1) / (R1 * R1)) / IMQ_INNER_PAD * IMQ_INNER_PAD;
      if (slice < IMQ_INNER_PAD) return fail(IMQ_ERR_UNSUPPORTED);
    }
    for (int64_t k0 = 0; k0 < gr.k_len_padded; k0 += slice) {
      if (pl->n_steps >= kMaxJobs) return fail(IMQ_ERR_UNSUPPORTED);
      const int i = pl->n_steps++;
      pl->step_k0[i] = gr.k_offset + k0;
      pl->step_klen[i] = (gr.k_len_padded - k0) < slice ? (gr.k_len_padded - k0) : slice;
      pl->step_first[i] = 1;
      pl->step_after[i] = -1;
      pl->step_drain_shift[i] = sh;
      ++pl->n_chunks;
    }
    // only a chunk whose state bound allows Horner can take further groups
    open_chunk = fits_horner && slice == gr.k_len_padded;
  }
  I.workspace_bytes = align_up((size_t)(I.M_unp * I.K_unp), 1024) + align_up((size_t)(I.N_unp * I.K_unp), 1024);

  // ---- stage 2: maps ----
  size_t off2 = 0;
  const size_t o_tK = off2; off2 = align_up(off2 + (size_t)I.K_unp * 4, 256);
  const size_t o_lAk = off2; off2 = align_up(off2 + (size_t)I.K_unp, 256);
  const size_t o_lBk = off2; off2 = align_up(off2 + (size_t)I.K_unp, 256);
  const size_t o_blk = off2; off2 = align_up(off2 + (size_t)(I.K_unp / 16) * 4, 256);
  size_t o_perm = 0, o_pinv = 0, o_tJ = 0;
  if (permuted) {
    o_perm = off2; off2 = align_up(off2 + (size_t)K * 4, 256);
    o_pinv = off2; off2 = align_up(off2 + (size_t)K * 4, 256);
    o_tJ = off2; off2 = align_up(off2 + (size_t)I.K_unp * 4, 256);
  }
  size_t o_posA = 0, o_srcA = 0, o_gLA = 0, o_gNA = 0, o_posB = 0, o_srcB = 0, o_gLB = 0, o_gNB = 0;
  if (a_outer) {
    o_posA = off2; off2 = align_up(off2 + (size_t)M * 4, 256);
    o_srcA = off2; off2 = align_up(off2 + (size_t)I.M_unp * 4, 256);
    o_gLA = off2; off2 = align_up(off2 + (size_t)pl->n_grp_a * 4, 256);
    o_gNA = off2; off2 = align_up(off2 + (size_t)pl->n_grp_a * 4, 256);
  }
  if (b_outer) {
    o_posB = off2; off2 = align_up(off2 + (size_t)N * 4, 256);
    o_srcB = off2; off2 = align_up(off2 + (size_t)I.N_unp * 4, 256);
    o_gLB = off2; off2 = align_up(off2 + (size_t)pl->n_grp_b * 4, 256);
    o_gNB = off2; off2 = align_up(off2 + (size_t)pl->n_grp_b * 4, 256);
  }
  char* b2 = nullptr;
  if (cudaMallocFromPoolAsync((void**)&b2, off2 > 0 ? off2 : 256, ds->pool, st) != cudaSuccess)
    return fail(IMQ_ERR_CUDA);
  pl->dev_block2 = b2;
  pl->dev_bytes += off2;
  InnerSeg* dsegs = reinterpret_cast<InnerSeg*>(blk1 + o_segs);
  OuterClass* dcls = reinterpret_cast<OuterClass*>(blk1 + o_cls);
  pl->tK = reinterpret_cast<int32_t*>(b2 + o_tK);
  pl->lAk = reinterpret_cast<int8_t*>(b2 + o_lAk);
  pl->lBk = reinterpret_cast<int8_t*>(b2 + o_lBk);
  pl->blk16 = reinterpret_cast<int32_t*>(b2 + o_blk);
  pl->perm = permuted ? reinterpret_cast<int32_t*>(b2 + o_perm) : nullptr;
  pl->pinv = permuted ? reinterpret_cast<int32_t*>(b2 + o_pinv) : nullptr;
  pl->tJ = permuted ? reinterpret_cast<int32_t*>(b2 + o_tJ) : pl->tK;
  if (a_outer) {
    pl->posA = reinterpret_cast<int32_t*>(b2 + o_posA);
    pl->srcA = reinterpret_cast<int32_t*>(b2 + o_srcA);
    pl->grpA_L = reinterpret_cast<int32_t*>(b2 + o_gLA);
    pl->grpA_n = reinterpret_cast<int32_t*>(b2 + o_gNA);
  }
  if (b_outer) {
    pl->posB = reinterpret_cast<int32_t*>(b2 + o_posB);
    pl->srcB = reinterpret_cast<int32_t*>(b2 + o_srcB);
    pl->grpB_L = reinterpret_cast<int32_t*>(b2 + o_gLB);
    pl->grpB_n = reinterpret_cast<int32_t*>(b2 + o_gNB);
  }
  if (ng > 0 || ncls > 0) {
    MapsArgs m;
    const int nE = (maxla + 1) * ew;
    m.inline_tables = (nseg <= kParamSegs && ncls <= kParamCls && ng <= kParamGrps && nE <= kParamE) ? 1 : 0;
    if (m.inline_tables) {
      memcpy(m.t.segs, hsegs, sizeof(InnerSeg) * (size_t)nseg);
      memcpy(m.t.cls, hcls, sizeof(OuterClass) * (size_t)ncls);
      memcpy(m.t.grps, hgrps, sizeof(InnerGroup) * (size_t)ng);
      memcpy(m.t.E, hE, sizeof(int32_t) * (size_t)nE);
    } else {
      // one upload from pinned staging (an asynchronous copy; pageable memory would be staged by the
      // driver first); the staging is reused once the previous plan's upload has completed
      if (cudaEventSynchronize(pin.tables_done) != cudaSuccess) return fail(IMQ_ERR_CUDA);
      char* stg = static_cast<char*>(pin.tables);
      memcpy(stg, hsegs, sizeof(InnerSeg) * (size_t)nseg);
      memcpy(stg + (o_cls - o_segs), hcls, sizeof(OuterClass) * (size_t)ncls);
      memcpy(stg + (o_grps - o_segs), hgrps, sizeof(InnerGroup) * (size_t)ng);
      memcpy(stg + (o_E - o_segs), hE, sizeof(int32_t) * (size_t)nE);
      if (cudaMemcpyAsync(dsegs, stg, (o_E - o_segs) + sizeof(int32_t) * (size_t)nE, cudaMemcpyHostToDevice,
                          st) != cudaSuccess ||
          cudaEventRecord(pin.tables_done, st) != cudaSuccess)
        return fail(IMQ_ERR_CUDA);
    }
    m.grps = reinterpret_cast<const InnerGroup*>(blk1 + o_grps);
    m.cls = dcls;
    m.ngrp = ng;
    m.segs = dsegs;
    m.E = reinterpret_cast<const int32_t*>(blk1 + o_E);
    m.ew = ew;
    m.maxla = maxla;
    m.maxlb = maxlb;
    m.lva = pl->lv_a_col;
    m.lvb = pl->lv_b_row;
    m.a_inner = a_inner;
    m.b_inner = b_inner;
    m.K = K;
    m.perm = pl->perm;
    m.pinv = pl->pinv;
    m.tK = pl->tK;
    m.tJ = pl->tJ;
    m.lAk = pl->lAk;
    m.lBk = pl->lBk;
    m.blk16 = pl->blk16;
    m.a = {cls_a0, a_outer ? cls_a1 - cls_a0 : 0, pl->lv_a_row, M, IMQ_A_GROUP, pl->posA, pl->srcA,
           pl->grpA_L, pl->grpA_n};
    m.b = {cls_b0, b_outer ? cls_b1 - cls_b0 : 0, pl->lv_b_col, N, IMQ_B_GROUP, pl->posB, pl->srcB,
           pl->grpB_L, pl->grpB_n};
    const int blocks = ng + m.a.ncls + m.b.ncls;
    if (job.batched && kBatchMaps) {
      job.has_maps = true;
      job.order_blocks = permuted ? maxla * maxlb : 0;
      job.maps_blocks = blocks;
      job.maps = m;
    } else {
      if (permuted) k_plan_order<<<maxla * maxlb, 1024, 0, st>>>(m);
      if (blocks > 0) k_plan_maps<<<blocks, 1024, 0, st>>>(m);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return fail(IMQ_ERR_CUDA);
#ifdef IMQ_DEBUG
  {
    // the exponent groups on the host: contiguous, padded to IMQ_INNER_PAD, filling K_unp
    int64_t next = 0;
    for (int g = 0; g < ng; ++g) {
      const imq_group& gr = pl->groups[g];
      if (gr.k_offset != next || gr.k_len > gr.k_len_padded || gr.k_len_padded % IMQ_INNER_PAD ||
          gr.k_len_padded - gr.k_len >= IMQ_INNER_PAD)
        return fail(IMQ_ERR_BOUNDS);
      next += gr.k_len_padded;
    }
    if (next != I.K_unp) return fail(IMQ_ERR_BOUNDS);
    CheckArgs c;
    memset(&c, 0, sizeof(c));
    c.K = K;
    c.K_unp = I.K_unp;
    c.a_inner = a_inner;
    c.b_inner = b_inner;
    c.lva = pl->lv_a_col;
    c.lvb = pl->lv_b_row;
    c.tK = pl->tK;
    c.tJ = pl->tJ;
    c.perm = pl->perm;
    c.pinv = pl->pinv;
    c.lAk = pl->lAk;
    c.lBk = pl->lBk;
    c.blk16 = pl->blk16;
    c.ng = ng;
    for (int g = 0; g < ng; ++g)
      c.grp[g] = CheckGroup{pl->groups[g].k_offset, pl->groups[g].k_len, pl->groups[g].k_len_padded, pl->groups[g].e};
    c.o[0] = CheckOuter{a_outer ? 1 : 0, M, I.M_unp, pl->n_grp_a, pl->lv_a_row, pl->posA, pl->srcA, pl->grpA_L,
                        pl->grpA_n};
    c.o[1] = CheckOuter{b_outer ? 1 : 0, N, I.N_unp, pl->n_grp_b, pl->lv_b_col, pl->posB, pl->srcB, pl->grpB_L,
                        pl->grpB_n};
    c.status = ds->status;
    k_plan_check<<<(unsigned)ds->num_sms, 256, 0, st>>>(c);
    if (cudaGetLastError() != cudaSuccess) return fail(IMQ_ERR_CUDA);
  }
#endif
  *out = pl;
  return IMQ_OK;
}

imq_status build_plans(int batch, const void* A, int64_t strideA, const void* B, int64_t strideB, imq_dtype it,
                       int64_t M, int64_t K, int64_t N, int32_t transA, int64_t lda, int32_t transB, int64_t ldb,
                       int32_t b, imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                       const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** out, cudaStream_t st);

// Stage 1 of a batch of plans: the summaries and column maxima cleared, the line maxima, the level
// kernels -- one launch each for the whole batch.
imq_status launch_stage1_batch(std::vector<PlanJob>& jobs, imq_dtype it, DeviceState* ds, cudaStream_t st) {
  std::vector<ZeroSpan> zero;
  std::vector<LineMaxJob> lm;
  std::vector<LevelArgs> la;
  std::vector<int> nblk;
  int64_t max_rows = 1, max_cols = 0;
  int max_blk = 1;
  int64_t max_bytes = 16;
  for (PlanJob& j : jobs) {
    for (int q = 0; q < j.nzero; ++q) {
      zero.push_back(j.zero[q]);
      max_bytes = j.zero[q].bytes > max_bytes ? j.zero[q].bytes : max_bytes;
    }
    for (int q = 0; q < j.nlm; ++q) {
      lm.push_back(j.lm[q]);
      max_rows = j.lm[q].rows > max_rows ? j.lm[q].rows : max_rows;
      max_cols = j.lm[q].cols > max_cols ? j.lm[q].cols : max_cols;
    }
    la.push_back(j.la);
    nblk.push_back((int)j.la.nblk);
    max_blk = (int)j.la.nblk > max_blk ? (int)j.la.nblk : max_blk;
  }
  void* dz = nullptr;
  void* dl = nullptr;
  void* da = nullptr;
  void* dn = nullptr;
  imq_status s = upload_table(zero.data(), sizeof(ZeroSpan) * zero.size(), &dz, st);
  if (s == IMQ_OK && !lm.empty()) s = upload_table(lm.data(), sizeof(LineMaxJob) * lm.size(), &dl, st);
  if (s == IMQ_OK) s = upload_table(la.data(), sizeof(LevelArgs) * la.size(), &da, st);
  if (s == IMQ_OK) s = upload_table(nblk.data(), sizeof(int) * nblk.size(), &dn, st);
  if (s == IMQ_OK) {
    const int64_t zb = (max_bytes / 16 + 255) / 256;
    k_zero_batch<<<dim3((unsigned)(zb < 64 ? zb : 64), (unsigned)zero.size()), 256, 0, st>>>(
        static_cast<const ZeroSpan*>(dz));
    if (!lm.empty()) {
      // about eight blocks per SM over the whole batch, at most one per row
      int64_t gx = ((int64_t)ds->num_sms * 8 + (int64_t)lm.size() - 1) / (int64_t)lm.size();
      if (gx > max_rows) gx = max_rows;
      const size_t smem = (size_t)max_cols * 4;
      const dim3 g((unsigned)gx, (unsigned)lm.size());
      if (it == IMQ_I16) {
        if (ensure_smem(reinterpret_cast<const void*>(k_line_max_batch<int16_t>), smem) != cudaSuccess) s = IMQ_ERR_CUDA;
        else k_line_max_batch<int16_t><<<g, 256, smem, st>>>(static_cast<const LineMaxJob*>(dl));
      } else {
        if (ensure_smem(reinterpret_cast<const void*>(k_line_max_batch<int32_t>), smem) != cudaSuccess) s = IMQ_ERR_CUDA;
        else k_line_max_batch<int32_t><<<g, 256, smem, st>>>(static_cast<const LineMaxJob*>(dl));
      }
    }
    if (s == IMQ_OK)
      k_levels_batch<<<dim3((unsigned)max_blk, (unsigned)la.size()), 256, 0, st>>>(static_cast<const LevelArgs*>(da),
                                                                                  static_cast<const int*>(dn));
    if (cudaGetLastError() != cudaSuccess) s = IMQ_ERR_CUDA;
  }
  for (void* p : {dz, dl, da, dn})
    if (p) cudaFreeAsync(p, st);
  return s;
}

// Stage 2 of a batch of plans: the order kernels, then the maps kernels, one launch each per 64 plans (the
// argument table of 64 plans stays within one staging buffer of the upload).
imq_status launch_stage2_batch(std::vector<PlanJob>& jobs, cudaStream_t st) {
  std::vector<MapsArgs> all;
  std::vector<int> order_blocks, maps_blocks;
  for (PlanJob& j : jobs) {
    if (!j.has_maps) continue;
    all.push_back(j.maps);
    order_blocks.push_back(j.order_blocks);
    maps_blocks.push_back(j.maps_blocks);
  }
  constexpr size_t kChunk = 64;
  for (size_t c0 = 0; c0 < all.size(); c0 += kChunk) {
    const size_t n = all.size() - c0 < kChunk ? all.size() - c0 : kChunk;
    int max_order = 0, max_maps = 0;
    for (size_t i = c0; i < c0 + n; ++i) {
      max_order = order_blocks[i] > max_order ? order_blocks[i] : max_order;
      max_maps = maps_blocks[i] > max_maps ? maps_blocks[i] : max_maps;
    }
    if (max_order == 0 && max_maps == 0) continue;
    void* dt = nullptr;
    imq_status s = upload_table(all.data() + c0, sizeof(MapsArgs) * n, &dt, st);
    if (s != IMQ_OK) return s;
    const MapsArgs* t = static_cast<const MapsArgs*>(dt);
    if (max_order > 0) k_plan_order_batch<<<dim3((unsigned)max_order, (unsigned)n), 1024, 0, st>>>(t);
    if (max_maps > 0) k_plan_maps_batch<<<dim3((unsigned)max_maps, (unsigned)n), 1024, 0, st>>>(t);
    s = cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
    cudaFreeAsync(dt, st);
    if (s != IMQ_OK) return s;
  }
  return IMQ_OK;
}

// See internal.h.
bool b_group_positions(const imq_plan_t* pl, std::vector<float>* pos) {
  if (!(pl->info.dir_b & IMQ_DIR_OUTER) || pl->n_grp_b <= 0 || !pl->host_tables) return false;
  const InnerSeg* hsegs = static_cast<const InnerSeg*>(pl->host_tables);
  const OuterClass* hcls = reinterpret_cast<const OuterClass*>(hsegs + kLv * kLv);
  pos->assign((size_t)pl->n_grp_b, 0.0f);
  for (int c = pl->cls_b0; c < pl->cls_b1; ++c) {
    const OuterClass& k = hcls[c];
    const int64_t ng = (k.count + k.per - 1) / k.per;
    for (int64_t g = 0; g < ng && k.grp0 + g < pl->n_grp_b; ++g) {
      const double first = (double)(g * k.per), n_in = (double)(g < ng - 1 ? k.per : k.count - (ng - 1) * k.per);
      (*pos)[(size_t)(k.grp0 + g)] = (float)((first + 0.5 * n_in) / (double)k.count);
    }
  }
  return true;
}

// Builds a plan; see imq_plan in include/imq.h.
imq_status build_plan(const void* A, const void* B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                      int32_t transA, int64_t lda, int32_t transB, int64_t ldb, int32_t b,
                      imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                      const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** out,
                      cudaStream_t st) {
  const int64_t sa = 0, sb = 0;
  return build_plans(1, A, sa, B, sb, it, M, K, N, transA, lda, transB, ldb, b, strategy, a_rowmax, a_colmax,
                     b_rowmax, b_colmax, out, st);
}

// Plans of `batch` equal-shaped problems: problem h reads A + h * strideA, B + h * strideB (elements)
// and the maxima vectors at h times their lengths.  Every stage 1 is queued first, then the summaries
// are waited for together, then every stage 2 runs: one host round trip for the whole batch.
imq_status build_plans(int batch, const void* A, int64_t strideA, const void* B, int64_t strideB, imq_dtype it,
                       int64_t M, int64_t K, int64_t N, int32_t transA, int64_t lda, int32_t transB, int64_t ldb,
                       int32_t b, imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                       const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** out, cudaStream_t st) {
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  int dev;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  Pinned& pin = g_pinned[dev & 63];
  std::lock_guard<std::mutex> lock(pin.mu);
  s = pinned_ready(pin, batch);
  if (s != IMQ_OK) return s;
  const size_t esz = it == IMQ_I16 ? 2 : 4;
  const bool have_max = a_rowmax && a_colmax && b_rowmax && b_colmax;
  std::vector<PlanJob> jobs((size_t)batch);
  for (int h = 0; h < batch; ++h) out[h] = nullptr;
  auto drop = [&](int upto, imq_status e) {
    // level kernels already queued write into the pinned summary slots: let them finish first
    cudaStreamSynchronize(st);
    for (int h = 0; h < upto; ++h)
      if (jobs[h].pl) plan_fail(jobs[h].pl, e, st);
    for (int h = 0; h < batch; ++h)
      if (out[h]) {
        imq_plan_destroy(out[h]);
        out[h] = nullptr;
      }
    return e;
  };
  // A batch queues each kind of plan kernel once for all its plans (the hybrid's choice kernels stay per
  // plan; the debug build's index checks follow each plan's maps, so there stage 2 stays per plan too).
  // (up to 256 plans: their stage-1 argument tables stay within one staging buffer of the upload)
  const bool batched = batch > 1 && batch <= 256 && strategy != IMQ_HYBRID &&
                       (have_max || (M <= 32768 && K <= 32768 && N <= 32768));
  for (int h = 0; h < batch; ++h) {
    PlanJob& j = jobs[h];
    j.batched = batched;
    j.A = static_cast<const char*>(A) + (size_t)h * strideA * esz;
    j.B = static_cast<const char*>(B) + (size_t)h * strideB * esz;
    j.it = it;
    j.M = M;
    j.K = K;
    j.N = N;
    j.transA = transA;
    j.lda = lda;
    j.transB = transB;
    j.ldb = ldb;
    j.b = b;
    j.strategy = strategy;
    j.a_rowmax = have_max ? a_rowmax + (size_t)h * M : nullptr;
    j.a_colmax = have_max ? a_colmax + (size_t)h * K : nullptr;
    j.b_rowmax = have_max ? b_rowmax + (size_t)h * K : nullptr;
    j.b_colmax = have_max ? b_colmax + (size_t)h * N : nullptr;
    j.slot = h;
    s = plan_begin(j, pin, ds, dev, st);
    if (s != IMQ_OK) return drop(h, s);
  }
  if (batched) {
    s = launch_stage1_batch(jobs, it, ds, st);
    if (s != IMQ_OK) return drop(batch, s);
  }
  std::vector<Summary> sums((size_t)batch);
  for (int h = 0; h < batch; ++h) {
    s = plan_wait(jobs[h], pin, st, &sums[h]);
    if (s != IMQ_OK) return drop(batch, s);
  }
  for (int h = 0; h < batch; ++h) {
    s = plan_finish(jobs[h], sums[h], pin, ds, st, &out[h]);
    if (s != IMQ_OK) return drop(batch, s);
  }
  if (batched) {
    s = launch_stage2_batch(jobs, st);
    if (s != IMQ_OK) return drop(batch, s);
  }
  return IMQ_OK;
}

}  // namespace imq
