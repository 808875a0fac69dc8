// rtn.cu -- percentile selection and round-to-nearest quantisation (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Problem" / "Approach" and the measured-effects rows on beta and p.  The scale of a group
// maps its nearest-rank p-quantile q of |x| to beta; entries are rounded to the nearest integer
// (ties to even) after one fp32 multiply and are NOT clipped, so heavy hitters stay far outside
// +-beta.  q is found exactly by a radix select on the order-preserving bit keys of |x| (the IEEE bit
// pattern of a non-negative float orders like an unsigned integer), 8 key bits per pass from the top.
//
// Kernels
//   k_rtn_rows    one CTA per stored row (grid-stride): the row is staged in shared memory once, the
//                 select passes and the quantisation read it from there (one HBM read, one write).
//                 Also used for per-tensor groups with the scale taken from the tensor select.
//   k_rtn_cols    one CTA per 16 stored columns: histograms per column in shared memory, the column
//                 slab is streamed once per pass (re-reads hit L2) and once more to quantise.
//   k_tensor_*    per-tensor select: global 256-bin histograms per pass, then k_rtn_rows.
// Side outputs: max |x_int| per stored row and column, the line statistics the unpack plan needs.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

constexpr int kThreads = 256;
constexpr int kColsPerCta = 16;

struct TensorState {
  unsigned long long krem;  // rank still to be found (1-based) inside the current prefix
  uint32_t prefix, mask;    // key bits fixed so far
  uint32_t maxkey, nonfinite;
  float s, delta, q;
  uint32_t pad_;
  uint32_t hist[256];
};

template <typename T>
struct Key;
template <>
struct Key<uint16_t> {  // bfloat16 bit patterns
  static constexpr int kBits = 15;
  static constexpr uint32_t kInf = 0x7F80u;
  __device__ static uint32_t key(uint16_t u) { return u & 0x7FFFu; }
  __device__ static float value(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }
  __device__ static float from_key(uint32_t k) { return __uint_as_float(k << 16); }
};
template <>
struct Key<uint32_t> {  // float32 bit patterns
  static constexpr int kBits = 31;
  static constexpr uint32_t kInf = 0x7F800000u;
  __device__ static uint32_t key(uint32_t u) { return u & 0x7FFFFFFFu; }
  __device__ static float value(uint32_t u) { return __uint_as_float(u); }
  __device__ static float from_key(uint32_t k) { return __uint_as_float(k); }
};

__host__ __device__ constexpr int num_passes(int bits) { return (bits + 7) / 8; }
__device__ __forceinline__ int pass_shift(int bits, int i) {
  const int s = bits - 8 * (i + 1);
  return s > 0 ? s : 0;
}
__device__ __forceinline__ uint32_t pass_width_mask(int bits, int i) {
  const int hi = bits - 8 * i;
  return (1u << (hi - pass_shift(bits, i))) - 1u;
}

// One warp.  Finds the smallest bucket d with hist[0] + ... + hist[d] >= k (hist has 256 buckets,
// `stride` words apart).  Lane 0 returns true and writes d and the count of keys below bucket d.
__device__ bool warp_select(const uint32_t* hist, int stride, unsigned long long k, int* d_out,
                            unsigned long long* below_out) {
  const int lane = threadIdx.x & 31;
  uint32_t c[8];
  unsigned long long local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = hist[(lane * 8 + j) * stride];
    local += c[j];
  }
  unsigned long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const unsigned long long excl = incl - local;
  const unsigned ball = __ballot_sync(0xffffffffu, excl < k && k <= incl);
  const int src = ball ? __ffs(ball) - 1 : 31;
  int d = 255;
  unsigned long long below = 0;
  if (lane == src) {
    unsigned long long cum = excl;
    d = lane * 8 + 7;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (cum + c[j] >= k) {
        d = lane * 8 + j;
        break;
      }
      cum += c[j];
    }
    below = cum;
  }
  d = __shfl_sync(0xffffffffu, d, src);
  below = __shfl_sync(0xffffffffu, below, src);
  if (lane == 0) {
    *d_out = d;
    *below_out = below;
  }
  return lane == 0;
}

__device__ __forceinline__ void scale_from_q(float q, float qmax, int beta, float* s, float* d) {
  if (q == 0.0f) q = qmax;
  if (q == 0.0f) {
    *s = 1.0f;
    *d = 1.0f;
  } else {
    *s = __fdiv_rn((float)beta, q);
    *d = __fdiv_rn(q, (float)beta);
  }
}

// Quantises one value; returns |v| (0 on a range error, which is recorded).
template <bool kOut16>
__device__ __forceinline__ uint32_t quant_one(float x, float s, void* out, int64_t idx, int32_t* status) {
  const float y = __fmul_rn(x, s);
  int32_t v = 0;
  if (fabsf(y) < 2147483648.0f) {
    v = __float2int_rn(y);
  } else {
    set_status(status, IMQ_ERR_RANGE);
  }
  uint32_t a = v < 0 ? (uint32_t)(-(int64_t)v) : (uint32_t)v;
  if (kOut16) {
    if (a > 32767u) {
      set_status(status, IMQ_ERR_RANGE);
      v = 0;
      a = 0;
    }
    static_cast<int16_t*>(out)[idx] = (int16_t)v;
  } else {
    static_cast<int32_t*>(out)[idx] = v;
  }
  return a;
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  uint32_t r = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, red[w]);
  return r;
}

// ------------------------------------------------------------------------------------------------
// per stored row (kSelect) or per tensor (scale from the tensor state)
// ------------------------------------------------------------------------------------------------
template <typename T, bool kSelect, bool kOut16>
__global__ void __launch_bounds__(kThreads) k_rtn_rows(
    const T* __restrict__ X, int64_t rows, int64_t cols, int64_t ld, unsigned long long krank, int beta,
    void* __restrict__ Xint, int64_t ldq, float* __restrict__ delta, float* __restrict__ qval,
    int32_t* __restrict__ rowmax, int32_t* __restrict__ colmax, const TensorState* __restrict__ ts,
    int vec, int32_t* status) {
  extern __shared__ __align__(16) unsigned char dsm[];
  T* row = reinterpret_cast<T*>(dsm);
  const int64_t row_bytes = (cols * (int64_t)sizeof(T) + 15) / 16 * 16;
  uint32_t* cmax = reinterpret_cast<uint32_t*>(dsm + row_bytes);
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[kThreads / 32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ unsigned long long s_k;
  __shared__ float s_s;
  __shared__ int s_ok;
  const int tid = threadIdx.x;
  constexpr int V = 16 / sizeof(T);

  if (colmax)
    for (int64_t c = tid; c < cols; c += kThreads) cmax[c] = 0;

  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* xr = X + r * ld;
    uint32_t mk = 0, bad = 0;
    if (vec) {
      const uint4* src = reinterpret_cast<const uint4*>(xr);
      uint4* dst = reinterpret_cast<uint4*>(row);
      for (int64_t c = tid; c < cols / V; c += kThreads) {
        const uint4 w = __ldcs(src + c);
        dst[c] = w;
        const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const uint32_t k = Key<T>::key(e[j]);
          mk = max(mk, k);
          bad |= (k >= Key<T>::kInf);
        }
      }
    } else {
      for (int64_t c = tid; c < cols; c += kThreads) {
        const T u = xr[c];
        row[c] = u;
        const uint32_t k = Key<T>::key(u);
        mk = max(mk, k);
        bad |= (k >= Key<T>::kInf);
      }
    }
    mk = block_max_u32(mk, red);
    bad = block_max_u32(bad, red);

    if (kSelect) {
      if (tid == 0) {
        s_prefix = 0;
        s_mask = 0;
        s_k = krank;
      }
      for (int pass = 0; pass < num_passes(Key<T>::kBits); ++pass) {
        hist[tid] = 0;
        __syncthreads();
        const uint32_t pre = s_prefix, msk = s_mask;
        const int sh = pass_shift(Key<T>::kBits, pass);
        for (int64_t c = tid; c < cols; c += kThreads) {
          const uint32_t k = Key<T>::key(row[c]);
          if ((k & msk) == pre) atomicAdd(&hist[(k >> sh) & 0xFFu], 1u);
        }
        __syncthreads();
        if (tid < 32) {
          int d;
          unsigned long long below;
          if (warp_select(hist, 1, s_k, &d, &below)) {
            s_prefix = pre | ((uint32_t)d << sh);
            s_mask = msk | (pass_width_mask(Key<T>::kBits, pass) << sh);
            s_k -= below;
          }
        }
        __syncthreads();
      }
    }
    if (tid == 0) {
      float s, d;
      if (kSelect) {
        const float q = Key<T>::from_key(s_prefix);
        scale_from_q(q, Key<T>::from_key(mk), beta, &s, &d);
        delta[r] = d;
        if (qval) qval[r] = q;
      } else {
        s = ts->s;
      }
      if (bad) set_status(status, IMQ_ERR_NONFINITE);
      s_s = s;
      s_ok = !bad;
    }
    __syncthreads();
    const float s = s_s;
    uint32_t rmx = 0;
    if (s_ok) {
      for (int64_t c = tid; c < cols; c += kThreads) {
        const uint32_t a = quant_one<kOut16>(Key<T>::value(row[c]), s, Xint, r * ldq + c, status);
        rmx = max(rmx, a);
        if (colmax) cmax[c] = max(cmax[c], a);
      }
    }
    rmx = block_max_u32(rmx, red);
    if (tid == 0 && rowmax) rowmax[r] = (int32_t)rmx;
    __syncthreads();
  }
  if (colmax) {
    __syncthreads();
    for (int64_t c = tid; c < cols; c += kThreads)
      if (cmax[c]) atomicMax(colmax + c, (int32_t)cmax[c]);
  }
}

// ------------------------------------------------------------------------------------------------
// per stored column: one CTA per kColsPerCta columns
// ------------------------------------------------------------------------------------------------
template <typename T, bool kOut16>
__global__ void __launch_bounds__(kThreads) k_rtn_cols(
    const T* __restrict__ X, int64_t rows, int64_t cols, int64_t ld, unsigned long long krank, int beta,
    void* __restrict__ Xint, int64_t ldq, float* __restrict__ delta, float* __restrict__ qval,
    int32_t* __restrict__ rowmax, int32_t* __restrict__ colmax, int32_t* status) {
  constexpr int CW = kColsPerCta;
  constexpr int RS = kThreads / CW;  // rows per sweep
  __shared__ uint32_t hist[256 * CW];  // [bucket][column]
  __shared__ uint32_t s_prefix[CW], s_mask[CW], s_maxkey[CW], s_cmax[CW];
  __shared__ unsigned long long s_k[CW];
  __shared__ float s_s[CW];
  __shared__ uint32_t s_bad;
  const int tid = threadIdx.x, cc = tid % CW, rsub = tid / CW;
  const int64_t c = (int64_t)blockIdx.x * CW + cc;
  const bool cval = c < cols;
  if (tid < CW) {
    s_prefix[tid] = 0;
    s_mask[tid] = 0;
    s_maxkey[tid] = 0;
    s_cmax[tid] = 0;
    s_k[tid] = krank;
  }
  if (tid == 0) s_bad = 0;
  for (int pass = 0; pass < num_passes(Key<T>::kBits); ++pass) {
    for (int i = tid; i < 256 * CW; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t pre = s_prefix[cc], msk = s_mask[cc];
    const int sh = pass_shift(Key<T>::kBits, pass);
    uint32_t mk = 0, bad = 0;
    if (cval) {
      for (int64_t r = rsub; r < rows; r += RS) {
        const uint32_t k = Key<T>::key(X[r * ld + c]);
        if (pass == 0) {
          mk = max(mk, k);
          bad |= (k >= Key<T>::kInf);
        }
        if ((k & msk) == pre) atomicAdd(&hist[((k >> sh) & 0xFFu) * CW + cc], 1u);
      }
    }
    if (pass == 0) {
      if (mk) atomicMax(&s_maxkey[cc], mk);
      if (bad) atomicOr(&s_bad, 1u);
    }
    __syncthreads();
    const int warp = tid >> 5;
    for (int col = warp; col < CW; col += kThreads / 32) {
      int d;
      unsigned long long below;
      if (warp_select(hist + col, CW, s_k[col], &d, &below)) {
        s_prefix[col] = s_prefix[col] | ((uint32_t)d << sh);
        s_mask[col] = s_mask[col] | (pass_width_mask(Key<T>::kBits, pass) << sh);
        s_k[col] -= below;
      }
    }
    __syncthreads();
  }
  if (tid < CW && (int64_t)blockIdx.x * CW + tid < cols) {
    const int64_t cg = (int64_t)blockIdx.x * CW + tid;
    float s, d;
    const float q = Key<T>::from_key(s_prefix[tid]);
    scale_from_q(q, Key<T>::from_key(s_maxkey[tid]), beta, &s, &d);
    delta[cg] = d;
    if (qval) qval[cg] = q;
    s_s[tid] = s;
  }
  if (tid == 0 && s_bad) set_status(status, IMQ_ERR_NONFINITE);
  __syncthreads();
  if (s_bad) return;
  const float s = s_s[cc];
  uint32_t cmx = 0;
  for (int64_t r0 = 0; r0 < rows; r0 += RS) {
    const int64_t r = r0 + rsub;
    uint32_t a = 0;
    if (cval && r < rows) {
      a = quant_one<kOut16>(Key<T>::value(X[r * ld + c]), s, Xint, r * ldq + c, status);
      cmx = max(cmx, a);
    }
    // max over the CW columns of this row (CW consecutive lanes)
#pragma unroll
    for (int o = CW / 2; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (rowmax && cc == 0 && r < rows && a) atomicMax(rowmax + r, (int32_t)a);
  }
  atomicMax(&s_cmax[cc], cmx);
  __syncthreads();
  if (colmax && tid < CW && (int64_t)blockIdx.x * CW + tid < cols)
    colmax[(int64_t)blockIdx.x * CW + tid] = (int32_t)s_cmax[tid];
}

// ------------------------------------------------------------------------------------------------
// per tensor
// ------------------------------------------------------------------------------------------------
__global__ void k_tensor_init(TensorState* ts, unsigned long long k) {
  uint32_t* w = reinterpret_cast<uint32_t*>(ts);
  for (int i = threadIdx.x; i < (int)(sizeof(TensorState) / 4); i += blockDim.x) w[i] = 0;
  __syncthreads();
  if (threadIdx.x == 0) ts->krem = k;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_tensor_hist(const T* __restrict__ X, int64_t rows,
                                                          int64_t cols, int64_t ld, TensorState* ts,
                                                          int pass) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[kThreads / 32];
  const int tid = threadIdx.x;
  hist[tid] = 0;
  __syncthreads();
  const uint32_t pre = ts->prefix, msk = ts->mask;
  const int sh = pass_shift(Key<T>::kBits, pass);
  uint32_t mk = 0, bad = 0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* xr = X + r * ld;
    for (int64_t c = tid; c < cols; c += kThreads) {
      const uint32_t k = Key<T>::key(xr[c]);
      if (pass == 0) {
        mk = max(mk, k);
        bad |= (k >= Key<T>::kInf);
      }
      if ((k & msk) == pre) atomicAdd(&hist[(k >> sh) & 0xFFu], 1u);
    }
  }
  __syncthreads();
  if (hist[tid]) atomicAdd(&ts->hist[tid], hist[tid]);
  if (pass == 0) {
    mk = block_max_u32(mk, red);
    bad = block_max_u32(bad, red);
    if (tid == 0) {
      if (mk) atomicMax(&ts->maxkey, mk);
      if (bad) atomicOr(&ts->nonfinite, 1u);
    }
  }
}

template <typename T>
__global__ void k_tensor_select(TensorState* ts, int pass, int last, int beta, float* delta,
                                float* qval, int32_t* status) {
  int d;
  unsigned long long below;
  const int sh = pass_shift(Key<T>::kBits, pass);
  const bool lead = warp_select(ts->hist, 1, ts->krem, &d, &below);
  __syncwarp();
  for (int i = threadIdx.x; i < 256; i += 32) ts->hist[i] = 0;
  if (lead) {
    ts->prefix |= (uint32_t)d << sh;
    ts->mask |= pass_width_mask(Key<T>::kBits, pass) << sh;
    ts->krem -= below;
    if (last) {
      const float q = Key<T>::from_key(ts->prefix);
      float s, dl;
      scale_from_q(q, Key<T>::from_key(ts->maxkey), beta, &s, &dl);
      ts->s = s;
      ts->delta = dl;
      ts->q = q;
      delta[0] = dl;
      if (qval) qval[0] = q;
      if (ts->nonfinite) {
        set_status(status, IMQ_ERR_NONFINITE);
        ts->s = 0.0f;
      }
    }
  }
}

__global__ void k_fill_f32(float* p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

int64_t nearest_rank(int64_t n, double p) {
  if (n <= 0) return 1;
  int64_t k = (int64_t)ceil(p * (double)n);
  if (k < 1) k = 1;
  if (k > n) k = n;
  return k;
}

template <typename T, bool kOut16>
imq_status run(const T* X, int64_t rows, int64_t cols, int64_t ld, imq_gran g, double p,
               int32_t beta, void* Xint, int64_t ldq, float* delta, float* qval, int32_t* rowmax,
               int32_t* colmax, DeviceState* ds, cudaStream_t st) {
  const int sms = ds->num_sms;
  if (g == IMQ_PER_COL) {
    const unsigned long long k = (unsigned long long)nearest_rank(rows, p);
    const int64_t grid = (cols + kColsPerCta - 1) / kColsPerCta;
    k_rtn_cols<T, kOut16><<<(unsigned)grid, kThreads, 0, st>>>(X, rows, cols, ld, k, beta, Xint, ldq,
                                                               delta, qval, rowmax, colmax, ds->status);
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  // staged rows
  const size_t row_bytes = (size_t)((cols * (int64_t)sizeof(T) + 15) / 16 * 16);
  const size_t smem = row_bytes + (colmax ? (size_t)cols * 4 : 0);
  if (smem > 200 * 1024) return IMQ_ERR_UNSUPPORTED;
  const bool vec = (cols % (16 / (int64_t)sizeof(T)) == 0) && (ld % (16 / (int64_t)sizeof(T)) == 0) &&
                   ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  int per_sm = (int)((200 * 1024) / (smem + 2048));
  if (per_sm > 8) per_sm = 8;
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = rows < (int64_t)sms * per_sm ? rows : (int64_t)sms * per_sm;
  if (g == IMQ_PER_ROW) {
    auto kern = k_rtn_rows<T, true, kOut16>;
    IMQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<(unsigned)grid, kThreads, smem, st>>>(X, rows, cols, ld,
                                                 (unsigned long long)nearest_rank(cols, p), beta, Xint, ldq,
                                                 delta, qval, rowmax, colmax, nullptr, vec, ds->status);
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  // per tensor
  if (!ds->scratch) IMQ_CUDA_TRY(cudaMalloc(&ds->scratch, sizeof(TensorState)));
  TensorState* ts = static_cast<TensorState*>(ds->scratch);
  k_tensor_init<<<1, 256, 0, st>>>(ts, (unsigned long long)nearest_rank(rows * cols, p));
  const int64_t hgrid = rows < (int64_t)sms * 8 ? rows : (int64_t)sms * 8;
  const int np = num_passes(Key<T>::kBits);
  for (int pass = 0; pass < np; ++pass) {
    k_tensor_hist<T><<<(unsigned)hgrid, kThreads, 0, st>>>(X, rows, cols, ld, ts, pass);
    k_tensor_select<T><<<1, 32, 0, st>>>(ts, pass, pass == np - 1, beta, delta, qval, ds->status);
  }
  auto kern = k_rtn_rows<T, false, kOut16>;
  IMQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  kern<<<(unsigned)grid, kThreads, smem, st>>>(X, rows, cols, ld, 0ull, beta, Xint, ldq, delta, qval,
                                               rowmax, colmax, ts, vec, ds->status);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

}  // namespace

imq_status launch_rtn_quantize(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               imq_gran g, double p, int32_t beta, void* Xint, imq_dtype it,
                               int64_t ldq, float* delta, float* qval, int32_t* rowmax,
                               int32_t* colmax, cudaStream_t st) {
  if (rows < 0 || cols < 0 || ld < cols || ldq < cols || !(p > 0.0 && p <= 1.0) || beta < 1 ||
      beta > (1 << 24))
    return IMQ_ERR_ARG;
  if (xt != IMQ_F32 && xt != IMQ_BF16) return IMQ_ERR_ARG;
  if (it != IMQ_I16 && it != IMQ_I32) return IMQ_ERR_ARG;
  if (g != IMQ_PER_TENSOR && g != IMQ_PER_ROW && g != IMQ_PER_COL) return IMQ_ERR_ARG;
  const int64_t ngroups = g == IMQ_PER_TENSOR ? 1 : (g == IMQ_PER_ROW ? rows : cols);
  if (!delta && ngroups > 0) return IMQ_ERR_ARG;
  if ((!X || !Xint) && rows > 0 && cols > 0) return IMQ_ERR_ARG;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (rowmax && rows > 0) IMQ_CUDA_TRY(cudaMemsetAsync(rowmax, 0, (size_t)rows * 4, st));
  if (colmax && cols > 0) IMQ_CUDA_TRY(cudaMemsetAsync(colmax, 0, (size_t)cols * 4, st));
  if (rows == 0 || cols == 0) {
    // every group is empty: q = max = 0, so s = Delta = 1 and there is nothing to quantise
    if (ngroups > 0) {
      k_fill_f32<<<1, 256, 0, st>>>(delta, ngroups, 1.0f);
      if (qval) k_fill_f32<<<1, 256, 0, st>>>(qval, ngroups, 0.0f);
    }
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  const bool o16 = it == IMQ_I16;
  if (xt == IMQ_BF16) {
    const uint16_t* x = static_cast<const uint16_t*>(X);
    return o16 ? run<uint16_t, true>(x, rows, cols, ld, g, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st)
               : run<uint16_t, false>(x, rows, cols, ld, g, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st);
  }
  const uint32_t* x = static_cast<const uint32_t*>(X);
  return o16 ? run<uint32_t, true>(x, rows, cols, ld, g, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st)
             : run<uint32_t, false>(x, rows, cols, ld, g, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st);
}

}  // namespace imq
