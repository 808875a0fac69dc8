// rtn.cu -- percentile selection and round-to-nearest quantisation (sm_100a).
//
// Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
// summary), "Problem" / "Approach" and the measured-effects rows on beta and p.  The scale of a group
// maps its nearest-rank p-quantile q of |x| to beta; entries are rounded to the nearest integer
// (ties to even) after one fp32 multiply and are NOT clipped, so heavy hitters stay far outside
// +-beta.  q is found exactly on the order-preserving bit keys of |x| (the IEEE bit pattern of a
// non-negative float orders like an unsigned integer): bf16 groups of 1024 entries or more by a sample
// select (a sample brackets the rank, one pass counts below the bracket and histograms inside it),
// smaller bf16 groups by bisection on the key, fp32 groups by radix passes of 8 key bits.
//
// Kernels
//   k_rtn_rows    one warp per stored row: the row is staged in the warp's shared-memory buffer once,
//                 the select and the quantisation read it from there (one HBM read, one write); rows
//                 are dealt to the CTAs in turn.  bf16 to int16: quantised in place, the CTA folds the
//                 column maxima of each round of rows without atomics.  Also used for per-tensor
//                 groups with the scale taken from the tensor select.
//   k_rtn_cols_staged  one CTA per 16 (or 8, 4) stored columns: the column slab is staged in shared
//                 memory (one HBM read), one warp per column, optional transposed output (a K x N
//                 weight quantised per output channel straight into N x K); bf16 to int16 quantised in
//                 place with the row maxima folded over the CTA's columns.
//   k_rtn_cols    the same for columns too tall to stage: the slab is streamed once per pass (re-reads
//                 hit L2) and once more to quantise.
//   k_tensor_*    per-tensor select: global 256-bin histograms per pass, then k_rtn_rows.
// Side outputs: max |x_int| per stored row and column, the line statistics the unpack plan needs.  The
// maxima that cross CTAs are written as per-CTA partials to per-call scratch (stream-ordered, from the
// library's pool) and reduced by a second small kernel (no global atomics).
#include <math.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace imq {
namespace {

constexpr int kThreads = 256;
constexpr int kColsPerCta = 16;
// Per-warp select scratch in 32-bit words: the 256-bin histogram of the fp32 radix passes, or the
// one-bin-per-key histogram of the sampled bf16 select (keys lo .. lo + kSelWords - 1).
constexpr int kSelWords = 384;
// bf16 groups with at least this many entries take the sampled select; smaller ones bisect directly.
constexpr int kSampledMin = 1024;
constexpr int kSampleSize = 128;  // 4 keys per lane

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

// Scale and step from the selected q; q == 0 falls back to the group maximum qmax.  Returns the q the
// scale was derived from (reported as qval).
__device__ __forceinline__ float scale_from_q(float q, float qmax, int beta, float* s, float* d) {
  if (q == 0.0f) q = qmax;
  if (q == 0.0f) {
    *s = 1.0f;
    *d = 1.0f;
  } else {
    *s = __fdiv_rn((float)beta, q);
    *d = __fdiv_rn(q, (float)beta);
  }
  return q;
}

// Quantises one value; returns |v| (0 on a range error, which is recorded).
// clip > 0: the clipping comparison variant, the scaled value clamped to [-clip, clip] (clip = beta).
template <bool kOut16>
__device__ __forceinline__ uint32_t quant_one(float x, float s, void* out, int64_t idx, int32_t* status,
                                              int clip) {
  float y = __fmul_rn(x, s);
  if (clip) y = fminf(fmaxf(y, -(float)clip), (float)clip);
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

// Copies n16 16-byte pieces from global memory (streaming loads) to shared memory, lane-strided over
// one warp, with kBatch loads in flight per lane before their stores: a store waits for its load, so a
// plain copy loop would keep a single load per lane in flight and pay one memory latency per piece.
template <int kBatch>
__device__ __forceinline__ void warp_copy16(const uint4* __restrict__ src, uint4* dst, int n16, int lane) {
  for (int c0 = lane; c0 < n16; c0 += 32 * kBatch) {
    uint4 buf[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int c = c0 + 32 * j;
      if (c < n16) buf[j] = __ldcs(src + c);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int c = c0 + 32 * j;
      if (c < n16) dst[c] = buf[j];
    }
  }
}

// ------------------------------------------------------------------------------------------------
// warp-level routines over one group of n values held contiguously in shared memory (16-byte aligned)
// ------------------------------------------------------------------------------------------------
// Exact nearest-rank select: the k-th smallest key (1-based) by 8-bit radix passes on a warp-private
// 256-bin histogram.  Returns the key; every lane gets it.
template <typename T>
__device__ uint32_t warp_select_key(const T* a, int n, unsigned long long k, uint32_t* hist) {
  constexpr int V = 16 / sizeof(T);
  const int lane = threadIdx.x & 31;
  uint32_t pre = 0, msk = 0;
  for (int pass = 0; pass < num_passes(Key<T>::kBits); ++pass) {
#pragma unroll
    for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
    __syncwarp();
    const int sh = pass_shift(Key<T>::kBits, pass);
    const int nv = n / V;
    for (int i = lane; i < nv; i += 32) {
      const uint4 w = reinterpret_cast<const uint4*>(a)[i];
      const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const uint32_t key = Key<T>::key(e[j]);
        if ((key & msk) == pre) atomicAdd(&hist[(key >> sh) & 0xFFu], 1u);
      }
    }
    for (int i = nv * V + lane; i < n; i += 32) {
      const uint32_t key = Key<T>::key(a[i]);
      if ((key & msk) == pre) atomicAdd(&hist[(key >> sh) & 0xFFu], 1u);
    }
    __syncwarp();
    int d;
    unsigned long long below;
    warp_select(hist, 1, k, &d, &below);
    d = __shfl_sync(0xffffffffu, d, 0);
    below = __shfl_sync(0xffffffffu, below, 0);
    pre |= (uint32_t)d << sh;
    msk |= pass_width_mask(Key<T>::kBits, pass) << sh;
    k -= below;
    __syncwarp();
  }
  return pre;
}

// Largest key of the group and whether any key is non-finite (every lane gets both).
template <typename T>
__device__ void warp_key_stats(const T* a, int n, uint32_t* mk_out, uint32_t* bad_out) {
  constexpr int V = 16 / sizeof(T);
  const int lane = threadIdx.x & 31;
  uint32_t mk = 0;
  const int nv = n / V;
  for (int i = lane; i < nv; i += 32) {
    const uint4 w = reinterpret_cast<const uint4*>(a)[i];
    const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
    for (int j = 0; j < V; ++j) mk = max(mk, Key<T>::key(e[j]));
  }
  for (int i = nv * V + lane; i < n; i += 32) mk = max(mk, Key<T>::key(a[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mk = max(mk, __shfl_xor_sync(0xffffffffu, mk, o));
  *mk_out = mk;
  *bad_out = mk >= Key<T>::kInf;
}

// Exact nearest-rank select for bf16 keys, without atomics: the k-th smallest 15-bit key is built
// from the top bit down, bit b being set when fewer than k keys lie below (answer | 2^b).  Two keys are
// counted per 32-bit word: with both sign bits forced to 1, (0x8000 + key) - t keeps bit 15 of its half
// exactly when key >= t and never borrows from the other half.  Each half-word counter sees at most
// n / 64 + 4 keys (n <= 100 000 here: a group fits the shared-memory stage), far below 2^16.
__device__ uint32_t warp_select_key_bf16(const uint16_t* a, int n, unsigned long long k) {
  const int lane = threadIdx.x & 31;
  const int nv = n / 8;
  uint32_t ans = 0;
  for (int b = 14; b >= 0; --b) {
    const uint32_t t = ans | (1u << b);
    const uint32_t t2 = t | (t << 16);
    // four independent counters, so that consecutive words do not wait on one another's add
    uint32_t c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll 4
    for (int i = lane; i < nv; i += 32) {
      const uint4 w = reinterpret_cast<const uint4*>(a)[i];
      c0 += (((w.x | 0x80008000u) - t2) >> 15) & 0x00010001u;
      c1 += (((w.y | 0x80008000u) - t2) >> 15) & 0x00010001u;
      c2 += (((w.z | 0x80008000u) - t2) >> 15) & 0x00010001u;
      c3 += (((w.w | 0x80008000u) - t2) >> 15) & 0x00010001u;
    }
    const uint32_t acc = (c0 + c1) + (c2 + c3);
    uint32_t ge = (acc & 0xFFFFu) + (acc >> 16);
    for (int i = nv * 8 + lane; i < n; i += 32) ge += (a[i] & 0x7FFFu) >= t ? 1u : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ge += __shfl_xor_sync(0xffffffffu, ge, o);
    const unsigned long long below = (unsigned long long)n - ge;
    if (below < k) ans = t;
  }
  return ans;
}

// Per 16-bit half of two packed keys (sign bits of w forced to 1, t2 = t * 0x10001, t <= 0x7FFF): 1 in
// bit 0 (low half) and bit 16 (high half) where the key is >= t.  (0x8000 + key) - t lies in [1, 0xFFFF]
// for keys and t below 2^15, so bit 15 of each half is set exactly when key >= t and no half borrows.
__device__ __forceinline__ uint32_t ge_pair(uint32_t w_signed, uint32_t t2) {
  return ((w_signed - t2) >> 15) & 0x00010001u;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Largest bf16 key of a group and whether any key is non-finite, two keys per 32-bit word.
__device__ void warp_key_stats_bf16(const uint16_t* a, int n, uint32_t* mk_out, uint32_t* bad_out) {
  const int lane = threadIdx.x & 31;
  const int nv = n / 8;
  uint32_t m0 = 0, m1 = 0;
  for (int i = lane; i < nv; i += 32) {
    const uint4 w = reinterpret_cast<const uint4*>(a)[i];
    m0 = max_u16x2(m0, max_u16x2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu));
    m1 = max_u16x2(m1, max_u16x2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
  }
  m0 = max_u16x2(m0, m1);
  uint32_t mk = max(m0 & 0xFFFFu, m0 >> 16);
  for (int i = nv * 8 + lane; i < n; i += 32) mk = max(mk, (uint32_t)(a[i] & 0x7FFFu));
  mk = __reduce_max_sync(0xffffffffu, mk);
  *mk_out = mk;
  *bad_out = mk >= Key<uint16_t>::kInf;
}

// Exact nearest-rank select for bf16 keys by sampling (the SampleSelect scheme of Ribizel and Anzt,
// "Parallel selection on GPUs", 2019, on one warp), which also returns the group's largest key:
//   1. kSampleSize keys at evenly spaced positions; lo = the sample order statistic whose rank lies
//      2.5 binomial standard deviations (+1.5) below the target rank k * S / n (bisection on the key
//      value over the sample, which the lanes hold in registers);
//   2. one pass over the group counts the keys below lo, histograms the keys in [lo, lo + kSelWords - 1]
//      into the warp's scratch (one bin per key value) and takes the largest key;
//   3. if the bracket holds (fewer than k keys below lo, at least k up to the histogram's top) the answer
//      is the bin where the running count reaches k; otherwise the group is bisected in full.
// The sample only steers the work: every answer is the exact k-th smallest key.
__device__ uint32_t warp_select_key_bf16_sampled(const uint16_t* a, int n, unsigned long long k, uint32_t* hist,
                                                  uint32_t* mk_out) {
  const int lane = threadIdx.x & 31;
  constexpr unsigned kFull = 0xffffffffu;
  // ---- 1. sample: keys j and j + 32 of sample slice m in word m (positions at the slice midpoints)
  uint32_t sw[kSampleSize / 64];
#pragma unroll
  for (int m = 0; m < kSampleSize / 64; ++m) {
    const int j0 = 64 * m + lane, j1 = j0 + 32;
    // (2j + 1) n < 2^31 for the groups staged here (n below 2^21)
    const uint32_t k0 = a[((2u * j0 + 1u) * (uint32_t)n) / (2u * kSampleSize)] & 0x7FFFu;
    const uint32_t k1 = a[((2u * j1 + 1u) * (uint32_t)n) / (2u * kSampleSize)] & 0x7FFFu;
    sw[m] = k0 | (k1 << 16);
  }
#pragma unroll
  for (int j = 0; j < kSelWords / 32; ++j) hist[j * 32 + lane] = 0;
  uint32_t smn = 0xFFFFFFFFu, smx = 0;
#pragma unroll
  for (int m = 0; m < kSampleSize / 64; ++m) {
    smn = min_u16x2(smn, sw[m]);
    smx = max_u16x2(smx, sw[m]);
    sw[m] |= 0x80008000u;
  }
  smn = __reduce_min_sync(kFull, min(smn & 0xFFFFu, smn >> 16));
  smx = __reduce_max_sync(kFull, max(smx & 0xFFFFu, smx >> 16));
  const float pk = (float)((double)k / (double)n);
  const int r_lo = (int)floorf(pk * (float)kSampleSize - 2.5f * sqrtf((float)kSampleSize * pk * (1.0f - pk)) - 1.5f);
  uint32_t lo = 0;
  if (r_lo >= 1) {
    // the r_lo-th smallest sample key: answer in [l, h], #{sample < mid} decides the half
    uint32_t l = smn, h = smx;
    while (l < h) {
      const uint32_t mid = (l + h + 1) >> 1, t2 = mid * 0x10001u;
      uint32_t g = 0;
#pragma unroll
      for (int m = 0; m < kSampleSize / 64; ++m) g += ge_pair(sw[m], t2);
      const uint32_t below = kSampleSize - __reduce_add_sync(kFull, (g & 0xFFFFu) + (g >> 16));
      if (below < (uint32_t)r_lo) l = mid; else h = mid - 1;
    }
    lo = l;
  }
  const uint32_t hi = min(lo + (uint32_t)kSelWords - 1u, 0x7FFFu);
  __syncwarp();
  // ---- 2. count below lo, histogram [lo, hi], largest key
  const uint32_t lo2 = lo * 0x10001u, hi2 = (hi | 0x8000u) * 0x10001u;
  const int nv = n / 8;
  uint32_t ge = 0, mx2 = 0;
  for (int i = lane; i < nv; i += 32) {
    const uint4 w4 = reinterpret_cast<const uint4*>(a)[i];
    const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t kk = ws[q] & 0x7FFF7FFFu;
      const uint32_t gl = ((kk | 0x80008000u) - lo2) & 0x80008000u;  // bit 15 / 31: key >= lo
      const uint32_t c = gl & (hi2 - kk);                               // bit 15 / 31: lo <= key <= hi
      ge += gl >> 15;
      mx2 = max_u16x2(mx2, kk);
      if (c & 0x8000u) atomicAdd(&hist[(kk & 0xFFFFu) - lo], 1u);
      if (c & 0x80000000u) atomicAdd(&hist[(kk >> 16) - lo], 1u);
    }
  }
  uint32_t mk = max(mx2 & 0xFFFFu, mx2 >> 16);
  uint32_t ge_tail = 0;
  for (int i = nv * 8 + lane; i < n; i += 32) {
    const uint32_t key = a[i] & 0x7FFFu;
    mk = max(mk, key);
    ge_tail += key >= lo ? 1u : 0u;
    if (key >= lo && key <= hi) atomicAdd(&hist[key - lo], 1u);
  }
  mk = __reduce_max_sync(kFull, mk);
  *mk_out = mk;
  const uint32_t n_ge = __reduce_add_sync(kFull, (ge & 0xFFFFu) + (ge >> 16) + ge_tail);
  const unsigned long long below = (unsigned long long)n - n_ge;
  __syncwarp();
  // ---- 3. running count over the bins: lane owns bins [12 lane, 12 lane + 12)
  constexpr int kPer = kSelWords / 32;
  uint32_t c[kPer], own = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    c[j] = hist[lane * kPer + j];
    own += c[j];
  }
  uint32_t incl = own;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t total = __shfl_sync(kFull, incl, 31);
  __syncwarp();
  if (!(below < k && k <= below + total)) return warp_select_key_bf16(a, n, k);
  const uint32_t r = (uint32_t)(k - below);
  const unsigned ball = __ballot_sync(kFull, incl - own < r && r <= incl);
  const int src = __ffs(ball) - 1;
  uint32_t bin = 0;
  if (lane == src) {
    uint32_t cum = incl - own;
    bin = lane * kPer + kPer - 1;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (cum + c[j] >= r) {
        bin = lane * kPer + j;
        break;
      }
      cum += c[j];
    }
  }
  return lo + __shfl_sync(kFull, bin, src);
}

// Largest key (mk) and the k-th smallest key of a group in shared memory: sampled select for bf16
// groups of kSampledMin entries and more (which returns the largest key as well), a key-statistics pass
// and bisection for smaller bf16 groups, radix passes for f32.  `scratch` is the warp's kSelWords words.
// bad: the group holds a non-finite value.
template <typename T>
__device__ __forceinline__ uint32_t stats_and_select(const T* a, int n, unsigned long long k, uint32_t* scratch,
                                                     uint32_t* mk, uint32_t* bad) {
  if constexpr (sizeof(T) == 2) {
    uint32_t key;
    if (n >= kSampledMin) {
      key = warp_select_key_bf16_sampled(a, n, k, scratch, mk);
    } else {
      warp_key_stats_bf16(a, n, mk, bad);
      key = warp_select_key_bf16(a, n, k);
    }
    *bad = *mk >= Key<T>::kInf;
    return key;
  } else {
    warp_key_stats(a, n, mk, bad);
    return warp_select_key(a, n, k, scratch);
  }
}

// Largest key of a group and whether any key is non-finite (groups that are not selected on).
template <typename T>
__device__ __forceinline__ void key_stats(const T* a, int n, uint32_t* mk_out, uint32_t* bad_out) {
  if constexpr (sizeof(T) == 2)
    warp_key_stats_bf16(a, n, mk_out, bad_out);
  else
    warp_key_stats(a, n, mk_out, bad_out);
}

// x * s rounded to the nearest integer, ties to even: the arithmetic of quant_one, without the store.
template <bool kOut16>
__device__ __forceinline__ int32_t quant_val(float x, float s, int32_t* status, int clip) {
  float y = __fmul_rn(x, s);
  if (clip) y = fminf(fmaxf(y, -(float)clip), (float)clip);
  int32_t v = 0;
  if (fabsf(y) < 2147483648.0f) {
    v = __float2int_rn(y);
  } else {
    set_status(status, IMQ_ERR_RANGE);
  }
  if (kOut16 && (v > 32767 || v < -32767)) {
    set_status(status, IMQ_ERR_RANGE);
    v = 0;
  }
  return v;
}

// Quantises 8 consecutive entries of a 16-byte aligned group in shared memory and stores them with
// 16-byte stores at out[idx .. idx+7] (idx a multiple of 8, out 16-byte aligned); a[j] = |value j|.
// The conversion saturates (a NaN never gets here: its group is refused first), so an entry out of the
// output's range shows in a[j] as a magnitude above 32767 (int16) or of at least 2^31 - 1 (int32: no
// float below 2^31 rounds to 2^31 - 1); range_error() on the group's largest a[j] reports it.
template <typename T, bool kOut16>
__device__ __forceinline__ void quant8(const T* src, float s, void* out, int64_t idx, int clip,
                                       uint32_t (&a)[8]) {
  // the 8 entries as 32-bit words (bf16: two per word, low half first), kept in registers
  uint32_t wd[8];
  {
    const uint4 w0 = reinterpret_cast<const uint4*>(src)[0];
    wd[0] = w0.x; wd[1] = w0.y; wd[2] = w0.z; wd[3] = w0.w;
    if (sizeof(T) == 4) {
      const uint4 w1 = reinterpret_cast<const uint4*>(src)[1];
      wd[4] = w1.x; wd[5] = w1.y; wd[6] = w1.z; wd[7] = w1.w;
    }
  }
  int32_t v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const T e = sizeof(T) == 2 ? (T)((wd[j >> 1] >> (16 * (j & 1))) & 0xFFFFu) : (T)wd[j];
    float y = __fmul_rn(Key<T>::value(e), s);
    if (clip) y = fminf(fmaxf(y, -(float)clip), (float)clip);
    v[j] = __float2int_rn(y);
    a[j] = v[j] < 0 ? 0u - (uint32_t)v[j] : (uint32_t)v[j];
  }
  if (kOut16) {
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) pk[j] = ((uint32_t)v[2 * j] & 0xFFFFu) | ((uint32_t)v[2 * j + 1] << 16);
    *reinterpret_cast<uint4*>(static_cast<int16_t*>(out) + idx) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  } else {
    int32_t* o = static_cast<int32_t*>(out) + idx;
    reinterpret_cast<int4*>(o)[0] = make_int4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<int4*>(o)[1] = make_int4(v[4], v[5], v[6], v[7]);
  }
}

// True when a quantised magnitude from quant8 lies outside the output type's range.
template <bool kOut16>
__device__ __forceinline__ bool range_error(uint32_t amax) {
  return kOut16 ? amax > 32767u : amax >= 0x7FFFFFFFu;
}

// Quantises a bf16 group held in shared memory (n a multiple of 8, 16-byte aligned) into int16 at
// out[0 .. n) (16-byte aligned), 8 entries per lane and step, and overwrites each staged entry with its
// |x_int| (16 bits) so that line maxima across the group can be folded afterwards without atomics.
__device__ __forceinline__ void quant_bf16_inplace(uint16_t* grp, int n, float s, int clip, int16_t* out) {
  const int lane = threadIdx.x & 31;
  for (int g = lane; g < n / 8; g += 32) {
    const uint4 w = reinterpret_cast<const uint4*>(grp)[g];
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
    uint32_t pv[4], pa[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float y0 = __fmul_rn(__uint_as_float(wd[q] << 16), s);
      float y1 = __fmul_rn(__uint_as_float(wd[q] & 0xFFFF0000u), s);
      if (clip) {
        y0 = fminf(fmaxf(y0, -(float)clip), (float)clip);
        y1 = fminf(fmaxf(y1, -(float)clip), (float)clip);
      }
      const int32_t v0 = __float2int_rn(y0), v1 = __float2int_rn(y1);
      const uint32_t a0 = v0 < 0 ? 0u - (uint32_t)v0 : (uint32_t)v0, a1 = v1 < 0 ? 0u - (uint32_t)v1 : (uint32_t)v1;
      pv[q] = __byte_perm((uint32_t)v0, (uint32_t)v1, 0x5410);
      pa[q] = __byte_perm(a0, a1, 0x5410);
    }
    *reinterpret_cast<uint4*>(out + g * 8) = make_uint4(pv[0], pv[1], pv[2], pv[3]);
    reinterpret_cast<uint4*>(grp)[g] = make_uint4(pa[0], pa[1], pa[2], pa[3]);
  }
}

// Largest |x_int| of a group from its largest |x| (xmax): a correctly rounded multiply and rint are
// monotone and odd, so the group's largest quantised magnitude is rint(fl(xmax * s)) (clamped with the
// clipping variant).  Sets *range when it lies outside the output type (int16: above 32767, int32: at or
// above 2^31).
template <bool kOut16>
__device__ __forceinline__ uint32_t group_max_int(float xmax, float s, int clip, bool* range) {
  float y = __fmul_rn(xmax, s);
  if (clip) y = fminf(y, (float)clip);
  *range = kOut16 ? !(y < 32767.5f) : !(y < 2147483648.0f);
  return *range ? 0u : (uint32_t)__float2int_rn(y);
}

// Raises m[0..7] (16-byte aligned shared memory) to a[j] where a[j] is larger: a plain read first, so
// that the atomic is only paid where the maximum actually grows.
__device__ __forceinline__ void max8_shared(uint32_t* m, const uint32_t (&a)[8]) {
  const uint4 m0 = reinterpret_cast<const uint4*>(m)[0], m1 = reinterpret_cast<const uint4*>(m)[1];
  const uint32_t mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (a[j] > mm[j]) atomicMax(&m[j], a[j]);
}

// ------------------------------------------------------------------------------------------------
// per stored row (kSelect) or per tensor (scale from the tensor state): one warp per row.  Each warp
// stages its row in its own shared-memory buffer, builds its own 256-bin histograms (warp-aggregated
// increments) and selects with warp scans, so no block barrier is involved.  Column maxima of the
// CTA's rows are kept in shared memory and written once per CTA to `part` (reduced afterwards).
// ------------------------------------------------------------------------------------------------
template <typename T, bool kSelect, bool kOut16>
__global__ void __launch_bounds__(kThreads) k_rtn_rows(
    const T* __restrict__ X, int64_t rows, int64_t cols, int64_t ld, unsigned long long krank, int beta,
    void* __restrict__ Xint, int64_t ldq, int trans_out, float* __restrict__ delta, float* __restrict__ qval,
    int32_t* __restrict__ rowmax, int32_t* __restrict__ part, const TensorState* __restrict__ ts, int vec,
    int nwarps, int32_t* status, int clip) {
  extern __shared__ __align__(16) unsigned char dsm[];
  const int64_t row_bytes = (cols * (int64_t)sizeof(T) + 15) / 16 * 16;
  uint32_t* cmax = reinterpret_cast<uint32_t*>(dsm);                  // [cols]
  const int64_t cmax_bytes = part ? (cols * 4 + 15) / 16 * 16 : 0;  // same layout as the host
  __shared__ uint32_t hist_all[kThreads / 32][kSelWords];
  __shared__ int s_done[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  T* row = reinterpret_cast<T*>(dsm + cmax_bytes + warp * row_bytes);
  uint32_t* hist = hist_all[warp];
  constexpr int V = 16 / sizeof(T);
  if (part)
    for (int64_t c = tid; c < cols; c += blockDim.x) cmax[c] = 0;
  __syncthreads();
  const int n = (int)cols;
  // vectorised quantisation: whole 8-entry groups, contiguous and 16-byte aligned output rows
  const bool vq = !trans_out && n % 8 == 0 && ldq % 8 == 0 && (reinterpret_cast<uintptr_t>(Xint) & 15) == 0;
  // bf16 in, int16 out: rows quantised in place (|x_int| kept in the staged row), and the CTA folds
  // each round of nwarps rows into its column maxima, every thread owning whole 8-column groups
  const bool inplace = sizeof(T) == 2 && kOut16 && vq;
  // rows are dealt to the CTAs in turn (row r to CTA r mod gridDim.x), so that every SM gets the same
  // number of rows to within one per CTA; round j of a CTA takes its rows j*nwarps .. j*nwarps+nwarps-1
  for (int64_t j0 = 0; j0 * gridDim.x + blockIdx.x < rows; j0 += nwarps) {
    const int64_t r = (j0 + warp) * gridDim.x + blockIdx.x;
    int done = 0;
    if (warp < nwarps && r < rows) {
      const T* xr = X + r * ld;
      if (vec) {
        warp_copy16<8>(reinterpret_cast<const uint4*>(xr), reinterpret_cast<uint4*>(row), n / V, lane);
      } else {
        for (int c = lane; c < n; c += 32) row[c] = xr[c];
      }
      __syncwarp();
      uint32_t mk, bad;
      float s;
      if (kSelect) {
        const float q = Key<T>::from_key(stats_and_select(row, n, krank, hist, &mk, &bad));
        float dl;
        const float qu = scale_from_q(q, Key<T>::from_key(mk), beta, &s, &dl);
        if (lane == 0) {
          delta[r] = dl;
          if (qval) qval[r] = qu;
        }
      } else {
        key_stats(row, n, &mk, &bad);
        s = ts->s;
      }
      __syncwarp();
      if (bad) {
        if (lane == 0) set_status(status, IMQ_ERR_NONFINITE);
      } else if (inplace) {
        quant_bf16_inplace(reinterpret_cast<uint16_t*>(row), n, s, clip, static_cast<int16_t*>(Xint) + r * ldq);
        bool range;
        const uint32_t rmx = group_max_int<kOut16>(Key<T>::from_key(mk), s, clip, &range);
        if (lane == 0) {
          if (range) set_status(status, IMQ_ERR_RANGE);
          if (rowmax) rowmax[r] = (int32_t)rmx;
        }
        done = 1;
      } else {
        uint32_t rmx = 0;
        if (vq) {
          // 8 consecutive entries per lane and step: 16-byte shared loads and global stores
          for (int g = lane; g < n / 8; g += 32) {
            uint32_t a[8];
            quant8<T, kOut16>(row + g * 8, s, Xint, r * ldq + g * 8, clip, a);
#pragma unroll
            for (int j = 0; j < 8; ++j) rmx = max(rmx, a[j]);
            if (part) max8_shared(cmax + g * 8, a);
          }
        } else {
          for (int c = lane; c < n; c += 32) {
            const uint32_t a = quant_one<kOut16>(Key<T>::value(row[c]), s, Xint,
                                                 trans_out ? c * ldq + r : r * ldq + c, status, clip);
            rmx = max(rmx, a);
            if (part && a > cmax[c]) atomicMax(&cmax[c], a);
          }
        }
        rmx = __reduce_max_sync(0xffffffffu, rmx);
        if (lane == 0 && vq && range_error<kOut16>(rmx)) set_status(status, IMQ_ERR_RANGE);
        if (lane == 0 && rowmax) rowmax[r] = (int32_t)rmx;
      }
      __syncwarp();
    }
    if (inplace && part) {
      if (lane == 0) s_done[warp] = done;
      __syncthreads();
      for (int g = tid; g < n / 8; g += blockDim.x) {
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
        for (int w = 0; w < nwarps; ++w) {
          if (!s_done[w]) continue;
          const uint4 a = reinterpret_cast<const uint4*>(dsm + cmax_bytes + w * row_bytes)[g];
          m0 = max_u16x2(m0, a.x);
          m1 = max_u16x2(m1, a.y);
          m2 = max_u16x2(m2, a.z);
          m3 = max_u16x2(m3, a.w);
        }
        uint4* cm = reinterpret_cast<uint4*>(cmax) + 2 * g;
        uint4 c0 = cm[0], c1 = cm[1];
        c0.x = max(c0.x, m0 & 0xFFFFu); c0.y = max(c0.y, m0 >> 16);
        c0.z = max(c0.z, m1 & 0xFFFFu); c0.w = max(c0.w, m1 >> 16);
        c1.x = max(c1.x, m2 & 0xFFFFu); c1.y = max(c1.y, m2 >> 16);
        c1.z = max(c1.z, m3 & 0xFFFFu); c1.w = max(c1.w, m3 >> 16);
        cm[0] = c0;
        cm[1] = c1;
      }
      __syncthreads();
    }
  }
  if (part) {
    __syncthreads();
    int32_t* mine = part + (int64_t)blockIdx.x * cols;
    for (int64_t c = tid; c < cols; c += blockDim.x) mine[c] = (int32_t)cmax[c];
  }
}

// ------------------------------------------------------------------------------------------------
// per stored row, bf16, the row in registers: one CTA of NT threads per row, thread t holding the
// 16-byte vectors t, t + NT, ... (VPT of them) of every row it processes, so that it also owns the same
// columns in every row and keeps their maxima in its registers.  The exact nearest-rank select is a
// two-pass radix select on the 15-bit keys of |x| (the bf16 bit pattern without its sign orders like the
// magnitude): a 256-bin shared histogram of the high 8 key bits picks the bucket holding rank k, a 128-bin
// histogram of the low 7 bits of that bucket's keys picks the key.  The row is read from HBM once and
// written once; the shared memory is two small histograms, so several CTAs share an SM.
// Requires n % 8 == 0, 16-byte aligned rows (X, ld, Xint, ldq) and no transposed output.
// ------------------------------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ uint32_t block_reduce_max(uint32_t v, uint32_t* red) {
  v = __reduce_max_sync(0xffffffffu, v);
  if constexpr (NT == 32) {
    return v;
  } else {
    const int warp = threadIdx.x >> 5;
    __syncthreads();  // red is free
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) m = max(m, red[w]);
    return m;
  }
}

template <int NT, int VPT, bool kOut16>
__global__ void __launch_bounds__(NT) k_rtn_rows_reg(const uint16_t* __restrict__ X, int64_t rows, int n, int64_t ld,
                                                     unsigned long long krank, int beta, void* __restrict__ Xint,
                                                     int64_t ldq, float* __restrict__ delta, float* __restrict__ qval,
                                                     int32_t* __restrict__ rowmax, int32_t* __restrict__ part,
                                                     int32_t* status, int clip) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[NT / 32];
  __shared__ int s_sel[2];
  __shared__ unsigned long long s_below;
  const int tid = threadIdx.x;
  const int nvec = n / 8;
  constexpr int CW = kOut16 ? 4 : 8;  // column maxima words per vector: two 16-bit or one 32-bit per entry
  uint32_t cm[VPT][CW];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int c = 0; c < CW; ++c) cm[j][c] = 0;
  // Rows are dealt to the CTAs in turn.  With kPrefetch the loads of a CTA's next row are issued as soon as
  // its current row is in registers, so that they complete while the current row is selected and
  // quantised (registers for two rows); otherwise each row is loaded when its turn comes.
  constexpr bool kPrefetch = VPT <= 6;
  uint4 w[VPT];
  auto load_row = [&](int64_t rr, uint4 (&dst)[VPT]) {
    const uint16_t* xr = X + rr * ld;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * NT;
      dst[j] = v < nvec ? __ldcs(reinterpret_cast<const uint4*>(xr) + v) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  if (kPrefetch && (int64_t)blockIdx.x < rows) load_row(blockIdx.x, w);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    uint4 wn[VPT];
    if constexpr (kPrefetch) {
      if (r + gridDim.x < rows) load_row(r + gridDim.x, wn);
    } else {
      load_row(r, w);
    }
    // largest key of this thread's entries, two 15-bit keys per word at a time
    uint32_t kmax2 = 0;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      kmax2 = __vmaxu2(kmax2, w[j].x & 0x7FFF7FFFu);
      kmax2 = __vmaxu2(kmax2, w[j].y & 0x7FFF7FFFu);
      kmax2 = __vmaxu2(kmax2, w[j].z & 0x7FFF7FFFu);
      kmax2 = __vmaxu2(kmax2, w[j].w & 0x7FFF7FFFu);
    }
    const uint32_t kmax = max(kmax2 & 0xFFFFu, kmax2 >> 16);
    const uint32_t bad = kmax >= 0x7F80u;  // an Inf or NaN among this thread's entries (padding is zero)
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    const uint32_t rkmax = block_reduce_max<NT>(kmax, red);  // also orders the zeroing before the counts
    if (NT == 32) __syncwarp();
    // pass A: high 8 key bits
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      if (tid + j * NT >= nvec) continue;
      const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        atomicAdd(&hist[(ww[q] & 0x7FFFu) >> 7], 1u);
        atomicAdd(&hist[((ww[q] >> 16) & 0x7FFFu) >> 7], 1u);
      }
    }
    __syncthreads();
    if (tid < 32) {
      int d;
      unsigned long long below;
      if (warp_select(hist, 1, krank, &d, &below)) {
        s_sel[0] = d;
        s_below = below;
      }
    }
    __syncthreads();
    const uint32_t bucket = (uint32_t)s_sel[0];
    const unsigned long long krem = krank - s_below;
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    // pass B: low 7 key bits of the keys in that bucket
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      if (tid + j * NT >= nvec) continue;
      const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t k0 = ww[q] & 0x7FFFu, k1 = (ww[q] >> 16) & 0x7FFFu;
        if ((k0 >> 7) == bucket) atomicAdd(&hist[k0 & 127u], 1u);
        if ((k1 >> 7) == bucket) atomicAdd(&hist[k1 & 127u], 1u);
      }
    }
    __syncthreads();
    if (tid < 32) {
      int d;
      unsigned long long below;
      if (warp_select(hist, 1, krem, &d, &below)) s_sel[1] = d;
    }
    // the bad flag of the whole row, which also publishes s_sel[1]
    const uint32_t rbad = block_reduce_max<NT>(bad, red);
    if (NT == 32) __syncwarp();
    const uint32_t qkey = (bucket << 7) | (uint32_t)s_sel[1];
    float s, dl;
    const float qu = scale_from_q(__uint_as_float(qkey << 16), __uint_as_float(rkmax << 16), beta, &s, &dl);
    if (tid == 0) {
      delta[r] = dl;
      if (qval) qval[r] = qu;
    }
    if (rbad) {
      if (tid == 0) set_status(status, IMQ_ERR_NONFINITE);
    } else {
      bool range;
      const uint32_t rmx = group_max_int<kOut16>(__uint_as_float(rkmax << 16), s, clip, &range);
      if (tid == 0) {
        if (range) set_status(status, IMQ_ERR_RANGE);
        if (rowmax) rowmax[r] = (int32_t)rmx;
      }
      char* orow = static_cast<char*>(Xint) + r * ldq * (kOut16 ? 2 : 4);
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = tid + j * NT;
        if (v >= nvec) continue;
        const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
        int32_t q[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float y0 = __fmul_rn(__uint_as_float(ww[e] << 16), s);
          float y1 = __fmul_rn(__uint_as_float(ww[e] & 0xFFFF0000u), s);
          if (clip) {
            y0 = fminf(fmaxf(y0, -(float)clip), (float)clip);
            y1 = fminf(fmaxf(y1, -(float)clip), (float)clip);
          }
          q[2 * e] = __float2int_rn(y0);
          q[2 * e + 1] = __float2int_rn(y1);
        }
        if constexpr (kOut16) {
          uint32_t pv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pv[e] = __byte_perm((uint32_t)q[2 * e], (uint32_t)q[2 * e + 1], 0x5410);
            const uint32_t a0 = (uint32_t)abs(q[2 * e]), a1 = (uint32_t)abs(q[2 * e + 1]);
            cm[j][e] = max_u16x2(cm[j][e], __byte_perm(a0, a1, 0x5410));
          }
          __stcs(reinterpret_cast<uint4*>(orow) + v, make_uint4(pv[0], pv[1], pv[2], pv[3]));
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) cm[j][e] = max(cm[j][e], q[e] < 0 ? 0u - (uint32_t)q[e] : (uint32_t)q[e]);
          int4* o = reinterpret_cast<int4*>(orow) + 2 * v;
          __stcs(o, make_int4(q[0], q[1], q[2], q[3]));
          __stcs(o + 1, make_int4(q[4], q[5], q[6], q[7]));
        }
      }
    }
    if constexpr (kPrefetch) {
#pragma unroll
      for (int j = 0; j < VPT; ++j) w[j] = wn[j];
    }
  }
  if (part) {
    int32_t* mine = part + (int64_t)blockIdx.x * n;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * NT;
      if (v >= nvec) continue;
      int4* o = reinterpret_cast<int4*>(mine + (int64_t)v * 8);
      if constexpr (kOut16) {
        o[0] = make_int4((int)(cm[j][0] & 0xFFFFu), (int)(cm[j][0] >> 16), (int)(cm[j][1] & 0xFFFFu),
                         (int)(cm[j][1] >> 16));
        o[1] = make_int4((int)(cm[j][2] & 0xFFFFu), (int)(cm[j][2] >> 16), (int)(cm[j][3] & 0xFFFFu),
                         (int)(cm[j][3] >> 16));
      } else {
        o[0] = make_int4((int)cm[j][0], (int)cm[j][1], (int)cm[j][2], (int)cm[j][3]);
        o[1] = make_int4((int)cm[j][4], (int)cm[j][5], (int)cm[j][6], (int)cm[j][7]);
      }
    }
  }
}

// Word k (0..3) of a 16-byte vector (k known at compile time after unrolling).
__device__ __forceinline__ uint32_t word_of(const uint4& v, int k) {
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// bf16 transpose in registers: X (rows x cols, leading dimension ld) into Y (cols x rows, dense).  A
// thread moves one 8 x 8 block: eight 16-byte row loads, the 8 x 8 transpose of its 16-bit entries by
// byte permutes (one per output word: the same half of one word of two consecutive input rows), eight
// 16-byte stores.  A warp covers 64 rows x 32 columns (lane = 4 column blocks x 8 row blocks), so that a
// load instruction reads 64 contiguous bytes of each of 8 rows and a store instruction 128 contiguous
// bytes of each of 4 output rows; a CTA of 8 warps covers 64 rows x 256 columns.  No shared memory.
// rows and cols are multiples of 8; X, ld and Y 16-byte aligned.
__global__ void __launch_bounds__(256) k_transpose_bf16(const uint16_t* __restrict__ X, int64_t rows, int64_t cols,
                                                        int64_t ld, uint16_t* __restrict__ Y) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t r = (int64_t)blockIdx.y * 64 + (lane >> 2) * 8;
  const int64_t c = (int64_t)blockIdx.x * 256 + warp * 32 + (lane & 3) * 8;
  if (r >= rows || c >= cols) return;  // blocks are whole: rows and cols are multiples of 8
  uint4 w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = __ldcs(reinterpret_cast<const uint4*>(X + (r + i) * ld + c));
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // output row c + j holds entries (r + 0..7, c + j): word j/2 of every input row, low half for even j
    const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = __byte_perm(word_of(w[2 * q], j >> 1), word_of(w[2 * q + 1], j >> 1), sel);
    *reinterpret_cast<uint4*>(Y + (c + j) * rows + r) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------------------------------------
// per stored column, slab staged in shared memory: CW columns x all rows are read from HBM once and
// stored transposed (each column contiguous); then one warp per column runs the same select and
// quantisation as a row.  With trans_out the quantised column is written as one contiguous output row
// (a K x N weight quantised per output channel straight into N x K).  Row maxima of the CTA's columns
// go to `part` (reduced afterwards); column maxima are written directly.
// ------------------------------------------------------------------------------------------------
template <typename T, int CW, bool kOut16>
__global__ void __launch_bounds__(CW * 32, 1) k_rtn_cols_staged(
    const T* __restrict__ X, int64_t rows, int64_t cols, int64_t ld, unsigned long long krank, int beta,
    void* __restrict__ Xint, int64_t ldq, int trans_out, float* __restrict__ delta, float* __restrict__ qval,
    int32_t* __restrict__ part, int32_t* __restrict__ colmax, int vec, int32_t* status, int clip) {
  extern __shared__ __align__(16) unsigned char dsm[];
  const int n = (int)rows;
  const int colstride = (n + 7) / 8 * 8;  // elements; keeps every column 16-byte aligned
  T* S = reinterpret_cast<T*>(dsm);       // [CW][colstride]
  uint32_t* rmax = reinterpret_cast<uint32_t*>(dsm + (size_t)CW * colstride * sizeof(T));  // [rows]
  __shared__ uint32_t hist_all[CW][kSelWords];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t c0 = (int64_t)blockIdx.x * CW;
  const int ncol = cols - c0 < CW ? (int)(cols - c0) : CW;
  for (int r = tid; r < n; r += CW * 32) rmax[r] = 0;
  // stage: 16-byte loads along the rows, transposed stores into the columns
  constexpr int V = 16 / sizeof(T);
  constexpr int SEG = CW / V;  // 16-byte pieces per slab row (0 when a slab row is narrower)
  constexpr int SEGD = SEG > 0 ? SEG : 1;  // divisor of the branch below, which SEG = 0 never takes
  if (SEG > 0 && vec && ncol == CW) {
    // kB loads in flight per thread before their transposed stores (see warp_copy16)
    constexpr int kB = 8;
    for (int i0 = tid; i0 < n * SEG; i0 += CW * 32 * kB) {
      uint4 buf[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int i = i0 + b * CW * 32;
        if (i < n * SEG) buf[b] = __ldcs(reinterpret_cast<const uint4*>(X + (i / SEGD) * ld + c0) + i % SEGD);
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int i = i0 + b * CW * 32;
        if (i < n * SEG) {
          const int r = i / SEGD, sg = i % SEGD;
          const T* e = reinterpret_cast<const T*>(&buf[b]);
#pragma unroll
          for (int j = 0; j < V; ++j) S[(sg * V + j) * colstride + r] = e[j];
        }
      }
    }
  } else {
    for (int i = tid; i < n * CW; i += CW * 32) {
      const int r = i / CW, k = i % CW;
      S[k * colstride + r] = k < ncol ? X[r * ld + c0 + k] : (T)0;
    }
  }
  __syncthreads();
  // vectorised quantisation when the column is written as one contiguous, aligned output row
  const bool vq = trans_out && n % 8 == 0 && ldq % 8 == 0 && (reinterpret_cast<uintptr_t>(Xint) & 15) == 0;
  // bf16 in, int16 out: columns quantised in place (|x_int| kept in the staged column) and the row maxima
  // folded afterwards over the CTA's columns, every thread owning whole 8-row groups
  const bool inplace = sizeof(T) == 2 && kOut16 && vq;
  __shared__ int s_done[CW];
  if (warp < ncol) {
    T* col = S + warp * colstride;
    const int64_t c = c0 + warp;
    uint32_t mk, bad;
    const float q = Key<T>::from_key(stats_and_select(col, n, krank, hist_all[warp], &mk, &bad));
    float s, dl;
    const float qu = scale_from_q(q, Key<T>::from_key(mk), beta, &s, &dl);
    if (lane == 0) {
      delta[c] = dl;
      if (qval) qval[c] = qu;
      if (bad) set_status(status, IMQ_ERR_NONFINITE);
    }
    __syncwarp();
    if (inplace) {
      uint32_t cmx = 0;
      if (!bad) {
        quant_bf16_inplace(reinterpret_cast<uint16_t*>(col), n, s, clip, static_cast<int16_t*>(Xint) + c * ldq);
        bool range;
        cmx = group_max_int<kOut16>(Key<T>::from_key(mk), s, clip, &range);
        if (lane == 0 && range) set_status(status, IMQ_ERR_RANGE);
      }
      if (lane == 0) {
        s_done[warp] = bad ? 0 : 1;
        if (colmax) colmax[c] = (int32_t)cmx;
      }
    } else {
      uint32_t cmx = 0;
      if (!bad && vq) {
        for (int g = lane; g < n / 8; g += 32) {
          uint32_t a[8];
          quant8<T, kOut16>(col + g * 8, s, Xint, c * ldq + g * 8, clip, a);
#pragma unroll
          for (int j = 0; j < 8; ++j) cmx = max(cmx, a[j]);
          if (part) max8_shared(rmax + g * 8, a);
        }
      } else if (!bad) {
        for (int r = lane; r < n; r += 32) {
          const uint32_t a = quant_one<kOut16>(Key<T>::value(col[r]), s, Xint, trans_out ? c * ldq + r : r * ldq + c,
                                               status, clip);
          cmx = max(cmx, a);
          if (part && a > rmax[r]) atomicMax(&rmax[r], a);
        }
      }
      cmx = __reduce_max_sync(0xffffffffu, cmx);
      if (lane == 0 && !bad && vq && range_error<kOut16>(cmx)) set_status(status, IMQ_ERR_RANGE);
      if (lane == 0 && colmax) colmax[c] = (int32_t)cmx;
    }
  }
  if (part) {
    __syncthreads();
    int32_t* mine = part + (int64_t)blockIdx.x * rows;
    if (inplace) {
      // row maxima of this CTA's columns: 8 rows per thread and step, 16-byte reads of each column
      for (int g = tid; g < n / 8; g += CW * 32) {
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
        for (int w = 0; w < ncol; ++w) {
          if (!s_done[w]) continue;
          const uint4 a = *reinterpret_cast<const uint4*>(S + w * colstride + g * 8);
          m0 = max_u16x2(m0, a.x);
          m1 = max_u16x2(m1, a.y);
          m2 = max_u16x2(m2, a.z);
          m3 = max_u16x2(m3, a.w);
        }
        int4* o = reinterpret_cast<int4*>(mine + g * 8);
        o[0] = make_int4((int)(m0 & 0xFFFFu), (int)(m0 >> 16), (int)(m1 & 0xFFFFu), (int)(m1 >> 16));
        o[1] = make_int4((int)(m2 & 0xFFFFu), (int)(m2 >> 16), (int)(m3 & 0xFFFFu), (int)(m3 >> 16));
      }
    } else {
      for (int r = tid; r < n; r += CW * 32) mine[r] = (int32_t)rmax[r];
    }
  }
}

// ------------------------------------------------------------------------------------------------
// per stored column: one CTA per kColsPerCta columns
// ------------------------------------------------------------------------------------------------
template <typename T, bool kOut16>
__global__ void __launch_bounds__(kThreads) k_rtn_cols(
    const T* __restrict__ X, int64_t rows, int64_t cols, int64_t ld, unsigned long long krank, int beta,
    void* __restrict__ Xint, int64_t ldq, int trans_out, float* __restrict__ delta, float* __restrict__ qval,
    int32_t* __restrict__ part, int32_t* __restrict__ colmax, int32_t* status, int clip) {
  constexpr int CW = kColsPerCta;
  int32_t* prow = part ? part + (int64_t)blockIdx.x * rows : nullptr;  // this CTA's row maxima
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
    for (int64_t r0 = 0; r0 < rows; r0 += RS) {
      const int64_t r = r0 + rsub;
      const bool in = cval && r < rows;
      const uint32_t k = in ? Key<T>::key(X[r * ld + c]) : 0u;
      if (pass == 0 && in) {
        mk = max(mk, k);
        bad |= (k >= Key<T>::kInf);
      }
      warp_count(hist, ((k >> sh) & 0xFFu) * CW + cc, in && (k & msk) == pre);
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
    const float qu = scale_from_q(q, Key<T>::from_key(s_maxkey[tid]), beta, &s, &d);
    delta[cg] = d;
    if (qval) qval[cg] = qu;
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
      a = quant_one<kOut16>(Key<T>::value(X[r * ld + c]), s, Xint, trans_out ? c * ldq + r : r * ldq + c, status,
                            clip);
      cmx = max(cmx, a);
    }
    // max over the CW columns of this row (CW consecutive lanes)
#pragma unroll
    for (int o = CW / 2; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (prow && cc == 0 && r < rows) prow[r] = (int32_t)a;
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
      const float qu = scale_from_q(q, Key<T>::from_key(ts->maxkey), beta, &s, &dl);
      ts->s = s;
      ts->delta = dl;
      ts->q = q;
      delta[0] = dl;
      if (qval) qval[0] = qu;
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

// Per-call scratch from the library's stream-ordered pool, allocated and freed on the call's stream:
// the free is ordered after every kernel of the call that uses it, and calls on different streams never
// share it, so they may run concurrently.
struct StreamScratch {
  void* p = nullptr;
  cudaStream_t st = nullptr;
  imq_status alloc(DeviceState* ds, size_t bytes, cudaStream_t s) {
    st = s;
    return cudaMallocFromPoolAsync(&p, bytes > 0 ? bytes : 16, ds->pool, s) == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  ~StreamScratch() {
    if (p) cudaFreeAsync(p, st);
  }
};

// Launch shape of the per-row kernel k_rtn_rows: one warp per row, the row buffers of the CTA's warps
// plus (when column maxima are wanted) its column maxima in shared memory, as many CTAs as fit on an SM
// (at most 4), and one CTA per row up to every resident slot (rows are dealt to the CTAs in turn).
// Returns false when one row and the column maxima do not fit the shared-memory budget.
struct RowsShape {
  int64_t grid;
  int nwarps;
  size_t smem;
};
bool rows_launch_shape(int64_t rows, int64_t cols, size_t elem, bool want_colmax, int sms, RowsShape* out) {
  const size_t row_bytes = (size_t)((cols * (int64_t)elem + 15) / 16 * 16);
  const size_t cmax_bytes = want_colmax ? (size_t)((cols * 4 + 15) / 16 * 16) : 0;
  constexpr size_t kBudget = 200 * 1024;
  if (cmax_bytes + row_bytes > kBudget) return false;
  int nwarps = (int)((kBudget - cmax_bytes) / row_bytes);
  if (nwarps > kThreads / 32) nwarps = kThreads / 32;
  const size_t smem = cmax_bytes + (size_t)nwarps * row_bytes;
  int per_sm = (int)(kBudget / (smem + kThreads / 32 * kSelWords * 4 + 1024));
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 4) per_sm = 4;
  out->grid = rows < (int64_t)sms * per_sm ? rows : (int64_t)sms * per_sm;
  out->nwarps = nwarps;
  out->smem = smem;
  return true;
}

int64_t nearest_rank(int64_t n, double p) {
  if (n <= 0) return 1;
  int64_t k = (int64_t)ceil(p * (double)n);
  if (k < 1) k = 1;
  if (k > n) k = n;
  return k;
}

template <typename T, int CW, bool kOut16>
imq_status run_cols_staged(const T* X, int64_t rows, int64_t cols, int64_t ld, unsigned long long k, int32_t beta,
                           void* Xint, int64_t ldq, int trans_out, float* delta, float* qval, int32_t* rowmax,
                           int32_t* colmax, int clip, DeviceState* ds, cudaStream_t st) {
  const size_t colstride = (size_t)(rows + 7) / 8 * 8;
  const size_t smem = (size_t)CW * colstride * sizeof(T) + (size_t)rows * 4;
  const bool vec = (ld % (16 / (int64_t)sizeof(T)) == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  const int64_t grid = (cols + CW - 1) / CW;
  int32_t* part = nullptr;
  StreamScratch sp;
  if (rowmax) {
    if (sp.alloc(ds, (size_t)grid * rows * 4, st) != IMQ_OK) return IMQ_ERR_CUDA;
    part = static_cast<int32_t*>(sp.p);
  }
  auto kern = k_rtn_cols_staged<T, CW, kOut16>;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  kern<<<(unsigned)grid, CW * 32, smem, st>>>(X, rows, cols, ld, k, beta, Xint, ldq, trans_out, delta, qval, part,
                                              colmax, vec ? 1 : 0, ds->status, clip);
  if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
  return rowmax ? launch_reduce_max(part, grid, rows, rowmax, st) : IMQ_OK;
}

// The register-resident per-row kernel for bf16 rows of n entries (n % 8 == 0, n <= 16384, 16-byte
// aligned rows of X and Xint): NT threads per row and VPT 16-byte vectors per thread.  rowmax / colmax
// are over the rows and columns of the matrix given here (the caller swaps them for a transposed input).
template <int NT, int VPT, bool kOut16>
imq_status launch_rows_reg(const uint16_t* X, int64_t rows, int n, int64_t ld, unsigned long long k, int32_t beta,
                           void* Xint, int64_t ldq, float* delta, float* qval, int32_t* rowmax, int32_t* colmax,
                           int clip, DeviceState* ds, cudaStream_t st) {
  auto kern = k_rtn_rows_reg<NT, VPT, kOut16>;
  int per_sm = 0;
  IMQ_CUDA_TRY(blocks_per_sm(reinterpret_cast<const void*>(kern), NT, 0, &per_sm));
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = rows < (int64_t)ds->num_sms * per_sm ? rows : (int64_t)ds->num_sms * per_sm;
  int32_t* part = nullptr;
  StreamScratch sp;
  if (colmax) {
    if (sp.alloc(ds, (size_t)grid * n * 4, st) != IMQ_OK) return IMQ_ERR_CUDA;
    part = static_cast<int32_t*>(sp.p);
  }
  kern<<<(unsigned)grid, NT, 0, st>>>(X, rows, n, ld, k, beta, Xint, ldq, delta, qval, rowmax, part, ds->status, clip);
  if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
  return colmax ? launch_reduce_max(part, grid, n, colmax, st) : IMQ_OK;
}

// True (and *status set) when the register-resident kernel takes this shape; false leaves it to the
// staged kernels.
template <bool kOut16>
bool try_rows_reg(const uint16_t* X, int64_t rows, int64_t n, int64_t ld, unsigned long long k, int32_t beta,
                  void* Xint, int64_t ldq, float* delta, float* qval, int32_t* rowmax, int32_t* colmax, int clip,
                  DeviceState* ds, cudaStream_t st, imq_status* status) {
  if (n % 8 != 0 || n > 16384 || ld % 8 != 0 || ldq % 8 != 0 || (reinterpret_cast<uintptr_t>(X) & 15) ||
      (reinterpret_cast<uintptr_t>(Xint) & 15))
    return false;
  const int nvec = (int)(n / 8), nn = (int)n;
  if (nvec <= 32)
    *status = launch_rows_reg<32, 1, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else if (nvec <= 128)
    *status = launch_rows_reg<128, 1, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else if (nvec <= 256)
    *status = launch_rows_reg<256, 1, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else if (nvec <= 512)
    *status = launch_rows_reg<256, 2, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else if (nvec <= 1024)
    *status = launch_rows_reg<256, 4, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else if (nvec <= 1536)
    *status = launch_rows_reg<256, 6, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  else
    *status = launch_rows_reg<256, 8, kOut16>(X, rows, nn, ld, k, beta, Xint, ldq, delta, qval, rowmax, colmax, clip, ds, st);
  return true;
}

template <typename T, bool kOut16>
imq_status run(const T* X, int64_t rows, int64_t cols, int64_t ld, imq_gran g, double p,
               int32_t beta, void* Xint, int64_t ldq, int trans_out, float* delta, float* qval, int32_t* rowmax,
               int32_t* colmax, int clip, DeviceState* ds, cudaStream_t st) {
  const int sms = ds->num_sms;
  if constexpr (sizeof(T) == 2) {
    // bf16 rows: the register-resident kernel; bf16 columns into the transposed layout: a transpose,
    // then the same kernel on the rows of the transpose (its row and column maxima swapped)
    imq_status rs = IMQ_OK;
    if (g == IMQ_PER_ROW && !trans_out &&
        try_rows_reg<kOut16>(X, rows, cols, ld, (unsigned long long)nearest_rank(cols, p), beta, Xint, ldq, delta,
                             qval, rowmax, colmax, clip, ds, st, &rs))
      return rs;
    if (g == IMQ_PER_COL && trans_out && rows % 8 == 0 && cols % 8 == 0 && rows <= 16384 && ld % 8 == 0 &&
        ldq % 8 == 0 && !(reinterpret_cast<uintptr_t>(X) & 15) && !(reinterpret_cast<uintptr_t>(Xint) & 15)) {
      StreamScratch tp;
      if (tp.alloc(ds, (size_t)rows * cols * 2, st) != IMQ_OK) return IMQ_ERR_CUDA;
      uint16_t* Y = static_cast<uint16_t*>(tp.p);
      const dim3 tg((unsigned)((cols + 255) / 256), (unsigned)((rows + 63) / 64));
      k_transpose_bf16<<<tg, 256, 0, st>>>(reinterpret_cast<const uint16_t*>(X), rows, cols, ld, Y);
      if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
      if (try_rows_reg<kOut16>(Y, cols, rows, rows, (unsigned long long)nearest_rank(rows, p), beta, Xint, ldq, delta,
                               qval, colmax, rowmax, clip, ds, st, &rs))
        return rs;
    }
  }
  if (g == IMQ_PER_COL) {
    const unsigned long long k = (unsigned long long)nearest_rank(rows, p);
    // the slab of 16 (or 8) columns is staged in shared memory when it fits (plus the row maxima)
    constexpr size_t kSlab = 192 * 1024;
    const size_t colb = (size_t)(rows + 7) / 8 * 8 * sizeof(T);
    if (16 * colb + (size_t)rows * 4 <= kSlab)
      return run_cols_staged<T, 16, kOut16>(X, rows, cols, ld, k, beta, Xint, ldq, trans_out, delta, qval, rowmax,
                                            colmax, clip, ds, st);
    if (8 * colb + (size_t)rows * 4 <= kSlab)
      return run_cols_staged<T, 8, kOut16>(X, rows, cols, ld, k, beta, Xint, ldq, trans_out, delta, qval, rowmax,
                                           colmax, clip, ds, st);
    if (4 * colb + (size_t)rows * 4 <= kSlab)
      return run_cols_staged<T, 4, kOut16>(X, rows, cols, ld, k, beta, Xint, ldq, trans_out, delta, qval, rowmax,
                                           colmax, clip, ds, st);
    const int64_t grid = (cols + kColsPerCta - 1) / kColsPerCta;
    int32_t* part = nullptr;
    StreamScratch sp;
    if (rowmax) {
      if (sp.alloc(ds, (size_t)grid * rows * 4, st) != IMQ_OK) return IMQ_ERR_CUDA;
      part = static_cast<int32_t*>(sp.p);
    }
    k_rtn_cols<T, kOut16><<<(unsigned)grid, kThreads, 0, st>>>(X, rows, cols, ld, k, beta, Xint, ldq, trans_out,
                                                               delta, qval, part, colmax, ds->status, clip);
    if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
    return rowmax ? launch_reduce_max(part, grid, rows, rowmax, st) : IMQ_OK;
  }
  RowsShape sh;
  if (!rows_launch_shape(rows, cols, sizeof(T), colmax != nullptr, sms, &sh)) return IMQ_ERR_UNSUPPORTED;
  const int64_t grid = sh.grid;
  const int nwarps = sh.nwarps;
  const size_t smem = sh.smem;
  const bool vec = (cols % (16 / (int64_t)sizeof(T)) == 0) && (ld % (16 / (int64_t)sizeof(T)) == 0) &&
                   ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  int32_t* part = nullptr;
  StreamScratch sp, sts;
  if (colmax) {
    if (sp.alloc(ds, (size_t)grid * cols * 4, st) != IMQ_OK) return IMQ_ERR_CUDA;
    part = static_cast<int32_t*>(sp.p);
  }
  TensorState* ts = nullptr;
  if (g == IMQ_PER_TENSOR) {
    if (sts.alloc(ds, sizeof(TensorState), st) != IMQ_OK) return IMQ_ERR_CUDA;
    ts = static_cast<TensorState*>(sts.p);
    k_tensor_init<<<1, 256, 0, st>>>(ts, (unsigned long long)nearest_rank(rows * cols, p));
    const int64_t hgrid = rows < (int64_t)sms * 8 ? rows : (int64_t)sms * 8;
    const int np = num_passes(Key<T>::kBits);
    for (int pass = 0; pass < np; ++pass) {
      k_tensor_hist<T><<<(unsigned)hgrid, kThreads, 0, st>>>(X, rows, cols, ld, ts, pass);
      k_tensor_select<T><<<1, 32, 0, st>>>(ts, pass, pass == np - 1, beta, delta, qval, ds->status);
    }
    auto kern = k_rtn_rows<T, false, kOut16>;
    IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
    kern<<<(unsigned)grid, kThreads, smem, st>>>(X, rows, cols, ld, 0ull, beta, Xint, ldq, trans_out, delta, qval,
                                                 rowmax, part, ts, vec, nwarps, ds->status, clip);
  } else {
    auto kern = k_rtn_rows<T, true, kOut16>;
    IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
    kern<<<(unsigned)grid, kThreads, smem, st>>>(X, rows, cols, ld, (unsigned long long)nearest_rank(cols, p), beta,
                                                 Xint, ldq, trans_out, delta, qval, rowmax, part, nullptr, vec, nwarps,
                                                 ds->status, clip);
  }
  if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
  return colmax ? launch_reduce_max(part, grid, cols, colmax, st) : IMQ_OK;
}

}  // namespace

imq_status launch_rtn_quantize(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               imq_gran g, double p, int32_t beta, void* Xint, imq_dtype it,
                               int64_t ldq, int32_t trans_out, float* delta, float* qval, int32_t* rowmax,
                               int32_t* colmax, uint32_t flags, cudaStream_t st) {
  if (trans_out != 0 && trans_out != 1) return IMQ_ERR_ARG;
  if (flags & ~(uint32_t)IMQ_RTN_CLIP) return IMQ_ERR_ARG;
  const int clip = (flags & IMQ_RTN_CLIP) ? beta : 0;
  if (rows < 0 || cols < 0 || ld < cols || ldq < (trans_out ? rows : cols) || !(p > 0.0 && p <= 1.0) || beta < 1 ||
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
  // every entry of rowmax / colmax is written by the kernels (directly or by a reduction)
  if (rows == 0 || cols == 0) {
    // every group is empty: q = max = 0, so s = Delta = 1 and there is nothing to quantise
    if (rowmax && rows > 0) IMQ_CUDA_TRY(cudaMemsetAsync(rowmax, 0, (size_t)rows * 4, st));
    if (colmax && cols > 0) IMQ_CUDA_TRY(cudaMemsetAsync(colmax, 0, (size_t)cols * 4, st));
    if (ngroups > 0) {
      k_fill_f32<<<1, 256, 0, st>>>(delta, ngroups, 1.0f);
      if (qval) k_fill_f32<<<1, 256, 0, st>>>(qval, ngroups, 0.0f);
    }
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  const bool o16 = it == IMQ_I16;
  if (xt == IMQ_BF16) {
    const uint16_t* x = static_cast<const uint16_t*>(X);
    return o16 ? run<uint16_t, true>(x, rows, cols, ld, g, p, beta, Xint, ldq, trans_out, delta, qval, rowmax, colmax, clip, ds, st)
               : run<uint16_t, false>(x, rows, cols, ld, g, p, beta, Xint, ldq, trans_out, delta, qval, rowmax, colmax, clip, ds, st);
  }
  const uint32_t* x = static_cast<const uint32_t*>(X);
  return o16 ? run<uint32_t, true>(x, rows, cols, ld, g, p, beta, Xint, ldq, trans_out, delta, qval, rowmax, colmax, clip, ds, st)
             : run<uint32_t, false>(x, rows, cols, ld, g, p, beta, Xint, ldq, trans_out, delta, qval, rowmax, colmax, clip, ds, st);
}

// ------------------------------------------------------------------------------------------------
// Allocation-free per-row quantiser (imq_rtn_quantize_rows_noalloc).
//
// Callers whose own allocator has reserved the free device memory cannot let the library's pool grow
// for the per-call scratch above.  For them the per-CTA column maxima of k_rtn_rows go to one fixed array in this module's device image,
// mapped by the CUDA runtime when the module loads.  Its device address is looked up once per device,
// on the first call with that device current.  Every call on a device shares the array, so calls whose
// executions overlap race on it.  Nothing in it has to start at zero: each CTA writes its whole slice
// of partial maxima before k_reduce_max reads them.
// ------------------------------------------------------------------------------------------------
namespace {
constexpr size_t kNoallocBytes = IMQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocBytes / sizeof(int32_t)];
std::atomic<int32_t*> g_noalloc_ptr[64];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (looked up on the first call there).  The
// look-up may load the module, which a stream capture in progress would not record: a first call on a
// device made while `st` is capturing is refused with IMQ_ERR_UNSUPPORTED before anything else happens.
imq_status noalloc_scratch(int32_t** out, cudaStream_t st) {
  int dev = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return IMQ_ERR_UNSUPPORTED;
  int32_t* ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    IMQ_CUDA_TRY(cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone) return IMQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    ptr = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (!ptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return IMQ_ERR_CUDA;
      ptr = static_cast<int32_t*>(p);
      g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
    }
  }
  *out = ptr;
  return IMQ_OK;
}

// The per-row branch of run() with the partials taken from the scratch array: same launch shape, same
// kernel, so the results are those of imq_rtn_quantize with g = IMQ_PER_ROW, trans_out = 0.
template <typename T, bool kOut16>
imq_status run_rows_noalloc(const T* X, int64_t rows, int64_t cols, int64_t ld, double p, int32_t beta,
                            void* Xint, int64_t ldq, float* delta, float* qval, int32_t* rowmax, int32_t* colmax,
                            DeviceState* ds, cudaStream_t st) {
  // the launch shape of the allocating per-row path, from the same helper
  RowsShape sh;
  if (!rows_launch_shape(rows, cols, sizeof(T), colmax != nullptr, ds->num_sms, &sh)) return IMQ_ERR_UNSUPPORTED;
  const int64_t grid = sh.grid;
  const int nwarps = sh.nwarps;
  const size_t smem = sh.smem;
  const bool vec = (cols % (16 / (int64_t)sizeof(T)) == 0) && (ld % (16 / (int64_t)sizeof(T)) == 0) &&
                   ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  int32_t* part = nullptr;
  if (colmax) {
    // checked before anything is launched: the kernel writes grid x cols partials
    if ((uint64_t)grid * (uint64_t)cols * sizeof(int32_t) > kNoallocBytes) return IMQ_ERR_UNSUPPORTED;
    imq_status e = noalloc_scratch(&part, st);
    if (e != IMQ_OK) return e;
  }
  auto kern = k_rtn_rows<T, true, kOut16>;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), smem));
  kern<<<(unsigned)grid, kThreads, smem, st>>>(X, rows, cols, ld, (unsigned long long)nearest_rank(cols, p), beta,
                                               Xint, ldq, 0, delta, qval, rowmax, part, nullptr, vec, nwarps,
                                               ds->status, 0);
  if (cudaGetLastError() != cudaSuccess) return IMQ_ERR_CUDA;
  return colmax ? launch_reduce_max(part, grid, cols, colmax, st) : IMQ_OK;
}
}  // namespace

imq_status launch_rtn_quantize_rows_noalloc(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                            double p, int32_t beta, void* Xint, imq_dtype it, int64_t ldq,
                                            float* delta, float* qval, int32_t* rowmax, int32_t* colmax,
                                            cudaStream_t st) {
  if (rows < 0 || cols < 0 || ld < cols || ldq < cols || !(p > 0.0 && p <= 1.0) || beta < 1 || beta > (1 << 24))
    return IMQ_ERR_ARG;
  if (xt != IMQ_F32 && xt != IMQ_BF16) return IMQ_ERR_ARG;
  if (it != IMQ_I16 && it != IMQ_I32) return IMQ_ERR_ARG;
  if (!delta && rows > 0) return IMQ_ERR_ARG;
  if ((!X || !Xint) && rows > 0 && cols > 0) return IMQ_ERR_ARG;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (rows == 0 || cols == 0) {
    // every row is empty: q = max = 0, so s = Delta = 1 and there is nothing to quantise
    if (rowmax && rows > 0) IMQ_CUDA_TRY(cudaMemsetAsync(rowmax, 0, (size_t)rows * 4, st));
    if (colmax && cols > 0) IMQ_CUDA_TRY(cudaMemsetAsync(colmax, 0, (size_t)cols * 4, st));
    if (rows > 0) {
      k_fill_f32<<<1, 256, 0, st>>>(delta, rows, 1.0f);
      if (qval) k_fill_f32<<<1, 256, 0, st>>>(qval, rows, 0.0f);
    }
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  const bool o16 = it == IMQ_I16;
  if (xt == IMQ_BF16) {
    const uint16_t* x = static_cast<const uint16_t*>(X);
    return o16 ? run_rows_noalloc<uint16_t, true>(x, rows, cols, ld, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st)
               : run_rows_noalloc<uint16_t, false>(x, rows, cols, ld, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st);
  }
  const uint32_t* x = static_cast<const uint32_t*>(X);
  return o16 ? run_rows_noalloc<uint32_t, true>(x, rows, cols, ld, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st)
             : run_rows_noalloc<uint32_t, false>(x, rows, cols, ld, p, beta, Xint, ldq, delta, qval, rowmax, colmax, ds, st);
}

// ------------------------------------------------------------------------------------------------
// Fused per-row RTN and unpack (imq_rtn_quantize_unpack).  One warp per row of X: the row is staged in
// shared memory, its percentile selected and its values quantised (as in k_rtn_rows) into an int16 row
// that never leaves shared memory; the warp then writes the row's unpacked line in the plan's layout (a
// 16-position block the plan marked contiguous is one digit plane of 16 consecutive entries, computed
// from two 16-byte reads; any other block is gathered entry by entry).  With a staging order the int16
// row is held in that order (entry t at staging position pinv[t]), which the plan's runs refer to.  Each
// quantised entry is checked
// against the plan's maximum |A[:, t]|: one above it may need a digit the layout does not hold, or break
// the plan's accumulator bound, and sets IMQ_ERR_PLAN.
// ------------------------------------------------------------------------------------------------
namespace {
struct FusedArgs {
  int64_t rows, cols, ld;  // X, row-major
  int64_t K_unp;
  const int32_t* pinv;  // staging position of each inner index (null: the identity)
  const int32_t* tJ;    // staging position of the index at each inner position
  const int8_t* lAk;
  const int32_t* blk16;
  const int32_t* amax;  // [cols] max |A[:, t]| of the plan
  int32_t bm1;
  unsigned long long krank;
  int32_t beta;
  float* delta;
  int8_t* out;
  int32_t* status;
};

// Bytes of shared memory one warp of k_rtn_unpack_rows uses: the staged row and, for fp32 input or a
// staging order, a separate int16 row (a bf16 row in index order is quantised in place: each lane reads
// its 8 entries before writing their 8 int16 values at the same address).
template <typename T>
__host__ __device__ constexpr int64_t fused_warp_bytes(int64_t cols, bool permuted) {
  return (cols * (int64_t)sizeof(T) + 15) / 16 * 16 + (sizeof(T) == 2 && !permuted ? 0 : (cols * 2 + 31) / 32 * 32);
}
constexpr int64_t kFusedMetaMaxChunks = 4096;

template <typename T>
__global__ void __launch_bounds__(kThreads) k_rtn_unpack_rows(const T* __restrict__ X, FusedArgs f, int nwarps,
                                                              int meta_smem) {
  extern __shared__ __align__(16) unsigned char dsm[];
  const int64_t row_bytes = (f.cols * (int64_t)sizeof(T) + 15) / 16 * 16;
  const int64_t wbytes = fused_warp_bytes<T>(f.cols, f.pinv != nullptr);
  __shared__ uint32_t hist_all[kThreads / 32][kSelWords];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nchunk = f.K_unp / 16;
  // [rows of nwarps warps][block starts, int32 x nchunk][first inner levels, int8 x nchunk]
  int32_t* s_blk = reinterpret_cast<int32_t*>(dsm + (int64_t)nwarps * wbytes);
  int8_t* s_lk0 = reinterpret_cast<int8_t*>(s_blk + nchunk);
  if (meta_smem) {
    for (int64_t c = tid; c < nchunk; c += blockDim.x) {
      s_blk[c] = f.blk16[c];
      s_lk0[c] = f.lAk[c * 16];
    }
    __syncthreads();
  }
  if (warp >= nwarps) return;
  T* row = reinterpret_cast<T*>(dsm + (int64_t)warp * wbytes);
  int16_t* qv = sizeof(T) == 2 && !f.pinv ? reinterpret_cast<int16_t*>(row)
                                          : reinterpret_cast<int16_t*>(dsm + (int64_t)warp * wbytes + row_bytes);
  uint32_t* hist = hist_all[warp];
  constexpr int V = 16 / sizeof(T);
  const int n = (int)f.cols;
  const bool vec = (f.cols % V == 0) && (f.ld % V == 0) && ((reinterpret_cast<uintptr_t>(X) & 15) == 0);
  // rows dealt to the CTAs in turn (row r to CTA r mod gridDim.x): every SM gets the same number of rows
  // to within one per CTA
  for (int64_t r = (int64_t)warp * gridDim.x + blockIdx.x; r < f.rows; r += (int64_t)gridDim.x * nwarps) {
    const T* xr = X + r * f.ld;
    if (vec) {
      warp_copy16<8>(reinterpret_cast<const uint4*>(xr), reinterpret_cast<uint4*>(row), n / V, lane);
    } else {
      for (int c = lane; c < n; c += 32) row[c] = xr[c];
    }
    __syncwarp();
    uint32_t mk, bad;
    const float q = Key<T>::from_key(stats_and_select(row, n, f.krank, hist, &mk, &bad));
    float s, dl;
    scale_from_q(q, Key<T>::from_key(mk), f.beta, &s, &dl);
    if (lane == 0) f.delta[r] = dl;
    if (bad) {
      if (lane == 0) set_status(f.status, IMQ_ERR_NONFINITE);
      continue;
    }
    // quantise into the int16 row, 8 entries per lane and step where the row allows, checking coverage
    bool over = false;
    const int n8 = (n % 8 == 0) ? n / 8 : 0;
    for (int g = lane; g < n8; g += 32) {
      uint32_t wd[8];
      {
        const uint4 w0 = reinterpret_cast<const uint4*>(row + g * 8)[0];
        wd[0] = w0.x; wd[1] = w0.y; wd[2] = w0.z; wd[3] = w0.w;
        if (sizeof(T) == 4) {
          const uint4 w1 = reinterpret_cast<const uint4*>(row + g * 8)[1];
          wd[4] = w1.x; wd[5] = w1.y; wd[6] = w1.z; wd[7] = w1.w;
        }
      }
      const int4 m0 = *reinterpret_cast<const int4*>(f.amax + g * 8);
      const int4 m1 = *reinterpret_cast<const int4*>(f.amax + g * 8 + 4);
      const int32_t mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
      int32_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const T e = sizeof(T) == 2 ? (T)((wd[j >> 1] >> (16 * (j & 1))) & 0xFFFFu) : (T)wd[j];
        v[j] = quant_val<true>(Key<T>::value(e), s, f.status, 0);
        over |= (v[j] < 0 ? -v[j] : v[j]) > mm[j];
      }
      if (f.pinv) {
        const int4 j0 = *reinterpret_cast<const int4*>(f.pinv + g * 8);
        const int4 j1 = *reinterpret_cast<const int4*>(f.pinv + g * 8 + 4);
        const int32_t jj[8] = {j0.x, j0.y, j0.z, j0.w, j1.x, j1.y, j1.z, j1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) qv[jj[j]] = (int16_t)v[j];
      } else {
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) pk[j] = ((uint32_t)v[2 * j] & 0xFFFFu) | ((uint32_t)v[2 * j + 1] << 16);
        *reinterpret_cast<uint4*>(qv + g * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    for (int c = n8 * 8 + lane; c < n; c += 32) {
      const int32_t v = quant_val<true>(Key<T>::value(row[c]), s, f.status, 0);
      over |= (v < 0 ? -v : v) > f.amax[c];
      qv[f.pinv ? f.pinv[c] : c] = (int16_t)v;
    }
    if (over) set_status(f.status, IMQ_ERR_PLAN);
    __syncwarp();
    // the unpacked line of row r, 16 inner positions per lane and step
    int8_t* orow = f.out + r * f.K_unp;
    for (int64_t c = lane; c < nchunk; c += 32) {
      const int32_t t0 = meta_smem ? s_blk[c] : f.blk16[c];
      const int64_t p = c * 16;
      uint4 o;
      if (t0 >= 0) {
        const uint4 w0 = *reinterpret_cast<const uint4*>(qv + t0), w1 = *reinterpret_cast<const uint4*>(qv + t0 + 8);
        const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        o = digits16_i16(w, meta_smem ? s_lk0[c] : f.lAk[p], f.bm1);
      } else {
        const int4* tq = reinterpret_cast<const int4*>(f.tJ + p);
        const int4 ta = tq[0], tb = tq[1], tc = tq[2], td = tq[3];
        const int32_t tt[16] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w,
                                tc.x, tc.y, tc.z, tc.w, td.x, td.y, td.z, td.w};
        const int4 lq = *reinterpret_cast<const int4*>(f.lAk + p);
        const int8_t* ll = reinterpret_cast<const int8_t*>(&lq);
        uint32_t w[4];
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          uint32_t packed = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int e = qd * 4 + k;
            const int32_t d = tt[e] >= 0 ? digit_of((int32_t)qv[tt[e]], ll[e], f.bm1) : 0;
            packed |= ((uint32_t)(uint8_t)(int8_t)d) << (8 * k);
          }
          w[qd] = packed;
        }
        o = make_uint4(w[0], w[1], w[2], w[3]);
      }
      *reinterpret_cast<uint4*>(orow + p) = o;
    }
    __syncwarp();
  }
}

template <typename T>
imq_status run_rtn_unpack(const T* X, const FusedArgs& f, DeviceState* ds, cudaStream_t st) {
  const int64_t per_warp = fused_warp_bytes<T>(f.cols, f.pinv != nullptr);
  const int64_t nchunk = f.K_unp / 16;
  const int meta_smem = nchunk <= kFusedMetaMaxChunks ? 1 : 0;
  const size_t meta = meta_smem ? (size_t)nchunk * 5 : 0;
  constexpr size_t kBudget = 200 * 1024;
  if ((size_t)per_warp + meta > kBudget) return IMQ_ERR_UNSUPPORTED;
  // eight warps per CTA while their rows fit in about a third of the budget (several CTAs per SM)
  int nwarps = (int)((kBudget / 3 - meta) / per_warp);
  if (nwarps < 1) nwarps = (int)((kBudget - meta) / per_warp) >= 1 ? 1 : 0;
  if (nwarps < 1) return IMQ_ERR_UNSUPPORTED;
  if (nwarps > kThreads / 32) nwarps = kThreads / 32;
  const size_t smem = (size_t)nwarps * per_warp + meta;
  int per_sm = (int)(kBudget / (smem + kThreads / 32 * kSelWords * 4 + 1024));
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 4) per_sm = 4;
  // one CTA per row up to every resident slot: rows are dealt to the CTAs in turn
  const int64_t grid = f.rows < (int64_t)ds->num_sms * per_sm ? f.rows : (int64_t)ds->num_sms * per_sm;
  IMQ_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(k_rtn_unpack_rows<T>), smem));
  k_rtn_unpack_rows<T><<<(unsigned)grid, kThreads, smem, st>>>(X, f, nwarps, meta_smem);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}
}  // namespace

imq_status launch_rtn_quantize_unpack(const imq_plan_t* pl, const void* X, imq_dtype xt, int64_t ld, double p,
                                      int32_t beta, int8_t* A_unp, float* delta, cudaStream_t st) {
  if (!pl) return IMQ_ERR_ARG;
  const imq_plan_info& I = pl->info;
  if (I.dir_a & IMQ_DIR_OUTER) return IMQ_ERR_ARG;  // A's lines would depend on the new values
  if (xt != IMQ_F32 && xt != IMQ_BF16) return IMQ_ERR_ARG;
  if (ld < I.K || !(p > 0.0 && p <= 1.0) || beta < 1 || beta > (1 << 24)) return IMQ_ERR_ARG;
  if (I.M > 0 && !delta) return IMQ_ERR_ARG;
  if (I.M > 0 && I.K > 0 && (!X || !A_unp)) return IMQ_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(A_unp) & 15) != 0) return IMQ_ERR_ARG;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  if (I.M == 0) return IMQ_OK;
  if (I.K == 0) {
    // empty rows: q = max = 0, so Delta = 1, and A' has no columns
    k_fill_f32<<<1, 256, 0, st>>>(delta, I.M, 1.0f);
    return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
  }
  FusedArgs f;
  f.rows = I.M;
  f.cols = I.K;
  f.ld = ld;
  f.K_unp = I.K_unp;
  f.pinv = pl->pinv;
  f.tJ = pl->tJ;
  f.lAk = pl->lAk;
  f.blk16 = pl->blk16;
  f.amax = pl->max_a_col;
  f.bm1 = I.b - 1;
  f.krank = (unsigned long long)nearest_rank(I.K, p);
  f.beta = beta;
  f.delta = delta;
  f.out = A_unp;
  f.status = ds->status;
  if (xt == IMQ_BF16) return run_rtn_unpack<uint16_t>(static_cast<const uint16_t*>(X), f, ds, st);
  return run_rtn_unpack<uint32_t>(static_cast<const uint32_t*>(X), f, ds, st);
}

}  // namespace imq
