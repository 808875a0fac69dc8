// api.cu -- the C ABI declared in include/imq.h: argument checks, per-device state, status word.
#include <stdlib.h>
#include <string.h>

#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace imq {
imq_status build_plan(const void* A, const void* B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                      int32_t transA, int64_t lda, int32_t transB, int64_t ldb, int32_t b,
                      imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                      const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** out, cudaStream_t st);

namespace {
__device__ int32_t g_status;  // the per-device status word (one instance per device)
DeviceState g_dev[64];
std::mutex g_dev_mu;
}  // namespace

imq_status device_state(DeviceState** out) {
  int dev = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return IMQ_ERR_UNSUPPORTED;
  DeviceState& d = g_dev[dev];
  if (!d.init.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!d.init.load(std::memory_order_relaxed)) {
      void* p = nullptr;
      IMQ_CUDA_TRY(cudaGetSymbolAddress(&p, g_status));
      IMQ_CUDA_TRY(cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev));
      cudaMemPoolProps props;
      memset(&props, 0, sizeof(props));
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      IMQ_CUDA_TRY(cudaMemPoolCreate(&d.pool, &props));
      uint64_t keep = UINT64_MAX;
      IMQ_CUDA_TRY(cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep));
      d.status = static_cast<int32_t*>(p);
      d.init.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return IMQ_OK;
}


namespace {
std::mutex g_smem_mu;
std::map<std::pair<int, const void*>, size_t> g_smem_set;  // (device, kernel) -> limit already set
}  // namespace

cudaError_t ensure_smem(const void* fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_smem_mu);
  size_t& have = g_smem_set[{dev, fn}];
  if (have >= bytes && have > 0) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

cudaError_t blocks_per_sm(const void* fn, int threads, size_t smem, int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, size_t>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, fn, threads, smem);
  const auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, fn, threads, smem);
  if (e == cudaSuccess) cache[key] = *out;
  return e;
}

namespace {
constexpr int kStageRing = 8;
constexpr size_t kStageBytes = 256 * 1024;
struct Staging {
  void* buf[kStageRing] = {};
  cudaEvent_t done[kStageRing] = {};
  int next = 0;
  std::mutex mu;
};
Staging g_staging[64];
}  // namespace

imq_status upload_table(const void* host, size_t bytes, void** dev, cudaStream_t st) {
  *dev = nullptr;
  if (bytes > kStageBytes) return IMQ_ERR_UNSUPPORTED;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  int d = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&d));
  Staging& sg = g_staging[d & 63];
  std::lock_guard<std::mutex> lock(sg.mu);
  const int k = sg.next;
  sg.next = (k + 1) % kStageRing;
  if (!sg.buf[k]) {
    IMQ_CUDA_TRY(cudaMallocHost(&sg.buf[k], kStageBytes));
    IMQ_CUDA_TRY(cudaEventCreateWithFlags(&sg.done[k], cudaEventDisableTiming));
  } else {
    IMQ_CUDA_TRY(cudaEventSynchronize(sg.done[k]));  // the buffer's previous upload has been read
  }
  IMQ_CUDA_TRY(cudaMallocFromPoolAsync(dev, bytes > 0 ? bytes : 16, ds->pool, st));
  memcpy(sg.buf[k], host, bytes);
  if (cudaMemcpyAsync(*dev, sg.buf[k], bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaEventRecord(sg.done[k], st) != cudaSuccess) {
    cudaFreeAsync(*dev, st);
    *dev = nullptr;
    return IMQ_ERR_CUDA;
  }
  return IMQ_OK;
}

namespace {
// Block of 32 x 32 threads: x = 32 consecutive entries (coalesced), y = one of 32 slices of the partials
// (four loads of a thread in flight); the slices are combined in shared memory.
__global__ void __launch_bounds__(1024) k_reduce_max(const int32_t* __restrict__ part, int64_t nparts, int64_t n,
                                                     int32_t* __restrict__ out) {
  __shared__ int32_t red[32][33];
  const int64_t i = (int64_t)blockIdx.x * 32 + threadIdx.x;
  int32_t m = 0;
  if (i < n) {
    int64_t p = threadIdx.y;
    for (; p + 96 < nparts; p += 128) {
      const int32_t a = __ldcs(part + p * n + i), b = __ldcs(part + (p + 32) * n + i);
      const int32_t c = __ldcs(part + (p + 64) * n + i), d = __ldcs(part + (p + 96) * n + i);
      m = max(max(m, a), max(b, max(c, d)));
    }
    for (; p < nparts; p += 32) m = max(m, __ldcs(part + p * n + i));
  }
  red[threadIdx.y][threadIdx.x] = m;
  __syncthreads();
  if (threadIdx.y == 0 && i < n) {
    for (int y = 1; y < 32; ++y) m = max(m, red[y][threadIdx.x]);
    out[i] = m;
  }
}

// One mbarrier that nothing arrives at, waited on by the library's bounded wait: the wait gives up after
// timeout_ns, raises the abort flag and records IMQ_ERR_TIMEOUT, and the kernel returns.
__global__ void k_check_bounded_wait(int32_t* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_addr(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(smem_addr(&bar), 0, &abort_flag, status, timeout_ns);
  __syncthreads();
}
}  // namespace

imq_status launch_reduce_max(const int32_t* part, int64_t nparts, int64_t n, int32_t* out, cudaStream_t st) {
  if (n == 0) return IMQ_OK;
  DeviceState* ds;
  imq_status s = device_state(&ds);
  if (s != IMQ_OK) return s;
  (void)ds;
  k_reduce_max<<<(unsigned)((n + 31) / 32), dim3(32, 32), 0, st>>>(part, nparts, n, out);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

}  // namespace imq

using imq::DeviceState;

extern "C" {

imq_status imq_rtn_quantize(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld, imq_gran g,
                            double p, int32_t beta, void* Xint, imq_dtype it, int64_t ldq, int32_t trans_out,
                            float* delta, float* qval, int32_t* rowmax, int32_t* colmax, imq_stream_t stream) {
  return imq::launch_rtn_quantize(X, xt, rows, cols, ld, g, p, beta, Xint, it, ldq, trans_out, delta, qval, rowmax,
                                  colmax, 0u, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_rtn_quantize_ex(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld, imq_gran g,
                               double p, int32_t beta, void* Xint, imq_dtype it, int64_t ldq, int32_t trans_out,
                               float* delta, float* qval, int32_t* rowmax, int32_t* colmax, uint32_t flags,
                               imq_stream_t stream) {
  return imq::launch_rtn_quantize(X, xt, rows, cols, ld, g, p, beta, Xint, it, ldq, trans_out, delta, qval, rowmax,
                                  colmax, flags, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_rtn_quantize_rows_noalloc(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                         double p, int32_t beta, void* Xint, imq_dtype it, int64_t ldq,
                                         float* delta, float* qval, int32_t* rowmax, int32_t* colmax,
                                         imq_stream_t stream) {
  return imq::launch_rtn_quantize_rows_noalloc(X, xt, rows, cols, ld, p, beta, Xint, it, ldq, delta, qval, rowmax,
                                               colmax, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_plan(const void* A, const void* B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                    int32_t transA, int64_t lda, int32_t transB, int64_t ldb, int32_t b, imq_strategy strategy,
                    const int32_t* a_rowmax, const int32_t* a_colmax, const int32_t* b_rowmax,
                    const int32_t* b_colmax, imq_plan_t** plan, imq_stream_t stream) {
  if (!plan) return IMQ_ERR_ARG;
  *plan = nullptr;
  if (it != IMQ_I16 && it != IMQ_I32) return IMQ_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || b < 2 || b > 8) return IMQ_ERR_ARG;
  if (M > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return IMQ_ERR_UNSUPPORTED;
  if ((int)strategy < 0 || (int)strategy > (int)IMQ_HYBRID) return IMQ_ERR_ARG;
  if (transA != 0 && transA != 1) return IMQ_ERR_ARG;
  if (transB != 0 && transB != 1) return IMQ_ERR_ARG;
  if (lda < (transA ? M : K) || ldb < (transB ? K : N)) return IMQ_ERR_ARG;
  if ((M > 0 && K > 0 && !A) || (K > 0 && N > 0 && !B)) return IMQ_ERR_ARG;
  return imq::build_plan(A, B, it, M, K, N, transA, lda, transB, ldb, b, strategy, a_rowmax, a_colmax, b_rowmax,
                         b_colmax, plan, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_plan_info_get(const imq_plan_t* plan, imq_plan_info* info) {
  if (!plan || !info) return IMQ_ERR_ARG;
  *info = plan->info;
  return IMQ_OK;
}

imq_status imq_plan_levels(const imq_plan_t* plan, int8_t* a_row, int8_t* a_col, int8_t* b_row, int8_t* b_col) {
  if (!plan) return IMQ_ERR_ARG;
  const imq_plan_info& I = plan->info;
  int dev = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  IMQ_CUDA_TRY(cudaSetDevice(plan->device));
  cudaError_t e = cudaSuccess;
  if (a_row && I.M) e = cudaMemcpy(a_row, plan->lv_a_row, (size_t)I.M, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && a_col && I.K) e = cudaMemcpy(a_col, plan->lv_a_col, (size_t)I.K, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && b_row && I.K) e = cudaMemcpy(b_row, plan->lv_b_row, (size_t)I.K, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && b_col && I.N) e = cudaMemcpy(b_col, plan->lv_b_col, (size_t)I.N, cudaMemcpyDeviceToHost);
  cudaSetDevice(dev);
  return e == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

namespace {
// Host copy of one OUTER map: the source line of every unpacked line (device srcX) and its level, which
// follows from the group's level L: the L lines of one source are consecutive inside a group of G.
imq_status outer_map_to_host(const int32_t* d_src, const int32_t* d_grpL, int64_t n_unp, int64_t n_grp, int G,
                             int32_t* src, int8_t* lvl) {
  int32_t* s = src;
  int32_t* tmp = nullptr;
  if (!s) {
    tmp = static_cast<int32_t*>(malloc((size_t)(n_unp > 0 ? n_unp : 1) * 4));
    if (!tmp) return IMQ_ERR_CUDA;
    s = tmp;
  }
  int32_t* gl = static_cast<int32_t*>(malloc((size_t)(n_grp > 0 ? n_grp : 1) * 4));
  cudaError_t e = gl ? cudaSuccess : cudaErrorMemoryAllocation;
  if (e == cudaSuccess && n_unp) e = cudaMemcpy(s, d_src, (size_t)n_unp * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && n_grp) e = cudaMemcpy(gl, d_grpL, (size_t)n_grp * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && lvl)
    for (int64_t u = 0; u < n_unp; ++u) lvl[u] = s[u] < 0 ? 0 : (int8_t)((u % G) % gl[u / G]);
  free(gl);
  free(tmp);
  return e == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}
}  // namespace

imq_status imq_plan_maps(const imq_plan_t* plan, int32_t* tK, int8_t* lAk, int8_t* lBk, int32_t* srcA, int8_t* lvlA,
                         int32_t* srcB, int8_t* lvlB) {
  if (!plan) return IMQ_ERR_ARG;
  const imq_plan_info& I = plan->info;
  int dev = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  IMQ_CUDA_TRY(cudaSetDevice(plan->device));
  imq_status s = IMQ_OK;
  cudaError_t e = cudaDeviceSynchronize();  // the maps kernel runs on the caller's stream
  if (e == cudaSuccess && tK && I.K_unp) e = cudaMemcpy(tK, plan->tK, (size_t)I.K_unp * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && lAk && I.K_unp) e = cudaMemcpy(lAk, plan->lAk, (size_t)I.K_unp, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && lBk && I.K_unp) e = cudaMemcpy(lBk, plan->lBk, (size_t)I.K_unp, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) s = IMQ_ERR_CUDA;
  if (s == IMQ_OK) {
    if (I.dir_a & IMQ_DIR_OUTER) {
      s = outer_map_to_host(plan->srcA, plan->grpA_L, I.M_unp, plan->n_grp_a, IMQ_A_GROUP, srcA, lvlA);
    } else {
      for (int64_t u = 0; u < I.M_unp; ++u) {
        if (srcA) srcA[u] = (int32_t)u;
        if (lvlA) lvlA[u] = 0;
      }
    }
  }
  if (s == IMQ_OK) {
    if (I.dir_b & IMQ_DIR_OUTER) {
      s = outer_map_to_host(plan->srcB, plan->grpB_L, I.N_unp, plan->n_grp_b, IMQ_B_GROUP, srcB, lvlB);
    } else {
      for (int64_t w = 0; w < I.N_unp; ++w) {
        if (srcB) srcB[w] = (int32_t)w;
        if (lvlB) lvlB[w] = 0;
      }
    }
  }
  cudaSetDevice(dev);
  return s;
}

imq_status imq_plan_groups(const imq_plan_t* plan, imq_group* groups, int32_t max_groups, int32_t* n_out) {
  if (!plan || !n_out || (max_groups > 0 && !groups)) return IMQ_ERR_ARG;
  const int n = plan->info.n_groups;
  for (int i = 0; i < n && i < max_groups; ++i) groups[i] = plan->groups[i];
  *n_out = n;
  return IMQ_OK;
}

imq_status imq_plan_destroy(imq_plan_t* plan) {
  if (!plan) return IMQ_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaSetDevice(plan->device);
  cudaError_t e1 = cudaSuccess, e2 = cudaSuccess;
  if (plan->dev_block) e1 = cudaFreeAsync(plan->dev_block, 0);
  if (plan->dev_block2) e2 = cudaFreeAsync(plan->dev_block2, 0);
  cudaSetDevice(dev);
  free(plan->host_tables);
  delete plan;
  return (e1 == cudaSuccess && e2 == cudaSuccess) ? IMQ_OK : IMQ_ERR_CUDA;
}

imq_status imq_unpack(const imq_plan_t* plan, const void* A, const void* B, int8_t* A_unp, int8_t* B_unp_t,
                      imq_stream_t stream) {
  if (!plan) return IMQ_ERR_ARG;
  const imq_plan_info& I = plan->info;
  if (I.K_unp > 0 && ((I.M_unp > 0 && !A_unp) || (I.N_unp > 0 && !B_unp_t))) return IMQ_ERR_ARG;
  if ((I.M > 0 && I.K > 0 && !A) || (I.K > 0 && I.N > 0 && !B)) return IMQ_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(A_unp) & 15) || (reinterpret_cast<uintptr_t>(B_unp_t) & 15)) return IMQ_ERR_ARG;
  return imq::launch_unpack(plan, A, B, A_unp, B_unp_t, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_rtn_quantize_unpack(const imq_plan_t* plan, const void* X, imq_dtype xt, int64_t ld, double p,
                                   int32_t beta, int8_t* A_unp, float* deltaA, imq_stream_t stream) {
  return imq::launch_rtn_quantize_unpack(plan, X, xt, ld, p, beta, A_unp, deltaA,
                                         reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_gemm_unpacked(const imq_plan_t* plan, const int8_t* A_unp, const int8_t* B_unp_t, const float* deltaA,
                             imq_gran gA, const float* deltaB, imq_gran gB, void* Cint, imq_dtype ct, int64_t ldc,
                             float* Cf, int64_t ldcf, imq_stream_t stream) {
  if (!plan) return IMQ_ERR_ARG;
  return imq::launch_gemm(plan, A_unp, B_unp_t, deltaA, gA, deltaB, gB, Cint, ct, ldc, Cf, ldcf,
                          reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_unpacked_gemm(const imq_plan_t* plan, const void* A, const void* B, const float* deltaA, imq_gran gA,
                             const float* deltaB, imq_gran gB, void* Cint, imq_dtype ct, int64_t ldc, float* Cf,
                             int64_t ldcf, void* workspace, size_t workspace_bytes, imq_stream_t stream) {
  if (!plan) return IMQ_ERR_ARG;
  const imq_plan_info& I = plan->info;
  if (workspace_bytes < I.workspace_bytes) return IMQ_ERR_BUFFER;
  if (I.workspace_bytes > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 1023))) return IMQ_ERR_ARG;
  // argument checks of the GEMM first, so a bad call launches nothing
  if (!Cint && !Cf) return IMQ_ERR_ARG;
  if (Cint && ct == IMQ_I32 && I.acc_bits > 32) return IMQ_ERR_RANGE;
  int8_t* Au = static_cast<int8_t*>(workspace);
  const size_t a_bytes = ((size_t)(I.M_unp * I.K_unp) + 1023) / 1024 * 1024;
  int8_t* Bu = Au ? Au + a_bytes : nullptr;
  imq_status s = imq_unpack(plan, A, B, Au, Bu, stream);
  if (s != IMQ_OK) return s;
  return imq_gemm_unpacked(plan, Au, Bu, deltaA, gA, deltaB, gB, Cint, ct, ldc, Cf, ldcf, stream);
}

imq_status imq_plan_unpack(const void* A, const void* B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                           int32_t transA, int64_t lda, int32_t transB, int64_t ldb, int32_t b,
                           imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                           const int32_t* b_rowmax, const int32_t* b_colmax, void* workspace,
                           size_t workspace_bytes, imq_plan_t** plan, imq_stream_t stream) {
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 1023)) return IMQ_ERR_ARG;
  imq_status s = imq_plan(A, B, it, M, K, N, transA, lda, transB, ldb, b, strategy, a_rowmax, a_colmax, b_rowmax,
                          b_colmax, plan, stream);
  if (s != IMQ_OK) return s;
  const imq_plan_info& I = (*plan)->info;
  if (I.workspace_bytes > 0 && (!workspace || workspace_bytes < I.workspace_bytes)) return IMQ_ERR_BUFFER;
  int8_t* Au = static_cast<int8_t*>(workspace);
  const size_t a_bytes = ((size_t)(I.M_unp * I.K_unp) + 1023) / 1024 * 1024;
  return imq_unpack(*plan, A, B, Au, Au ? Au + a_bytes : nullptr, stream);
}

imq_status imq_level_cover(const int32_t* maxima, int64_t n, int32_t b, int32_t cap, int32_t* out,
                           imq_stream_t stream) {
  if (n < 0 || b < 2 || b > 8 || cap < 0 || (n > 0 && (!maxima || !out))) return IMQ_ERR_ARG;
  return imq::launch_level_cover(maxima, n, b, cap, out, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_plan_batched(int32_t batch, const void* A, int64_t strideA, const void* B, int64_t strideB, imq_dtype it,
                            int64_t M, int64_t K, int64_t N, int32_t transA, int64_t lda, int32_t transB, int64_t ldb,
                            int32_t b, imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                            const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** plans,
                            imq_stream_t stream) {
  if (!plans || batch < 0) return IMQ_ERR_ARG;
  for (int32_t h = 0; h < batch; ++h) plans[h] = nullptr;
  if (batch == 0) return IMQ_OK;
  if (it != IMQ_I16 && it != IMQ_I32) return IMQ_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || b < 2 || b > 8 || strideA < 0 || strideB < 0) return IMQ_ERR_ARG;
  if (M > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return IMQ_ERR_UNSUPPORTED;
  if ((int)strategy < 0 || (int)strategy > (int)IMQ_HYBRID) return IMQ_ERR_ARG;
  if ((transA != 0 && transA != 1) || (transB != 0 && transB != 1)) return IMQ_ERR_ARG;
  if (lda < (transA ? M : K) || ldb < (transB ? K : N)) return IMQ_ERR_ARG;
  if ((M > 0 && K > 0 && !A) || (K > 0 && N > 0 && !B)) return IMQ_ERR_ARG;
  return imq::build_plans(batch, A, strideA, B, strideB, it, M, K, N, transA, lda, transB, ldb, b, strategy,
                          a_rowmax, a_colmax, b_rowmax, b_colmax, plans, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
size_t align1k(size_t x) { return (x + 1023) / 1024 * 1024; }

// The batch workspace: for each plan its A' then its B'^T, each from a 1024-byte boundary.
imq_status batch_layout(int32_t batch, imq_plan_t* const* plans, size_t* offsets, size_t* total) {
  if (batch < 0 || (batch > 0 && !plans)) return IMQ_ERR_ARG;
  size_t off = 0;
  for (int32_t h = 0; h < batch; ++h) {
    if (!plans[h]) return IMQ_ERR_ARG;
    const imq_plan_info& I = plans[h]->info;
    if (offsets) offsets[2 * h] = off;
    off += align1k((size_t)(I.M_unp * I.K_unp));
    if (offsets) offsets[2 * h + 1] = off;
    off += align1k((size_t)(I.N_unp * I.K_unp));
  }
  *total = off;
  return IMQ_OK;
}

// Same device, same shapes, b, layouts and strategy: the plans of one imq_plan_batched call.
bool same_batch(int32_t batch, imq_plan_t* const* plans) {
  const imq_plan_t* p0 = plans[0];
  for (int32_t h = 1; h < batch; ++h) {
    const imq_plan_t* p = plans[h];
    if (p->device != p0->device || p->it != p0->it || p->transA != p0->transA || p->transB != p0->transB ||
        p->lda != p0->lda || p->ldb != p0->ldb || p->info.M != p0->info.M || p->info.K != p0->info.K ||
        p->info.N != p0->info.N || p->info.b != p0->info.b)
      return false;
  }
  return true;
}
}  // namespace

imq_status imq_batch_workspace(int32_t batch, imq_plan_t* const* plans, size_t* offsets, size_t* total_bytes) {
  if (!total_bytes) return IMQ_ERR_ARG;
  return batch_layout(batch, plans, offsets, total_bytes);
}

imq_status imq_unpack_batched(int32_t batch, imq_plan_t* const* plans, const void* A, int64_t strideA, const void* B,
                              int64_t strideB, void* workspace, size_t workspace_bytes, imq_stream_t stream) {
  if (batch == 0) return IMQ_OK;
  size_t total = 0;
  std::vector<size_t> off((size_t)batch * 2);
  imq_status s = batch_layout(batch, plans, off.data(), &total);
  if (s != IMQ_OK) return s;
  if (!same_batch(batch, plans)) return IMQ_ERR_ARG;
  if (workspace_bytes < total) return IMQ_ERR_BUFFER;
  if (total > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 1023))) return IMQ_ERR_ARG;
  if (strideA < 0 || strideB < 0) return IMQ_ERR_ARG;
  const imq_plan_info& I0 = plans[0]->info;
  if ((I0.M > 0 && I0.K > 0 && !A) || (I0.K > 0 && I0.N > 0 && !B)) return IMQ_ERR_ARG;
  const size_t esz = plans[0]->it == IMQ_I16 ? 2 : 4;
  std::vector<const void*> pa((size_t)batch), pb((size_t)batch);
  std::vector<int8_t*> wa((size_t)batch), wb((size_t)batch);
  for (int32_t h = 0; h < batch; ++h) {
    pa[h] = static_cast<const char*>(A) + (size_t)h * strideA * esz;
    pb[h] = static_cast<const char*>(B) + (size_t)h * strideB * esz;
    wa[h] = static_cast<int8_t*>(workspace) + off[2 * h];
    wb[h] = static_cast<int8_t*>(workspace) + off[2 * h + 1];
  }
  int dev = 0;
  IMQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != plans[0]->device) return IMQ_ERR_ARG;
  return imq::launch_unpack_batch(plans, batch, pa.data(), pb.data(), wa.data(), wb.data(),
                                  reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_gemm_unpacked_batched(int32_t batch, imq_plan_t* const* plans, const void* workspace,
                                     size_t workspace_bytes, const float* deltaA, int64_t strideDA, imq_gran gA,
                                     const float* deltaB, int64_t strideDB, imq_gran gB, void* Cint, int64_t strideC,
                                     imq_dtype ct, int64_t ldc, float* Cf, int64_t strideCf, int64_t ldcf,
                                     imq_stream_t stream) {
  if (batch == 0) return IMQ_OK;
  size_t total = 0;
  std::vector<size_t> off((size_t)batch * 2);
  imq_status s = batch_layout(batch, plans, off.data(), &total);
  if (s != IMQ_OK) return s;
  if (!same_batch(batch, plans)) return IMQ_ERR_ARG;
  if (workspace_bytes < total) return IMQ_ERR_BUFFER;
  if (total > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 1023))) return IMQ_ERR_ARG;
  if (strideDA < 0 || strideDB < 0 || strideC < 0 || strideCf < 0) return IMQ_ERR_ARG;
  const size_t csz = ct == IMQ_I64 ? 8 : 4;
  std::vector<imq::GemmSpec> specs((size_t)batch);
  for (int32_t h = 0; h < batch; ++h) {
    imq::GemmSpec& g = specs[h];
    g.plan = plans[h];
    g.Au = static_cast<const int8_t*>(workspace) + off[2 * h];
    g.Bu = static_cast<const int8_t*>(workspace) + off[2 * h + 1];
    g.dA = deltaA ? deltaA + (size_t)h * strideDA : nullptr;
    g.gA = gA;
    g.dB = deltaB ? deltaB + (size_t)h * strideDB : nullptr;
    g.gB = gB;
    g.C = Cint ? static_cast<char*>(Cint) + (size_t)h * strideC * csz : nullptr;
    g.ct = ct;
    g.ldc = ldc;
    g.Cf = Cf ? Cf + (size_t)h * strideCf : nullptr;
    g.ldcf = ldcf;
  }
  return imq::launch_gemm_multi(specs.data(), batch, reinterpret_cast<cudaStream_t>(stream));
}

imq_status imq_unpacked_gemm_batched(int32_t batch, imq_plan_t* const* plans, const void* A, int64_t strideA,
                                     const void* B, int64_t strideB, const float* deltaA, int64_t strideDA,
                                     imq_gran gA, const float* deltaB, int64_t strideDB, imq_gran gB, void* Cint,
                                     int64_t strideC, imq_dtype ct, int64_t ldc, float* Cf, int64_t strideCf,
                                     int64_t ldcf, void* workspace, size_t workspace_bytes, imq_stream_t stream) {
  imq_status s = imq_unpack_batched(batch, plans, A, strideA, B, strideB, workspace, workspace_bytes, stream);
  if (s != IMQ_OK) return s;
  return imq_gemm_unpacked_batched(batch, plans, workspace, workspace_bytes, deltaA, strideDA, gA, deltaB, strideDB,
                                   gB, Cint, strideC, ct, ldc, Cf, strideCf, ldcf, stream);
}

imq_status imq_check_bounded_wait(uint64_t timeout_ns, imq_stream_t stream) {
  if (timeout_ns < 1000ull || timeout_ns > 1000000000ull) return IMQ_ERR_ARG;
  DeviceState* ds;
  imq_status s = imq::device_state(&ds);
  if (s != IMQ_OK) return s;
  imq::k_check_bounded_wait<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ds->status, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? IMQ_OK : IMQ_ERR_CUDA;
}

imq_status imq_device_status(imq_stream_t stream, int32_t clear) {
  DeviceState* ds;
  imq_status s = imq::device_state(&ds);
  if (s != IMQ_OK) return s;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  IMQ_CUDA_TRY(cudaMemcpyAsync(&v, ds->status, 4, cudaMemcpyDeviceToHost, st));
  IMQ_CUDA_TRY(cudaStreamSynchronize(st));
  if (clear) {
    IMQ_CUDA_TRY(cudaMemsetAsync(ds->status, 0, 4, st));
    IMQ_CUDA_TRY(cudaStreamSynchronize(st));
  }
  return (imq_status)v;
}

const char* imq_status_str(imq_status s) {
  switch (s) {
    case IMQ_OK: return "ok";
    case IMQ_ERR_ARG: return "invalid argument";
    case IMQ_ERR_NONFINITE: return "non-finite input";
    case IMQ_ERR_RANGE: return "integer range exceeded";
    case IMQ_ERR_BUFFER: return "buffer too small";
    case IMQ_ERR_TIMEOUT: return "bounded wait timed out in a kernel";
    case IMQ_ERR_CUDA: return "CUDA runtime error";
    case IMQ_ERR_UNSUPPORTED: return "unsupported input";
    case IMQ_ERR_PLAN: return "input not covered by the plan";
    case IMQ_ERR_BOUNDS: return "plan index outside the plan's sizes (debug build)";
  }
  return "unknown status";
}

}  // extern "C"
