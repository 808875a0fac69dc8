// internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <vector>
#include <stddef.h>
#include <stdint.h>

#include "imq.h"

namespace imq {

constexpr int kMaxJobs = 128;  // accumulation jobs of one output tile

// Per-device state owned by the library: the status word address, the SM count and the memory pool.
struct DeviceState {
  int32_t* status = nullptr;   // device address of the status word of this device
  int num_sms = 0;
  // stream-ordered pool for plan memory and the quantiser's per-call scratch; it keeps what is freed
  // (no trim at synchronisation), so later calls reuse memory instead of mapping fresh pages
  cudaMemPool_t pool = nullptr;
  // set (release) after every field above; read with acquire before any of them is used
  std::atomic<bool> init{false};
};
imq_status device_state(DeviceState** out);
// Raises the dynamic shared-memory limit of kernel `fn` on the current device to at least `bytes`.  The
// attribute call costs microseconds of host time, so it is made only when no earlier call on this device
// already set a limit at least as large.
cudaError_t ensure_smem(const void* fn, size_t bytes);
// Resident blocks per SM of kernel fn at this block size and dynamic shared memory (the occupancy
// query, cached per device, kernel and configuration).
cudaError_t blocks_per_sm(const void* fn, int threads, size_t smem, int* out);
// Copies a small host table to new device memory from the library's pool, through pinned staging (a
// ring of buffers, each reused once its previous upload has completed), in stream order on `st`.  The
// caller frees *dev with cudaFreeAsync on `st` after the kernels that read it.
imq_status upload_table(const void* host, size_t bytes, void** dev, cudaStream_t st);
// out[i] = max over p < nparts of part[p * n + i] (int32, non-negative); nparts may be 0 (out = 0).
imq_status launch_reduce_max(const int32_t* part, int64_t nparts, int64_t n, int32_t* out, cudaStream_t st);

// Percentile + RTN quantisation (rtn.cu).
imq_status launch_rtn_quantize(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               imq_gran g, double p, int32_t beta, void* Xint, imq_dtype it,
                               int64_t ldq, int32_t trans_out, float* delta, float* qval, int32_t* rowmax,
                               int32_t* colmax, uint32_t flags, cudaStream_t stream);
// imq_rtn_quantize_rows_noalloc: the per-row quantiser with its scratch in a fixed device array.
imq_status launch_rtn_quantize_rows_noalloc(const void* X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                            double p, int32_t beta, void* Xint, imq_dtype it, int64_t ldq,
                                            float* delta, float* qval, int32_t* rowmax, int32_t* colmax,
                                            cudaStream_t stream);

// imq_level_cover (plan.cu).
imq_status launch_level_cover(const int32_t* maxima, int64_t n, int32_t b, int32_t cap, int32_t* out,
                              cudaStream_t stream);
// Line maxima of an integer matrix (plan.cu): logical rows and columns of a stored matrix.
imq_status launch_line_max(const void* X, imq_dtype it, int64_t rows, int64_t cols, int64_t ld,
                           int32_t* rowmax, int32_t* colmax, cudaStream_t stream);

}  // namespace imq

// The plan object (opaque in the public header).
struct imq_plan {
  imq_plan_info info;
  int device;
  // inputs the plan was made from
  const void* A;
  const void* B;
  imq_dtype it;
  int32_t transA, transB;
  int64_t lda, ldb;
  // one device allocation holding every array below
  void* dev_block;   // stage 1: line maxima, levels, summary
  void* dev_block2;  // stage 2: index maps
  size_t dev_bytes;
  void* host_tables; // segment and class tables copied to the device (kept until destroy)
  int32_t* max_a_row;
  int32_t* max_a_col;
  int32_t* max_b_row;
  int32_t* max_b_col;
  int8_t* lv_a_row;
  int8_t* lv_a_col;
  int8_t* lv_b_row;
  int8_t* lv_b_col;
  int32_t* tK;      // [K_unp] source inner index, -1 on padding
  int8_t* lAk;      // [K_unp] digit level of A at that inner position
  int8_t* lBk;      // [K_unp] digit level of B
  int32_t* perm;    // [K] staging order: the inner index at each staging position (indices grouped by
                    // their (A column, B row) level class); null when the order is the identity
  int32_t* pinv;    // [K] staging position of each inner index; null with perm
  int32_t* tJ;      // [K_unp] staging position of the index at each inner position, -1 on padding (tK
                    // itself when perm is null)
  int32_t* blk16;   // [K_unp/16] when positions 16c..16c+15 hold the indices at staging positions
                    // j0..j0+15 with one (lA, lB) pair: j0 if j0 % 16 == 0, else -(j0 + 2); otherwise -1
                    // (the unpackers stage a source line in staging order and copy runs)
  int32_t* posA;    // [M] first unpacked row of each source row (A OUTER)
  int32_t* srcA;    // [M_unp] source row of each unpacked row, -1 unused (A OUTER)
  int32_t* grpA_L;  // [M_unp / IMQ_A_GROUP] level of each row group
  int32_t* grpA_n;  // [...] number of source rows in the group
  int32_t* posB;    // [N]
  int32_t* srcB;    // [N_unp]
  int32_t* grpB_L;  // [N_unp / IMQ_B_GROUP]
  int32_t* grpB_n;
  int64_t n_grp_a, n_grp_b;
  int32_t cls_b0, cls_b1;  // B's OUTER level classes: entries cls_b0 .. cls_b1 - 1 of the host class table
  imq_group groups[IMQ_MAX_GROUPS];
  // GEMM schedule of one output tile (see gemm.cu): a sequence of steps, each one exponent group (or a
  // K-slice of one) accumulated into the tile's TMEM slot.  Consecutive steps of a chunk follow Horner's
  // rule (the slot is multiplied by R^(e_prev - e) between them); at the end of a chunk the slot is
  // drained into C, shifted by e_last * (b - 1).
  int32_t n_steps;
  int64_t step_k0[imq::kMaxJobs];     // first unpacked inner index (multiple of IMQ_INNER_PAD)
  int64_t step_klen[imq::kMaxJobs];   // inner length (multiple of IMQ_INNER_PAD)
  int32_t step_first[imq::kMaxJobs];  // 1: first step of its chunk (the MMA overwrites the slot)
  int32_t step_after[imq::kMaxJobs];  // >= 0: left shift applied to the slot after this step (Horner);
                                      // -1: the chunk ends here and the slot is drained
  int32_t step_drain_shift[imq::kMaxJobs];
  int32_t n_chunks;
};

namespace imq {
// Fused per-row RTN of X and unpack into the plan's A' layout (rtn.cu).
imq_status launch_rtn_quantize_unpack(const imq_plan_t* pl, const void* X, imq_dtype xt, int64_t ld, double p,
                                      int32_t beta, int8_t* A_unp, float* delta, cudaStream_t stream);
imq_status launch_unpack(const imq_plan_t* pl, const void* A, const void* B, int8_t* Au, int8_t* Bu,
                         cudaStream_t stream);
// The unpack of n plans made together (imq_plan_batched): as few launches as their kernels allow.
imq_status launch_unpack_batch(const imq_plan_t* const* pls, int n, const void* const* A, const void* const* B,
                               int8_t* const* Au, int8_t* const* Bu, cudaStream_t stream);
// Plans of `batch` equal-shaped problems with one host round trip (plan.cu).
imq_status build_plans(int batch, const void* A, int64_t strideA, const void* B, int64_t strideB, imq_dtype it,
                       int64_t M, int64_t K, int64_t N, int32_t transA, int64_t lda, int32_t transB, int64_t ldb,
                       int32_t b, imq_strategy strategy, const int32_t* a_rowmax, const int32_t* a_colmax,
                       const int32_t* b_rowmax, const int32_t* b_colmax, imq_plan_t** out, cudaStream_t st);
imq_status launch_gemm(const imq_plan_t* pl, const int8_t* Au, const int8_t* Bu, const float* dA,
                       imq_gran gA, const float* dB, imq_gran gB, void* C, imq_dtype ct,
                       int64_t ldc, float* Cf, int64_t ldcf, cudaStream_t stream);
// One GEMM problem: a plan, its unpacked operands, scales and outputs (the arguments of imq_gemm_unpacked).
struct GemmSpec {
  const imq_plan_t* plan;
  const int8_t* Au;
  const int8_t* Bu;
  const float* dA;
  imq_gran gA;
  const float* dB;
  imq_gran gB;
  void* C;
  imq_dtype ct;
  int64_t ldc;
  float* Cf;
  int64_t ldcf;
};
// For B unpacked OUTER: the relative position in N of each group of B'^T's lines, the middle rank of its
// sources within their level class over the class's size (sources are spread over N, so groups of equal
// position in different classes cover about the same output columns).  False when B is not OUTER (plan.cu).
bool b_group_positions(const imq_plan_t* pl, std::vector<float>* pos);
// The GEMMs of n problems in as few launches as the problem table allows (gemm.cu).
imq_status launch_gemm_multi(const GemmSpec* specs, int n, cudaStream_t stream);
}  // namespace imq

#define IMQ_CUDA_TRY(expr)                                    \
  do {                                                        \
    cudaError_t e_ = (expr);                                  \
    if (e_ != cudaSuccess) return IMQ_ERR_CUDA;               \
  } while (0)
