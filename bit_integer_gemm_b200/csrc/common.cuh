// common.cuh -- shared device helpers of the IM-Unpack CUDA library (sm_100a only).
//
// Inline-PTX wrappers for mbarriers, TMA bulk-tensor loads and the tcgen05 tensor-core / tensor-memory
// instructions, a bounded mbarrier wait that turns a would-be hang into an error status, and the
// per-device status word every kernel reports into.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "imq.h"

namespace imq {

// ------------------------------------------------------------------------------------------------
// status word: the first error a kernel meets is kept (atomicCAS from IMQ_OK)
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, (int32_t)IMQ_OK, code);
}

// ------------------------------------------------------------------------------------------------
// shared memory / barriers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------------------------------------
// clusters of two CTAs (the pair that shares one cta_group::2 MMA)
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier that may live in another CTA of the cluster.  The default (CTA-scope release)
// semantics: the arrive is used after tcgen05.wait + tcgen05.fence::before_thread_sync to hand tensor
// memory back to the MMA issuer, which orders the tcgen05 reads; a cluster-scope release would also
// wait for every prior global store of the thread to become visible, which that hand-over never needs.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Every thread of every CTA of the cluster arrives, then waits for all the others.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase of `bar` with the given parity.  Gives up (returns false) when *abort is set by
// another role, or after timeout_ns of wall time, in which case it raises *abort and records
// IMQ_ERR_TIMEOUT.  Every wait in the library's kernels goes through here.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int32_t* status, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > timeout_ns) {
        *abort = 1;
        set_status(status, IMQ_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Named barrier over `nthreads` threads (multiple of 32), id 1..15 (0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------------------------------------
// TMA.  Every tensor load here copies into the issuing CTA's own shared memory; none is multicast.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// The same load issued by either CTA of an MMA pair: the bytes land in the issuing CTA's own shared
// memory and complete_tx is signalled on `cluster_bar`, a barrier of the pair's leading CTA.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                                 uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}

// ------------------------------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor core
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, s8 x s8 -> s32, one CTA.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// The CTA-pair forms (cta_group::2).  Allocation, relinquish and release are issued by the same warp
// of both CTAs; the MMA and its commits only by the leading CTA.  D (M=256) spans both CTAs' tensor
// memory at the same address: each CTA holds 128 rows x N.  A comes 128 rows from each CTA's shared
// memory and B N/2 columns from each, at the same offsets as the descriptors give for the leader.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the barrier at offset `bar` of every CTA in `cta_mask` when the pair's prior MMAs
// issued by this thread have completed.
__device__ __forceinline__ void mma_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with 128-byte swizzle:
// rows of 128 bytes, 8-row swizzle atoms of 1024 bytes stacked densely (stride byte offset 1024).
// Fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30) (unused for swizzled K-major,
// set to 1), stride byte offset >> 4 [32,46), descriptor version 1 [46,48), base offset 0, layout
// SWIZZLE_128B (2) [61,64).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor of kind::i8: s32 accumulator, signed A and B, both K-major, M x N tile.
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ------------------------------------------------------------------------------------------------
// integer helpers shared by the quantiser, planner and unpacker kernels
// ------------------------------------------------------------------------------------------------
// Sign-magnitude base-2^(b-1) digit l of v: sgn(v) * ((|v| >> l(b-1)) & (2^(b-1) - 1)).
__device__ __forceinline__ int32_t digit_of(int32_t v, int32_t l, int32_t bm1) {
  const int32_t sh = l * bm1;
  if (sh >= 31) return 0;
  const uint32_t m = v < 0 ? (uint32_t)(-(int64_t)v) : (uint32_t)v;
  const int32_t d = (int32_t)((m >> sh) & ((1u << bm1) - 1u));
  return v < 0 ? -d : d;
}

// Warp-aggregated shared-memory increment: lanes with equal keys add their count once, so a hot bin
// costs one atomic per warp instead of one per lane.  Every lane of the warp must call it; `active`
// lanes contribute.
__device__ __forceinline__ void warp_count(uint32_t* base, uint32_t key, bool active) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, key);
  const int leader = __ffs(peers) - 1;
  if ((int)(threadIdx.x & 31) == leader) atomicAdd(base + key, (uint32_t)__popc(peers));
}

// Magnitudes and signs of 16 int16 entries held as 8 words (two entries per word, low half first):
// |entry| per half without a carry between halves, and per 4 entries a byte mask (0xFF where the entry
// is negative) in entry order.
struct Mag16 {
  uint32_t a[8];
  uint32_t neg[4];
};
__device__ __forceinline__ Mag16 mag16_i16(const uint32_t (&w)[8]) {
  Mag16 m;
  uint32_t S[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const uint32_t sgn = (w[h] >> 15) & 0x00010001u;  // 1 in each negative half
    S[h] = sgn * 0xFFFFu;                              // 0xFFFF in each negative half
    m.a[h] = (w[h] ^ S[h]) + sgn;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) m.neg[q] = __byte_perm(S[2 * q], S[2 * q + 1], 0x6420);
  return m;
}

// Digit l (base 2^bm1, sign-magnitude) of the 16 entries of m, as 16 bytes in entry order: the digit's
// bits are masked, then shifted down within each half; a byte permute gathers the four digits of two
// words; negative entries' digits are negated byte-wise as (0x80808080 - d) ^ 0x80808080 (a digit is at
// most 127, so no byte borrows).  Digits with l * bm1 >= 16 are zero for int16 magnitudes.
__device__ __forceinline__ uint4 digits16_from(const Mag16& m, int l, int bm1) {
  const int sh = l * bm1;
  if (sh >= 16) return make_uint4(0u, 0u, 0u, 0u);
  const uint32_t m2 = ((((1u << bm1) - 1u) << sh) & 0xFFFFu) * 0x00010001u;
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t d0 = (m.a[2 * q] & m2) >> sh, d1 = (m.a[2 * q + 1] & m2) >> sh;
    const uint32_t pd = __byte_perm(d0, d1, 0x6420);
    const uint32_t nd = (0x80808080u - pd) ^ 0x80808080u;
    o[q] = (pd & ~m.neg[q]) | (nd & m.neg[q]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Digit l of 16 int16 entries held as 8 words, as 16 bytes in entry order.
__device__ __forceinline__ uint4 digits16_i16(const uint32_t (&w)[8], int l, int bm1) {
  if (l * bm1 >= 16) return make_uint4(0u, 0u, 0u, 0u);
  return digits16_from(mag16_i16(w), l, bm1);
}

// Number of base-2^(b-1) digits of m (>= 1).
__device__ __forceinline__ int32_t level_of(uint32_t m, int32_t bm1) {
  if (m == 0) return 1;
  const int32_t bits = 32 - __clz(m);
  return (bits + bm1 - 1) / bm1;
}

}  // namespace imq
