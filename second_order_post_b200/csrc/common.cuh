// Shared helpers of libkronq: status plumbing, tensor-map creation and the
// sm_100a PTX wrappers (mbarrier, TMA bulk-tensor loads, tcgen05 MMA / TMEM).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kronq.h"

namespace kronq {

template <class T>
__host__ __device__ __forceinline__ T kq_min(T a, T b) { return a < b ? a : b; }
template <class T>
__host__ __device__ __forceinline__ T kq_max(T a, T b) { return a < b ? b : a; }

// ----------------------------------------------------------------- host side
// Counts every kernel the library launches (reported by kronq_kernel_launches).
void count_launch();

// Records a failed CUDA call (reported by kronq_last_cuda_error) and returns
// KRONQ_ERR_CUDA.
kronq_status cuda_fail(cudaError_t e);

#define KQ_CHECK_LAUNCH()                                                      \
  do {                                                                         \
    count_launch();                                                            \
    cudaError_t e_ = cudaGetLastError();                                       \
    if (e_ != cudaSuccess) return ::kronq::cuda_fail(e_);                      \
  } while (0)

#define KQ_CUDA(expr)                                                          \
  do {                                                                         \
    cudaError_t e_ = (expr);                                                   \
    if (e_ != cudaSuccess) return ::kronq::cuda_fail(e_);                      \
  } while (0)

#define KQ_TRY(expr)                                                           \
  do {                                                                         \
    kronq_status s_ = (expr);                                                  \
    if (s_ != KRONQ_OK) return s_;                                             \
  } while (0)

// Device ordinal check: the library runs on sm_100 only.
kronq_status require_sm100();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device. The attribute belongs to the device context, so it is set once per
// (device, kernel, size); thread-safe.
kronq_status set_max_dyn_smem(const void *func, int bytes);
template <class F>
inline kronq_status smem_attr(F *func, int bytes) {
  return set_max_dyn_smem(reinterpret_cast<const void *>(func), bytes);
}
// Lets a kernel launch with clusters of more than 8 CTAs (once per device).
kronq_status set_nonportable_cluster(const void *func);
template <class F>
inline kronq_status nonportable_cluster_attr(F *func) {
  return set_nonportable_cluster(reinterpret_cast<const void *>(func));
}

// 2D tiled tensor map over a row-major fp32/bf16 matrix: inner extent `inner`
// (contiguous), outer extent `outer`, row pitch `pitch_elems`, box
// {box_inner, box_outer}, zero fill out of bounds. Swizzle: TMAP_SW128
// (128-byte rows, 16-byte granules), TMAP_SW128_32B (128-byte rows, 32-byte
// granules), TMAP_SW64 (64-byte rows, 16-byte granules) or TMAP_NONE (the
// box lands row-major and unswizzled).
enum { TMAP_SW128 = 0, TMAP_SW128_32B = 1, TMAP_SW64 = 2, TMAP_NONE = 3 };
kronq_status make_tmap_2d(CUtensorMap *map, const void *base, bool bf16,
                          uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                          uint32_t box_inner, uint32_t box_outer,
                          int swz = TMAP_SW128);

inline cudaStream_t as_stream(kronq_stream_t s) {
  return reinterpret_cast<cudaStream_t>(s);
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Bounded device waits give up after this many nanoseconds of wall time and
// report KRONQ_ERR_TIMEOUT instead of spinning forever.
constexpr uint64_t kWaitLimitNs = 4000000000ull;
// Upper bound of the wait limit kronq_selftest_timeout accepts.
constexpr uint64_t kSelftestMaxNs = 1000000000ull;

// ----------------------------------------------------------------- device side
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// First error wins; later ones are dropped.
__device__ __forceinline__ void report(int32_t *info, int32_t code) {
  if (info) atomicCAS(info, 0, code);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same test, but the thread may sleep in hardware until the phase completes
// or about `ns` nanoseconds pass (no polling traffic on shared memory).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity,
                                                    uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete. Returns
// false (and leaves the barrier untouched) once *abort is set by another
// thread or the wall-time limit `limit_ns` passes; the caller then winds
// down. Between checks the thread sleeps on the barrier for up to 0.5 ms (1 us
// under limits below 1 ms).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint32_t nap = limit_ns < 1000000ull ? 1000u : 500000u;
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, nap)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA: 2D tiled load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map,
                                            uint64_t *bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Untiled bulk copy of `bytes` (multiple of 16; both addresses 16-byte
// aligned) global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src,
                                          uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk prefetch of `bytes` (multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map))
               : "memory");
}

// ---- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          smem_u32(dst_smem)),
      "r"(ncols)
      : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                   taddr),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D(tmem) (+)= A(smem) * B(smem)^T, one elected thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a_desc,
                                          uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once all previously issued tcgen05.mma of this thread finish.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns of TMEM -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
        "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for tcgen05 (version field 1; offsets in
// bytes). Layout type 2 = 128-byte swizzle with 16-byte granules (K-major
// operands, and MN-major 16-bit operands); layout type 4 = the same with
// 64-byte rows; layout type 1 = 128-byte swizzle with 32-byte granules, the
// only MN-major layout for 32-bit (tf32) operands (K groups of 4 rows
// instead of 8).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo,
                                          uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo,
                                                uint32_t sbo) {
  return sdesc(saddr, lbo, sbo, 2);
}

// Instruction descriptor: fp32 accumulate, operand formats (1 = bf16,
// 2 = tf32), majors (0 = K-major, 1 = MN-major), tile M x N.
__host__ __device__ constexpr uint32_t idesc_make(uint32_t fmt, uint32_t a_mn,
                                                  uint32_t b_mn, uint32_t M,
                                                  uint32_t N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn << 15) | (b_mn << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// The tf32 MMA reads an fp32 operand by dropping its 13 low mantissa bits
// (truncation, measured on sm_100a), so the raw slab already is the hi part;
// only lo = x - trunc(x) (exact in fp32, |lo| < 2^-10 |x|) has to be written.
// lo is stored rounded to the nearest tf32 value, so the MMA's own truncation
// of it costs nothing; per product the split then keeps a*b up to
// |a_lo b_lo| + 2^-22 (|a| |b_lo| + |a_lo| |b|) <= 1.5 * 2^-20 |a b|.
__device__ __forceinline__ float tf32_lo1(float x) {
  const float lo = x - __uint_as_float(__float_as_uint(x) & 0xffffe000u);
  // nearest tf32 value, ties away from zero (sign-magnitude bit pattern)
  return __uint_as_float((__float_as_uint(lo) + 0x1000u) & 0xffffe000u);
}
__device__ __forceinline__ float4 tf32_lo(float4 x) {
  return make_float4(tf32_lo1(x.x), tf32_lo1(x.y), tf32_lo1(x.z), tf32_lo1(x.w));
}

// ---- thread-block clusters (distributed shared memory)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives (release) and waits
// (acquire): shared-memory writes before it are visible cluster-wide after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address, in the shared::cluster window, of the same shared-memory offset in
// the cluster's CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace kronq
