// kda_prims.cuh -- PTX wrappers shared by the library's kernels: mbarriers
// (bounded waits), TMA tensor and bulk copies, cluster signalling, ldmatrix,
// mma.sync and conversions. Included once, by kda_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>

#include "../../include/kda.h"

namespace kda {

constexpr int D = KDA_HEAD_DIM;   // dk = dv = 128

// Wait budget for every mbarrier wait (cycles). A wait that runs out records
// a timeout and lets the thread continue, so no barrier is ever left waiting.
constexpr long long kWaitCycles = 1ll << 28;  // ~0.14 s at 1.9 GHz
// A waiting thread is suspended in hardware (up to this many ns per try)
// instead of spinning, so waiting warps leave the issue slots to the others.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ unsigned int g_wait_timeouts = 0;

// Device status word (bit 0: a cu_seqlens that is not a non-decreasing
// partition of [0, T)); read and cleared through the C ABI.
__device__ unsigned int g_device_flags = 0;
constexpr unsigned int kFlagBadCuSeqlens = 1u;

// Checks sequence `seq`'s boundaries of a packed batch of `nseq` sequences
// over T tokens and records a violation in the status word.
__device__ __forceinline__ void check_bounds(const int32_t* cu, int seq, int nseq, int64_t T) {
  const int64_t a = cu[seq], b = cu[seq + 1];
  const bool bad = a < 0 || b < a || b > T || (seq == 0 && a != 0) || (seq == nseq - 1 && b != T);
  if (bad) atomicOr(&g_device_flags, kFlagBadCuSeqlens);
}

// ---------------------------------------------------------------- primitives
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* m, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(m)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* m) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(m)) : "memory");
}

// One arrive per warp: __syncwarp orders every lane's prior shared-memory
// accesses before lane 0's release-arrive.
__device__ __forceinline__ void mbar_arrive_warp(unsigned long long* m) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(m);
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long* m, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(m)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
// Non-blocking probe: cheaper than a suspending try_wait when the phase has
// long completed, which is the common case for well-fed pipeline stages.
__device__ __forceinline__ bool mbar_test_wait(unsigned long long* m, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(m)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_wait(unsigned long long* m, uint32_t parity) {
  if (mbar_test_wait(m, parity)) return;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(m, parity)) return;
    if ((i & 63u) == 0 && clock64() - t0 > kWaitCycles) {
      atomicAdd(&g_wait_timeouts, 1u);
      return;
    }
  }
}

// 4-byte asynchronous copy (zero fill when src_bytes = 0) and the arrive that
// fires once this thread's copies have landed.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_arrive(unsigned long long* m) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(m)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* m, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(m)), "r"(bytes)
               : "memory");
}

// TMA tiled loads into this CTA's own shared memory. Out-of-range rows of the box are zero-filled.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            unsigned long long* m) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(m))
      : "memory");
}

__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// D += A(16x16 row-major fragment) * B(16x8 column fragment); bf16 in, fp32 acc.
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// (x, y) *= (a, b) as one packed fp32 multiply
__device__ __forceinline__ void mul2(float& x, float& y, float a, float b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"((static_cast<unsigned long long>(__float_as_uint(y)) << 32) | __float_as_uint(x)),
        "l"((static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a)));
  x = __uint_as_float(static_cast<uint32_t>(r));
  y = __uint_as_float(static_cast<uint32_t>(r >> 32));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}


// ---- cluster-scope signalling
__device__ __forceinline__ bool mbar_try_wait_cl(unsigned long long* m, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(m)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_wait_cl(unsigned long long* m, uint32_t parity) {
  if (mbar_try_wait_cl(m, parity)) return;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cl(m, parity)) return;
    if ((i & 63u) == 0 && clock64() - t0 > kWaitCycles) {
      atomicAdd(&g_wait_timeouts, 1u);
      return;
    }
  }
}

// Arrive on the mbarrier at the same shared-memory offset in CTA `rank` of the
// cluster. Relaxed: a "done" signal whose data (if any) was already made
// complete and visible by its sender, so it need not wait for this thread's
// outstanding global stores.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(unsigned long long* m, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(m)), "r"(rank));
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Generic-proxy shared-memory writes become visible to the bulk-copy engine.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bulk copy shared -> global as one bulk async-group.
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Bulk copy shared -> global without committing (the caller commits a group).
__device__ __forceinline__ void bulk_s2g_nc(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk async-groups are still pending
// (their writes to global memory completed).
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Bulk copy global -> shared, completion counted in bytes on the mbarrier.
__device__ __forceinline__ void bulk_g2s(void* sdst, const void* gsrc, uint32_t bytes, unsigned long long* m) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(sdst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(m))
      : "memory");
}

}  // namespace kda
