// Device helpers shared by the liboda kernels: bf16 unpacking, mbarrier / bulk-copy PTX
// wrappers for sm_100a, bounded waits, status reporting, and the per-device launch cache.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "oda.h"

namespace oda {

constexpr int kHeadDim = 128;
constexpr int kPage = 16;                                // tokens per KV page
constexpr int kRowBytes = kHeadDim * 2;                  // one bf16 row: 256 B
constexpr int kPageBytes = kPage * kRowBytes;            // one (page, KV head) run: 4 KB
constexpr unsigned long long kWaitNs = 1000000000ull;    // bounded waits give up after 1 s

// ---- status ------------------------------------------------------------------------------
__device__ __forceinline__ void report(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// ---- bf16 -> fp32 (a bf16 value is the high half of the fp32 with the same bits) ---------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// ---- softmax arithmetic -------------------------------------------------------------------
// Base-2 exponential, reciprocal and base-2 logarithm by the PTX approximate instructions
// (ex2.approx, rcp.approx, lg2.approx; flush to zero): a few ulp from the exact values, where
// the library calls take several times as many instructions. Softmax weights and rescale
// factors (arguments <= 0, results in [0, 1]), and the merges' 1 / L and log2 L for L >= 1,
// sit on the decode kernels' latency-bound chains.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- shared-memory barriers and 1-D bulk copies (TMA engine, no tensor map, no multicast) -
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async proxy before any bulk copy signals it.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's generic-proxy shared-memory accesses before later bulk copies into
// the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for a barrier phase, giving up after limit_ns. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// Global -> shared bulk copy completing on `bar` (byte count must be a multiple of 16 and
// both addresses 16-byte aligned). Streaming data: hint L2 to evict it first.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// 16-byte asynchronous global -> shared copy (no register staging; L2 only, .cg), and the
// wait for every such copy this thread has issued.
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Arrive on a merge ticket: gpu-scope acquire-release add by one thread, after a CTA
// barrier, publishes the CTA's partial and, for the last arrival, acquires all others.
__device__ __forceinline__ unsigned ticket_arrive(unsigned* t) {
  unsigned prev;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(t) : "memory");
  return prev;
}

// Thread-block cluster: this CTA's rank, a full cluster barrier (release / acquire), and a
// 4-byte store to / load from the shared memory of CTA `rank` at the address of a local
// variable.
__device__ __forceinline__ unsigned cluster_ctarank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// The halves of a cluster barrier (all threads of every CTA of the cluster): arrive with
// release, arrive without ordering (after fence_barrier_init it publishes mbarrier
// initialisation), and wait with acquire.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16-byte and 4-byte stores into the shared memory of a CTA of the cluster (`dst` from
// cluster_addr), each completing its bytes on that CTA's mbarrier `bar` (also from
// cluster_addr): the receiver learns from the barrier phase that every expected byte landed.
__device__ __forceinline__ void st_async4(uint32_t dst, float4 v, uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void st_async1(uint32_t dst, float v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];"
               ::"r"(dst), "f"(v), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void dsmem_st(float* local, unsigned rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
// 16-byte store to the shared memory of CTA `rank` (`local` 16-byte aligned).
__device__ __forceinline__ void dsmem_st4(float* local, unsigned rank, float4 v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(remote), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
// The shared::cluster address of a variable of this CTA's shared memory in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* local, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  return remote;
}
// Bulk copy from this CTA's shared memory to a CTA of the cluster (addresses from
// cluster_addr), completing `bytes` on that CTA's mbarrier (16-byte aligned, multiple of 16).
__device__ __forceinline__ void bulk_to_cluster(uint32_t dst, const void* src, uint32_t bytes,
                                                uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "r"(smem_addr(src)), "r"(bytes), "r"(bar)
      : "memory");
}
// Arrive (release, cluster scope) on an mbarrier of a CTA of the cluster (address from
// cluster_addr). A copy into another CTA's shared memory completes only on that CTA's
// mbarrier -- bulk async-groups do not track it -- so the receiver tells the sender this way
// that the sender's source buffer may be written again.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
               : "memory");
}
// Wait (bounded) for a phase of this CTA's mbarrier that copies from other CTAs of the cluster
// complete: acquire at cluster scope. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
  auto try_wait = [&]() {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
  };
  if (try_wait()) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (try_wait()) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ float dsmem_ld(const float* local, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote));
  return v;
}

// ---- global counters between the CTAs of one launch (persistent kernels) ---------------
// Release-add by one thread after a CTA barrier publishes the CTA's earlier global writes;
// an acquire load that sees the count makes them visible to the loading thread, and a CTA
// barrier after it to the rest of its CTA.
__device__ __forceinline__ void counter_release_add(unsigned* c, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(c), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned counter_acquire_load(const unsigned* c) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
  return v;
}

// Spin (one thread) until *c >= target (counts compared modulo 2^32), *abort becomes non-zero
// or limit_ns pass. Returns 1 when the count was reached, 0 on abort or timeout; the caller
// raises the abort word on a timeout so that every other waiter of the launch stops at once.
__device__ __forceinline__ unsigned counter_relaxed_load(const unsigned* c) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acquire_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
// (polls with relaxed loads; the fence after the count is seen gives the acquire)
__device__ __forceinline__ int counter_wait(const unsigned* c, unsigned target,
                                            const unsigned* abort, unsigned long long limit_ns) {
  if ((int)(counter_relaxed_load(c) - target) >= 0) {
    fence_acquire_gpu();
    return 1;
  }
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if ((int)(counter_relaxed_load(c) - target) >= 0) {
        fence_acquire_gpu();
        return 1;
      }
    if (counter_relaxed_load(abort) != 0u) return 0;
    if (global_ns() - t0 > limit_ns) return 0;
  }
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// ---- programmatic dependent launch -------------------------------------------------------
// Wait until every prerequisite grid has completed and its writes are visible (returns at
// once for a kernel launched without a programmatic dependency).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel in the stream start its own pre-wait prologue.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- host side: CUDA error bookkeeping ---------------------------------------------------
void note_cuda_error(int err);  // remembered for oda_last_cuda_error()

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ODA_OK;
  note_cuda_error(static_cast<int>(e));
  return ODA_ERR_CUDA;
}

// ---- host side: per-device launch facts --------------------------------------------------
struct DeviceInfo {
  int device = -1;
  int sms = 0;
};

// Streaming-multiprocessor count of the current device (cached per device).
int current_device_info(DeviceInfo* info);

}  // namespace oda
