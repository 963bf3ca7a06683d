// ptx.cuh -- inline-PTX wrappers for sm_100a: mbarrier, TMA, tcgen05 / TMEM.
//
// Written for this library from the public PTX ISA.  Every device-side wait
// is bounded in time: past its limit it records DEV_TIMEOUT in a global flag
// and returns false, so a kernel can unwind instead of hanging.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace moezc {

// Device-side error codes written to the workspace flag.
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- dependent launch
// Kernels are launched with programmatic stream serialisation: a kernel may
// start while its predecessor in the stream is finishing.  Everything before
// griddep_wait() must not touch global memory a predecessor writes or reads;
// after it, all predecessors' writes are visible.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Let the next kernel in the stream start launching.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// The time bound of the device waits counts this SM's own clock (clock64),
// not the global nanosecond timer: reads of that timer were measured to take
// microseconds when the SMs of a grid read it together, as waiting CTAs do.
// A limit of L ns is taken as 2 L cycles, so that at SM clocks up to 2 GHz
// (B200 runs at most 1965 MHz) a wait lasts at least L ns.
constexpr long long kWaitCyclesPerNs = 2;
__device__ __forceinline__ long long wait_cycles(long long limit_ns) {
  return limit_ns > (1LL << 61) ? (1LL << 62) : limit_ns * kWaitCyclesPerNs;
}

// Wait until the phase of `bar` with the given parity has completed, for at
// most `limit_ns` nanoseconds (as above).  On running out, record DEV_TIMEOUT
// in *err (unless an error is already there) and return false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit_ns,
                                          int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  const long long lim = wait_cycles(limit_ns);
  while (true) {
    for (int i = 0; i < 16; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
    }
    if (clock64() - t0 > lim) {
      atomicCAS(err, DEV_OK, DEV_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA
// Prefetch the box at (x, y) of a 2-D tensor map into L2 (no shared memory,
// no barrier: a hint that completes on its own).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared (this CTA), completing on `bar`.
// c0 is the innermost (contiguous) coordinate in elements, c1 the row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(c0), "r"(c1)
      : "memory");
}

// L2 cache policies (createpolicy): evict-last for data that later CTAs
// re-read, evict-first for data read or written once.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// tma_load_2d with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t c0, int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

// 16-byte global store with an L2 cache policy, not allocated in L1.
__device__ __forceinline__ void st_global_v4_hint(void* ptr, const uint4& v, uint64_t policy) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;"
               ::"l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy)
               : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Allocate `ncols` TMEM columns (power of two >= 32); the address is written
// to shared memory at `dst`.  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
      ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 16 columns of 32-bit TMEM -> 16 registers per thread
// (thread i of the warp reads lane (warp%4)*32 + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major bf16 tile written by TMA with
// 128-byte swizzle: rows of 64 elements (128 B), 8-row groups 1024 B apart.
// The tile base must be 1024-byte aligned; advancing along K inside the
// 128-byte row is done by adding the byte offset to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);        // start address
  desc |= static_cast<uint64_t>(1) << 16;                        // leading byte offset (unused)
  desc |= static_cast<uint64_t>(1024 >> 4) << 32;                // stride byte offset
  desc |= static_cast<uint64_t>(1) << 46;                        // descriptor version (sm100)
  desc |= static_cast<uint64_t>(2) << 61;                        // 128-byte swizzle
  return desc;
}

// Instruction descriptor: kind::f16, A and B bf16 K-major, D fp32, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A format: bf16
         | (1u << 10)         // B format: bf16
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------- block-scaled FP8
// D[tmem] (+)= (A * sa) * (B * sb)^T, kind::mxf8f6f4 with block scaling: A and
// B E4M3, K-major, K = 32 per instruction; one UE8M0 scale per row of A and
// per column of B for the 32 elements, read from TMEM at sfa / sfb (the byte
// within each 32-bit TMEM word is chosen by the instruction descriptor).
__device__ __forceinline__ void umma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor of umma_mxf8: E4M3 x E4M3 -> fp32, UE8M0 scales,
// M x N, scale bytes sfa_id / sfb_id of the TMEM words (the 32-element block
// of the 4 that one 32-bit word holds).
__host__ __device__ constexpr uint32_t idesc_mxf8(uint32_t M, uint32_t N, uint32_t sfa_id,
                                                 uint32_t sfb_id) {
  return (sfb_id << 4)        // B scale-factor byte
         | (0u << 7)          // A format: E4M3
         | (0u << 10)         // B format: E4M3
         | ((N >> 3) << 17)   // N / 8
         | (1u << 23)         // scale format: UE8M0
         | ((M >> 4) << 24)   // M / 16
         | (sfa_id << 29);    // A scale-factor byte
}

// Copy 32 rows x 16 bytes of shared memory (a 512-byte scale atom) into 4
// TMEM columns of all four lane quadrants (lane i % 32 of each quadrant gets
// row i).  Asynchronous, ordered with this thread's later tcgen05.mma.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Shared-memory descriptor of a 512-byte scale atom for tmem_cp_atom: 32
// rows of 16 bytes, no swizzle (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_atom(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);   // start address
  desc |= static_cast<uint64_t>(128 >> 4) << 32;           // stride byte offset (8-row groups)
  desc |= static_cast<uint64_t>(1) << 46;                  // descriptor version (sm100)
  return desc;                                             // layout: no swizzle
}

// Untiled bulk copy global -> shared (this CTA), completing on `bar`: both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address, in the cluster's shared window, of the same shared-memory offset
// in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// All threads of the cluster (each warp converged).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// A 32-bit store into a cluster-window shared-memory address (may be a
// peer CTA's), and a poll of this CTA's word that such stores update: wait
// until it is at least `target` for at most limit_ns, then go on either way
// (for pacing only -- nothing may depend on the wait having succeeded).
__device__ __forceinline__ void st_cluster_u32(uint32_t cl_addr, uint32_t v) {
  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(cl_addr), "r"(v)
               : "memory");
}
__device__ __forceinline__ uint32_t ld_cluster_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.relaxed.cluster.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p))
               : "memory");
  return v;
}
__device__ __forceinline__ void pace_until_shared(const void* p, uint32_t target,
                                                  long long limit_ns) {
  if (ld_cluster_u32(p) >= target) return;
  const long long t0 = clock64();
  const long long lim = wait_cycles(limit_ns);
  while (ld_cluster_u32(p) < target) {
    if (clock64() - t0 > lim) return;
  }
}

// Counters in global memory that CTAs of one grid publish progress through:
// the writer stores its data, fences and adds; the reader waits (bounded) for
// the count with acquire loads and then orders its later bulk-tensor (async
// proxy) reads after what it has seen.
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Wait until *p >= target for at most limit_ns; on running out record
// DEV_TIMEOUT in *err and return false.
__device__ __forceinline__ bool wait_count_geq(const int* p, int target, long long limit_ns,
                                               int* err) {
  if (ld_acquire_gpu(p) >= target) return true;
  const long long t0 = clock64();
  const long long lim = wait_cycles(limit_ns);
  while (true) {
    __nanosleep(128);
    if (ld_acquire_gpu(p) >= target) return true;
    if (clock64() - t0 > lim) {
      atomicCAS(err, DEV_OK, DEV_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

}  // namespace moezc
