// step.cuh -- per-element steps of the layer shared by the standalone
// kernels and the phases of the persistent decode step (run by the one-grid
// expert GEMMs, gemm_tcgen05.cu), so that both compute the same bits: the
// routing of one token, the summation of the router's K slices, the combine
// of one 8-feature chunk, the block-scaled FP8 quantisation of 32 elements;
// and the phases themselves with their bounded grid barrier.
#pragma once

#include <cfloat>
#include <climits>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moezc {

// ------------------------------------------------------------------ route
// (LongCat-Flash write-up, section "Zero-computation experts": softmax router
// over the N FFN and Z zero-computation experts, the expert bias shifting
// only the selection, K picks per token.)
// fp32 -> uint32 with the same order (larger float -> larger key); the key 0
// is below every float's key and marks a taken or absent expert.
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// A lane's candidate list: its three best slots in the order (key desc,
// slot asc), with their probabilities.
struct Top3 {
  uint32_t k0, k1, k2;
  int i0, i1, i2;
  float p0, p1, p2;
};

// The three best of this lane's slots that come after (lk, li) in the order
// (key desc, slot asc); lk = UINT32_MAX, li = -1 takes all slots.  Slots are
// scanned in ascending order and displace only on a strictly larger key, so
// equal keys keep the lower slot (the lower expert index) first.
template <int VPL>
__device__ __forceinline__ Top3 lane_top3(const uint32_t (&key)[VPL], const float (&p)[VPL],
                                          uint32_t lk, int li) {
  Top3 c{0u, 0u, 0u, 0, 0, 0, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const uint32_t k = key[i];
    const bool after = k < lk || (k == lk && i > li);
    if (!after) continue;
    if (k > c.k0) {
      c.k2 = c.k1; c.i2 = c.i1; c.p2 = c.p1;
      c.k1 = c.k0; c.i1 = c.i0; c.p1 = c.p0;
      c.k0 = k; c.i0 = i; c.p0 = p[i];
    } else if (k > c.k1) {
      c.k2 = c.k1; c.i2 = c.i1; c.p2 = c.p1;
      c.k1 = k; c.i1 = i; c.p1 = p[i];
    } else if (k > c.k2) {
      c.k2 = k; c.i2 = i; c.p2 = p[i];
    }
  }
  return c;
}

// Softmax, biased top-K, gates and zsum of one token from its logits l
// (lane + 32 i), by one warp; picks are counted in hist (shared memory).
//
// Top-K: each lane keeps its three best slots; a round is two warp
// reductions (max key, then the lowest expert index among the lanes holding
// it) and the winning lane pops its list.  A lane whose list runs dry
// rescans its slots for the three best after the last one it gave.
template <int VPL>
__device__ __forceinline__ void route_token(float (&l)[VPL], const float* __restrict__ bias,
                                            const float* __restrict__ offset, int E, int N, int K,
                                            int lane, int64_t t, int* __restrict__ idx,
                                            float* __restrict__ gate, float* __restrict__ zsum,
                                            int* hist) {
  float mx = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    if (j < E) {
      if (offset) l[i] += offset[j];
      mx = fmaxf(mx, l[i]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float p[VPL];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    p[i] = (j < E) ? expf(l[i] - mx) : 0.f;
    sum += p[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    p[i] = p[i] / sum;
    // A NaN score (only from non-finite logits) ranks below every real
    // score but above a taken or absent expert, so each round still picks
    // a valid index.
    const float sc = p[i] + (j < E ? bias[j] : 0.f);
    key[i] = (j < E) ? order_key(sc == sc ? sc : -FLT_MAX) : 0u;
  }

  Top3 c = lane_top3<VPL>(key, p, 0xffffffffu, -1);
  float zs = 0.f;
  for (int k = 0; k < K; ++k) {
    // the largest score; among equal scores the lowest expert index
    const uint32_t mk = __reduce_max_sync(0xffffffffu, c.k0);
    const uint32_t cand = (c.k0 == mk) ? static_cast<uint32_t>(lane + 32 * c.i0) : 0xffffffffu;
    const int jw = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
    const float pw = __shfl_sync(0xffffffffu, c.p0, jw & 31);
    if (jw >= N) zs += pw;
    if (lane == 0) {
      idx[t * K + k] = jw;
      gate[t * K + k] = pw;
      atomicAdd(&hist[jw], 1);
    }
    if (lane == (jw & 31)) {
      const uint32_t lk = c.k0;
      const int li = c.i0;
      c.k0 = c.k1; c.i0 = c.i1; c.p0 = c.p1;
      c.k1 = c.k2; c.i1 = c.i2; c.p1 = c.p2;
      c.k2 = 0u;
      if (c.k0 == 0u) c = lane_top3<VPL>(key, p, lk, li);
    }
  }
  if (lane == 0) zsum[t] = zs;
}

// One logit summed over the router GEMM's K slices (at p, p + stride, ...),
// in slice order.  The loads of SLICE_GROUP slices are issued together before
// their adds, so a logit waits for ceil(splits / SLICE_GROUP) round trips to
// L2 rather than one per slice.
__device__ __forceinline__ float slice_sum(const float* __restrict__ p, int64_t stride,
                                           int splits) {
  constexpr int SLICE_GROUP = 8;
  float acc = p[0];
  for (int sp = 1; sp < splits; sp += SLICE_GROUP) {
    float a[SLICE_GROUP];
#pragma unroll
    for (int u = 0; u < SLICE_GROUP; ++u)
      a[u] = sp + u < splits ? p[static_cast<int64_t>(sp + u) * stride] : 0.f;
#pragma unroll
    for (int u = 0; u < SLICE_GROUP; ++u)
      if (sp + u < splits) acc += a[u];
  }
  return acc;
}

// Two logits at once (p0 and p1, each loaded only where its flag is set),
// each summed over the slices in slice order as slice_sum does, with every
// slice load of both in flight together (splits <= 32: one round trip).
__device__ __forceinline__ void slice_sum2(const float* __restrict__ p0, bool has0,
                                           const float* __restrict__ p1, bool has1,
                                           int64_t stride, int splits, float& s0, float& s1) {
  constexpr int GROUP = 32;
  float acc0 = has0 ? p0[0] : 0.f, acc1 = has1 ? p1[0] : 0.f;
  for (int sp = 1; sp < splits; sp += GROUP) {
    float a0[GROUP], a1[GROUP];
#pragma unroll
    for (int u = 0; u < GROUP; ++u) {
      const bool in = sp + u < splits;
      const int64_t o = static_cast<int64_t>(sp + u) * stride;
      a0[u] = in && has0 ? p0[o] : 0.f;
      a1[u] = in && has1 ? p1[o] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < GROUP; ++u) {
      if (sp + u < splits) {
        acc0 += a0[u];
        acc1 += a1[u];
      }
    }
  }
  s0 = acc0;
  s1 = acc1;
}

// ------------------------------------------------------------------ dispatch
// Exclusive prefix sum of v over a CTA of NT threads, with the CTA's total in
// *total (warp_sums: NT / 32 ints of shared memory).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  constexpr int W = NT / 32;
  static_assert(W <= 32 && NT % 32 == 0, "block_excl_scan: 32 to 1024 threads");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < W ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < W; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < W) warp_sums[lane] = w;   // inclusive prefix over warps
  }
  __syncthreads();
  const int base = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[W - 1];
  __syncthreads();
  return base + incl - v;
}

// ------------------------------------------------------------------ combine
// a[i] += g * (8 bf16 features in v), fp32 fused multiply-add.
__device__ __forceinline__ void acc8(float (&a)[8], const uint4& v, float g) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), a[2 * i]);
    a[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xFFFF0000u), a[2 * i + 1]);
  }
}

// One 8-feature chunk c of out_t = bf16(zsum_t x_t + sum_k gate_k Y[slot_k]):
// fp32 accumulation in a fixed order (the zero-expert term first, then the
// token's FFN picks in k order: sl / gt hold the n picks with slot >= 0), one
// rounding to bf16.
__device__ __forceinline__ uint4 combine_chunk(const uint4* __restrict__ x,
                                               const uint4* __restrict__ Y, int64_t t, int c,
                                               int d8, float z, const int* sl, const float* gt,
                                               int n) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = 0.f;
  acc8(a, x[t * d8 + c], z);
  for (int k = 0; k < n; ++k) acc8(a, Y[static_cast<int64_t>(sl[k]) * d8 + c], gt[k]);
  uint4 o;
  uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
    ow[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return o;
}

// ------------------------------------------------------------------ FP8 (E4M3, 1 x 32 blocks)
// UE8M0 byte of the smallest power of two 2^k with amax <= 448 * 2^k (amax > 0,
// finite).  With amax = (1 + m / 2^23) 2^(E - 127) and 448 = 1.75 * 2^8:
// k = E - 135, plus one when the significand exceeds 1.75 (m > 0x600000).
// Subnormal amax (and anything needing k < -127) takes the floor 2^-127.
__device__ __forceinline__ uint32_t ue8m0_of_amax(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int E = static_cast<int>((bits >> 23) & 0xFF);
  if (amax == 0.f || E == 0xFF) return 127u;   // zero, or a NaN / infinity in the block
  if (E == 0) return 0u;
  int k = E - 135 + ((bits & 0x7FFFFF) > 0x600000u ? 1 : 0);
  k = k < -127 ? -127 : (k > 127 ? 127 : k);
  return static_cast<uint32_t>(k + 127);
}

// 2^-k as a float, exactly (k in [-127, 127]).
__device__ __forceinline__ float inv_pow2(int k) {
  return k <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - k) << 23)
                  : __uint_as_float(0x00400000u);   // 2^-127 (subnormal)
}

// Byte offset, in the token tiles' scale atoms, of the scales of the token
// at place pos of token tile `tile` (d / 128 contraction groups of two
// 512-byte atoms each; block b of the row adds (b / 4) * 2 * SF_ATOM_BYTES +
// b % 4).
__device__ __forceinline__ int64_t token_sf_base(int64_t tile, int pos, int d) {
  return tile * (d / 128) * (2 * SF_ATOM_BYTES) + (pos / 128) * SF_ATOM_BYTES + (pos % 32) * 16 +
         ((pos % 128) / 32) * 4;
}

// 32 bf16 values (8 per uint4) -> their E4M3 codes (4 per uint32) and the
// block's UE8M0 scale byte.  value / 2^k is exact in fp32, and the
// conversion rounds to nearest, ties to even (it never saturates:
// |value| / 2^k <= 448).
__device__ __forceinline__ uint32_t quantize32(const uint4 (&v)[4], uint32_t (&codes)[8]) {
  float f[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[q * 8 + 2 * i] = bf16_lo(w[i]);
      f[q * 8 + 2 * i + 1] = bf16_hi(w[i]);
    }
  }
  float amax = 0.f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float a = fabsf(f[i]);
    finite = finite && (__float_as_uint(a) < 0x7F800000u);
    amax = fmaxf(amax, a);
  }
  const uint32_t sf = finite ? ue8m0_of_amax(amax) : 127u;
  const float inv = inv_pow2(static_cast<int>(sf) - 127);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_fp8_storage_t c =
          __nv_cvt_float_to_fp8(f[4 * i + j] * inv, __NV_SATFINITE, __NV_E4M3);
      word |= static_cast<uint32_t>(c) << (8 * j);
    }
    codes[i] = word;
  }
  return sf;
}

// ------------------------------------------------------------------ grid barrier
// All CTAs of a grid that is resident as a whole (a cooperative launch): each
// CTA adds one to *ctr once its threads are here and waits, for at most
// limit_ns, until *ctr reaches `target` (gridDim.x times the number of
// barriers passed so far; the counter is zero at launch).  Writes before the
// barrier (also, with PROXY, those that bulk-tensor copies read afterwards:
// the proxy fences) are visible after it.
//
// A CTA whose wait runs out records DEV_TIMEOUT in *err, and -- as does a CTA
// that arrives with arrive_ok false (its own work failed) -- adds
// STEP_POISON to the counter.  A CTA that sees the poison returns false as
// well: it came from a CTA that skipped work which the phase after this
// barrier may read.  Returns true when the work after the barrier may run.
constexpr int STEP_POISON = 1 << 16;

template <bool PROXY = true>
__device__ __forceinline__ bool grid_barrier(int* ctr, int target, long long limit_ns, int* err,
                                             volatile int* ok_sh, bool arrive_ok) {
  if (PROXY) fence_proxy_async_global();
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, arrive_ok ? 1 : 1 + STEP_POISON);
    bool ok = wait_count_geq(ctr, target, limit_ns, err);
    if (ok) {
      ok = ld_acquire_gpu(ctr) < STEP_POISON;
    } else {
      __threadfence();
      atomicAdd(ctr, STEP_POISON);
    }
    *ok_sh = (ok && arrive_ok) ? 1 : 0;
    if (PROXY) fence_proxy_async_global();
  }
  __syncthreads();
  return *ok_sh != 0;
}

// ------------------------------------------------------------------ persistent decode step
// The phases the one-grid expert GEMMs run around their tiles when
// StepParams::on (kernels.cuh).  Every block calls each phase with all its
// threads and takes its work by blockIdx.x.  What other blocks of the grid
// wrote before a grid barrier is read after it with plain loads (the
// barrier's acquire makes those writes visible; no block reads such words
// before the barrier that publishes them, so no stale line sits in L1).  ws
// is the GEMM's epilogue staging area (shared memory that no bulk copy
// touches).

// route: tokens blockIdx.x, + gridDim.x, ...; the whole block routes one
// token, with the bits of route_token (one warp per token):
//   * each thread sums the router's K slices of its one or two logits (j =
//     tid, tid + NT) in slice order, all slice loads in flight at once;
//   * the maximum over the block (exact in any order);
//   * e_j = expf(l_j - max), summed in route_token's order: lane L of warp 0
//     adds e_L, e_{L+32}, ... in turn, then the same xor-shuffle tree;
//   * p_j = e_j / sum and the selection key of p_j + b_j, as route_token;
//   * the K picks in the order (key desc, index asc) that route_token's
//     rounds also follow: each warp lists the best K of its own values, and
//     warp 0 merges the sorted lists, adding zero-expert gates into zsum in
//     pick order and counting picks straight into the global histogram.
// (Shared memory: 2 * MOE_MAX_E_INTERNAL floats, the warps' lists, scratch.)
template <int NT>
__device__ __forceinline__ void step_route(const StepParams& sp, uint8_t* ws) {
  constexpr int W = NT / 32;
  constexpr int MK = MOE_MAX_K_INTERNAL;
  static_assert(2 * NT >= MOE_MAX_E_INTERNAL, "step_route: two logits per thread");
  float* e_s = reinterpret_cast<float*>(ws);                               // [E]
  float* p_s = e_s + MOE_MAX_E_INTERNAL;                                   // [E]
  uint32_t* ck = reinterpret_cast<uint32_t*>(p_s + MOE_MAX_E_INTERNAL);    // [W][MK] keys
  int* cj = reinterpret_cast<int*>(ck + W * MK);                           // [W][MK] indices
  float* red = reinterpret_cast<float*>(cj + W * MK);                      // [W + 1]
  const int E = sp.E, K = sp.K, N = sp.N;
  const int64_t stride = static_cast<int64_t>(sp.T) * E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j0 = threadIdx.x, j1 = threadIdx.x + NT;
  const bool v0 = j0 < E, v1 = j1 < E;
  const float b0 = v0 ? sp.bias[j0] : 0.f, b1 = v1 ? sp.bias[j1] : 0.f;
  const float o0 = v0 && sp.offset ? sp.offset[j0] : 0.f;
  const float o1 = v1 && sp.offset ? sp.offset[j1] : 0.f;
  for (int t = blockIdx.x; t < sp.T; t += gridDim.x) {
    const float* base = sp.logits + static_cast<int64_t>(t) * E;
    float l0 = 0.f, l1 = 0.f;
    slice_sum2(base + j0, v0, base + j1, v1, stride, sp.splits, l0, l1);
    if (sp.offset) {
      l0 += o0;
      l1 += o1;
    }
    float mx = -FLT_MAX;
    if (v0) mx = fmaxf(mx, l0);
    if (v1) mx = fmaxf(mx, l1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < W; ++w) mx = fmaxf(mx, red[w]);
    const float e0 = v0 ? expf(l0 - mx) : 0.f;
    const float e1 = v1 ? expf(l1 - mx) : 0.f;
    if (v0) e_s[j0] = e0;
    if (v1) e_s[j1] = e1;
    __syncthreads();
    if (warp == 0) {
      float sum = 0.f;
      for (int j = lane; j < E; j += 32) sum += e_s[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) red[W] = sum;
    }
    __syncthreads();
    const float sum = red[W];
    uint32_t k0 = 0u, k1 = 0u;
    if (v0) {
      const float p = e0 / sum;
      const float sc = p + b0;
      k0 = order_key(sc == sc ? sc : -FLT_MAX);
      p_s[j0] = p;
    }
    if (v1) {
      const float p = e1 / sum;
      const float sc = p + b1;
      k1 = order_key(sc == sc ? sc : -FLT_MAX);
      p_s[j1] = p;
    }
    // this warp's best K: a round takes the largest key, among equal keys
    // the lowest index (a lane's own two: j0 < j1)
    for (int k = 0; k < K; ++k) {
      const bool second = k1 > k0;
      const uint32_t bk = second ? k1 : k0;
      const int bj = second ? j1 : j0;
      const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
      const int jw = static_cast<int>(
          __reduce_min_sync(0xffffffffu, bk == mk ? static_cast<uint32_t>(bj) : 0xffffffffu));
      if (lane == 0) {
        ck[warp * MK + k] = mk;
        cj[warp * MK + k] = jw;
      }
      if (bj == jw) {
        if (second) k1 = 0u; else k0 = 0u;
      }
    }
    __syncthreads();
    if (warp == 0) {
      // merge: lane w follows warp w's list; lane k keeps pick k, and the
      // picks are stored, and counted, by all lanes at once afterwards
      int pos = 0;
      uint32_t hk = lane < W ? ck[lane * MK] : 0u;
      int hj = lane < W ? cj[lane * MK] : INT_MAX;
      float zs = 0.f;
      int my_j = -1;
      float my_p = 0.f;
      for (int k = 0; k < K; ++k) {
        const uint32_t mk = __reduce_max_sync(0xffffffffu, hk);
        const int jw = static_cast<int>(
            __reduce_min_sync(0xffffffffu, hk == mk ? static_cast<uint32_t>(hj) : 0xffffffffu));
        const float pw = p_s[jw];
        if (jw >= N) zs += pw;
        if (lane == k) {
          my_j = jw;
          my_p = pw;
        }
        if (hj == jw) {
          ++pos;
          hk = pos < K ? ck[lane * MK + pos] : 0u;
          hj = pos < K ? cj[lane * MK + pos] : INT_MAX;
        }
      }
      if (lane < K) {
        sp.idx[static_cast<int64_t>(t) * K + lane] = my_j;
        sp.gate[static_cast<int64_t>(t) * K + lane] = my_p;
        atomicAdd(sp.cnt + my_j, 1);
      }
      if (lane == 0) sp.zsum[t] = zs;
    }
    __syncthreads();
  }
}

// The first gate/up tile whose weights a block prefetches into L2 while the
// tokens are dispatched: tile blockIdx.x, which some block takes in the
// grid's first round (tiles come from the counter in order), its first
// `stages` contraction steps of both A blocks (maps a0 / a1, rows of
// `a_rows` per expert, `kelems` contraction elements per step).
struct TilePrefetch {
  const CUtensorMap* a0;
  const CUtensorMap* a1;
  int mblocks, a_rows, kelems, stages;
};

// assign + permute.  Every block derives from the histogram each FFN
// expert's first row (count rounded up to 16) and first token tiles (of
// GEMM_BN tokens, and of FP8_BN for FP8 gate/up), as the assign kernel does
// (block 0 also stores them for the tiles), and prefetches the weights of
// its first-round tile (pf).  Then for each token of the block: a slot for
// each FFN pick (an atomicAdd on the expert's fill counter; slot -1 for
// zero-expert picks) and the token's row copied into its slots -- bf16, or
// quantised once into FP8 codes and scale atoms.  (Which slot of its expert
// a token gets does not change any result: a token's GEMM columns are
// independent of the others'.)
template <int NT, bool FP8>
__device__ __forceinline__ void step_assign_permute(const StepParams& sp, uint8_t* ws,
                                                    const TilePrefetch& pf) {
  const int N = sp.N, K = sp.K, d = sp.d;
  int* off_s = reinterpret_cast<int*>(ws);   // [N] first row
  int* cnt_s = off_s + N;                    // [N]
  int* gtp_s = cnt_s + N;                    // [N] first gate/up token tile (FP8: of FP8_BN)
  int* scan_s = gtp_s + N;                   // [32]
  int* sl_s = scan_s + 32;                   // [32] slots of the token's FFN picks, k order
  int* tile_s = sl_s + 32;                   // [32] FP8: the slot's token tile
  int* pos_s = tile_s + 32;                  // [32] FP8: its place in the tile
  int* n_s = pos_s + 32;
  // The block's first token: its picks (warp 0, lane k) and its row (bf16:
  // chunks tid, tid + NT; FP8: block of 32 tid) are loaded before the scans,
  // so that their latency overlaps them; later tokens load in turn.
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x;
  const bool first = t0 < sp.T;
  const int g0 = first && threadIdx.x < 32 && lane < K
                     ? sp.idx[static_cast<int64_t>(t0) * K + lane] : -1;
  constexpr int XR = 2;
  uint4 xr[FP8 ? 4 : XR];
  {
    const uint4* src0 = reinterpret_cast<const uint4*>(sp.x) + static_cast<int64_t>(t0) * (d / 8);
#pragma unroll
    for (int i = 0; i < (FP8 ? 4 : XR); ++i) {
      const int c = FP8 ? static_cast<int>(threadIdx.x) * 4 + i : static_cast<int>(threadIdx.x) + i * NT;
      const bool in = first && (FP8 ? static_cast<int>(threadIdx.x) < d / 32 : c < d / 8);
      xr[i] = in ? src0[c] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  int carry_r = 0, carry_t = 0, carry_t8 = 0;
  for (int base = 0; base < N; base += NT) {
    const int g = base + static_cast<int>(threadIdx.x);
    const int c = g < N ? sp.cnt[g] : 0;
    int tot_r, tot_t, tot_t8 = 0;
    const int off = block_excl_scan<NT>((c + 15) / 16 * 16, scan_s, &tot_r);
    const int ttp = block_excl_scan<NT>((c + GEMM_BN - 1) / GEMM_BN, scan_s, &tot_t);
    const int ttp8 = FP8 ? block_excl_scan<NT>((c + FP8_BN - 1) / FP8_BN, scan_s, &tot_t8) : 0;
    if (g < N) {
      off_s[g] = carry_r + off;
      cnt_s[g] = c;
      gtp_s[g] = FP8 ? carry_t8 + ttp8 : carry_t + ttp;
      if (blockIdx.x == 0) {
        sp.grp_off[g] = carry_r + off;
        sp.grp_ttp[g] = carry_t + ttp;
        if (FP8) sp.grp_ttp8[g] = carry_t8 + ttp8;
      }
    }
    carry_r += tot_r;
    carry_t += tot_t;
    carry_t8 += tot_t8;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    sp.grp_off[N] = carry_r;
    sp.grp_ttp[N] = carry_t;
    if (FP8) sp.grp_ttp8[N] = carry_t8;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // gate/up tile u = blockIdx.x, decoded as the tiles decode it: expert
    // g (the last whose first tile is at or below u's token tile), then the
    // weight block
    const int gtotal = FP8 ? carry_t8 : carry_t;
    const int u = blockIdx.x;
    if (u < gtotal * pf.mblocks) {
      const int tt = u / pf.mblocks;
      int lo = 0, hi = N - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gtp_s[mid] <= tt) lo = mid; else hi = mid - 1;
      }
      const int ttp0 = gtp_s[lo];
      const int ntt = (lo + 1 < N ? gtp_s[lo + 1] : gtotal) - ttp0;
      const int v = u - ttp0 * pf.mblocks;
      const int m = ntt == 2 ? v >> 1 : v % pf.mblocks;
      const int row = lo * pf.a_rows + m * GEMM_BM;
      for (int k = 0; k < pf.stages; ++k) {
        tma_prefetch_l2_2d(pf.a0, k * pf.kelems, row);
        tma_prefetch_l2_2d(pf.a1, k * pf.kelems, row);
      }
    }
  }
  for (int t = blockIdx.x; t < sp.T; t += gridDim.x) {
    const bool pre = first && t == t0;
    if (threadIdx.x < 32) {
      const int g = pre ? g0 : (lane < K ? sp.idx[static_cast<int64_t>(t) * K + lane] : -1);
      const bool ffn = g >= 0 && g < N;
      int s = -1;
      if (ffn) s = off_s[g] + atomicAdd(sp.fill + g, 1);
      if (lane < K) sp.slot[static_cast<int64_t>(t) * K + lane] = s;
      const unsigned m = __ballot_sync(0xffffffffu, ffn);
      if (ffn) {
        const int k = __popc(m & ((1u << lane) - 1u));
        sl_s[k] = s;
        if (FP8) {
          const int count = cnt_s[g];
          const int tsz = even_tile_size(count, (count + FP8_BN - 1) / FP8_BN, FP8_BN);
          const int u = s - off_s[g];
          const int j = u / tsz;
          tile_s[k] = gtp_s[g] + j;
          pos_s[k] = u - j * tsz;
        }
      }
      if (lane == 0) *n_s = __popc(m);
    }
    __syncthreads();
    const int n = *n_s;
    if (FP8) {
      const int nb = d / 32;
      const uint4* src = reinterpret_cast<const uint4*>(sp.x) + static_cast<int64_t>(t) * (d / 8);
      uint4* Xp8 = reinterpret_cast<uint4*>(sp.Xp8);
      for (int b = threadIdx.x; b < nb; b += NT) {
        const bool held = pre && b == static_cast<int>(threadIdx.x);
        uint4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = held ? xr[q] : src[b * 4 + q];
        uint32_t c[8];
        const uint32_t sc = quantize32(v, c);
        const uint4 c0 = make_uint4(c[0], c[1], c[2], c[3]);
        const uint4 c1 = make_uint4(c[4], c[5], c[6], c[7]);
        const int64_t sf_off = static_cast<int64_t>(b / 4) * (2 * SF_ATOM_BYTES) + (b % 4);
        for (int k = 0; k < n; ++k) {
          uint4* dst = Xp8 + (static_cast<int64_t>(sl_s[k]) * d + static_cast<int64_t>(b) * 32) / 16;
          dst[0] = c0;
          dst[1] = c1;
          sp.sfx[token_sf_base(tile_s[k], pos_s[k], d) + sf_off] = static_cast<uint8_t>(sc);
        }
      }
    } else {
      const int d8 = d / 8;
      const uint4* src = reinterpret_cast<const uint4*>(sp.x) + static_cast<int64_t>(t) * d8;
      uint4* Xp = reinterpret_cast<uint4*>(sp.Xp);
#pragma unroll
      for (int i = 0; i < XR; ++i) {
        const int c = static_cast<int>(threadIdx.x) + i * NT;
        if (c < d8) {
          const uint4 v = pre ? xr[i] : src[c];
          for (int k = 0; k < n; ++k) Xp[static_cast<int64_t>(sl_s[k]) * d8 + c] = v;
        }
      }
      for (int c = threadIdx.x + XR * NT; c < d8; c += NT) {
        const uint4 v = src[c];
        for (int k = 0; k < n; ++k) Xp[static_cast<int64_t>(sl_s[k]) * d8 + c] = v;
      }
    }
    __syncthreads();
  }
}

// combine: items (token, part of its row) over the grid, the parts chosen as
// the combine kernel chooses them; per item warp 0 gathers the token's FFN
// picks in k order, and every thread combines 8-feature chunks.
template <int NT>
__device__ __forceinline__ void step_combine(const StepParams& sp, uint8_t* ws) {
  int* sl_s = reinterpret_cast<int*>(ws);               // [32]
  float* gt_s = reinterpret_cast<float*>(sl_s + 32);    // [32]
  int* n_s = sl_s + 64;
  float* z_s = reinterpret_cast<float*>(sl_s + 65);
  const int d8 = sp.d / 8, K = sp.K;
  int parts = (static_cast<int>(gridDim.x) + sp.T - 1) / sp.T;
  if (parts > 8) parts = 8;
  while (parts > 1 && d8 / parts < 128) --parts;
  const int items = sp.T * parts;
  const int lane = threadIdx.x & 31;
  const uint4* x = reinterpret_cast<const uint4*>(sp.x);
  const uint4* Y = reinterpret_cast<const uint4*>(sp.Y);
  uint4* out = reinterpret_cast<uint4*>(sp.out);
  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const int t = it / parts, part = it - t * parts;
    if (threadIdx.x < 32) {
      const int64_t row = static_cast<int64_t>(t) * K;
      const int s = lane < K ? sp.slot[row + lane] : -1;
      const float g = lane < K ? sp.gate[row + lane] : 0.f;
      const unsigned m = __ballot_sync(0xffffffffu, s >= 0);
      if (s >= 0) {
        const int k = __popc(m & ((1u << lane) - 1u));
        sl_s[k] = s;
        gt_s[k] = g;
      }
      if (lane == 0) {
        *n_s = __popc(m);
        *z_s = sp.zsum[t];
      }
    }
    __syncthreads();
    const int n = *n_s;
    const float z = *z_s;
    const int c_begin = static_cast<int>(static_cast<int64_t>(d8) * part / parts);
    const int c_end = static_cast<int>(static_cast<int64_t>(d8) * (part + 1) / parts);
    for (int c = c_begin + threadIdx.x; c < c_end; c += NT)
      out[static_cast<int64_t>(t) * d8 + c] = combine_chunk(x, Y, t, c, d8, z, sl_s, gt_s, n);
    __syncthreads();
  }
}

}  // namespace moezc
