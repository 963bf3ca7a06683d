// route.cu -- softmax router, expert bias and top-K with the zero-expert
// short-circuit.
//
// LongCat-Flash write-up ("Meituan's large model goes viral for its speed",
// section "Zero-computation experts"): R is a softmax router over the N FFN
// experts plus the Z zero-computation experts; the expert bias b_i adjusts the
// routing scores; each token picks K experts.  Per token t (one warp):
//
//   p_t = softmax(logits_t + offset)      over all E experts, fp32
//   s_t = p_t + b                         selection score
//   picks: K rounds of a warp-wide argmax of s (ties -> lower expert index):
//          scores become order-preserving uint32 keys, each lane keeps a
//          list of its three best slots, a round is two warp reductions (max
//          key, then min index among the lanes holding it), and the winning
//          lane pops its list (rescanning its slots only when it runs dry)
//   gate_{t,k} = p_t at pick k            (unbiased, not renormalised)
//   zsum_t     = sum of the gates of zero-expert picks (index >= N)
//
// Zero-expert picks go no further than zsum_t: the combine adds zsum_t * x_t,
// so identity experts never enter dispatch or the FFN GEMMs.  The expert-load
// histogram counts picks of all E experts, first in shared memory per block,
// then one global atomic per touched expert per block.
#include <cfloat>
#include <climits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moezc {
namespace {

constexpr int ROUTE_WARPS = 8;

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

// One warp per token, up to ROUTE_WARPS tokens (tps) per block and step of
// a grid-stride loop over a single wave of resident blocks; a block
// histogram in shared memory is flushed once per block.  SLICED: the router
// GEMM left `splits` K slices of partial logits, summed for each logit in
// slice order: by each warp for its own token when there are many tokens,
// else (tps < ROUTE_WARPS tokens per block, so that the slices are read by
// many SMs at once) by all threads of the block into shared memory.
template <int VPL, bool SLICED>
__global__ void __launch_bounds__(ROUTE_WARPS * 32)
route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
             const float* __restrict__ offset, int64_t T, int E, int N, int K,
             int* __restrict__ idx, float* __restrict__ gate, float* __restrict__ zsum,
             int* __restrict__ cnt, int splits, int tps) {
  extern __shared__ int smem_i[];
  int* hist = smem_i;                                         // [E]
  float* lsum = reinterpret_cast<float*>(smem_i + E);         // [tps][E] (SLICED)
  for (int j = threadIdx.x; j < E; j += blockDim.x) hist[j] = 0;
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t split_stride = T * E;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * tps; t0 < T;
       t0 += static_cast<int64_t>(gridDim.x) * tps) {
    const int64_t t = t0 + warp;
    const bool mine = warp < tps && t < T;
    float l[VPL];
    if (SLICED && tps == ROUTE_WARPS) {
      // many tokens: each warp sums its own token's slices in registers
      if (mine) {
        const float* lrow = logits + t * E;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int j = lane + 32 * i;
          l[i] = (j < E) ? lrow[j] : 0.f;
        }
#pragma unroll 4
        for (int sp = 1; sp < splits; ++sp) {
          const float* srow = lrow + sp * split_stride;
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            const int j = lane + 32 * i;
            if (j < E) l[i] += srow[j];
          }
        }
      }
    } else if (SLICED) {
      // Few tokens: every thread sums some of the block's logits over the
      // slices, in slice order.  The loads of SLICE_GROUP slices are issued
      // together before their adds, so a logit waits for ceil(splits /
      // SLICE_GROUP) round trips to L2 rather than one per slice.
      constexpr int SLICE_GROUP = 8;
      const int V = static_cast<int>(T - t0 < tps ? T - t0 : tps) * E;
      const float* base = logits + t0 * E;
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        float acc = base[v];
        for (int sp = 1; sp < splits; sp += SLICE_GROUP) {
          float a[SLICE_GROUP];
#pragma unroll
          for (int u = 0; u < SLICE_GROUP; ++u)
            a[u] = sp + u < splits ? base[static_cast<int64_t>(sp + u) * split_stride + v] : 0.f;
#pragma unroll
          for (int u = 0; u < SLICE_GROUP; ++u)
            if (sp + u < splits) acc += a[u];
        }
        lsum[v] = acc;
      }
      __syncthreads();
      if (mine) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int j = lane + 32 * i;
          l[i] = (j < E) ? lsum[warp * E + j] : 0.f;
        }
      }
    } else if (mine) {
      const float* lrow = logits + t * E;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int j = lane + 32 * i;
        l[i] = (j < E) ? lrow[j] : 0.f;
      }
    }
    if (mine) route_token<VPL>(l, bias, offset, E, N, K, lane, t, idx, gate, zsum, hist);
    if (SLICED && tps < ROUTE_WARPS) __syncthreads();   // lsum is refilled next step
  }
  __syncthreads();
  for (int j = threadIdx.x; j < E; j += blockDim.x)
    if (hist[j]) atomicAdd(&cnt[j], hist[j]);
}

template <int VPL, bool SLICED>
cudaError_t launch_route_kernel(const float* logits, const float* b, const float* offset,
                                int64_t T, int E, int N, int K, int* idx, float* gate,
                                float* zsum, int* cnt, cudaStream_t stream, int splits) {
  const int sms = device_sms();
  // tokens per block step: ROUTE_WARPS, or for sliced logits of few tokens
  // fewer, so that about two blocks per SM share the slice sums
  int tps = ROUTE_WARPS;
  if (SLICED) {
    const int64_t want = (T + 2LL * sms - 1) / (2LL * sms);
    tps = static_cast<int>(want < 1 ? 1 : (want > ROUTE_WARPS ? ROUTE_WARPS : want));
  }
  const size_t smem =
      E * sizeof(int) + (SLICED && tps < ROUTE_WARPS ? static_cast<size_t>(tps) * E * sizeof(float) : 0);
  if (smem > 48 * 1024) {
    const cudaError_t e = smem_limit<route_kernel<VPL, SLICED>>(static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // one wave of resident blocks, each walking many token steps, so the
  // per-block histogram zeroing and flush are paid once per block
  const int per_sm = blocks_per_sm<route_kernel<VPL, SLICED>>(ROUTE_WARPS * 32, smem);
  const int64_t want = (T + tps - 1) / tps;
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(route_kernel<VPL, SLICED>, dim3(grid), dim3(ROUTE_WARPS * 32), smem, stream,
                    logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, splits, tps);
}

template <int VPL>
cudaError_t launch_route_vpl(const float* logits, const float* b, const float* offset, int64_t T,
                             int E, int N, int K, int* idx, float* gate, float* zsum, int* cnt,
                             cudaStream_t stream, int splits) {
  if (splits > 1)
    return launch_route_kernel<VPL, true>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt,
                                          stream, splits);
  return launch_route_kernel<VPL, false>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt,
                                         stream, splits);
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* b, const float* offset, int64_t T,
                         int E, int N, int K, int* idx, float* gate, float* zsum, int* cnt,
                         cudaStream_t stream, int splits) {
  if (T <= 0) return cudaSuccess;
  if (splits < 1) splits = 1;
#define MOEZC_ROUTE(V)                                                                     \
  if (E <= 32 * (V))                                                                       \
    return launch_route_vpl<V>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream, \
                               splits);
  MOEZC_ROUTE(1)
  MOEZC_ROUTE(2)
  MOEZC_ROUTE(3)
  MOEZC_ROUTE(4)
  MOEZC_ROUTE(6)
  MOEZC_ROUTE(8)
  MOEZC_ROUTE(12)
  MOEZC_ROUTE(16)
  MOEZC_ROUTE(24)
#undef MOEZC_ROUTE
  return launch_route_vpl<32>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream, splits);
}

}  // namespace moezc
