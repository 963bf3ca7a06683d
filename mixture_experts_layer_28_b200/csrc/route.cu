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
#include "kernels.cuh"
#include "ptx.cuh"
#include "step.cuh"

namespace moezc {
namespace {

constexpr int ROUTE_WARPS = 8;

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
      // slices, in slice order (slice_sum).
      const int V = static_cast<int>(T - t0 < tps ? T - t0 : tps) * E;
      const float* base = logits + t0 * E;
      for (int v = threadIdx.x; v < V; v += blockDim.x)
        lsum[v] = slice_sum(base + v, split_stride, splits);
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
