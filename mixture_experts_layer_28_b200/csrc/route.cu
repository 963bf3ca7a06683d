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
//   picks: K rounds of a warp-wide argmax of s (ties -> lower expert index)
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

namespace moezc {
namespace {

constexpr int ROUTE_WARPS = 8;

template <int VPL>  // logits per lane: E <= 32 * VPL
__global__ void __launch_bounds__(ROUTE_WARPS * 32)
route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
             const float* __restrict__ offset, int64_t T, int E, int N, int K,
             int* __restrict__ idx, float* __restrict__ gate, float* __restrict__ zsum,
             int* __restrict__ cnt) {
  extern __shared__ int hist[];  // [E]
  for (int j = threadIdx.x; j < E; j += blockDim.x) hist[j] = 0;
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * ROUTE_WARPS + warp; t < T;
       t += static_cast<int64_t>(gridDim.x) * ROUTE_WARPS) {
    const float* lrow = logits + t * E;
    float p[VPL], s[VPL];
    float mx = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane + 32 * i;
      float l = -FLT_MAX;
      if (j < E) {
        l = lrow[j];
        if (offset) l += offset[j];
      }
      p[i] = l;
      mx = fmaxf(mx, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane + 32 * i;
      p[i] = (j < E) ? expf(p[i] - mx) : 0.f;
      sum += p[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane + 32 * i;
      p[i] *= inv;
      // A NaN score (only from non-finite logits) ranks below every real
      // score but above a taken or absent expert, so each round still picks
      // a valid index.
      const float sc = p[i] + (j < E ? bias[j] : 0.f);
      s[i] = (j < E) ? (sc == sc ? sc : -FLT_MAX) : -INFINITY;
    }

    float zs = 0.f;
    for (int k = 0; k < K; ++k) {
      // best of this lane (values visited in increasing index: strict > keeps the lower one)
      float bs = -INFINITY, bp = 0.f;
      int bj = INT_MAX;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        if (s[i] > bs) { bs = s[i]; bj = lane + 32 * i; bp = p[i]; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        const float op = __shfl_xor_sync(0xffffffffu, bp, o);
        if (os > bs || (os == bs && oj < bj)) { bs = os; bj = oj; bp = op; }
      }
      // remove the winner from its lane
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i == bj) s[i] = -INFINITY;
      if (bj >= N) zs += bp;
      if (lane == 0) {
        idx[t * K + k] = bj;
        gate[t * K + k] = bp;
        atomicAdd(&hist[bj], 1);
      }
    }
    if (lane == 0) zsum[t] = zs;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < E; j += blockDim.x)
    if (hist[j]) atomicAdd(&cnt[j], hist[j]);
}

template <int VPL>
cudaError_t launch_route_vpl(const float* logits, const float* b, const float* offset, int64_t T,
                             int E, int N, int K, int* idx, float* gate, float* zsum, int* cnt,
                             cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (T + ROUTE_WARPS - 1) / ROUTE_WARPS;
  // a few tokens per warp so the per-block histogram flush is amortised
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  route_kernel<VPL><<<grid, ROUTE_WARPS * 32, E * sizeof(int), stream>>>(
      logits, b, offset, T, E, N, K, idx, gate, zsum, cnt);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const float* logits, const float* b, const float* offset, int64_t T,
                         int E, int N, int K, int* idx, float* gate, float* zsum, int* cnt,
                         cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (E <= 128) return launch_route_vpl<4>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream);
  if (E <= 256) return launch_route_vpl<8>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream);
  if (E <= 512) return launch_route_vpl<16>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream);
  return launch_route_vpl<32>(logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, stream);
}

}  // namespace moezc
