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
//          scores become order-preserving uint32 keys, each lane keeps its
//          best slot, a round is two warp reductions (max key, then min
//          index among the lanes holding it), and only the winning lane
//          rescans its slots
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

// Best key of this lane's VPL slots (lower slot on equal keys), as a tree so
// the dependency depth is log2(VPL).
template <int VPL>
__device__ __forceinline__ void lane_best(const uint32_t (&key)[VPL], const float (&p)[VPL],
                                          uint32_t& bk, int& bi, float& bp) {
  uint32_t k[VPL];
  int ix[VPL];
  float pv[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) { k[i] = key[i]; ix[i] = i; pv[i] = p[i]; }
#pragma unroll
  for (int w = 1; w < VPL; w <<= 1) {
#pragma unroll
    for (int i = 0; i + w < VPL; i += 2 * w) {
      if (k[i + w] > k[i]) { k[i] = k[i + w]; ix[i] = ix[i + w]; pv[i] = pv[i + w]; }
    }
  }
  bk = k[0];
  bi = ix[0];
  bp = pv[0];
}

template <int VPL, bool SPLIT>  // logits per lane: E <= 32 * VPL; SPLIT: sum K slices
__global__ void __launch_bounds__(ROUTE_WARPS * 32)
route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
             const float* __restrict__ offset, int64_t T, int E, int N, int K,
             int* __restrict__ idx, float* __restrict__ gate, float* __restrict__ zsum,
             int* __restrict__ cnt, int splits) {
  extern __shared__ int hist[];  // [E]
  for (int j = threadIdx.x; j < E; j += blockDim.x) hist[j] = 0;
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t split_stride = T * E;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * ROUTE_WARPS + warp; t < T;
       t += static_cast<int64_t>(gridDim.x) * ROUTE_WARPS) {
    const float* lrow = logits + t * E;
    // logits: the router GEMM's K slices summed in slice order
    float l[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane + 32 * i;
      l[i] = (j < E) ? lrow[j] : 0.f;
    }
    // (unrolled by 4 so that several slices' loads are in flight at once;
    // the sum is still taken in slice order)
#pragma unroll 4
    for (int sp = 1; SPLIT && sp < splits; ++sp) {
      const float* srow = lrow + sp * split_stride;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int j = lane + 32 * i;
        if (j < E) l[i] += srow[j];
      }
    }
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

    uint32_t bk;
    int bi;
    float bp;
    lane_best<VPL>(key, p, bk, bi, bp);
    float zs = 0.f;
    for (int k = 0; k < K; ++k) {
      // the largest score; among equal scores the lowest expert index
      const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t cand = (bk == mk) ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu;
      const int jw = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
      const float pw = __shfl_sync(0xffffffffu, bp, jw & 31);
      if (jw >= N) zs += pw;
      if (lane == 0) {
        idx[t * K + k] = jw;
        gate[t * K + k] = pw;
        atomicAdd(&hist[jw], 1);
      }
      if (lane == (jw & 31)) {
        const int iw = jw >> 5;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (i == iw) key[i] = 0u;
        lane_best<VPL>(key, p, bk, bi, bp);
      }
    }
    if (lane == 0) zsum[t] = zs;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < E; j += blockDim.x)
    if (hist[j]) atomicAdd(&cnt[j], hist[j]);
}

template <int VPL, bool SPLIT>
cudaError_t launch_route_kernel(const float* logits, const float* b, const float* offset,
                               int64_t T, int E, int N, int K, int* idx, float* gate,
                               float* zsum, int* cnt, cudaStream_t stream, int splits) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one wave of resident blocks, each warp walking many tokens, so the
  // per-block histogram zeroing and flush are paid once per block
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_kernel<VPL, SPLIT>,
                                                    ROUTE_WARPS * 32, E * sizeof(int)) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t want = (T + ROUTE_WARPS - 1) / ROUTE_WARPS;
  const int64_t cap = static_cast<int64_t>(sms) * per_sm;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_pdl(route_kernel<VPL, SPLIT>, dim3(grid), dim3(ROUTE_WARPS * 32), E * sizeof(int),
                    stream, logits, b, offset, T, E, N, K, idx, gate, zsum, cnt, splits);
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
