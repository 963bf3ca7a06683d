// combine.cu -- weighted combine of the expert outputs.
//
// LongCat-Flash write-up ("Meituan's large model goes viral for its speed",
// section "Zero-computation experts"): the layer's output is the
// gate-weighted sum of the picked experts' outputs, and a zero-computation
// expert's output is its input.  So, per token t,
//
//   out_t = bf16( zsum_t * x_t + sum_{k : slot_{t,k} >= 0} gate_{t,k} * Y[slot_{t,k}] )
//
// with zsum_t the router's sum of zero-expert gates.  fp32 accumulation in a
// fixed order (zero experts first, then picks k = 0..K-1), one rounding to
// bf16: the result does not depend on where the dispatch put a token's rows.
// One CTA per token and part of the row (few tokens: several parts, so that
// more SMs keep loads in flight); each thread handles 8 features at a time
// with 16-byte loads.
#include "kernels.cuh"
#include "ptx.cuh"
#include "step.cuh"

namespace moezc {
namespace {

__global__ void combine_kernel(const uint4* __restrict__ x, const uint4* __restrict__ Y,
                               const int* __restrict__ slot, const float* __restrict__ gate,
                               const float* __restrict__ zsum, int d8, int K,
                               uint4* __restrict__ out) {
  const int64_t t = blockIdx.x;
  const int part = blockIdx.y, parts = gridDim.y;   // this CTA's share of the row
  const int c_begin = static_cast<int>(static_cast<int64_t>(d8) * part / parts);
  const int c_end = static_cast<int>(static_cast<int64_t>(d8) * (part + 1) / parts);
  __shared__ int sl[MOE_MAX_K_INTERNAL];
  __shared__ float gt[MOE_MAX_K_INTERNAL];
  __shared__ int nffn;
  griddep_wait();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int k = 0; k < K; ++k) {
      const int s = slot[t * K + k];
      if (s >= 0) { sl[n] = s; gt[n] = gate[t * K + k]; ++n; }
    }
    nffn = n;
  }
  __syncthreads();
  const float z = zsum[t];
  const int n = nffn;
  for (int c = c_begin + threadIdx.x; c < c_end; c += blockDim.x)
    out[t * d8 + c] = combine_chunk(x, Y, t, c, d8, z, sl, gt, n);
  // many waves of CTAs: let dependents launch only as the last ones finish
  griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* x, const __nv_bfloat16* Y, const int* slot,
                           const float* gate, const float* zsum, int64_t T, int d, int K,
                           __nv_bfloat16* out, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int d8 = d / 8;
  // few tokens: split each row over up to 8 CTAs (at least 128 vectors each)
  // so that about two CTAs per SM are busy
  const int64_t want = (2LL * device_sms() + T - 1) / T;
  int parts = static_cast<int>(want < 8 ? want : 8);
  while (parts > 1 && d8 / parts < 128) --parts;
  if (parts < 1) parts = 1;
  const int per = (d8 + parts - 1) / parts;
  const int threads = per < 256 ? ((per + 31) / 32) * 32 : 256;
  return launch_pdl(combine_kernel, dim3(static_cast<unsigned>(T), parts), dim3(threads), 0, stream,
                    reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(Y), slot,
                    gate, zsum, d8, K, reinterpret_cast<uint4*>(out));
}

}  // namespace moezc
