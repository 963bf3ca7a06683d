// fp8.cu -- block-scaled FP8 (E4M3) operands of the gate/up GEMM.
//
// LongCat-Flash write-up ("Meituan's large model goes viral for its speed",
// section "System-level optimisation", its quantisation paragraph): the model
// quantises at fine-grained block level, as DeepSeek-V3 does, and keeps the
// down projection (whose input activations reach extreme magnitudes) in
// higher precision.  The block form used here is the one the tensor cores'
// block-scaled FP8 MMA applies in hardware: one power-of-two scale per 32
// consecutive elements along the contraction (a weight row's or a token's),
// the smallest with amax / scale <= 448, so that no element saturates; the
// elements are E4M3 codes of value / scale, rounded to nearest, ties to even.
// An all-zero block, or one holding a NaN or an infinity, gets scale 1.
// Scales are stored as UE8M0 bytes (2^(byte - 127)), clamped to 2^-127 for
// blocks whose amax is below 448 * 2^-127 (no bf16 block is above the top of
// the range).
//
//   quantize weights   W [rows, cols] bf16 -> codes [rows, cols] and scales in
//                      the 512-byte atoms the GEMM copies into TMEM
//   permute (FP8)      each token row is quantised once, its codes go to the
//                      token's FFN slots of Xp8 and its scales to the atoms
//                      of the gate/up token tiles that hold those slots
#include "kernels.cuh"
#include "ptx.cuh"
#include "step.cuh"

namespace moezc {
namespace {

__global__ void fp8_quantize_weights_kernel(const uint4* __restrict__ W, int64_t rows, int cols,
                                            uint4* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int nb = cols / 32;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nb) return;
  const int64_t r = i / nb;
  const int kb = static_cast<int>(i - r * nb);
  const uint4* src = W + (r * cols + static_cast<int64_t>(kb) * 32) / 8;
  uint4 v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) v[q] = src[q];
  uint32_t c[8];
  const uint32_t s = quantize32(v, c);
  uint4* dst = codes + (r * cols + static_cast<int64_t>(kb) * 32) / 16;
  dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
  dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
  sf[sf_atom_offset(r, kb, cols / 128)] = static_cast<uint8_t>(s);
}

// One CTA per token: thread b quantises 32-element blocks b, b + blockDim.x, ...
// of the row and writes them to every FFN slot of the token.
__global__ void permute_fp8_kernel(const uint4* __restrict__ x, const int* __restrict__ idx,
                                   const int* __restrict__ slot, const int* __restrict__ cnt,
                                   const int* __restrict__ grp_off,
                                   const int* __restrict__ grp_ttp8, int d, int K, int N,
                                   uint4* __restrict__ Xp8, uint8_t* __restrict__ sfx) {
  const int64_t t = blockIdx.x;
  __shared__ int64_t row_s[MOE_MAX_K_INTERNAL];   // slot's first code byte, or -1
  __shared__ int64_t sf_s[MOE_MAX_K_INTERNAL];    // the slot's atom row base in sfx
  __shared__ int npick;
  griddep_wait();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int k = 0; k < K; ++k) {
      const int g = idx[t * K + k];
      const int s = slot[t * K + k];
      if (g < 0 || g >= N || s < 0) continue;
      const int count = cnt[g];
      const int ttp0 = grp_ttp8[g];
      const int ntt = grp_ttp8[g + 1] - ttp0;
      const int tsz = even_tile_size(count, ntt, FP8_BN);
      const int u = s - grp_off[g];
      const int j = u / tsz;
      const int pos = u - j * tsz;                 // the token's place in its tile
      const int64_t tile = ttp0 + j;
      row_s[n] = static_cast<int64_t>(s) * d;
      sf_s[n] = token_sf_base(tile, pos, d);
      ++n;
    }
    npick = n;
  }
  __syncthreads();
  const int nb = d / 32;
  const uint4* src = x + t * (d / 8);
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = src[b * 4 + q];
    uint32_t c[8];
    const uint32_t s = quantize32(v, c);
    const uint4 c0 = make_uint4(c[0], c[1], c[2], c[3]);
    const uint4 c1 = make_uint4(c[4], c[5], c[6], c[7]);
    // block b: contraction group b / 4 (one 1024-byte pair of atoms per group), byte b % 4
    const int64_t sf_off = static_cast<int64_t>(b / 4) * (2 * SF_ATOM_BYTES) + (b % 4);
    for (int k = 0; k < npick; ++k) {
      uint4* dst = Xp8 + (row_s[k] + static_cast<int64_t>(b) * 32) / 16;
      dst[0] = c0;
      dst[1] = c1;
      sfx[sf_s[k] + sf_off] = static_cast<uint8_t>(s);
    }
  }
  // many waves: the dependent GEMM launches only as the last CTAs finish
  griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_fp8_quantize_weights(const __nv_bfloat16* W, int64_t rows, int cols,
                                        uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  const int64_t n = rows * (cols / 32);
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  fp8_quantize_weights_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0,
                                stream>>>(reinterpret_cast<const uint4*>(W), rows, cols,
                                          reinterpret_cast<uint4*>(codes), sf);
  return cudaGetLastError();
}

cudaError_t launch_permute_fp8(const __nv_bfloat16* x, const int* idx, const int* slot,
                               const int* cnt, const int* grp_off, const int* grp_ttp8, int64_t T,
                               int d, int K, int N, uint8_t* Xp8, uint8_t* sfx,
                               cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int nb = d / 32;
  const int threads = nb < 256 ? ((nb + 31) / 32) * 32 : 256;
  return launch_pdl(permute_fp8_kernel, dim3(static_cast<unsigned>(T)), dim3(threads), 0, stream,
                    reinterpret_cast<const uint4*>(x), idx, slot, cnt, grp_off, grp_ttp8, d, K,
                    N, reinterpret_cast<uint4*>(Xp8), sfx);
}

}  // namespace moezc
