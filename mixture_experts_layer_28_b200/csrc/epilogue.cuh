// epilogue.cuh -- shared-memory staged stores of GEMM results.
//
// A warp holds a 32-feature x up-to-32-token block of results (thread =
// feature, register i = token i).  The block goes through a per-warp staging
// tile in shared memory, transposed to token-major rows, and leaves as
// coalesced 16-byte stores.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace moezc {

// One warp's 32 features x ncol tokens of fp32 results (thread = feature,
// v[i] = token i) -> bf16 rows out[i * ld + 0..31] for i < rows, through a
// [32 tokens][32 features] staging tile: 2-byte shared stores by feature,
// then 16-byte loads and global stores, four lanes per 64-byte row; a
// non-zero l2_policy (createpolicy) is attached to the global stores.
__device__ __forceinline__ void stage_store_bf16(uint8_t* stg, int lane, const uint32_t (&v)[32],
                                                 int ncol, int rows, __nv_bfloat16* out,
                                                 int64_t ld, uint64_t l2_policy) {
  __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(stg);
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i < ncol) st[i * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = (lane >> 2) + 8 * k;
    const int part = lane & 3;
    if (r < rows) {
      const uint4 val = *reinterpret_cast<const uint4*>(stg + r * 64 + part * 16);
      if (l2_policy)
        st_global_v4_hint(out + r * ld + part * 8, val, l2_policy);
      else
        *reinterpret_cast<uint4*>(out + r * ld + part * 8) = val;
    }
  }
  __syncwarp();
}

// As stage_store_bf16, from results already rounded to bf16 and packed in
// pairs (v[i] holds tokens 2i and 2i+1 in its low and high halves).
__device__ __forceinline__ void stage_store_bf16x2(uint8_t* stg, int lane, const uint32_t (&v)[16],
                                                   int ncol, int rows, __nv_bfloat16* out,
                                                   int64_t ld, uint64_t l2_policy) {
  uint16_t* st = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (2 * i < ncol) {
      st[(2 * i) * 32 + lane] = static_cast<uint16_t>(v[i] & 0xFFFFu);
      st[(2 * i + 1) * 32 + lane] = static_cast<uint16_t>(v[i] >> 16);
    }
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = (lane >> 2) + 8 * k;
    const int part = lane & 3;
    if (r < rows) {
      const uint4 val = *reinterpret_cast<const uint4*>(stg + r * 64 + part * 16);
      if (l2_policy)
        st_global_v4_hint(out + r * ld + part * 8, val, l2_policy);
      else
        *reinterpret_cast<uint4*>(out + r * ld + part * 8) = val;
    }
  }
  __syncwarp();
}

// fp32 variant for the router's logits: features ebase + 0..31 of rows
// tok_base + i, features >= E dropped; 128-byte rows, eight lanes per row,
// staged 16 tokens at a time (2 KB).
__device__ __forceinline__ void stage_store_f32(uint8_t* stg, int lane, const uint32_t (&v)[32],
                                                int ncol, int rows, float* out, int tok_base,
                                                int ld, int ebase, int E) {
  uint32_t* st = reinterpret_cast<uint32_t*>(stg);
  const bool vec = (ld % 4 == 0) && (ebase + 32 <= E);
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (hf * 16 >= ncol) break;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (hf * 16 + i < ncol) st[i * 32 + lane] = v[hf * 16 + i];
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = (lane >> 3) + 4 * k;
      const int row = hf * 16 + r;
      const int part = lane & 7;
      if (row < rows) {
        float* dst = out + static_cast<int64_t>(tok_base + row) * ld + ebase + part * 4;
        const uint4 val = *reinterpret_cast<const uint4*>(stg + r * 128 + part * 16);
        if (vec) {
          *reinterpret_cast<uint4*>(dst) = val;
        } else {
          const uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (ebase + part * 4 + e < E) dst[e] = __uint_as_float(w[e]);
        }
      }
    }
    __syncwarp();
  }
}

}  // namespace moezc
