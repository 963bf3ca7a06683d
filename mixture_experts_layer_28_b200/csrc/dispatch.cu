// dispatch.cu -- counting-sort dispatch of (token, pick) pairs to FFN experts.
//
// Only picks of the N FFN experts are dispatched; a zero-computation expert
// returns its input (LongCat-Flash write-up "Meituan's large model goes viral
// for its speed", section "Zero-computation experts"), so its picks were
// already folded into zsum by the router and get slot -1 here.
//
//   assign    first every CTA takes, from the expert-load histogram, each
//             FFN expert's rows (count rounded up to 16) and token tiles
//             (ceil(count / 256), and for the FP8 gate/up GEMM ceil(count /
//             240)); exclusive prefix sums give the expert's first row in the
//             permuted buffers (rows rounded up to 16 per expert, or not at
//             all for a dispatch to other ranks, whose rows travel packed)
//             (grp_off) and its first GEMM token tile (grp_ttp, grp_ttp8),
//             which CTA 0 also stores for the GEMMs
//             (the GEMM grid walks grp_ttp).  Then one thread per (token,
//             pick): lanes of a warp that picked the same expert are grouped
//             with __match_any_sync and take their slots with one atomicAdd
//             per group (warp-aggregated atomics) on per-expert fill
//             counters that the router GEMM zeroed.
//   permute   one CTA per token (per part of its row for few tokens): copies
//             x_t (16-byte vectors) to each of its FFN slots of Xp, the B
//             operand of the gate/up GEMM.
// The histogram itself is integer and comes from the router, so it is exact.
#include "kernels.cuh"
#include "ptx.cuh"
#include "step.cuh"

namespace moezc {
namespace {

constexpr int ASSIGN_THREADS = 256;

__global__ void __launch_bounds__(ASSIGN_THREADS)
assign_slots_kernel(const int* __restrict__ cnt, const int* __restrict__ idx, int64_t pairs,
                    int N, int* __restrict__ grp_off, int* __restrict__ grp_ttp,
                    int* __restrict__ fill, int* __restrict__ slot, int* __restrict__ grp_ttp8,
                    int pad, int* __restrict__ row_expert) {
  __shared__ int off_s[MOE_MAX_E_INTERNAL];
  __shared__ int warp_sums[32];
  griddep_wait();
  // experts' first rows (and, in CTA 0, first token tiles) from the histogram
  int carry_rows = 0, carry_tiles = 0, carry_tiles8 = 0;
  for (int base = 0; base < N; base += ASSIGN_THREADS) {
    const int g = base + threadIdx.x;
    const int c = g < N ? cnt[g] : 0;
    int tot_rows, tot_tiles = 0, tot_tiles8 = 0;
    const int off = block_excl_scan<ASSIGN_THREADS>((c + pad - 1) / pad * pad, warp_sums, &tot_rows);
    if (g < N) off_s[g] = carry_rows + off;
    if (blockIdx.x == 0) {
      const int ttp = block_excl_scan<ASSIGN_THREADS>((c + GEMM_BN - 1) / GEMM_BN, warp_sums, &tot_tiles);
      if (g < N) {
        grp_off[g] = carry_rows + off;
        grp_ttp[g] = carry_tiles + ttp;
      }
      if (grp_ttp8) {   // (uniform over the CTA)
        const int t8 = block_excl_scan<ASSIGN_THREADS>((c + FP8_BN - 1) / FP8_BN, warp_sums, &tot_tiles8);
        if (g < N) grp_ttp8[g] = carry_tiles8 + t8;
      }
    }
    carry_rows += tot_rows;
    carry_tiles += tot_tiles;
    carry_tiles8 += tot_tiles8;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    grp_off[N] = carry_rows;
    grp_ttp[N] = carry_tiles;
    if (grp_ttp8) grp_ttp8[N] = carry_tiles8;
  }
  __syncthreads();

  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool valid = i < pairs;
  const int e = valid ? idx[i] : -1;
  const bool ffn = valid && e >= 0 && e < N;
  const unsigned act = __ballot_sync(0xffffffffu, ffn);
  int s = -1;
  if (ffn) {
    const unsigned peers = __match_any_sync(act, e);
    const int leader = __ffs(peers) - 1;
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int base = 0;
    if (lane == leader) base = atomicAdd(&fill[e], __popc(peers));
    base = __shfl_sync(peers, base, leader);
    s = off_s[e] + base + rank;
    if (row_expert) row_expert[s] = e;
  }
  if (valid) slot[i] = s;
  griddep_launch_dependents();   // as the last CTAs finish (several waves)
}

__global__ void permute_kernel(const uint4* __restrict__ x, const int* __restrict__ slot,
                               int d8, int K, uint4* __restrict__ Xp) {
  const int64_t t = blockIdx.x;
  const int part = blockIdx.y, parts = gridDim.y;   // this CTA's share of the row
  const int c_begin = static_cast<int>(static_cast<int64_t>(d8) * part / parts);
  const int c_end = static_cast<int>(static_cast<int64_t>(d8) * (part + 1) / parts);
  __shared__ int sl[MOE_MAX_K_INTERNAL];
  griddep_wait();
  if (threadIdx.x < K) sl[threadIdx.x] = slot[t * K + threadIdx.x];
  __syncthreads();
  const uint4* src = x + t * d8;
  for (int c = c_begin + threadIdx.x; c < c_end; c += blockDim.x) {
    const uint4 v = src[c];
    for (int k = 0; k < K; ++k) {
      const int s = sl[k];
      if (s >= 0) Xp[static_cast<int64_t>(s) * d8 + c] = v;
    }
  }
  // Many waves of CTAs: the dependent GEMM (one 216 KB CTA per SM) may
  // launch only as the last CTAs finish, or its early CTAs would take SMs
  // from this kernel's later waves.
  griddep_launch_dependents();
}

// Caller-given routing of R rows, one pick each: idx = expert - base, gate
// 1, zsum 0, and the histogram (cnt zeroed before the launch).  A row whose
// expert lies outside [base, base + N) is not dispatched (its output row is
// zero).
__global__ void given_routing_kernel(const int* __restrict__ expert, int64_t R, int base, int N,
                                     int* __restrict__ idx, float* __restrict__ gate,
                                     float* __restrict__ zsum, int* __restrict__ cnt) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= R) return;
  const int e = expert[i] - base;
  const bool ok = e >= 0 && e < N;
  idx[i] = ok ? e : -1;
  gate[i] = 1.0f;
  zsum[i] = 0.0f;
  if (ok) atomicAdd(cnt + e, 1);
}

__global__ void add_counts_kernel(const int* __restrict__ cnt, int E, int* __restrict__ total) {
  griddep_wait();
  griddep_launch_dependents();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < E) total[j] += cnt[j];
}

}  // namespace

cudaError_t launch_add_counts(const int* cnt, int E, int* total, cudaStream_t stream) {
  return launch_pdl(add_counts_kernel, dim3((E + 255) / 256), dim3(256), 0, stream, cnt, E, total);
}

cudaError_t launch_assign_slots(const int* cnt, const int* idx, int64_t pairs, int N,
                                int* grp_off, int* grp_ttp, int* fill, int* slot,
                                cudaStream_t stream, int* grp_ttp8, int pad, int* row_expert) {
  const int64_t blocks = pairs > 0 ? (pairs + ASSIGN_THREADS - 1) / ASSIGN_THREADS : 1;
  return launch_pdl(assign_slots_kernel, dim3(static_cast<unsigned>(blocks)), dim3(ASSIGN_THREADS),
                    0, stream, cnt, idx, pairs, N, grp_off, grp_ttp, fill, slot, grp_ttp8, pad,
                    row_expert);
}

cudaError_t launch_given_routing(const int* expert, int64_t R, int base, int N, int* idx,
                                 float* gate, float* zsum, int* cnt, cudaStream_t stream) {
  if (R <= 0) return cudaSuccess;
  return launch_pdl(given_routing_kernel, dim3(static_cast<unsigned>((R + 255) / 256)), dim3(256),
                    0, stream, expert, R, base, N, idx, gate, zsum, cnt);
}

cudaError_t launch_permute(const __nv_bfloat16* x, const int* slot, int64_t T, int d, int K,
                           __nv_bfloat16* Xp, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int d8 = d / 8;
  // few tokens: split each row over up to 8 CTAs (at least 128 vectors each)
  const int64_t want = (2LL * device_sms() + T - 1) / T;
  int parts = static_cast<int>(want < 8 ? want : 8);
  while (parts > 1 && d8 / parts < 128) --parts;
  if (parts < 1) parts = 1;
  const int per = (d8 + parts - 1) / parts;
  const int threads = per < 256 ? ((per + 31) / 32) * 32 : 256;
  return launch_pdl(permute_kernel, dim3(static_cast<unsigned>(T), parts), dim3(threads), 0, stream,
                    reinterpret_cast<const uint4*>(x), slot, d8, K, reinterpret_cast<uint4*>(Xp));
}

}  // namespace moezc
