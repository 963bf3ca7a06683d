// gemm_pair.cu -- the expert GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// Same contractions as gemm_tcgen05.cu for the FFN experts of the MoE layer
// with zero-computation experts (LongCat-Flash write-up "Meituan's large
// model goes viral for its speed", section "Zero-computation experts"), with
// the weights as the MMA's A operand as in the write-up's "SwapAB" kernels,
// but on a pair of SMs: one MMA of M = 256 weight rows x N = up to 256 tokens
// reads its A rows 128 + 128 and its B tokens N/2 + N/2 from the two CTAs'
// shared memory and leaves each CTA 128 rows x N fp32 in its own TMEM.
//
// Per CTA that is 32 KB of operands per 64-wide K step for 4.2 MFLOP -- the
// same operand reuse as the single-SM kernel's 64 KB for 8.4 MFLOP -- but the
// accumulator needs only 256 TMEM columns, so it is double-buffered: the
// epilogue of tile i runs while the MMAs of tile i+1 fill the other buffer,
// and the smaller stages give a six-deep TMA ring.
//
//   gate/up  CTA r's 128 A rows are W_gate and W_up rows of the same 64
//            features (m*128 + r*64 + 0..63): TMEM lanes 0..63 hold gate,
//            64..127 up.  Warps of lane quadrants 0/1 (gate) and 2/3 (up)
//            pair up, swap their halves through shared memory and each
//            writes H = SiLU(gate) * up for half of the tokens.
//   down     CTA r's A rows are W_down rows m*256 + r*128 + 0..127.
//
// Roles per CTA (384 threads): warp 0 TMA producer (both CTAs, completion
// counted on the even CTA's barrier), warp 1 MMA issuer (even CTA only),
// warp 2 TMEM allocator (both), warps 4..11 epilogue (both).  All waits are
// time-bounded; on running out a CTA records the error, drains what it has in
// flight and leaves through the same cluster barrier.
#include "epilogue.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace moezc {
namespace {

constexpr long long PAIR_DRAIN_NS = 2000000000LL;

struct PairTile {
  int g, m, tok0, count, nmma, half_rows, brow, a_row_gate_or_down, a_row_up;
};

template <int MODE>
__device__ __forceinline__ PairTile pair_tile(const GemmParams& p, int t, uint32_t rank) {
  // Tiles of one expert come in groups of `mg` weight blocks: all of the
  // expert's token tiles for blocks 0..mg-1, then for the next mg blocks, so
  // the pairs running at the same time share fewer weight blocks more often.
  PairTile tl;
  const int mg = p.mgroup > 0 ? p.mgroup : p.mblocks;
  int lo = 0, hi = p.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.grp_ttp + mid) * p.mblocks <= t) lo = mid; else hi = mid - 1;
  }
  tl.g = lo;
  const int ttp0 = __ldg(p.grp_ttp + lo);
  const int ntt = __ldg(p.grp_ttp + lo + 1) - ttp0;   // token tiles of this expert
  const int tl_local = t - ttp0 * p.mblocks;
  const int grp = tl_local / (ntt * mg);
  const int rem = tl_local - grp * (ntt * mg);
  const int j = rem / mg;
  tl.m = grp * mg + (rem - j * mg);
  tl.count = __ldg(p.grp_count + lo);
  tl.tok0 = j * GEMM_BN;
  const int ntok = min(GEMM_BN, tl.count - tl.tok0);
  tl.nmma = (ntok + 15) & ~15;
  tl.half_rows = tl.nmma >> 1;
  // this CTA's half of the tokens
  tl.brow = __ldg(p.grp_off + lo) + tl.tok0 + static_cast<int>(rank) * tl.half_rows;
  if (MODE == MODE_GATEUP) {
    tl.a_row_gate_or_down = tl.g * p.a_rows + tl.m * GEMM_BM + static_cast<int>(rank) * 64;
    tl.a_row_up = tl.a_row_gate_or_down;
  } else {
    tl.a_row_gate_or_down = tl.g * p.a_rows + tl.m * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM;
    tl.a_row_up = 0;
  }
  return tl;
}

template <int MODE>
__global__ void __launch_bounds__(PAIR_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[PAIR_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[PAIR_STAGES];
  __shared__ __align__(8) uint64_t acc_full_bar[2];
  __shared__ __align__(8) uint64_t acc_empty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* epi = smem + PAIR_STAGES * PAIR_STAGE_BYTES;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full_bar[b], 1);
      mbar_init(&acc_empty_bar[b], 2 * PAIR_EPI_WARPS);   // one per epilogue warp, both CTAs
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  __syncwarp();
  if (warp == 2) {
    tmem_alloc_pair(&tmem_base_sh, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before any cross-CTA use
  tc_fence_after();
  griddep_wait();       // the previous kernel's results are visible from here
  griddep_launch_dependents();
  const uint32_t tmem = tmem_base_sh;
  const int ntiles = __ldg(p.grp_ttp + p.G) * p.mblocks;
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, last_par = 0;
      for (int t = cl; t < ntiles && !abort_sh; t += ncl) {
        const PairTile tl = pair_tile<MODE>(p, t, rank);
        const int nbox = (tl.half_rows + GEMM_B_BOX_ROWS - 1) / GEMM_B_BOX_ROWS;
        const uint32_t cta_bytes = PAIR_A_BYTES + nbox * GEMM_B_BOX_ROWS * GEMM_BK * 2;
        for (int ks = 0; ks < p.ksteps; ++ks) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, p.wait_ns, p.err)) {
            abort_sh = 1;
            break;
          }
          uint8_t* st = smem + stage * PAIR_STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * cta_bytes);
          armed |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          const int kc = ks * GEMM_BK;
          if (MODE == MODE_GATEUP) {
            tma_load_2d_pair(st, &tmA0, bar, kc, tl.a_row_gate_or_down);            // 64 gate rows
            tma_load_2d_pair(st + PAIR_A_BYTES / 2, &tmA1, bar, kc, tl.a_row_up);   // 64 up rows
          } else {
            tma_load_2d_pair(st, &tmA0, bar, kc, tl.a_row_gate_or_down);            // 128 rows
          }
          uint8_t* sb = st + PAIR_A_BYTES;
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d_pair(sb + bx * GEMM_B_BOX_ROWS * GEMM_BK * 2, &tmB, bar, kc,
                             tl.brow + bx * GEMM_B_BOX_ROWS);
          if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Drain: the even CTA's full barriers count both CTAs' copies; the odd
      // CTA sees its copies consumed through its empty barriers.
      for (int s = 0; s < PAIR_STAGES; ++s)
        if (armed & (1u << s))
          mbar_wait(leader ? &full_bar[s] : &empty_bar[s], (last_par >> s) & 1, PAIR_DRAIN_NS,
                    p.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = cl; t < ntiles && !abort_sh; t += ncl, ++local) {
        const PairTile tl = pair_tile<MODE>(p, t, rank);
        const int buf = local & 1, use = local >> 1;
        if (use > 0 && !mbar_wait(&acc_empty_bar[buf], (use - 1) & 1, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(2 * GEMM_BM, tl.nmma);
        const uint32_t dt = tmem + buf * 256;
        bool ok = true;
        for (int ks = 0; ks < p.ksteps; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * PAIR_STAGE_BYTES);
          const uint64_t ad = smem_desc_sw128(st);
          const uint64_t bd = smem_desc_sw128(st + PAIR_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk)
            umma_bf16_pair(dt, ad + 2 * kk, bd + 2 * kk, idesc, (ks | kk) != 0 ? 1u : 0u);
          umma_commit_pair_mc(&empty_bar[stage], 0x3);
          if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) { abort_sh = 1; break; }
        umma_commit_pair_mc(&acc_full_bar[buf], 0x3);
      }
      umma_commit_pair(&drain_bar);
      mbar_wait(&drain_bar, 0, PAIR_DRAIN_NS, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant
    const int half = (warp - 4) >> 2;   // which 32-column chunks
    const uint64_t pol_out = p.l2_stream ? l2_policy_evict_first() : 0;
    const uint32_t acc_empty_cl0 = mapa_shared(smem_u32(&acc_empty_bar[0]), 0);
    const uint32_t acc_empty_cl1 = mapa_shared(smem_u32(&acc_empty_bar[1]), 0);
    int local = 0;
    for (int t = cl; t < ntiles && !abort_sh; t += ncl, ++local) {
      const PairTile tl = pair_tile<MODE>(p, t, rank);
      const int buf = local & 1, use = local >> 1;
      if (!mbar_wait(&acc_full_bar[buf], use & 1, p.wait_ns, p.err)) {
        abort_sh = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      const int64_t row_of_tok0 = static_cast<int64_t>(__ldg(p.grp_off + tl.g)) + tl.tok0;
      for (int c0 = half * 32; c0 < tl.nmma; c0 += 64) {
        const bool wide = c0 + 32 <= tl.nmma;
        const int ncol = wide ? 32 : 16;
        uint32_t r[32];
        tmem_ld16(tq + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
        if (wide) tmem_ld16(tq + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
        tmem_ld_wait();
        const int tok_base = tl.tok0 + c0;
        if (MODE == MODE_GATEUP) {
          // gate warps (q 0/1) pair with up warps (q 2/3) of the same features
          const int pr = (q & 1) + 2 * half;
          const bool is_gate = q < 2;
          uint8_t* pb = epi + pr * PAIR_XCHG_BYTES;
          float* xg = reinterpret_cast<float*>(pb);
          float* xu = reinterpret_cast<float*>(pb + 4096);
          // Each warp writes its 32 x ncol values, both read the other's,
          // then each stages and stores half of the tokens through its own
          // half of the swap buffer (same warp, so no further barrier).
          float* mine = is_gate ? xg : xu;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < ncol) mine[i * 32 + lane] = __uint_as_float(r[i]);
          named_bar_sync(1 + pr, 64);   // both halves written
          const int nmine = ncol >> 1;
          const int start = is_gate ? 0 : nmine;
          uint32_t h[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g = xg[(start + i) * 32 + lane];
            const float u = xu[(start + i) * 32 + lane];
            h[i] = __float_as_uint(g * __frcp_rn(1.0f + __expf(-g)) * u);
          }
#pragma unroll
          for (int i = 16; i < 32; ++i) h[i] = 0u;
          named_bar_sync(1 + pr, 64);   // both done reading the swap buffer
          const int rows = min(nmine, tl.count - (tok_base + start));
          const int f = tl.m * GEMM_BM + static_cast<int>(rank) * 64 + (q & 1) * 32;
          if (rows > 0)
            stage_store_bf16(reinterpret_cast<uint8_t*>(mine), lane, h, nmine, rows,
                             out + (row_of_tok0 + c0 + start) * p.out_ld + f, p.out_ld,
                             pol_out);
        } else {
          const int rows = min(ncol, tl.count - tok_base);
          const int f = tl.m * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM + q * 32;
          uint8_t* stg = epi + (warp - 4) * 2048;
          stage_store_bf16(stg, lane, r, ncol, rows, out + (row_of_tok0 + c0) * p.out_ld + f,
                           p.out_ld, pol_out);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? acc_empty_cl1 : acc_empty_cl0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the pair's MMAs, copies and remote arrivals are over
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_gemm_pair(GemmMode mode, const CUtensorMap& a0, const CUtensorMap& a1,
                             const CUtensorMap& b, const GemmParams& p, int clusters,
                             cudaStream_t stream) {
  if (clusters <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(PAIR_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (mode == MODE_GATEUP) {
    e = smem_limit<gemm_pair_kernel<MODE_GATEUP>>(PAIR_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<MODE_GATEUP>, a0, a1, b, p);
  } else if (mode == MODE_DOWN) {
    e = smem_limit<gemm_pair_kernel<MODE_DOWN>>(PAIR_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<MODE_DOWN>, a0, a1, b, p);
  } else {
    return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moezc
