// gemm_tcgen05.cu -- grouped "SwapAB" GEMM on the 5th-generation tensor cores.
//
// The three contractions of the MoE layer with zero-computation experts
// (LongCat-Flash write-up "Meituan's large model goes viral for its speed",
// section "Zero-computation experts"; SwiGLU expert form per the layer's
// definition in moe_zc.h) run on this one engine:
//
//   router   logits[t, e]  = x_t . W_r[e]                  (fp32 out)
//   gate/up  H[s, i]       = SiLU(Xp_s . W_gate[e,i]) * (Xp_s . W_up[e,i])
//   down     Y[s, j]       = H_s . W_down[e, j]
//
// where s runs over the slots of the tokens routed to FFN expert e.  As in the
// write-up's section on custom kernels ("SwapAB"), the weights are the left
// operand: an A block is 128 weight rows (MMA M = 128) and the tokens of one
// expert are the right operand (MMA N = 16..256 in steps of 16), so an expert
// hit by a handful of decode tokens costs an N = 16 MMA rather than a padded
// 128-row one.
//
// A tile is (expert g, token tile j, weight block m): one or two A blocks
// (gate and up rows of block m; two consecutive 128-row blocks of W_down or
// W_r; or a single block) against up to 256 tokens.  Each A block gives one
// 128 x N fp32 accumulator in TMEM; 256-token tiles keep the MMA at N = 256,
// the shape whose operand traffic the tensor core and L2 sustain (128-token
// tiles and single-block down tiles were measured slower).
//
// Persistent, warp-specialised CTA (512 threads, one per SM):
//   warp 0      TMA producer: A blocks [128 x 64] and B boxes (one [256 x 64]
//               box for a full token tile, else [32 x 64] boxes), 128-byte
//               swizzle, into a 3-stage shared-memory ring
//   warp 1      MMA issuer: tcgen05.mma kind::f16, commits free the stage
//   warp 2      TMEM allocator (512 columns)
//   warps 4..15 epilogue, three per TMEM lane quadrant: tcgen05.ld ->
//               fp32 math -> bf16 in registers -> shared staging ->
//               coalesced 16-byte global stores
// The epilogue hands TMEM back as soon as it has read it, before it stores:
//   * one-block tiles use 256 columns, so two accumulator buffers alternate
//     and a tile's epilogue overlaps the next tile's MMAs;
//   * two-block tiles fill all 512 columns; the epilogue releases the first
//     accumulator, then the second, and the issuer starts the next tile's
//     first-block MMAs on up to GEMM_STAGES loaded stages before it needs
//     the second accumulator back.
// Batches of at most 64 tokens (decode) stream weights: there the gate/up and
// down tiles run in one persistent grid (MODE_FUSED, see gemm_kernel), so the
// SMs that the last, part-filled round of gate/up tiles leaves idle stream
// down weights of the experts whose H rows are already complete; the same
// grid also routes, dispatches and combines (the decode step's phases,
// step.cuh).
// That grid and the prefill-sized gate/up and down launches take their tiles
// in order from a global counter (the producer takes each and hands it to
// the MMA issuer and the epilogue through a small shared-memory queue), so
// the tiles running at any moment are neighbours in tile order -- those that
// share a weight block or a token tile overlap in time and re-read it from
// L2 -- and SMs that stream faster take more tiles.
// Every wait is time-bounded (ptx.cuh); on running out the CTA drains its
// in-flight copies and MMAs, frees TMEM and returns with the error flag set.
#include "epilogue.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "step.cuh"

namespace moezc {
namespace {

constexpr long long DRAIN_NS = 2000000000LL;  // bound of the drain waits at exit
constexpr long long PACE_NS = 50000LL;        // longest wait for the partner CTA's tile start
constexpr int TILE_Q = 4;                      // depth of the producer's tile queue

struct Tile {
  int k0, k1;   // k-step range of this tile
  int split;    // router: K slice index
  int g;        // group (expert)
  int m;        // weight block
  int tok0;     // first token of the tile inside its group
  int ntok;     // valid tokens in the tile
  int nmma;     // MMA N: ntok rounded up to 16
  int brow0;    // first B row
  int count;    // tokens in the group
  int ntt;      // token tiles of the group
  bool has_a1;  // second A block present
  int a0_row, a1_row;
  int r0;       // router / down: A block 0's first row inside the group
  int ttile;    // expert GEMMs: the tile's index among all token tiles (FP8 scale atoms)
};

// The expert offsets and counts a tile is decoded from: written by earlier
// kernels (read-only here: the non-coherent path), or -- in the one grid
// that runs the whole decode step -- by this grid's own assign phase (COH):
// plain loads, which after the grid barrier's acquire see those writes and
// then hit in L1 (no block reads these words before that barrier).
template <bool COH>
__device__ __forceinline__ int ld_meta(const int* p) {
  return COH ? *p : __ldg(p);
}

__device__ __forceinline__ int router_tok_tile(const GemmParams& p) {
  return p.tok_tile > 0 ? p.tok_tile : GEMM_BN;
}

template <int MODE, bool COH = false>
__device__ __forceinline__ int total_tiles(const GemmParams& p) {
  if (MODE == MODE_ROUTER) {
    const int tt = router_tok_tile(p);
    return ((p.T + tt - 1) / tt) * p.mblocks * (p.ksplit > 1 ? p.ksplit : 1);
  }
  return ld_meta<COH>(p.grp_ttp + p.G) * p.mblocks;
}

// Group (expert) of expert-GEMM tile t: the largest g with ttp[g] <= t / mblocks
// (a group's tiles start at ttp[g] * mblocks).
template <bool COH = false>
__device__ __forceinline__ int group_of_tile(const GemmParams& p, int t) {
  const int tt = t / p.mblocks;
  int lo = 0, hi = p.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ld_meta<COH>(p.grp_ttp + mid) <= tt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int MODE, bool COH = false>
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int t) {
  Tile tl;
  tl.split = 0;
  tl.k0 = 0;
  tl.k1 = p.ksteps;
  if (MODE == MODE_ROUTER && p.ksplit > 1) {
    const int per = ((p.T + router_tok_tile(p) - 1) / router_tok_tile(p)) * p.mblocks;
    tl.split = t / per;
    t -= tl.split * per;
    tl.k0 = static_cast<int>(static_cast<long long>(p.ksteps) * tl.split / p.ksplit);
    tl.k1 = static_cast<int>(static_cast<long long>(p.ksteps) * (tl.split + 1) / p.ksplit);
  }
  const int tt = t / p.mblocks;
  tl.m = t - tt * p.mblocks;
  int j;
  if (MODE == MODE_ROUTER) {
    tl.g = 0;
    tl.ntt = 0;
    j = tt;
    tl.count = p.T;
    tl.brow0 = 0;
  } else {
    const int lo = group_of_tile<COH>(p, t);
    tl.g = lo;
    // Order inside the group: weight block fastest, so that the tiles of a
    // round of the persistent grid share a few weight blocks and token
    // tiles; but an expert with two token tiles goes weight block by weight
    // block with its two token tiles adjacent (tiles 2i and 2i + 1 read the
    // same weight block).
    const int ttp0 = ld_meta<COH>(p.grp_ttp + lo);
    const int ntt = ld_meta<COH>(p.grp_ttp + lo + 1) - ttp0;
    tl.ntt = ntt;
    const int u = t - ttp0 * p.mblocks;
    if (ntt == 2) {
      tl.m = u >> 1;
      j = u & 1;
    } else {
      j = u / p.mblocks;
      tl.m = u - j * p.mblocks;
    }
    tl.count = ld_meta<COH>(p.grp_count + lo);
    tl.brow0 = ld_meta<COH>(p.grp_off + lo);
  }
  // An expert's ntt = ceil(count / tile) token tiles share its tokens evenly
  // (sizes a multiple of 16): two tiles of similar size run side by side in
  // one round of the persistent grid and read the same weight blocks at the
  // same pace, so the second read of a block is an L2 hit.  (tile: GEMM_BN,
  // or FP8_BN for the FP8 gate/up GEMM, whose p.tok_tile says so.)
  int tsz = router_tok_tile(p);
  tl.ttile = 0;
  if (MODE != MODE_ROUTER) {
    tsz = even_tile_size(tl.count, tl.ntt, tsz);
    tl.ttile = ld_meta<COH>(p.grp_ttp + tl.g) + j;
  }
  tl.tok0 = j * tsz;
  tl.ntok = min(tsz, tl.count - tl.tok0);
  tl.nmma = (tl.ntok + 15) & ~15;
  tl.brow0 += tl.tok0;
  if (MODE == MODE_GATEUP) {
    tl.r0 = tl.m * GEMM_BM;
    tl.a0_row = tl.g * p.a_rows + tl.r0;             // W_gate rows
    tl.a1_row = tl.a0_row;                           // W_up rows
    tl.has_a1 = true;
  } else {
    const int r = tl.m * (p.single_a ? 1 : 2) * GEMM_BM;
    tl.r0 = r;
    tl.a0_row = tl.g * p.a_rows + r;
    tl.a1_row = tl.a0_row + GEMM_BM;
    tl.has_a1 = !p.single_a && (r + GEMM_BM) < p.a_rows;
  }
  return tl;
}

// Tile `it` of this CTA's list when tiles are not taken from a counter (the
// router, and the one-phase GEMMs of batches below the counter's size):
// tiles blockIdx.x + i * G of the n0.  (MODE_FUSED always takes its tiles
// from the counter.)
template <int MODE>
__device__ __forceinline__ bool tile_at(int it, int n0, int& tph, int& t) {
  tph = 0;
  t = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
  return t < n0;
}

// Tiles taken in order from p.tile_counter: the u-th is tile u of a
// one-phase mode; MODE_FUSED hands out its n0 gate/up tiles, then its down
// tiles in group order.  Gate/up tiles wait on nothing, and all of them are
// handed out before any down tile, so every down tile's wait ends.
template <int MODE>
__device__ __forceinline__ void dyn_tile(int u, int n0, int& tph, int& t) {
  tph = MODE == MODE_FUSED && u >= n0 ? 1 : 0;
  t = tph ? u - n0 : u;
}

// Tile t of the given phase (see tile_at).
template <int MODE>
__device__ __forceinline__ Tile phase_tile(const GemmParams& p, const GemmParams& p2, int tph,
                                           int t) {
  if (MODE == MODE_FUSED)
    return tph ? decode_tile<MODE_DOWN, true>(p2, t) : decode_tile<MODE_GATEUP, true>(p, t);
  return decode_tile<MODE>(p, t);
}


// One 64-wide K step of one A block: four K = 16 MMAs into accumulator d.
__device__ __forceinline__ void mma_kstep(uint32_t d, uint32_t a_smem, uint32_t b_smem,
                                          uint32_t idesc, bool first) {
  const uint64_t ad = smem_desc_sw128(a_smem);
  const uint64_t bd = smem_desc_sw128(b_smem);
#pragma unroll
  for (int kk = 0; kk < GEMM_BK / 16; ++kk)
    umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (first && kk == 0) ? 0u : 1u);
}

// FP8 (block-scaled) gate/up tiles keep their scale factors in TMEM columns
// SF_TMEM_COL.. (behind the two FP8_BN-column accumulators): W_gate's atom
// at +0, W_up's at +4, the token tile's at +8 (tokens 0..127) and +12
// (128..239).  One set serves the stage whose MMAs come next: a
// tcgen05.cp and the tcgen05.mma issued after it by the same thread run in
// issue order, so each stage's copies simply precede its MMAs.
constexpr uint32_t SF_TMEM_COL = 2 * FP8_BN;
static_assert(SF_TMEM_COL + 16 <= 512, "scale-factor columns exceed TMEM");

__device__ __forceinline__ void sf_to_tmem(uint32_t sf_t, uint32_t sf_smem, bool two_tok) {
  tmem_cp_atom(sf_t, smem_desc_atom(sf_smem));
  tmem_cp_atom(sf_t + 4, smem_desc_atom(sf_smem + SF_ATOM_BYTES));
  tmem_cp_atom(sf_t + 8, smem_desc_atom(sf_smem + 2 * SF_ATOM_BYTES));
  if (two_tok) tmem_cp_atom(sf_t + 12, smem_desc_atom(sf_smem + 3 * SF_ATOM_BYTES));
}

// One FP8 stage (128 contraction elements) of one A block: four K = 32
// block-scaled MMAs into accumulator d, the k-th taking byte k of the scale
// words at sfa_t (the A block's rows) and sfb_t (the tokens).
__device__ __forceinline__ void mma_kstep_fp8(uint32_t d, uint32_t a_smem, uint32_t b_smem,
                                              uint32_t nmma, uint32_t sfa_t, uint32_t sfb_t,
                                              bool first) {
  const uint64_t ad = smem_desc_sw128(a_smem);
  const uint64_t bd = smem_desc_sw128(b_smem);
#pragma unroll
  for (uint32_t kb = 0; kb < FP8_BK / 32; ++kb)
    umma_mxf8(d, ad + 2 * kb, bd + 2 * kb, idesc_mxf8(GEMM_BM, nmma, kb, kb), sfa_t, sfb_t,
              (first && kb == 0) ? 0u : 1u);
}

// The epilogue chunks of warp group `group` (0..2) in its lane quadrant:
// columns group * 32 + j * 96 (j = 0..2) below nmma, 32 wide (16 for a
// ragged last chunk).
//
// Reads this warp's chunks of the accumulator at tacc (for gate/up also the
// up accumulator acc1 columns on), applies the epilogue math and rounds to
// bf16: hp[j][i] holds tokens 2i and 2i+1 of chunk j.
template <int MODE>
__device__ __forceinline__ void epi_read_bf16(uint32_t tacc, int group, int nmma,
                                              uint32_t (&hp)[3][16], uint32_t acc1 = 256) {
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int c0 = group * 32 + j * 32 * GEMM_EPI_GROUPS;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cc = c0 + 16 * hh;
      if (cc < nmma) {
        uint32_t r0[16], r1[16];
        tmem_ld16(tacc + cc, r0);
        if (MODE == MODE_GATEUP) tmem_ld16(tacc + acc1 + cc, r1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float g = __uint_as_float(r0[2 * i + h]);
            if (MODE == MODE_GATEUP) {
              const float u = __uint_as_float(r1[2 * i + h]);
              // SiLU(g) * u; the exponent is clamped so 1 + e^-g stays finite
              v[h] = __fdividef(g, 1.0f + __expf(-fmaxf(g, -80.0f))) * u;
            } else {
              v[h] = g;
            }
          }
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[0], v[1]);
          hp[j][8 * hh + i] = *reinterpret_cast<const uint32_t*>(&b2);
        }
      }
    }
  }
}

// Stores the chunks epi_read_bf16 produced: token rows of the tile's slots,
// 32 bf16 columns each from out (already offset to this warp's features).
__device__ __forceinline__ void epi_store_bf16(uint8_t* stg, int lane, int group, const Tile& tl,
                                               const uint32_t (&hp)[3][16], __nv_bfloat16* out,
                                               int64_t ld, uint64_t pol) {
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int c0 = group * 32 + j * 32 * GEMM_EPI_GROUPS;
    if (c0 < tl.nmma) {
      const int ncol = c0 + 32 <= tl.nmma ? 32 : 16;
      const int tok_base = tl.tok0 + c0;
      const int rows = min(ncol, tl.count - tok_base);
      const int64_t row0 = tl.brow0 - tl.tok0 + tok_base;   // first output row
      stage_store_bf16x2(stg, lane, hp[j], ncol, rows, out + row0 * ld, ld, pol);
    }
  }
}

// Router logits (fp32) of one accumulator: weight rows ebase + 0..31 of this
// warp's quadrant, chunk by chunk straight from TMEM to global memory.
__device__ __forceinline__ void epi_router_f32(uint32_t tacc, uint8_t* stg, int lane, int group,
                                               const Tile& tl, const GemmParams& p, int ebase) {
  float* out = static_cast<float*>(p.out) + tl.split * p.split_stride;
  for (int c0 = group * 32; c0 < tl.nmma; c0 += 32 * GEMM_EPI_GROUPS) {
    const bool wide = c0 + 32 <= tl.nmma;
    uint32_t r[32];
    tmem_ld16(tacc + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
    if (wide) tmem_ld16(tacc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
    tmem_ld_wait();
    const int ncol = wide ? 32 : 16;
    const int tok_base = tl.tok0 + c0;
    const int rows = min(ncol, tl.count - tok_base);
    stage_store_f32(stg, lane, r, ncol, rows, out, tok_base, p.out_ld, ebase, p.a_rows);
  }
}

// NST stages of SB bytes: two A blocks (2 * GEMM_A_BYTES), then the B rows
// (up to (SB - 2 * GEMM_A_BYTES) / 128 tokens).  The prefill shape has 3
// stages of 64 KB (256 tokens); batches of at most 64 tokens have 5 stages of
// 40 KB, so that more weight bytes are in flight per SM while they stream.
//
// MODE_FUSED runs the gate/up tiles (maps tmA0, tmA1, tmB; parameters p) and
// then the down tiles (maps tmA2 for both A blocks, tmB2; parameters p2) of
// one forward in one grid, so that the SMs left idle in the last, part-filled
// round of gate/up tiles already stream down weights.  A down tile of group g
// reads H rows that other CTAs write: its producer waits (bounded) until all
// GEMM_EPI_WARPS * mblocks * ntt epilogue warps of g's gate/up tiles have
// counted themselves in p.done[g].  No wait can close a cycle: gate/up tiles
// wait on nothing outside their CTA, a CTA has issued all loads of its
// earlier tiles before it waits for a down tile's group, the counter hands
// out every gate/up tile before any down tile, and the grid (one CTA per SM,
// at most one per SM of the device) is resident as a whole.
template <int MODE, int NST, int SB, bool FP8>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
            const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBf,
            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
            const GemmParams p, const GemmParams p2, const __grid_constant__ StepParams sp) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[NST];
  __shared__ __align__(8) uint64_t empty_bar[NST];
  // Accumulator hand-over.  One-block tiles: [b] = buffer b (TMEM columns
  // 256 b ..).  Two-block tiles: [0] / [1] = first / second accumulator.
  __shared__ __align__(8) uint64_t acc_full_bar[2];
  __shared__ __align__(8) uint64_t acc_empty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ uint32_t peer_tile_sh;   // p.pair_tiles: paced tiles the partner CTA has begun
  // Tiles taken from p.tile_counter: the producer takes each and hands it to
  // the MMA issuer and the epilogue warps through this queue (-1: no more).
  __shared__ volatile int tile_q[TILE_Q];
  __shared__ __align__(8) uint64_t tq_full[TILE_Q];
  __shared__ __align__(8) uint64_t tq_empty[TILE_Q];
  __shared__ volatile int bar_ok_sh;   // grid barriers of the decode step
  const bool dyn = MODE == MODE_FUSED ||
                   ((MODE == MODE_GATEUP || MODE == MODE_DOWN) && p.tile_counter != nullptr &&
                    !p.pair_tiles);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1024-byte aligned (128-byte swizzle atoms); an offset from smem_raw, so
  // that the compiler keeps every access through it in the shared state space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full_bar[b], 1);
      mbar_init(&acc_empty_bar[b], GEMM_EPI_THREADS);
    }
    mbar_init(&drain_bar, 1);
    for (int i = 0; i < TILE_Q; ++i) {
      mbar_init(&tq_full[i], 1);
      mbar_init(&tq_empty[i], 1 + GEMM_EPI_WARPS);
    }
    abort_sh = 0;
    peer_tile_sh = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBf);
    if (MODE == MODE_FUSED) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  __syncwarp();
  if (warp == 2) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (p.pair_tiles) cluster_sync_all();   // the partner's pacing word exists before any store
  tc_fence_after();
  // the prologue above overlaps the previous kernel; from here on its
  // results (routing, offsets, activations) are read
  griddep_wait();
  griddep_launch_dependents();
  if (MODE == MODE_ROUTER && blockIdx.x == 0) {
    // this forward's expert-load histogram and slot counters start at zero
    // (the previous forward's readers are done: griddep_wait)
    for (int i = threadIdx.x; i < p.nzero0; i += blockDim.x) p.zero0[i] = 0;
    for (int i = threadIdx.x; i < p.nzero1; i += blockDim.x) p.zero1[i] = 0;
  }
  // The whole decode step (sp.on): route, then assign and permute, each
  // followed by a grid barrier, before the expert tiles; the combine after
  // them.  Every block passes every barrier (a wait that runs out records
  // DEV_TIMEOUT), but the work after a failed one is skipped.
  uint8_t* ws = smem + NST * SB;   // the epilogue staging area
  bool step_ok = true;
  int nbar = 0;
  if (MODE == MODE_FUSED && sp.on) {
    const int G = static_cast<int>(gridDim.x);
    step_route<GEMM_THREADS>(sp, ws);
    step_ok = grid_barrier(sp.gbar, ++nbar * G, p.wait_ns, p.err, &bar_ok_sh, step_ok);
    if (step_ok) {
      // (bf16 only: measured -2 us at decode; FP8 tiles +1 us with it)
      const TilePrefetch pf{&tmA0, &tmA1, p.mblocks, p.a_rows, FP8 ? FP8_BK : GEMM_BK,
                            FP8 ? 0 : (p.ksteps < NST ? p.ksteps : NST)};
      step_assign_permute<GEMM_THREADS, FP8>(sp, ws, pf);
    }
    step_ok = grid_barrier(sp.gbar, ++nbar * G, p.wait_ns, p.err, &bar_ok_sh, step_ok);
    if (!step_ok && threadIdx.x == 0) abort_sh = 1;
    __syncthreads();
  }
  const uint32_t tmem = tmem_base_sh;
  const int ntiles = total_tiles<MODE == MODE_FUSED ? MODE_GATEUP : MODE, MODE == MODE_FUSED>(p);
  const int ntiles2 = MODE == MODE_FUSED ? total_tiles<MODE_DOWN, true>(p2) : 0;
  const int ndyn = ntiles + ntiles2;   // tiles the counter hands out
  // gate/up tiles always hold two blocks; router and down tiles hold one
  // when p.single_a is set (1 buffer of 512 columns, or 2 of 256)
  // (MODE_FUSED: both phases hold two blocks)
  const int nbuf = (MODE == MODE_GATEUP || MODE == MODE_FUSED || !p.single_a) ? 1 : 2;

  // Single-thread roles run on lane 0; the other lanes of their warp wait at
  // a __syncwarp so that every warp reaches the final CTA barrier converged.
  if (warp == 0) {
   if (lane == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0;          // stages armed at least once
    uint32_t last_par = 0;       // parity each stage was last armed with
    const uint64_t pol_stream = l2_policy_evict_first();
    // p.pair_tiles: the grid runs as 2-CTA clusters (the two SMs of a TPC),
    // CTA rank r of a cluster taking tiles t with t % 2 == r.  When tiles t
    // and t ^ 1 are the two token tiles of one weight block of an expert with
    // two token tiles (the common case when experts get a few hundred tokens
    // each), the CTAs start them together, so the weight bytes one of them
    // loads from DRAM are an L2 hit for the other: each stores into the
    // partner's shared memory how many such tiles it has begun and waits
    // until the partner has begun the same one -- for at most PACE_NS, after
    // which it goes on alone (pacing is only a hint: it never holds up or
    // fails the GEMM).  Experts with many token tiles share weight blocks
    // across each round of the grid anyway and are not paced.
    const uint32_t peer_word =
        p.pair_tiles ? mapa_shared(smem_u32(&peer_tile_sh), cluster_ctarank() ^ 1u) : 0u;
    uint32_t begun = 0;
    for (int it = 0; !abort_sh; ++it) {
      int tph, t;
      if (dyn) {
        // take the next tile of the grid and hand it to the other roles
        const int qs = it % TILE_Q;
        if (!mbar_wait(&tq_empty[qs], ((it / TILE_Q) & 1) ^ 1, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        const int u = atomicAdd(p.tile_counter, 1);
        tile_q[qs] = u < ndyn ? u : -1;
        mbar_arrive(&tq_full[qs]);
        if (u >= ndyn) break;
        dyn_tile<MODE>(u, ntiles, tph, t);
      } else if (!tile_at<MODE>(it, ntiles, tph, t)) {
        break;
      }
      const Tile tl = phase_tile<MODE>(p, p2, tph, t);
      const bool down_ph = MODE == MODE_FUSED && tph == 1;
      if (down_ph) {
        // group tl.g's H rows are all stored once every epilogue warp of its
        // gate/up tiles has counted itself; the acquire and the proxy fence
        // order this CTA's bulk copies of them after those stores
        const int need =
            GEMM_EPI_WARPS * p.mblocks *
            (ld_meta<true>(p.grp_ttp + tl.g + 1) - ld_meta<true>(p.grp_ttp + tl.g));
        if (!wait_count_geq(p.done + tl.g, need, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        fence_proxy_async_global();
      }
      const CUtensorMap* mA0 = down_ph ? &tmA2 : &tmA0;
      const CUtensorMap* mA1 = down_ph ? &tmA2 : &tmA1;
      const CUtensorMap* mB = down_ph ? &tmB2 : &tmB;
      // both CTAs evaluate the same predicate on the pair (t, t ^ 1)
      if (MODE != MODE_ROUTER && MODE != MODE_FUSED && p.pair_tiles && tl.ntt == 2 &&
          (t ^ 1) < ntiles &&
          group_of_tile(p, t ^ 1) == tl.g) {
        ++begun;
        st_cluster_u32(peer_word, begun);
        pace_until_shared(&peer_tile_sh, begun, PACE_NS);
      }
      // FP8 kernels run their gate/up tiles in FP8 (MODE_FUSED's down tiles
      // stay bf16): 128 contraction elements per stage instead of 64, in the
      // same 128-byte rows, plus the stage's scale atoms
      const bool f8 = FP8 && !down_ph;
      const int nbox = (tl.nmma + GEMM_B_BOX_ROWS - 1) / GEMM_B_BOX_ROWS;
      // a full token tile (the tile size: 256 tokens, 240 for FP8, the
      // router's own) in one copy of the b_full map, whose box has exactly
      // that many rows
      const int full_rows = router_tok_tile(p);
      const bool full_box = MODE != MODE_FUSED && p.b_box_full && tl.nmma == full_rows;
      const int sfb_atoms = tl.nmma > 128 ? 2 : 1;
      const uint32_t bytes = GEMM_A_BYTES * (tl.has_a1 ? 2 : 1) +
                             (full_box ? tl.nmma : nbox * GEMM_B_BOX_ROWS) * 128 +
                             (f8 ? (2 + sfb_atoms) * SF_ATOM_BYTES : 0);
      const int kstep = f8 ? FP8_BK : GEMM_BK;
      for (int ks = tl.k0; ks < tl.k1; ++ks) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        uint8_t* st = smem + stage * SB;
        mbar_arrive_expect_tx(&full_bar[stage], bytes);
        armed |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        const int kc = ks * kstep;
        // Streaming batches (decode) read every weight byte once: evict
        // first.  Prefill-sized batches keep the default policy (measured:
        // evict-last weights or evict-first tokens there cost ~4%).
        uint8_t* sb = st + 2 * GEMM_A_BYTES;
        if (p.l2_stream) {
          tma_load_2d_hint(st, mA0, &full_bar[stage], kc, tl.a0_row, pol_stream);
          if (tl.has_a1)
            tma_load_2d_hint(st + GEMM_A_BYTES, mA1, &full_bar[stage], kc, tl.a1_row, pol_stream);
          if (full_box) {
            tma_load_2d_hint(sb, &tmBf, &full_bar[stage], kc, tl.brow0, pol_stream);
          } else {
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d_hint(sb + bx * GEMM_B_BOX_ROWS * GEMM_BK * 2, mB, &full_bar[stage], kc,
                               tl.brow0 + bx * GEMM_B_BOX_ROWS, pol_stream);
          }
        } else {
          tma_load_2d(st, mA0, &full_bar[stage], kc, tl.a0_row);
          if (tl.has_a1) tma_load_2d(st + GEMM_A_BYTES, mA1, &full_bar[stage], kc, tl.a1_row);
          if (full_box) {
            tma_load_2d(sb, &tmBf, &full_bar[stage], kc, tl.brow0);
          } else {
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d(sb + bx * GEMM_B_BOX_ROWS * GEMM_BK * 2, mB, &full_bar[stage], kc,
                          tl.brow0 + bx * GEMM_B_BOX_ROWS);
          }
        }
        if (f8) {
          // scale atoms: W_gate's and W_up's 128 rows of this block, and the
          // token tile's one or two atoms, for these 4 blocks of 32
          uint8_t* sf = st + (SB - FP8_SF_STAGE_BYTES);
          const int64_t wa =
              (static_cast<int64_t>(tl.a0_row / GEMM_BM) * p.sf_kgroups + ks) * SF_ATOM_BYTES;
          bulk_load(sf, p.sfa0 + wa, SF_ATOM_BYTES, &full_bar[stage]);
          bulk_load(sf + SF_ATOM_BYTES, p.sfa1 + wa, SF_ATOM_BYTES, &full_bar[stage]);
          const int64_t tb =
              (static_cast<int64_t>(tl.ttile) * p.sf_kgroups + ks) * (2 * SF_ATOM_BYTES);
          bulk_load(sf + 2 * SF_ATOM_BYTES, p.sfb + tb, sfb_atoms * SF_ATOM_BYTES,
                    &full_bar[stage]);
        }
        if (++stage == NST) { stage = 0; phase ^= 1; }
      }
    }
    // Drain: every copy this thread started must land before the CTA exits.
    for (int s = 0; s < NST; ++s)
      if (armed & (1u << s)) mbar_wait(&full_bar[s], (last_par >> s) & 1, DRAIN_NS, p.err);
   }
   __syncwarp();
  } else if (warp == 1) {
   if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    for (int local = 0; !abort_sh; ++local) {
      int tph, t;
      if (dyn) {
        const int qs = local % TILE_Q;
        if (!mbar_wait(&tq_full[qs], (local / TILE_Q) & 1, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        const int u = tile_q[qs];
        mbar_arrive(&tq_empty[qs]);
        if (u < 0) break;
        dyn_tile<MODE>(u, ntiles, tph, t);
      } else if (!tile_at<MODE>(local, ntiles, tph, t)) {
        break;
      }
      const Tile tl = phase_tile<MODE>(p, p2, tph, t);
      const int buf = local % nbuf;
      const int use = local / nbuf;
      const uint32_t par = static_cast<uint32_t>(use - 1) & 1u;
      const uint32_t acc0 = tmem + buf * 256;
      if (use > 0 && !mbar_wait(&acc_empty_bar[buf], par, p.wait_ns, p.err)) {
        abort_sh = 1;
        break;
      }
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(GEMM_BM, tl.nmma);
      const int nk = tl.k1 - tl.k0;
      // FP8 gate/up tiles: block-scaled MMAs, the second accumulator FP8_BN
      // columns on (two FP8_BN-token accumulators and the scale columns fill
      // TMEM); bf16 tiles: 256 columns on
      const bool f8 = FP8 && !(MODE == MODE_FUSED && tph == 1);
      const uint32_t acc1 = acc0 + (f8 ? FP8_BN : 256);
      const uint32_t sf_t = tmem + SF_TMEM_COL;
      const bool two_tok = tl.nmma > 128;
      constexpr uint32_t SF_OFF = SB - FP8_SF_STAGE_BYTES;
      // first / second accumulator's k-step on the stage at st
      auto kstep0 = [&](uint32_t st, bool first) {
        if (f8) {
          sf_to_tmem(sf_t, st + SF_OFF, two_tok);
          mma_kstep_fp8(acc0, st, st + 2 * GEMM_A_BYTES, tl.nmma, sf_t, sf_t + 8, first);
        } else {
          mma_kstep(acc0, st, st + 2 * GEMM_A_BYTES, idesc, first);
        }
      };
      auto kstep1 = [&](uint32_t st, bool first, bool copy_sf) {
        if (f8) {
          if (copy_sf) sf_to_tmem(sf_t, st + SF_OFF, two_tok);
          mma_kstep_fp8(acc1, st + GEMM_A_BYTES, st + 2 * GEMM_A_BYTES, tl.nmma, sf_t + 4,
                        sf_t + 8, first);
        } else {
          mma_kstep(acc1, st + GEMM_A_BYTES, st + 2 * GEMM_A_BYTES, idesc, first);
        }
      };
      // Two-block tile after the first: the first npre loaded stages feed the
      // first accumulator alone; they are freed once the second accumulator
      // is back and has had its MMAs on them too (FP8: with their scale
      // atoms copied into TMEM again).
      const bool stagger = nbuf == 1 && use > 0;
      const int npre = stagger ? min(nk, NST) : 0;
      bool ok = true;
      const int stage0 = stage;
      for (int i = 0; i < npre; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, p.wait_ns, p.err)) { ok = false; break; }
        tc_fence_after();
        kstep0(smem_u32(smem + stage * SB), i == 0);
        if (++stage == NST) { stage = 0; phase ^= 1; }
      }
      if (ok && stagger) {
        if (!mbar_wait(&acc_empty_bar[1], par, p.wait_ns, p.err)) {
          ok = false;
        } else {
          tc_fence_after();
          int s = stage0;
          for (int i = 0; i < npre; ++i) {
            if (tl.has_a1) kstep1(smem_u32(smem + s * SB), i == 0, true);
            umma_commit(&empty_bar[s]);
            if (++s == NST) s = 0;
          }
        }
      }
      for (int i = npre; ok && i < nk; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, p.wait_ns, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + stage * SB);
        kstep0(st, i == 0);
        if (tl.has_a1) kstep1(st, i == 0, false);
        umma_commit(&empty_bar[stage]);
        if (++stage == NST) { stage = 0; phase ^= 1; }
      }
      if (!ok) { abort_sh = 1; break; }
      umma_commit(&acc_full_bar[buf]);
    }
    // Drain: all MMAs issued by this thread finish before TMEM is freed.
    umma_commit(&drain_bar);
    mbar_wait(&drain_bar, 0, DRAIN_NS, p.err);
   }
   __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // Twelve warps: warp w drains TMEM lanes (w % 4) * 32 .. +31 (the quadrant
    // its warp id may access) and every third 32-column chunk of the tile
    // (group = 0, 1 or 2), leaving through a per-warp staging tile in shared
    // memory as 16-byte coalesced stores of 64-byte (bf16) or 128-byte
    // (fp32) row pieces.
    const int q = warp & 3;
    const int group = (warp - 4) >> 2;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint8_t* stg = smem + NST * SB + (warp - 4) * GEMM_STG_BYTES;
    // H / Y rows are written once here; hint them only for streaming batches
    // whose next reader is another kernel (the one grid reads H back, and
    // the combine reads Y right after it: default policy)
    const uint64_t pol_out = p.l2_stream && MODE != MODE_FUSED ? l2_policy_evict_first() : 0;
    for (int local = 0; !abort_sh; ++local) {
      int tph, t;
      if (dyn) {
        const int qs = local % TILE_Q;
        if (!mbar_wait(&tq_full[qs], (local / TILE_Q) & 1, p.wait_ns, p.err)) {
          abort_sh = 1;
          break;
        }
        const int u = tile_q[qs];
        __syncwarp();
        if (lane == 0) mbar_arrive(&tq_empty[qs]);
        if (u < 0) break;
        dyn_tile<MODE>(u, ntiles, tph, t);
      } else if (!tile_at<MODE>(local, ntiles, tph, t)) {
        break;
      }
      const Tile tl = phase_tile<MODE>(p, p2, tph, t);
      const int buf = local % nbuf;
      if (!mbar_wait(&acc_full_bar[buf], (local / nbuf) & 1, p.wait_ns, p.err)) {
        abort_sh = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tq + buf * 256;
      const bool down_ph = MODE == MODE_FUSED && tph == 1;
      // router / down: this warp's first weight row of A block 0
      const int row_blk = tl.r0 + q * 32;
      if (MODE == MODE_ROUTER) {
        epi_router_f32(tacc, stg, lane, group, tl, p, row_blk);
        tc_fence_before();
        mbar_arrive(&acc_empty_bar[buf]);
        if (nbuf == 1) {
          if (tl.has_a1) epi_router_f32(tacc + 256, stg, lane, group, tl, p, row_blk + GEMM_BM);
          tc_fence_before();
          mbar_arrive(&acc_empty_bar[1]);
        }
      } else if (MODE == MODE_GATEUP || (MODE == MODE_FUSED && !down_ph)) {
        uint32_t hp[3][16];
        epi_read_bf16<MODE_GATEUP>(tacc, group, tl.nmma, hp, FP8 ? FP8_BN : 256);
        tc_fence_before();
        mbar_arrive(&acc_empty_bar[0]);
        mbar_arrive(&acc_empty_bar[1]);
        // (MODE_FUSED reads H back in this grid: default L2 policy)
        epi_store_bf16(stg, lane, group, tl, hp,
                       static_cast<__nv_bfloat16*>(p.out) + tl.m * GEMM_BM + q * 32, p.out_ld,
                       MODE == MODE_FUSED ? 0 : pol_out);
        if (MODE == MODE_FUSED) {
          // publish this warp's H rows of the tile to the down tiles of
          // tl.g: each lane's stores are made visible (also to bulk copies)
          // before lane 0 counts the warp in
          fence_proxy_async_global();
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.done + tl.g, 1);
        }
      } else {
        __nv_bfloat16* out =
            static_cast<__nv_bfloat16*>(MODE == MODE_FUSED ? p2.out : p.out) + row_blk;
        const int64_t out_ld = MODE == MODE_FUSED ? p2.out_ld : p.out_ld;
        // d % 128 == 64: the last weight block's upper 64 rows lie past d
        // (their accumulator lanes hold no output feature and are not stored)
        const int a_rows = MODE == MODE_FUSED ? p2.a_rows : p.a_rows;
        uint32_t hp[3][16];
        epi_read_bf16<MODE_DOWN>(tacc, group, tl.nmma, hp);
        tc_fence_before();
        mbar_arrive(&acc_empty_bar[buf]);
        if (row_blk < a_rows) epi_store_bf16(stg, lane, group, tl, hp, out, out_ld, pol_out);
        if (nbuf == 1) {
          if (tl.has_a1) epi_read_bf16<MODE_DOWN>(tacc + 256, group, tl.nmma, hp);
          tc_fence_before();
          mbar_arrive(&acc_empty_bar[1]);
          if (tl.has_a1 && row_blk + GEMM_BM < a_rows)
            epi_store_bf16(stg, lane, group, tl, hp, out + GEMM_BM, out_ld, pol_out);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while its partner may still store into its shared memory
  if (p.pair_tiles) cluster_sync_all();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (MODE == MODE_FUSED && sp.on) {
    // every Y row is stored once all blocks are here (the combine reads
    // them with plain loads: no proxy fence)
    step_ok = grid_barrier<false>(sp.gbar, ++nbar * static_cast<int>(gridDim.x), p.wait_ns,
                                  p.err, &bar_ok_sh, step_ok && !abort_sh);
    if (step_ok) step_combine<GEMM_THREADS>(sp, ws);
  }
}

// a2, b2, p2: MODE_FUSED's down phase (other modes: copies of a0, b, p).
// sp: the decode step's phases (MODE_FUSED; off elsewhere).
template <int MODE, int NST, int SB, bool FP8 = false>
cudaError_t launch_mode(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                        const CUtensorMap& b_full, const CUtensorMap& a2, const CUtensorMap& b2,
                        GemmParams p, const GemmParams& p2, int grid, cudaStream_t stream,
                        const StepParams& sp = StepParams{}) {
  constexpr int smem = NST * SB + GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024;
  const cudaError_t e = smem_limit<gemm_kernel<MODE, NST, SB, FP8>>(smem);
  if (e != cudaSuccess) return e;
  // pacing runs the grid as 2-CTA clusters: an even grid of at least two
  if (p.pair_tiles) {
    if (grid >= 2) {
      return launch_pdl_pairs(gemm_kernel<MODE, NST, SB, FP8>, dim3(grid & ~1),
                              dim3(GEMM_THREADS), smem, stream, a0, a1, b, b_full, a2, b2, p, p2,
                              StepParams{});
    }
    p.pair_tiles = 0;
  }
  // a down tile of the one grid may wait for any other block's gate/up
  // tiles: every block must be resident at once
  if (MODE == MODE_FUSED)
    return launch_pdl_coop(gemm_kernel<MODE, NST, SB, FP8>, dim3(grid), dim3(GEMM_THREADS), smem,
                           stream, a0, a1, b, b_full, a2, b2, p, p2, sp);
  return launch_pdl(gemm_kernel<MODE, NST, SB, FP8>, dim3(grid), dim3(GEMM_THREADS), smem, stream,
                    a0, a1, b, b_full, a2, b2, p, p2, StepParams{});
}

// The stage shapes: prefill (3 x 64 KB) and at most 64 tokens (5 x 40 KB).
template <int MODE>
cudaError_t launch_shape(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                         const CUtensorMap& b_full, const GemmParams& p, int grid,
                         cudaStream_t stream) {
  if (p.small_b)
    return launch_mode<MODE, GEMM_SMALL_STAGES, GEMM_SMALL_STAGE_BYTES>(a0, a1, b, b_full, a0, b, p,
                                                                         p, grid, stream);
  return launch_mode<MODE, GEMM_STAGES, GEMM_STAGE_BYTES>(a0, a1, b, b_full, a0, b, p, p, grid,
                                                          stream);
}

}  // namespace

cudaError_t launch_gemm(GemmMode mode, const CUtensorMap& a0, const CUtensorMap& a1,
                        const CUtensorMap& b, const CUtensorMap& b_full, const GemmParams& p,
                        int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  switch (mode) {
    case MODE_ROUTER: {
      GemmParams q = p;
      q.pair_tiles = 0;
      e = launch_shape<MODE_ROUTER>(a0, a1, b, b_full, q, grid, stream);
      break;
    }
    case MODE_GATEUP:
      e = launch_shape<MODE_GATEUP>(a0, a1, b, b_full, p, grid, stream);
      break;
    case MODE_DOWN:
      e = launch_shape<MODE_DOWN>(a0, a1, b, b_full, p, grid, stream);
      break;
    case MODE_FUSED:   // two phases: launch_gemm_fused
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// A decode step (step.on) wants the barrier counter, sizes the phases can
// hold in the staging area (N + Z <= MOE_MAX_E_INTERNAL, K <= 32) and its
// output buffers.
static bool step_args_ok(const StepParams& s, const GemmParams& pg, bool fp8) {
  if (!s.on) return true;
  return s.gbar && s.T > 0 && s.T <= GEMM_SMALL_B && s.E <= MOE_MAX_E_INTERNAL && s.N > 0 &&
         s.N <= s.E && s.K > 0 && s.K <= 32 && s.splits >= 1 && s.logits && s.bias && s.idx &&
         s.gate && s.zsum && s.cnt == pg.grp_count && s.slot && s.fill && s.grp_off == pg.grp_off &&
         s.grp_ttp && s.x && s.Y && s.out && (fp8 ? (s.Xp8 && s.sfx && s.grp_ttp8) : s.Xp != nullptr);
}

cudaError_t launch_gemm_fused(const CUtensorMap& wg, const CUtensorMap& wu, const CUtensorMap& xp,
                              const CUtensorMap& wd, const CUtensorMap& h, const GemmParams& pg,
                              const GemmParams& pd, int grid, cudaStream_t stream,
                              const StepParams& step) {
  if (grid <= 0) return cudaSuccess;
  if (grid > device_sms() || !pg.small_b || pg.pair_tiles || pg.b_box_full || pd.single_a ||
      pg.done == nullptr || pg.tile_counter == nullptr || !step_args_ok(step, pg, false))
    return cudaErrorInvalidValue;
  // (a refused cooperative launch leaves nothing queued: launch_mode's error
  // is returned as is, without cudaGetLastError, for the caller to clear)
  return launch_mode<MODE_FUSED, GEMM_SMALL_STAGES, GEMM_SMALL_STAGE_BYTES>(
      wg, wu, xp, xp, wd, h, pg, pd, grid, stream, step);
}

int fused_resident_blocks() {
  constexpr int smem = GEMM_SMALL_STAGES * GEMM_SMALL_STAGE_BYTES +
                       GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024;
  if (smem_limit<gemm_kernel<MODE_FUSED, GEMM_SMALL_STAGES, GEMM_SMALL_STAGE_BYTES, false>>(
          smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return blocks_per_sm<gemm_kernel<MODE_FUSED, GEMM_SMALL_STAGES, GEMM_SMALL_STAGE_BYTES, false>>(
             GEMM_THREADS, smem) *
         device_sms();
}

cudaError_t launch_gemm_gateup_fp8(const CUtensorMap& wg, const CUtensorMap& wu,
                                   const CUtensorMap& xp8, const CUtensorMap& xp8_full,
                                   const GemmParams& p, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  if (p.tok_tile != FP8_BN || !p.sfa0 || !p.sfa1 || !p.sfb || p.sf_kgroups != p.ksteps)
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (p.small_b)
    e = launch_mode<MODE_GATEUP, FP8_SMALL_STAGES, FP8_SMALL_STAGE_BYTES, true>(
        wg, wu, xp8, xp8_full, wg, xp8, p, p, grid, stream);
  else
    e = launch_mode<MODE_GATEUP, GEMM_STAGES, FP8_STAGE_BYTES, true>(wg, wu, xp8, xp8_full, wg,
                                                                      xp8, p, p, grid, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_fused_fp8(const CUtensorMap& wg, const CUtensorMap& wu,
                                  const CUtensorMap& xp8, const CUtensorMap& wd,
                                  const CUtensorMap& h, const GemmParams& pg,
                                  const GemmParams& pd, int grid, cudaStream_t stream,
                                  const StepParams& step) {
  if (grid <= 0) return cudaSuccess;
  if (grid > device_sms() || !pg.small_b || pg.pair_tiles || pg.b_box_full || pd.single_a ||
      pg.done == nullptr || pg.tile_counter == nullptr || pg.tok_tile != FP8_BN || !pg.sfa0 ||
      !pg.sfa1 || !pg.sfb || pg.sf_kgroups != pg.ksteps || !step_args_ok(step, pg, true))
    return cudaErrorInvalidValue;
  return launch_mode<MODE_FUSED, FP8_SMALL_STAGES, FP8_SMALL_STAGE_BYTES, true>(
      wg, wu, xp8, xp8, wd, h, pg, pd, grid, stream, step);
}

}  // namespace moezc
