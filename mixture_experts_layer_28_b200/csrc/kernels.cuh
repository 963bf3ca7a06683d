// kernels.cuh -- launchers of the five hot-path kernels (internal C++ API).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace moezc {

constexpr int MOE_MAX_K_INTERNAL = 32;   // most picks per token
constexpr int MOE_MAX_E_INTERNAL = 1024; // most experts (FFN + zero)

// Launch with programmatic stream serialisation (the kernel overlaps its
// predecessor's tail and orders itself with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// launch_pdl as a cooperative launch: the driver makes every block of the
// grid resident at once, or refuses the launch (cudaErrorCooperativeLaunchTooLarge).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once: later calls only read a per-device cache, so a forward makes
// no attribute calls after its first (e.g. while a caller captures it into a
// CUDA graph).
template <auto Kernel>
inline cudaError_t smem_limit(int bytes) {
  static int done[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = bytes;
  return e;
}

// Resident blocks per SM of a kernel at (threads, smem), cached per device
// for the last smem asked.
template <auto Kernel>
inline int blocks_per_sm(int threads, size_t smem) {
  static int cached[64] = {0};
  static size_t cached_smem[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  if (dev >= 0 && cached[dev] > 0 && cached_smem[dev] == smem) return cached[dev];
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  if (dev >= 0) {
    cached[dev] = n;
    cached_smem[dev] = smem;
  }
  return n;
}

// Launch with programmatic dependent launch (as launch_pdl) as clusters of
// two CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Multiprocessors of the current device (cached).
inline int device_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// The wait bound that moe_zc_test_inject set for the next call (0: none), and
// clear it; the forward and the no-allocation routing call take it.
long long take_injected_wait_ns();

// ------------------------------------------------------------------ GEMM
// One tcgen05 engine serves the three contractions of the layer.  Weights are
// the A operand (M = 128 rows per MMA, two A blocks per tile -> two fp32
// accumulators in TMEM); tokens are the B operand (N = 16..256 per tile).
// MODE_FUSED: the gate/up and down GEMMs of batches of at most GEMM_SMALL_B
// tokens in one persistent grid (launch_gemm_fused).
enum GemmMode : int { MODE_ROUTER = 0, MODE_GATEUP = 1, MODE_DOWN = 2, MODE_FUSED = 3 };

constexpr int GEMM_BM = 128;           // rows of one A block
constexpr int GEMM_BN = 256;           // tokens per tile at most
constexpr int GEMM_BK = 64;            // K per pipeline stage (128-byte rows)
constexpr int GEMM_STAGES = 3;
constexpr int GEMM_B_BOX_ROWS = 32;    // tokens per TMA box of B
constexpr int GEMM_EPI_GROUPS = 3;          // epilogue warps per TMEM lane quadrant
constexpr int GEMM_EPI_WARPS = 4 * GEMM_EPI_GROUPS;
constexpr int GEMM_EPI_THREADS = GEMM_EPI_WARPS * 32;
constexpr int GEMM_THREADS = 128 + GEMM_EPI_THREADS;
constexpr int GEMM_STG_BYTES = 32 * 32 * 2;  // per epilogue warp: 32 tokens x 32 bf16 (or 16 x 32 fp32)
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;
constexpr int GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;
constexpr int GEMM_STAGE_BYTES = 2 * GEMM_A_BYTES + GEMM_B_BYTES;
constexpr int GEMM_SMEM_BYTES =
    GEMM_STAGES * GEMM_STAGE_BYTES + GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024;
// Stage shape for batches of at most GEMM_SMALL_B tokens (decode): B rows
// need 8 KB, so five 40 KB stages keep twice the weight bytes in flight.
constexpr int GEMM_SMALL_B = 64;
constexpr int GEMM_SMALL_STAGES = 5;
constexpr int GEMM_SMALL_STAGE_BYTES = 2 * GEMM_A_BYTES + GEMM_SMALL_B * GEMM_BK * 2;
static_assert(GEMM_SMALL_STAGES * GEMM_SMALL_STAGE_BYTES + GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024 <=
                  227 * 1024 - 256,
              "small-batch stages exceed shared memory");

struct GemmParams {
  // Token groups (FFN experts).  For MODE_ROUTER there is one group of T
  // tokens starting at row 0 and the arrays are unused.
  const int* grp_count;   // [G] tokens in group g
  const int* grp_off;     // [G] first B row of group g (multiple of 16)
  const int* grp_ttp;     // [G+1] prefix sum of token tiles per group
  int G;
  int T;                  // MODE_ROUTER: tokens
  int ksteps;             // contraction length / GEMM_BK
  int ksplit;             // MODE_ROUTER: K split into this many slices (0 or 1: none);
                          // slice s writes its partial sums to out + s * split_stride
  long long split_stride;
  int single_a;           // MODE_ROUTER/MODE_DOWN: 1 = one 128-row A block per tile (no pair)
  int l2_stream;          // 1: weight and token tiles loaded, and outputs stored, with an
                          // L2 evict-first policy (decode: every weight byte is read once)
  int b_box_full;         // 1: a full token tile's B rows come in one GEMM_BN-row copy
  int tok_tile;           // MODE_ROUTER: tokens per tile (multiple of 16, <= GEMM_BN; 0: GEMM_BN)
  int pair_tiles;         // gate/up, down: 2-CTA clusters pace tiles t, t ^ 1 (even grid)
  int small_b;            // every token tile has at most GEMM_SMALL_B tokens: small-B stages
  int* zero0;             // MODE_ROUTER: CTA 0 clears zero0[0, nzero0) and zero1[0, nzero1)
  int* zero1;             //   once the previous kernel is done (the next forward's counters)
  int nzero0, nzero1;
  int mblocks;            // tiles along the weight rows of one group
  int a_rows;             // weight rows per group: E (router), I (gate/up), d (down)
  void* out;              // fp32 logits [T, E] | bf16 H [rows, I] | bf16 Y [rows, d]
  int out_ld;             // elements per output row
  int* err;               // device error flag
  long long wait_ns;      // bound of every pipeline wait
  // MODE_FUSED (set in the gate/up parameters): done[g] counts the epilogue
  // warps that have stored their part of a gate/up tile of group g (zeroed
  // before the launch); a down tile of group g starts once all of them have.
  int* done;
  // FP8 gate/up (block-scaled E4M3, FP8_BK contraction elements per stage):
  // the UE8M0 scale atoms of W_gate and W_up (rows of the weight matrices,
  // sf_atom_offset with kgroups = sf_kgroups) and of the token tiles (sfb:
  // two atoms per tile and contraction group, as launch_permute_fp8 writes).
  const uint8_t* sfa0;
  const uint8_t* sfa1;
  const uint8_t* sfb;
  int sf_kgroups;         // contraction length / FP8_BK
  // Gate/up and down launches without tile pacing: CTAs take tiles in order
  // from this counter (zero before the launch) instead of every G-th tile,
  // so the tiles running at any moment are neighbours in tile order (those
  // sharing a weight block or token tile overlap in time, and their reads
  // hit L2) and no CTA is left with a longer share; nullptr: fixed shares.
  int* tile_counter;
};

// The rest of a forward of at most GEMM_SMALL_B tokens, run by the one-grid
// expert GEMMs (launch_gemm_fused with step.on) around their tiles, as
// phases separated by grid barriers (the grid is resident as a whole):
//   route    the router's K slices summed and each token routed (softmax,
//            biased top-K, gates, zsum, histogram), as launch_route does
//   assign   expert offsets from the histogram (grp_off, grp_ttp and, for
//            FP8, grp_ttp8 stored for the tiles), a slot for each FFN pick
//            and the token copied into its slots (bf16 rows, or FP8 codes
//            and scale atoms), as launch_assign_slots and launch_permute(_fp8)
//   experts  the gate/up and down tiles
//   combine  out_t = zsum_t x_t + sum_k gate_{t,k} Y[slot_{t,k}], as launch_combine
// The histogram, fill counters and *gbar are zero at launch.
struct StepParams {
  int on;
  int T, E, N, K, d;
  const float* logits;       // [splits][T, E] partial router logits
  int splits;
  const float* bias;         // [E]
  const float* offset;       // [E] or null
  int* idx;                  // [T, K] out
  float* gate;               // [T, K] out
  float* zsum;               // [T] out
  int* cnt;                  // [E] histogram out
  int* slot;                 // [T, K] out
  int* fill;                 // [N] slot counters
  int* grp_off;              // [N + 1] out
  int* grp_ttp;              // [N + 1] out (GEMM_BN-token tiles)
  int* grp_ttp8;             // [N + 1] out (FP8_BN-token tiles), FP8 only
  const __nv_bfloat16* x;    // [T, d]
  __nv_bfloat16* Xp;         // bf16 permuted rows, or
  uint8_t* Xp8;              // FP8 codes and
  uint8_t* sfx;              //   scale atoms of the token tiles
  const __nv_bfloat16* Y;    // [rows, d] the down tiles' output
  __nv_bfloat16* out;        // [T, d]
  int* gbar;                 // grid barrier counter
};

// b: B map with GEMM_B_BOX_ROWS-row boxes; b_full: with GEMM_BN-row boxes,
// used for full token tiles when p.b_box_full is set.  With p.pair_tiles the
// grid (rounded down to even) runs as 2-CTA clusters.
cudaError_t launch_gemm(GemmMode mode, const CUtensorMap& a0, const CUtensorMap& a1,
                        const CUtensorMap& b, const CUtensorMap& b_full, const GemmParams& p,
                        int grid, cudaStream_t stream);

// Gate/up then down in one persistent grid of `grid` CTAs (batches of at most
// GEMM_SMALL_B tokens): wg, wu, xp as for the gate/up launch (parameters pg,
// with pg.done and pg.tile_counter set: the grid takes its tiles from the
// counter, zero at launch), wd and h as for the down launch (parameters pd).
// A cooperative launch: an error return (the grid cannot be resident at
// once) launches nothing, and the caller runs the two GEMMs as separate
// launches instead.
cudaError_t launch_gemm_fused(const CUtensorMap& wg, const CUtensorMap& wu, const CUtensorMap& xp,
                              const CUtensorMap& wd, const CUtensorMap& h, const GemmParams& pg,
                              const GemmParams& pd, int grid, cudaStream_t stream,
                              const StepParams& step);
// The FP8 gate/up GEMM (E4M3 maps of W_gate, W_up [N*I, d] with [128 x 128]
// boxes and of the quantised tokens Xp8 with [128 x 32] boxes, b_full with
// FP8_BN-row boxes; p.tok_tile = FP8_BN, p.grp_ttp the FP8_BN-tile prefix,
// p.ksteps = d / FP8_BK, scale atoms in p.sfa0 / p.sfa1 / p.sfb).
cudaError_t launch_gemm_gateup_fp8(const CUtensorMap& wg, const CUtensorMap& wu,
                                   const CUtensorMap& xp8, const CUtensorMap& xp8_full,
                                   const GemmParams& p, int grid, cudaStream_t stream);
// launch_gemm_fused with the gate/up phase in FP8 (maps and parameters as for
// launch_gemm_gateup_fp8); the down phase stays bf16.
cudaError_t launch_gemm_fused_fp8(const CUtensorMap& wg, const CUtensorMap& wu,
                                  const CUtensorMap& xp8, const CUtensorMap& wd,
                                  const CUtensorMap& h, const GemmParams& pg,
                                  const GemmParams& pd, int grid, cudaStream_t stream,
                                  const StepParams& step);
// Blocks of the one-grid expert GEMM kernel the current device holds at once
// (its occupancy times the multiprocessors).
int fused_resident_blocks();

// ------------------------------------------------------------------ FP8 gate/up
// Block-scaled FP8 (E4M3 elements, one power-of-two scale per 32 elements
// along the contraction, stored as a UE8M0 exponent byte: 2^(byte - 127)).
// The gate/up GEMM's scale factors reach the tensor cores through TMEM in
// 512-byte atoms: 128 rows x 4 consecutive 32-element blocks, the byte of row
// r and block k at (r % 32) * 16 + (r / 32) * 4 + k.
constexpr int FP8_BK = 128;            // contraction elements per pipeline stage (128-byte rows)
constexpr int FP8_BN = 240;            // tokens per gate/up tile (2 x 240 accumulator columns
                                       // + 16 scale-factor columns fill TMEM's 512)
constexpr int SF_ATOM_BYTES = 512;
constexpr int FP8_SF_STAGE_BYTES = 4 * SF_ATOM_BYTES;   // gate atom, up atom, two token atoms
constexpr int FP8_STAGE_BYTES = 2 * GEMM_A_BYTES + FP8_BN * FP8_BK + FP8_SF_STAGE_BYTES;
constexpr int FP8_SMALL_STAGES = 4;
constexpr int FP8_SMALL_STAGE_BYTES =
    ((2 * GEMM_A_BYTES + GEMM_SMALL_B * FP8_BK + 3 * SF_ATOM_BYTES) + 1023) & ~1023;
static_assert(3 * FP8_STAGE_BYTES + GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024 <= 227 * 1024,
              "FP8 stages exceed shared memory");
static_assert(FP8_SMALL_STAGES * FP8_SMALL_STAGE_BYTES + GEMM_EPI_WARPS * GEMM_STG_BYTES + 1024 <=
                  227 * 1024,
              "FP8 small-batch stages exceed shared memory");

// Tokens per token tile of an expert with `count` tokens cut into ntt tiles of
// at most tmax: the tiles share the tokens evenly (a multiple of 16 each),
// unless that would leave the last tile empty.
__host__ __device__ __forceinline__ int even_tile_size(int count, int ntt, int tmax) {
  if (ntt > 1) {
    const int even = (((count + ntt - 1) / ntt) + 15) & ~15;
    if (static_cast<long long>(ntt - 1) * even < count) return even;
  }
  return tmax;
}

// Byte offset, in a matrix's scale-factor atoms, of row r and contraction
// block kb (of 32 elements) when the matrix has kgroups = cols / 128 groups.
__host__ __device__ __forceinline__ int64_t sf_atom_offset(int64_t r, int kb, int kgroups) {
  return ((r / 128) * kgroups + kb / 4) * SF_ATOM_BYTES + (r % 32) * 16 + ((r % 128) / 32) * 4 +
         (kb % 4);
}

// W [rows, cols] bf16 (rows % 128 == 0, cols % 128 == 0) -> E4M3 codes
// [rows, cols] and UE8M0 scales in atoms (sf_atom_offset).
cudaError_t launch_fp8_quantize_weights(const __nv_bfloat16* W, int64_t rows, int cols,
                                        uint8_t* codes, uint8_t* sf, cudaStream_t stream);
// The FP8 permute: each token row is quantised once (E4M3 codes, 1 x 32
// blocks) and written to its FFN slots of Xp8; its scales go to the atoms of
// the gate/up token tiles holding those slots: tile j of expert g (FP8_BN
// token tiles, first tile grp_ttp8[g]) at sfx + (tile * d / 128 + kg) * 1024,
// the tile's token n as atom row n (two atoms: tokens 0..127, 128..239).
cudaError_t launch_permute_fp8(const __nv_bfloat16* x, const int* idx, const int* slot,
                               const int* cnt, const int* grp_off, const int* grp_ttp8, int64_t T,
                               int d, int K, int N, uint8_t* Xp8, uint8_t* sfx,
                               cudaStream_t stream);

// ------------------------------------------------------------------ router
// softmax over E logits (+offset), + bias, top-K, zero-gate sums, histogram.
// The logits may come as `splits` partial sums [splits][T][E], added in
// slice order.
cudaError_t launch_route(const float* logits, const float* b, const float* offset, int64_t T,
                         int E, int N, int K, int* idx, float* gate, float* zsum, int* cnt,
                         cudaStream_t stream, int splits = 1);

// ------------------------------------------------------------------ dispatch
// Slot assignment with the experts' row and tile offsets (grp_off, grp_ttp
// [N + 1], written by CTA 0) computed from the histogram cnt; fill [N] must
// be zero on entry (the router GEMM clears it).
// grp_ttp8 (optional, [N + 1]): the same prefix for FP8_BN-token tiles.
// pad: each expert's rows rounded up to a multiple of pad (16 for the GEMM
// buffers, 1 for packed rows); row_expert (optional): the expert of every
// assigned row.
cudaError_t launch_assign_slots(const int* cnt, const int* idx, int64_t pairs, int N,
                                int* grp_off, int* grp_ttp, int* fill, int* slot,
                                cudaStream_t stream, int* grp_ttp8 = nullptr, int pad = 16,
                                int* row_expert = nullptr);
// Routing given by the caller for R rows with one pick each (expert[i] -
// base; rows outside [0, N) are not dispatched): idx, gate 1, zsum 0 and
// the histogram cnt (zeroed by the caller).
cudaError_t launch_given_routing(const int* expert, int64_t R, int base, int N, int* idx,
                                 float* gate, float* zsum, int* cnt, cudaStream_t stream);
// total[j] += cnt[j] for j < E (histogram summed over the chunks of a forward)
cudaError_t launch_add_counts(const int* cnt, int E, int* total, cudaStream_t stream);
cudaError_t launch_permute(const __nv_bfloat16* x, const int* slot, int64_t T, int d, int K,
                           __nv_bfloat16* Xp, cudaStream_t stream);

// ------------------------------------------------------------------ combine
cudaError_t launch_combine(const __nv_bfloat16* x, const __nv_bfloat16* Y, const int* slot,
                           const float* gate, const float* zsum, int64_t T, int d, int K,
                           __nv_bfloat16* out, cudaStream_t stream);

}  // namespace moezc
