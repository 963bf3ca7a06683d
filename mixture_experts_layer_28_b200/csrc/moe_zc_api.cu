// moe_zc_api.cu -- the C ABI (include/moe_zc.h): argument checks, per-device
// workspace, TMA descriptors and the launch sequence of one forward.
//
// One forward of the MoE layer with zero-computation experts (LongCat-Flash
// write-up "Meituan's large model goes viral for its speed", section
// "Zero-computation experts") is, all on the caller's stream:
//
//   1  router GEMM        logits = x W_r^T              tcgen05, fp32 out
//                         (and clears this forward's histogram and counters)
//   2  route              softmax, + b, top-K, zsum, histogram
//   3  assign slots       per-expert row offsets and GEMM token tiles from
//                         the histogram; warp-aggregated atomics, FFN picks
//   4  permute            x rows -> Xp (grouped by expert)
//   5  gate/up GEMM       H = SiLU(Xp W_gate^T) * (Xp W_up^T)
//   6  down GEMM          Y = H W_down^T
//                         (batches of at most 64 tokens: 5 and 6 in one grid)
//   7  combine            out = zsum x + sum gate * Y
//
// No step reads anything back to the host: the GEMM tile lists are built on
// the device and walked by persistent kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/moe_zc.h"
#include "kernels.cuh"

namespace {

using namespace moezc;

constexpr int kMaxDevices = 16;
constexpr long long kWaitNs = 2000000000LL;  // 2 s bound of every pipeline wait

struct Buf {
  void* p = nullptr;
  size_t bytes = 0;
};

struct Ctx {
  bool init = false;
  int sms = 0;
  Buf logits, idx, gate, zsum, slot, cnt, fill, grp_off, grp_ttp, Xp, H, Y, err;
  // FP8 gate/up forwards: quantised tokens, their scale atoms per token tile,
  // and the experts' first FP8_BN-token tiles
  Buf Xp8, sfx, grp_ttp8;
  // host-buffer forwards: device staging for two chunks in and out, the
  // histogram summed over chunks, copy streams and their events
  Buf xin[2], yout[2], cnt_total;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
  bool counts_total = false;   // last forward was chunked: report cnt_total
  cudaEvent_t done = nullptr;
  bool has_result = false;
  bool done_valid = false;     // `done` marks the last forward (false: it was captured)
  int64_t T = 0;
  int d = 0, N = 0, Z = 0, K = 0, I = 0;
  int64_t rows_cap = 0;
  // Expert-load shape seen by earlier forwards, to choose the expert GEMMs'
  // launch without a host sync: after each prefill-sized forward its FFN
  // histogram is copied to pinned host memory behind an event; a later
  // forward reads it once the event has completed.
  int* hist_host = nullptr;          // pinned [MOE_ZC_MAX_E]
  cudaEvent_t hist_ev = nullptr;
  bool hist_pending = false;
  int hist_N = 0;
  bool pair_hint = false;            // most FFN pairs sit in experts with two token tiles
  bool spread_hint = false;          // at least half of the N FFN experts were hit
  bool one_grid_refused = false;     // the one-grid expert GEMMs' cooperative launch was refused
};

Ctx g_ctx[kMaxDevices];
std::mutex g_mu;

// Per-stage CUDA-event timing of forwards (moe_zc_profile / moe_zc_profile_read).
constexpr int kStages = 7;
constexpr int kRing = 256;
const char* const kStageNames[kStages] = {"router_gemm", "route",       "assign_slots",
                                          "permute",     "gateup_gemm", "down_gemm",
                                          "combine"};
struct Prof {
  bool on = false;
  int device = -1;
  int n = 0;          // forwards recorded since the last reset
  bool created = false;
  cudaEvent_t ev[kRing][kStages + 1];
};
Prof g_prof;
int g_fail_allocs = 0;
long long g_wait_ns_next = 0;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D bf16 tensor [rows, k] (row-major), box [box_rows, 64], 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t k, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(GEMM_BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D E4M3 (one byte per element) tensor [rows, k], box [box_rows, 128]
// (128-byte rows like the bf16 maps' 64 elements), 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t k, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(FP8_BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int ensure(Ctx& c, Buf& b, size_t bytes) {
  if (bytes == 0) bytes = 16;
  if (b.bytes >= bytes) return MOE_ZC_OK;
  if (g_fail_allocs > 0) {
    --g_fail_allocs;
    return MOE_ZC_ERR_OOM;
  }
  if (b.p) {
    // the previous forward may still read it
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ZC_ERR_CUDA;
    cudaFree(b.p);
    b.p = nullptr;
    b.bytes = 0;
  }
  if (cudaMalloc(&b.p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ZC_ERR_OOM;
  }
  b.bytes = bytes;
  (void)c;
  return MOE_ZC_OK;
}

int get_ctx(Ctx** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ZC_ERR_CUDA;
  Ctx& c = g_ctx[dev];
  if (!c.init) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    if (major != 10) return MOE_ZC_ERR_UNSUPPORTED;   // sm_100a only
    if (cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    if (cudaEventCreateWithFlags(&c.done, cudaEventDisableTiming) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    if (cudaEventCreateWithFlags(&c.hist_ev, cudaEventDisableTiming) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    if (cudaMallocHost(&c.hist_host, sizeof(int) * MOE_ZC_MAX_E) != cudaSuccess) {
      cudaGetLastError();
      c.hist_host = nullptr;   // the launch choice then keeps its default
    }
    c.init = true;
  }
  *out = &c;
  return MOE_ZC_OK;
}

// Router GEMM layout for T tokens: with few token tiles (decode) each tile is
// one 128-row block of W_r and K is split into slices so that the tiles fill
// the SMs, each slice at least 4 k-steps (256 of d); otherwise tiles pair two
// blocks and K is not split.
struct RouterPlan {
  int single_a, mblocks, splits;
  int tok_tile;    // tokens per tile
  int64_t tiles;   // token tiles x weight blocks (per slice)
};
RouterPlan router_plan(int64_t T, int E, int ksteps, int sms) {
  RouterPlan rp{0, (E + 2 * GEMM_BM - 1) / (2 * GEMM_BM), 1, GEMM_BN, 0};
  const int64_t ttiles = (T + GEMM_BN - 1) / GEMM_BN;
  rp.tiles = ttiles * rp.mblocks;
  if (rp.tiles >= sms) {
    // Many tiles: the token tile size (176..256 tokens) that finishes in the
    // least time, taking each wave of `sms` tiles to last as long as its
    // tile size (e.g. T = 16384, E = 768: 282 tiles of 176 tokens in two
    // waves rather than 192 of 256 in two, the second a third full).
    int64_t best = -1;
    for (int tt = GEMM_BN; tt >= 176; tt -= 16) {
      const int64_t tiles = (T + tt - 1) / tt * rp.mblocks;
      const int64_t cost = (tiles + sms - 1) / sms * tt;
      if (best < 0 || cost < best) {
        best = cost;
        rp.tok_tile = tt;
        rp.tiles = tiles;
      }
    }
  }
  if (rp.tiles > 0 && rp.tiles < sms / 2) {
    rp.single_a = 1;
    rp.mblocks = (E + GEMM_BM - 1) / GEMM_BM;
    rp.tiles = ttiles * rp.mblocks;
    int64_t s = sms / rp.tiles;
    const int64_t cap = ksteps / 4 > 0 ? ksteps / 4 : 1;
    if (s > cap) s = cap;
    rp.splits = s < 1 ? 1 : static_cast<int>(s);
  }
  return rp;
}

// The launch plan of a forward (moe_zc_plan; forward_impl takes its decisions
// from it).  The expert GEMMs' grids are sized from an upper bound of their
// tiles (every expert's last token tile may be partial), since the routing is
// not known on the host.
struct Plan {
  RouterPlan rp;
  int64_t router_grid = 0;
  bool one_grid = false;        // gate/up and down GEMMs in one persistent grid
  bool step = false;            // ... which also routes, dispatches and combines
  int64_t gateup_grid = 0, down_grid = 0, fused_grid = 0;
  int kernels = 0;
};
// test hook: 0 default, 1 never the one grid, 2 the one grid for the expert
// GEMMs only (route, dispatch and combine in their own kernels)
int g_one_grid_mode = 0;

// Counters that the router GEMM clears for each forward (see reserve_impl).
constexpr int kFillInts(int N) { return 2 * N + 5; }

Plan make_plan(int64_t T, int d, int N, int Z, int K, int I, int sms, int64_t resident,
               bool fp8 = false) {
  Plan pl;
  const int E = N + Z;
  pl.rp = router_plan(T, E, d / GEMM_BK, sms);
  const int64_t rg = pl.rp.tiles * pl.rp.splits;
  pl.router_grid = rg < sms ? rg : sms;
  if (T == 0) return pl;                         // a memset of the histogram only
  if (N == 0) {
    pl.kernels = 4;                              // router GEMM, route, assign, combine
    return pl;
  }
  const int64_t tiles_ub = (T * K + GEMM_BN - 1) / GEMM_BN + N;
  // (the FP8 gate/up GEMM cuts tokens into FP8_BN-token tiles)
  const int64_t g_tiles_ub = fp8 ? (T * K + FP8_BN - 1) / FP8_BN + N : tiles_ub;
  const int64_t g_ub = g_tiles_ub * (I / GEMM_BM);
  const int64_t d_ub = tiles_ub * ((d + 2 * GEMM_BM - 1) / (2 * GEMM_BM));
  pl.gateup_grid = g_ub < sms ? g_ub : sms;
  pl.down_grid = d_ub < sms ? d_ub : sms;
  pl.fused_grid = g_ub + d_ub < sms ? g_ub + d_ub : sms;
  pl.one_grid = T <= GEMM_SMALL_B && g_one_grid_mode != 1 && pl.fused_grid <= resident;
  // the one grid also runs route, assign, permute and combine: the router
  // GEMM and that grid are the whole forward
  pl.step = pl.one_grid && g_one_grid_mode != 2;
  pl.kernels = pl.step ? 2 : (pl.one_grid ? 6 : 7);
  return pl;
}

int reserve_impl(Ctx& c, int64_t T, int d, int N, int Z, int K, int I, bool fp8 = false) {
  const int64_t E = static_cast<int64_t>(N) + Z;
  const int64_t pairs = T * K;
  const int64_t rows_cap = N > 0 ? pairs + 15LL * N + 16 : 16;
  int s;
  const bool fresh_err = c.err.p == nullptr;
  if ((s = ensure(c, c.err, sizeof(int))) != MOE_ZC_OK) return s;
  if (fresh_err && cudaMemset(c.err.p, 0, sizeof(int)) != cudaSuccess) return MOE_ZC_ERR_CUDA;
  {
    const RouterPlan rp = router_plan(T, static_cast<int>(E), d / GEMM_BK, c.sms);
    if ((s = ensure(c, c.logits, static_cast<size_t>(T * E * rp.splits) * sizeof(float))) !=
        MOE_ZC_OK)
      return s;
  }
  if ((s = ensure(c, c.idx, static_cast<size_t>(pairs) * sizeof(int))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.gate, static_cast<size_t>(pairs) * sizeof(float))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.slot, static_cast<size_t>(pairs) * sizeof(int))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.zsum, static_cast<size_t>(T) * sizeof(float))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.cnt, static_cast<size_t>(E) * sizeof(int))) != MOE_ZC_OK) return s;
  // fill: [N + 1] slot counters, [N + 1] gate/up completion counters, the
  // gate/up and down GEMMs' tile counters, the decode step's grid barrier
  if ((s = ensure(c, c.fill, static_cast<size_t>(kFillInts(N)) * sizeof(int))) != MOE_ZC_OK)
    return s;
  if ((s = ensure(c, c.grp_off, static_cast<size_t>(N + 1) * sizeof(int))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.grp_ttp, static_cast<size_t>(N + 1) * sizeof(int))) != MOE_ZC_OK) return s;
  if (N > 0) {
    if ((s = ensure(c, c.Xp, static_cast<size_t>(rows_cap) * d * 2)) != MOE_ZC_OK) return s;
    if ((s = ensure(c, c.H, static_cast<size_t>(rows_cap) * I * 2)) != MOE_ZC_OK) return s;
    if ((s = ensure(c, c.Y, static_cast<size_t>(rows_cap) * d * 2)) != MOE_ZC_OK) return s;
  }
  if (fp8 && N > 0) {
    const int64_t tiles8 = (pairs + FP8_BN - 1) / FP8_BN + N;
    if ((s = ensure(c, c.Xp8, static_cast<size_t>(rows_cap) * d)) != MOE_ZC_OK) return s;
    if ((s = ensure(c, c.sfx, static_cast<size_t>(tiles8) * (d / FP8_BK) * 2 * SF_ATOM_BYTES)) !=
        MOE_ZC_OK)
      return s;
    if ((s = ensure(c, c.grp_ttp8, static_cast<size_t>(N + 1) * sizeof(int))) != MOE_ZC_OK)
      return s;
  }
  c.rows_cap = rows_cap;
  return MOE_ZC_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_args(const void* x, const void* W_r, const float* b, const void* W_gate,
               const void* W_up, const void* W_down, int64_t T, int32_t d, int32_t N, int32_t Z,
               int32_t K, int32_t I, const float* off, const void* out) {
  if (!W_r || !b) return MOE_ZC_ERR_INVALID_ARG;
  if (T != 0 && (!x || !out)) return MOE_ZC_ERR_INVALID_ARG;   // T == 0: may be NULL
  if (T < 0 || N < 0 || Z < 0 || d <= 0) return MOE_ZC_ERR_INVALID_ARG;
  const int64_t E = static_cast<int64_t>(N) + Z;
  if (E < 1 || K < 1 || K > E) return MOE_ZC_ERR_INVALID_ARG;
  if (N > 0 && (!W_gate || !W_up || !W_down || I <= 0)) return MOE_ZC_ERR_INVALID_ARG;
  if (K > MOE_ZC_MAX_K || E > MOE_ZC_MAX_E) return MOE_ZC_ERR_UNSUPPORTED;
  if (d % GEMM_BK != 0) return MOE_ZC_ERR_UNSUPPORTED;   // whole 64-wide K steps
  if (N > 0 && I % 128 != 0) return MOE_ZC_ERR_UNSUPPORTED;
  if (T * K + 16LL * N + 16 > (1LL << 31) - 1) return MOE_ZC_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(N) * (d > I ? d : I) > (1LL << 31) - 1) return MOE_ZC_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(W_r) || !aligned16(b) || !aligned16(out))  // NULL is aligned
    return MOE_ZC_ERR_UNSUPPORTED;
  if (off && !aligned16(off)) return MOE_ZC_ERR_UNSUPPORTED;
  if (N > 0 && (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down)))
    return MOE_ZC_ERR_UNSUPPORTED;
  return MOE_ZC_OK;
}

#define CK(expr)                                   \
  do {                                             \
    if ((expr) != cudaSuccess) {                   \
      cudaGetLastError();                          \
      return MOE_ZC_ERR_CUDA;                      \
    }                                              \
  } while (0)

// Records event `i` of the current profiled forward (no-op when profiling is off).
struct StageRec {
  cudaEvent_t* ev = nullptr;
  cudaStream_t st = nullptr;
  void mark(int i) const {
    if (ev) cudaEventRecord(ev[i], st);
  }
};

// Expert-load hints for later launch choices, without a host sync: a copy
// of the FFN histogram goes to pinned memory behind an event
// (queue_load_hints), and a later forward reads it once the event has
// completed (read_load_hints):
//   pair_hint    at least half of the FFN pairs sat in experts with two token
//                tiles (257..512 tokens): pace those tiles on 2-CTA clusters
//   spread_hint  at least half of the FFN experts were hit: a host-buffer
//                forward takes the batch in one chunk
int read_load_hints(Ctx& c, int N) {
  if (!c.hist_pending) return MOE_ZC_OK;
  const cudaError_t q = cudaEventQuery(c.hist_ev);
  if (q == cudaErrorNotReady) {
    cudaGetLastError();   // not an error: the copy is still on its way
    return MOE_ZC_OK;
  }
  CK(q);
  if (c.hist_N == N) {
    long long two = 0, all = 0;
    int hit = 0;
    for (int e = 0; e < N; ++e) {
      const int n = c.hist_host[e];
      all += n;
      hit += n > 0;
      if (n > GEMM_BN && n <= 2 * GEMM_BN) two += n;
    }
    c.pair_hint = all > 0 && 2 * two >= all;
    c.spread_hint = 2 * hit >= N;
  }
  c.hist_pending = false;
  return MOE_ZC_OK;
}

int queue_load_hints(Ctx& c, const int* cnt, int N, cudaStream_t st) {
  if (c.hist_pending || !c.hist_host) return MOE_ZC_OK;
  CK(cudaMemcpyAsync(c.hist_host, cnt, sizeof(int) * N, cudaMemcpyDeviceToHost, st));
  CK(cudaEventRecord(c.hist_ev, st));
  c.hist_pending = true;
  c.hist_N = N;
  return MOE_ZC_OK;
}

// FP8 gate/up weights of moe_zc_forward_fp8: E4M3 codes of W_gate and W_up
// (where the bf16 forward takes the bf16 matrices) and their scale atoms.
struct Fp8Gates {
  const uint8_t* gate_sf;
  const uint8_t* up_sf;
};

int check_fp8(const Fp8Gates* f8, int d, int N) {
  if (!f8 || N == 0) return MOE_ZC_OK;
  if (!f8->gate_sf || !f8->up_sf) return MOE_ZC_ERR_INVALID_ARG;
  if (d % FP8_BK != 0) return MOE_ZC_ERR_UNSUPPORTED;   // whole 128-element stages
  if (!aligned16(f8->gate_sf) || !aligned16(f8->up_sf)) return MOE_ZC_ERR_UNSUPPORTED;
  return MOE_ZC_OK;
}

// f8: NULL for the bf16 forward; else W_gate / W_up hold E4M3 codes and f8
// their scales (the FP8 gate/up GEMM; the down projection stays bf16).
// Routing given by the caller (moe_zc_experts): row i goes, with gate 1, to
// FFN expert expert[i] - base; there is no router (K = 1, Z = 0).
struct GivenRouting {
  const int32_t* expert;
  int base;
};

int forward_impl(const void* x, const void* W_r, const float* b, const void* W_gate,
                 const void* W_up, const void* W_down, int64_t T, int32_t d, int32_t N,
                 int32_t Z, int32_t K, int32_t I, const float* off, void* out, void* stream,
                 const Fp8Gates* f8 = nullptr, const GivenRouting* given = nullptr) {
  int s = check_args(x, W_r, b, W_gate, W_up, W_down, T, d, N, Z, K, I, off, out);
  if (s != MOE_ZC_OK) return s;
  if ((s = check_fp8(f8, d, N)) != MOE_ZC_OK) return s;
  if (N == 0) f8 = nullptr;
  Ctx* cp = nullptr;
  if ((s = get_ctx(&cp)) != MOE_ZC_OK) return s;
  Ctx& c = *cp;
  if ((s = reserve_impl(c, T, d, N, Z, K, N > 0 ? I : 128, f8 != nullptr)) != MOE_ZC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = N + Z;
  const long long wait_ns = g_wait_ns_next > 0 ? g_wait_ns_next : kWaitNs;
  g_wait_ns_next = 0;
  int* err = static_cast<int*>(c.err.p);
  int* cnt = static_cast<int*>(c.cnt.p);
  int* idx = static_cast<int*>(c.idx.p);
  float* gate = static_cast<float*>(c.gate.p);
  float* zsum = static_cast<float*>(c.zsum.p);
  int* slot = static_cast<int*>(c.slot.p);
  int* grp_off = static_cast<int*>(c.grp_off.p);
  int* grp_ttp = static_cast<int*>(c.grp_ttp.p);
  int* fill = static_cast<int*>(c.fill.p);

  // A forward captured into a CUDA graph by the caller records no events:
  // an event recorded during capture cannot be waited on afterwards.
  cudaStreamCaptureStatus capturing = cudaStreamCaptureStatusNone;
  CK(cudaStreamIsCapturing(st, &capturing));
  const bool captured = capturing != cudaStreamCaptureStatusNone;
  StageRec rec;
  int dev_now = -1;
  cudaGetDevice(&dev_now);
  if (!captured && g_prof.on && g_prof.device == dev_now && g_prof.n < kRing) {
    rec.ev = g_prof.ev[g_prof.n];
    rec.st = st;
  }
  rec.mark(0);
  // (a batch with tokens clears its histogram in the router GEMM)
  if (T == 0) CK(cudaMemsetAsync(cnt, 0, sizeof(int) * E, st));
  // Prefill-sized batches whose experts mostly get two token tiles (a few
  // hundred tokens each, as under balanced load) run the expert GEMMs as
  // 2-CTA clusters that pace those tiles; batches concentrated on a few
  // experts do better without (measured: +10% on balanced gate/up, -3% on
  // concentrated).  The choice follows the histogram of an earlier forward.
  if (!captured && (s = read_load_hints(c, N)) != MOE_ZC_OK) return s;
  const bool pace_tiles = N > 0 && T >= 1024 && c.pair_hint;
  const Plan plan = make_plan(T, d, N, Z, K, I, c.sms,
                              T > 0 && T <= GEMM_SMALL_B && N > 0 && !c.one_grid_refused
                                  ? fused_resident_blocks()
                                  : 0,
                              f8 != nullptr);
  int* grp_ttp8 = f8 ? static_cast<int*>(c.grp_ttp8.p) : nullptr;
  if (T > 0 && given) {
    // 1-2  the caller's routing: one pick per row, gate 1, no zero experts
    CK(cudaMemsetAsync(cnt, 0, sizeof(int) * E, st));
    CK(cudaMemsetAsync(fill, 0, sizeof(int) * kFillInts(N), st));
    CK(launch_given_routing(given->expert, T, given->base, N, idx, gate, zsum, cnt, st));
    rec.mark(1);
    rec.mark(2);
  }
  if (T > 0) {
    const RouterPlan rp = plan.rp;
    const int splits = rp.splits;
   if (!given) {
    // 1  router GEMM
    CUtensorMap mWr, mX;
    // x in boxes of 32 tokens, and of one full token tile (rp.tok_tile)
    CUtensorMap mXf;
    const bool full_ok = T >= rp.tok_tile;
    if (!make_map(&mWr, W_r, E, d, GEMM_BM) || !make_map(&mX, x, T, d, GEMM_B_BOX_ROWS) ||
        !make_map(&mXf, x, T, d, full_ok ? rp.tok_tile : GEMM_B_BOX_ROWS))
      return MOE_ZC_ERR_CUDA;
    GemmParams pr{};
    pr.G = 1;
    pr.T = static_cast<int>(T);
    pr.ksteps = d / GEMM_BK;
    pr.a_rows = E;
    pr.out = c.logits.p;
    pr.out_ld = E;
    pr.err = err;
    pr.wait_ns = wait_ns;
    // Few token tiles (decode): single blocks and K slices so that every SM
    // streams a part of W_r; the slices' partial logits are summed in slice
    // order by the route kernel (or the decode step's route phase).
    pr.mblocks = rp.mblocks;
    pr.single_a = rp.single_a;
    pr.tok_tile = rp.tok_tile;
    pr.ksplit = splits;
    pr.split_stride = T * E;
    pr.b_box_full = full_ok ? 1 : 0;
    pr.small_b = T <= GEMM_SMALL_B ? 1 : 0;
    pr.zero0 = cnt;
    pr.nzero0 = E;
    pr.zero1 = fill;
    pr.nzero1 = kFillInts(N);
    CK(launch_gemm(MODE_ROUTER, mWr, mWr, mX, mXf, pr, static_cast<int>(plan.router_grid), st));
    rec.mark(1);
   }
    // 2  route (unless the decode step's one grid does it)
    auto route = [&]() -> int {
      if (given) return MOE_ZC_OK;
      CK(launch_route(static_cast<const float*>(c.logits.p), b, off, T, E, N, K, idx, gate, zsum,
                      cnt, st, splits));
      rec.mark(2);
      return MOE_ZC_OK;
    };
    // 7  combine
    auto combine = [&]() -> int {
      CK(launch_combine(static_cast<const __nv_bfloat16*>(x),
                        static_cast<const __nv_bfloat16*>(c.Y.p), slot, gate, zsum, T, d, K,
                        static_cast<__nv_bfloat16*>(out), st));
      return MOE_ZC_OK;
    };
    if (N > 0) {
      // the expert GEMMs' maps and parameters (host only)
      CUtensorMap mWg, mWu, mXp;
      if (!make_map(&mWg, W_gate, static_cast<uint64_t>(N) * I, d, GEMM_BM) ||
          !make_map(&mWu, W_up, static_cast<uint64_t>(N) * I, d, GEMM_BM) ||
          !make_map(&mXp, c.Xp.p, c.rows_cap, d, GEMM_B_BOX_ROWS))
        return MOE_ZC_ERR_CUDA;
      // full 256-token boxes of the permuted tokens and of H
      CUtensorMap mXpf, mHf;
      const bool full_ok = c.rows_cap >= GEMM_BN;
      const uint32_t fbox = full_ok ? GEMM_BN : GEMM_B_BOX_ROWS;
      if (!make_map(&mXpf, c.Xp.p, c.rows_cap, d, fbox) ||
          !make_map(&mHf, c.H.p, c.rows_cap, I, fbox))
        return MOE_ZC_ERR_CUDA;
      GemmParams pg{};
      pg.grp_count = cnt;
      pg.grp_off = grp_off;
      pg.grp_ttp = grp_ttp;
      pg.G = N;
      pg.ksteps = d / GEMM_BK;
      pg.mblocks = I / GEMM_BM;
      pg.a_rows = I;
      pg.out = c.H.p;
      pg.out_ld = I;
      pg.err = err;
      pg.wait_ns = wait_ns;
      // decode-sized batches stream every weight byte once
      pg.l2_stream = T < 1024 ? 1 : 0;
      // at most 64 tokens per expert: five smaller stages, more weights in flight
      pg.small_b = T <= GEMM_SMALL_B ? 1 : 0;
      pg.b_box_full = full_ok ? 1 : 0;
      // prefill-sized batches: CTA pairs pace the two token tiles of a weight
      // block so that its second read is an L2 hit
      pg.pair_tiles = pace_tiles ? 1 : 0;
      // otherwise, for batches of many rounds of tiles, CTAs take tiles in
      // order from a counter (cleared with the slot counters by the router
      // GEMM, or by the given-routing memset).  Measured: gate/up -1..3% at
      // prefill and skewed; +2% on the 4096-token workload, whose 888 tiles
      // are six even rounds of 148, so smaller batches keep fixed shares.
      const bool by_counter = T >= 8192;
      pg.tile_counter = by_counter ? fill + 2 * N + 2 : nullptr;
      CUtensorMap mWd, mH;
      if (!make_map(&mWd, W_down, static_cast<uint64_t>(N) * d, I, GEMM_BM) ||
          !make_map(&mH, c.H.p, c.rows_cap, I, GEMM_B_BOX_ROWS))
        return MOE_ZC_ERR_CUDA;
      GemmParams pd = pg;
      pd.tile_counter = by_counter ? fill + 2 * N + 3 : nullptr;
      pd.ksteps = I / GEMM_BK;
      pd.mblocks = (d + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
      pd.a_rows = d;
      pd.out = c.Y.p;
      pd.out_ld = d;
      if (f8) {
        // the FP8 gate/up GEMM: E4M3 operands with 128 contraction elements
        // per stage, FP8_BN-token tiles, scale atoms (the down GEMM above
        // keeps the bf16 parameters)
        const bool full8 = c.rows_cap >= FP8_BN;
        if (!make_map_u8(&mWg, W_gate, static_cast<uint64_t>(N) * I, d, GEMM_BM) ||
            !make_map_u8(&mWu, W_up, static_cast<uint64_t>(N) * I, d, GEMM_BM) ||
            !make_map_u8(&mXp, c.Xp8.p, c.rows_cap, d, GEMM_B_BOX_ROWS) ||
            !make_map_u8(&mXpf, c.Xp8.p, c.rows_cap, d, full8 ? FP8_BN : GEMM_B_BOX_ROWS))
          return MOE_ZC_ERR_CUDA;
        pg.b_box_full = full8 ? 1 : 0;
        pg.tok_tile = FP8_BN;
        pg.grp_ttp = grp_ttp8;
        pg.ksteps = d / FP8_BK;
        pg.sf_kgroups = d / FP8_BK;
        pg.sfa0 = f8->gate_sf;
        pg.sfa1 = f8->up_sf;
        pg.sfb = static_cast<const uint8_t*>(c.sfx.p);
      }
      // At most 64 tokens: both expert GEMMs in one persistent grid, the
      // down tiles of an expert starting as soon as its H rows are stored
      // (the SMs that the last round of gate/up tiles leaves idle stream down
      // weights meanwhile).
      GemmParams pf = pg;
      pf.b_box_full = 0;
      pf.done = fill + N + 1;
      // tiles taken in order from a counter (cleared by the router GEMM or
      // the given-routing memset), so that SMs that stream faster take more
      // (measured: -2 us at decode, bf16 and FP8, against fixed shares)
      pf.tile_counter = fill + 2 * N + 2;
      auto one_grid_launch = [&](const StepParams& sp) {
        return f8 ? launch_gemm_fused_fp8(mWg, mWu, mXp, mWd, mH, pf, pd,
                                          static_cast<int>(plan.fused_grid), st, sp)
                  : launch_gemm_fused(mWg, mWu, mXp, mWd, mH, pf, pd,
                                      static_cast<int>(plan.fused_grid), st, sp);
      };
      // a refused cooperative launch (its blocks cannot all be resident)
      // queues nothing: the forward goes on with separate launches, and so do
      // the later ones
      auto refused = [&]() -> int {
        cudaGetLastError();
        if (captured) return MOE_ZC_ERR_CUDA;   // (the capture is invalidated)
        c.one_grid_refused = true;
        return MOE_ZC_OK;
      };
      bool stepped = false;
      if (plan.step && !given) {
        // 2-7  the rest of the forward in the one grid: route, assign and
        // permute, the expert tiles, combine
        StepParams sp{};
        sp.on = 1;
        sp.T = static_cast<int>(T);
        sp.E = E;
        sp.N = N;
        sp.K = K;
        sp.d = d;
        sp.logits = static_cast<const float*>(c.logits.p);
        sp.splits = splits;
        sp.bias = b;
        sp.offset = off;
        sp.idx = idx;
        sp.gate = gate;
        sp.zsum = zsum;
        sp.cnt = cnt;
        sp.slot = slot;
        sp.fill = fill;
        sp.grp_off = grp_off;
        sp.grp_ttp = grp_ttp;
        sp.grp_ttp8 = grp_ttp8;
        sp.x = static_cast<const __nv_bfloat16*>(x);
        sp.Xp = static_cast<__nv_bfloat16*>(c.Xp.p);
        sp.Xp8 = f8 ? static_cast<uint8_t*>(c.Xp8.p) : nullptr;
        sp.sfx = f8 ? static_cast<uint8_t*>(c.sfx.p) : nullptr;
        sp.Y = static_cast<const __nv_bfloat16*>(c.Y.p);
        sp.out = static_cast<__nv_bfloat16*>(out);
        sp.gbar = fill + 2 * N + 4;
        for (int i = 2; i <= 4; ++i) rec.mark(i);
        if (one_grid_launch(sp) == cudaSuccess) {
          for (int i = 5; i <= 6; ++i) rec.mark(i);
          stepped = true;
        } else if ((s = refused()) != MOE_ZC_OK) {
          return s;
        }
      }
      if (!stepped) {
        if ((s = route()) != MOE_ZC_OK) return s;
        // 3-4  dispatch
        CK(launch_assign_slots(cnt, idx, T * K, N, grp_off, grp_ttp, fill, slot, st, grp_ttp8));
        rec.mark(3);
        if (f8) {
          // each token row quantised once (E4M3, 1 x 32 blocks) into its slots
          CK(launch_permute_fp8(static_cast<const __nv_bfloat16*>(x), idx, slot, cnt, grp_off,
                                grp_ttp8, T, d, K, N, static_cast<uint8_t*>(c.Xp8.p),
                                static_cast<uint8_t*>(c.sfx.p), st));
        } else {
          CK(launch_permute(static_cast<const __nv_bfloat16*>(x), slot, T, d, K,
                            static_cast<__nv_bfloat16*>(c.Xp.p), st));
        }
        rec.mark(4);
        bool one_grid = plan.one_grid && !c.one_grid_refused;
        if (one_grid) {
          // 5-6  the expert GEMMs in the one grid
          if (one_grid_launch(StepParams{}) == cudaSuccess) {
            rec.mark(5);
            rec.mark(6);
          } else {
            if ((s = refused()) != MOE_ZC_OK) return s;
            one_grid = false;
          }
        }
        if (!one_grid) {
          // 5  gate/up GEMM
          if (f8)
            CK(launch_gemm_gateup_fp8(mWg, mWu, mXp, mXpf, pg, static_cast<int>(plan.gateup_grid),
                                      st));
          else
            CK(launch_gemm(MODE_GATEUP, mWg, mWu, mXp, mXpf, pg,
                           static_cast<int>(plan.gateup_grid), st));
          rec.mark(5);
          // 6  down GEMM
          CK(launch_gemm(MODE_DOWN, mWd, mWd, mH, mHf, pd, static_cast<int>(plan.down_grid), st));
          rec.mark(6);
        }
        if ((s = combine()) != MOE_ZC_OK) return s;
      }
    } else {
      if ((s = route()) != MOE_ZC_OK) return s;
      CK(launch_assign_slots(cnt, idx, T * K, N, grp_off, grp_ttp, fill, slot, st));
      for (int i = 3; i <= 6; ++i) rec.mark(i);
      if ((s = combine()) != MOE_ZC_OK) return s;
    }
  } else {
    for (int i = 1; i <= 6; ++i) rec.mark(i);
  }
  rec.mark(7);
  if (rec.ev) ++g_prof.n;
  if (!captured && N > 0 && T >= 1024 && (s = queue_load_hints(c, cnt, N, st)) != MOE_ZC_OK)
    return s;
  if (!captured) CK(cudaEventRecord(c.done, st));
  c.done_valid = !captured;
  c.has_result = true;
  c.counts_total = false;
  c.T = T;
  c.d = d;
  c.N = N;
  c.Z = Z;
  c.K = K;
  c.I = I;
  return MOE_ZC_OK;
}

int host_streams(Ctx& c) {
  if (c.s_in) return MOE_ZC_OK;
  CK(cudaStreamCreateWithFlags(&c.s_in, cudaStreamNonBlocking));
  CK(cudaStreamCreateWithFlags(&c.s_out, cudaStreamNonBlocking));
  CK(cudaEventCreateWithFlags(&c.ev_start, cudaEventDisableTiming));
  for (int i = 0; i < 2; ++i) {
    CK(cudaEventCreateWithFlags(&c.ev_in[i], cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&c.ev_comp[i], cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&c.ev_out[i], cudaEventDisableTiming));
  }
  return MOE_ZC_OK;
}

// The forward on host buffers: T tokens in chunks, each chunk copied in on
// one stream, computed on the caller's stream and copied out on a third, so
// that the copies of chunk c +- 1 overlap the kernels of chunk c.
int forward_host_impl(const void* x_host, const void* W_r, const float* b, const void* W_gate,
                      const void* W_up, const void* W_down, int64_t T, int32_t d, int32_t N,
                      int32_t Z, int32_t K, int32_t I, const float* off, void* out_host,
                      int64_t chunk, void* stream, const Fp8Gates* f8 = nullptr) {
  if (T < 0) return MOE_ZC_ERR_INVALID_ARG;
  if (T > 0 && (!x_host || !out_host)) return MOE_ZC_ERR_INVALID_ARG;
  // the device-side checks of one chunk (fake aligned buffers stand in)
  int s = check_args(reinterpret_cast<const void*>(16), W_r, b, W_gate, W_up, W_down, T, d, N,
                     Z, K, I, off, reinterpret_cast<void*>(16));
  if (s != MOE_ZC_OK) return s;
  if ((s = check_fp8(f8, d, N)) != MOE_ZC_OK) return s;
  Ctx* cp = nullptr;
  if ((s = get_ctx(&cp)) != MOE_ZC_OK) return s;
  Ctx& c = *cp;
  // Chunk sizes.  Given: chunk_tokens each.  Default: about T/4 (measured
  // best of uniform sizes at the prefill workload: 2048: 13.0 ms, 4096:
  // 12.1 ms, 8192: 12.8 ms per step), with the first and the last chunk
  // half as long, since the first copy in and the last copy out overlap
  // nothing (prefill: 2048, 4096, 4096, 4096, 2048).  But when earlier
  // forwards spread their tokens over most FFN experts, every chunk would
  // stream nearly all expert weights again: one chunk then (balanced
  // prefill: 18.3 ms per step against 27 ms in four).
  std::vector<int64_t> sizes;
  if (chunk > 0 || (c.spread_hint && c.hist_N == N)) {
    const int64_t step = chunk > 0 ? chunk : (T > 0 ? T : 1);
    for (int64_t t0 = 0; t0 < T; t0 += step) sizes.push_back(T - t0 < step ? T - t0 : step);
  } else {
    int64_t mid = ((T + 3) / 4 + 255) / 256 * 256;
    if (mid < 1024) mid = 1024;
    const int64_t end = mid / 2 / 256 * 256 >= 512 ? mid / 2 / 256 * 256 : 512;
    int64_t rem = T;
    if (rem > mid + end) {
      sizes.push_back(end);
      rem -= end;
      while (rem > mid + end) {
        sizes.push_back(mid);
        rem -= mid;
      }
      if (rem > mid) {
        sizes.push_back(rem - end);
        rem = end;
      }
    }
    if (rem > 0) sizes.push_back(rem);
  }
  chunk = 0;
  for (int64_t n : sizes) chunk = n > chunk ? n : chunk;
  const int E = N + Z;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(d) * 2;
  if (sizes.size() == 1) {
    // One chunk (e.g. a decode batch): nothing to overlap, so the copy in,
    // the forward and the copy out run in order on the caller's stream,
    // without the pipeline's side streams, events and summed histogram
    // (decode e2e 56-79 us over the device-resident step before, 43 us with
    // this path).
    if ((s = ensure(c, c.xin[0], T * row_bytes)) != MOE_ZC_OK) return s;
    if ((s = ensure(c, c.yout[0], T * row_bytes)) != MOE_ZC_OK) return s;
    CK(cudaMemcpyAsync(c.xin[0].p, x_host, T * row_bytes, cudaMemcpyHostToDevice, st));
    if ((s = forward_impl(c.xin[0].p, W_r, b, W_gate, W_up, W_down, T, d, N, Z, K, I, off,
                          c.yout[0].p, stream, f8)) != MOE_ZC_OK)
      return s;
    CK(cudaMemcpyAsync(out_host, c.yout[0].p, T * row_bytes, cudaMemcpyDeviceToHost, st));
    CK(cudaEventRecord(c.done, st));
    c.done_valid = true;
    return MOE_ZC_OK;
  }
  if ((s = host_streams(c)) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.cnt_total, sizeof(int) * E)) != MOE_ZC_OK) return s;
  for (int i = 0; i < 2 && T > 0; ++i) {
    if ((s = ensure(c, c.xin[i], chunk * row_bytes)) != MOE_ZC_OK) return s;
    if ((s = ensure(c, c.yout[i], chunk * row_bytes)) != MOE_ZC_OK) return s;
  }
  CK(cudaMemsetAsync(c.cnt_total.p, 0, sizeof(int) * E, st));
  CK(cudaEventRecord(c.ev_start, st));
  CK(cudaStreamWaitEvent(c.s_in, c.ev_start, 0));
  CK(cudaStreamWaitEvent(c.s_out, c.ev_start, 0));
  const char* xh = static_cast<const char*>(x_host);
  char* oh = static_cast<char*>(out_host);
  const int64_t nchunks = static_cast<int64_t>(sizes.size());
  int64_t t0 = 0;
  for (int64_t ci = 0; ci < nchunks; t0 += sizes[ci], ++ci) {
    const int bi = static_cast<int>(ci & 1);
    const int64_t n = sizes[ci];
    // copy in once the kernels of chunk ci-2 are done with this buffer
    if (ci >= 2) CK(cudaStreamWaitEvent(c.s_in, c.ev_comp[bi], 0));
    CK(cudaMemcpyAsync(c.xin[bi].p, xh + t0 * row_bytes, n * row_bytes, cudaMemcpyHostToDevice,
                       c.s_in));
    CK(cudaEventRecord(c.ev_in[bi], c.s_in));
    // compute once the input is here and chunk ci-2's output has left
    CK(cudaStreamWaitEvent(st, c.ev_in[bi], 0));
    if (ci >= 2) CK(cudaStreamWaitEvent(st, c.ev_out[bi], 0));
    s = forward_impl(c.xin[bi].p, W_r, b, W_gate, W_up, W_down, n, d, N, Z, K, I, off,
                     c.yout[bi].p, stream, f8);
    if (s != MOE_ZC_OK) return s;
    CK(launch_add_counts(static_cast<const int*>(c.cnt.p), E,
                         static_cast<int*>(c.cnt_total.p), st));
    CK(cudaEventRecord(c.ev_comp[bi], st));
    // copy out
    CK(cudaStreamWaitEvent(c.s_out, c.ev_comp[bi], 0));
    CK(cudaMemcpyAsync(oh + t0 * row_bytes, c.yout[bi].p, n * row_bytes, cudaMemcpyDeviceToHost,
                       c.s_out));
    CK(cudaEventRecord(c.ev_out[bi], c.s_out));
  }
  // the caller's stream completes only after every copy out
  for (int i = 0; i < 2 && i < nchunks; ++i) CK(cudaStreamWaitEvent(st, c.ev_out[i], 0));
  CK(cudaEventRecord(c.done, st));
  c.done_valid = true;
  c.has_result = true;
  c.counts_total = true;
  c.N = N;
  c.Z = Z;
  return MOE_ZC_OK;
}

int sync_impl(Ctx& c) {
  if (!c.has_result) return MOE_ZC_ERR_NO_RESULT;
  // after a captured forward its replays are the caller's: wait for the device
  if (c.done_valid) {
    CK(cudaEventSynchronize(c.done));
  } else {
    CK(cudaDeviceSynchronize());
  }
  int e = 0;
  CK(cudaMemcpy(&e, c.err.p, sizeof(int), cudaMemcpyDeviceToHost));
  if (e != 0) {
    CK(cudaMemset(c.err.p, 0, sizeof(int)));
    return MOE_ZC_ERR_TIMEOUT;
  }
  return MOE_ZC_OK;
}

}  // namespace

long long moezc::take_injected_wait_ns() {
  std::lock_guard<std::mutex> lk(g_mu);
  const long long v = g_wait_ns_next;
  g_wait_ns_next = 0;
  return v;
}

extern "C" {

int moe_zc_forward(const void* x, const void* W_r, const float* b, const void* W_gate,
                   const void* W_up, const void* W_down, int64_t T, int32_t d, int32_t N,
                   int32_t Z, int32_t K, int32_t I, void* out, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  return forward_impl(x, W_r, b, W_gate, W_up, W_down, T, d, N, Z, K, I, nullptr, out, stream);
}

int moe_zc_forward_ex(const void* x, const void* W_r, const float* b, const void* W_gate,
                      const void* W_up, const void* W_down, int64_t T, int32_t d, int32_t N,
                      int32_t Z, int32_t K, int32_t I, const float* logit_offset, void* out,
                      void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  return forward_impl(x, W_r, b, W_gate, W_up, W_down, T, d, N, Z, K, I, logit_offset, out,
                      stream);
}

int moe_zc_route(const void* x, const void* W_r, const float* b, const float* logit_offset,
                 int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t* idx,
                 float* gate, float* zsum, int32_t* counts, void* stream) {
  const void* f = reinterpret_cast<const void*>(16);   // stand-ins: no expert weights here
  int s = check_args(x, W_r, b, f, f, f, T, d, N, Z, K, 128, logit_offset, f);
  if (s != MOE_ZC_OK) return s;
  if (!counts || (T > 0 && (!idx || !gate || !zsum))) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* cp = nullptr;
  if ((s = get_ctx(&cp)) != MOE_ZC_OK) return s;
  Ctx& c = *cp;
  const int E = N + Z;
  const RouterPlan rp = router_plan(T, E, d / GEMM_BK, c.sms);
  const bool fresh_err = c.err.p == nullptr;
  if ((s = ensure(c, c.err, sizeof(int))) != MOE_ZC_OK) return s;
  if (fresh_err && cudaMemset(c.err.p, 0, sizeof(int)) != cudaSuccess) return MOE_ZC_ERR_CUDA;
  if ((s = ensure(c, c.logits, static_cast<size_t>(T * E * rp.splits) * sizeof(float))) !=
      MOE_ZC_OK)
    return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long wait_ns = g_wait_ns_next > 0 ? g_wait_ns_next : kWaitNs;
  g_wait_ns_next = 0;
  if (T == 0) {
    CK(cudaMemsetAsync(counts, 0, sizeof(int) * E, st));
  } else {
    CUtensorMap mWr, mX, mXf;
    const bool full_ok = T >= rp.tok_tile;
    if (!make_map(&mWr, W_r, E, d, GEMM_BM) || !make_map(&mX, x, T, d, GEMM_B_BOX_ROWS) ||
        !make_map(&mXf, x, T, d, full_ok ? rp.tok_tile : GEMM_B_BOX_ROWS))
      return MOE_ZC_ERR_CUDA;
    GemmParams pr{};
    pr.G = 1;
    pr.T = static_cast<int>(T);
    pr.ksteps = d / GEMM_BK;
    pr.a_rows = E;
    pr.out = c.logits.p;
    pr.out_ld = E;
    pr.err = static_cast<int*>(c.err.p);
    pr.wait_ns = wait_ns;
    pr.mblocks = rp.mblocks;
    pr.single_a = rp.single_a;
    pr.tok_tile = rp.tok_tile;
    pr.ksplit = rp.splits;
    pr.split_stride = T * E;
    pr.b_box_full = full_ok ? 1 : 0;
    pr.small_b = T <= GEMM_SMALL_B ? 1 : 0;
    pr.zero0 = counts;   // the router GEMM clears the histogram
    pr.nzero0 = E;
    const int64_t rg = rp.tiles * rp.splits;
    CK(launch_gemm(MODE_ROUTER, mWr, mWr, mX, mXf, pr, static_cast<int>(rg < c.sms ? rg : c.sms),
                   st));
    CK(launch_route(static_cast<const float*>(c.logits.p), b, logit_offset, T, E, N, K, idx, gate,
                    zsum, counts, st, rp.splits));
  }
  CK(cudaEventRecord(c.done, st));
  c.done_valid = true;
  c.has_result = true;
  return MOE_ZC_OK;
}

int moe_zc_dispatch(const void* x, const int32_t* idx, const int32_t* counts, int64_t T,
                    int32_t d, int32_t N, int32_t K, int32_t* slot, void* send,
                    int32_t* send_expert, void* stream) {
  if (T < 0 || N < 1 || K < 1 || K > MOE_ZC_MAX_K || N > MOE_ZC_MAX_E || d <= 0)
    return MOE_ZC_ERR_INVALID_ARG;
  if (T > 0 && (!x || !idx || !counts || !slot || !send || !send_expert))
    return MOE_ZC_ERR_INVALID_ARG;
  if (d % 8 != 0 || !aligned16(x) || !aligned16(send)) return MOE_ZC_ERR_UNSUPPORTED;
  if (T * K > (1LL << 31) - 1) return MOE_ZC_ERR_UNSUPPORTED;
  if (T == 0) return MOE_ZC_OK;
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* cp = nullptr;
  int s = get_ctx(&cp);
  if (s != MOE_ZC_OK) return s;
  Ctx& c = *cp;
  if ((s = ensure(c, c.fill, static_cast<size_t>(2 * N + 2) * sizeof(int))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.grp_off, static_cast<size_t>(N + 1) * sizeof(int))) != MOE_ZC_OK) return s;
  if ((s = ensure(c, c.grp_ttp, static_cast<size_t>(N + 1) * sizeof(int))) != MOE_ZC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* fill = static_cast<int*>(c.fill.p);
  CK(cudaMemsetAsync(fill, 0, sizeof(int) * (N + 1), st));
  // packed rows (no padding): expert e's rows follow expert e - 1's, so the
  // rows bound for each rank's contiguous range of experts are contiguous
  CK(launch_assign_slots(counts, idx, T * K, N, static_cast<int*>(c.grp_off.p),
                         static_cast<int*>(c.grp_ttp.p), fill, slot, st, nullptr, 1, send_expert));
  CK(launch_permute(static_cast<const __nv_bfloat16*>(x), slot, T, d, K,
                    static_cast<__nv_bfloat16*>(send), st));
  return MOE_ZC_OK;
}

int moe_zc_experts(const void* x_rows, const int32_t* expert, int32_t expert_base, int64_t R,
                   int32_t d, int32_t N, int32_t I, const void* W_gate, const void* W_up,
                   const void* W_down, void* y, void* stream) {
  if (R > 0 && !expert) return MOE_ZC_ERR_INVALID_ARG;
  if (N < 1) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  const void* f = reinterpret_cast<const void*>(16);   // no router: stand-ins
  const GivenRouting given{expert, expert_base};
  return forward_impl(x_rows, f, static_cast<const float*>(f), W_gate, W_up, W_down, R, d, N, 0,
                      1, I, nullptr, y, stream, nullptr, &given);
}

int moe_zc_combine(const void* x, const void* y_rows, const int32_t* slot, const float* gate,
                   const float* zsum, int64_t T, int32_t d, int32_t K, void* out, void* stream) {
  if (T < 0 || K < 1 || K > MOE_ZC_MAX_K || d <= 0) return MOE_ZC_ERR_INVALID_ARG;
  if (T > 0 && (!x || !slot || !gate || !zsum || !out)) return MOE_ZC_ERR_INVALID_ARG;
  if (d % 8 != 0 || !aligned16(x) || !aligned16(y_rows) || !aligned16(out))
    return MOE_ZC_ERR_UNSUPPORTED;
  CK(launch_combine(static_cast<const __nv_bfloat16*>(x),
                    static_cast<const __nv_bfloat16*>(y_rows), slot, gate, zsum, T, d, K,
                    static_cast<__nv_bfloat16*>(out), static_cast<cudaStream_t>(stream)));
  return MOE_ZC_OK;
}

int moe_zc_forward_fp8(const void* x, const void* W_r, const float* b, const void* W_gate8,
                       const void* W_gate_sf, const void* W_up8, const void* W_up_sf,
                       const void* W_down, int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K,
                       int32_t I, const float* logit_offset, void* out, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  const Fp8Gates f8{static_cast<const uint8_t*>(W_gate_sf), static_cast<const uint8_t*>(W_up_sf)};
  return forward_impl(x, W_r, b, W_gate8, W_up8, W_down, T, d, N, Z, K, I, logit_offset, out,
                      stream, &f8);
}

int moe_zc_forward_host_fp8(const void* x_host, const void* W_r, const float* b,
                            const void* W_gate8, const void* W_gate_sf, const void* W_up8,
                            const void* W_up_sf, const void* W_down, int64_t T, int32_t d,
                            int32_t N, int32_t Z, int32_t K, int32_t I,
                            const float* logit_offset, void* out_host, int64_t chunk_tokens,
                            void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  const Fp8Gates f8{static_cast<const uint8_t*>(W_gate_sf), static_cast<const uint8_t*>(W_up_sf)};
  return forward_host_impl(x_host, W_r, b, W_gate8, W_up8, W_down, T, d, N, Z, K, I,
                           logit_offset, out_host, chunk_tokens, stream, &f8);
}

int moe_zc_fp8_quantize_weights(const void* W, int64_t rows, int32_t cols, void* codes,
                                void* scales, void* stream) {
  if (!W || !codes || !scales || rows < 1 || cols < 1) return MOE_ZC_ERR_INVALID_ARG;
  if (rows % GEMM_BM != 0 || cols % FP8_BK != 0) return MOE_ZC_ERR_UNSUPPORTED;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return MOE_ZC_ERR_UNSUPPORTED;
  CK(launch_fp8_quantize_weights(static_cast<const __nv_bfloat16*>(W), rows, cols,
                                 static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                 static_cast<cudaStream_t>(stream)));
  return MOE_ZC_OK;
}

int moe_zc_forward_host(const void* x_host, const void* W_r, const float* b,
                        const void* W_gate, const void* W_up, const void* W_down, int64_t T,
                        int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I,
                        const float* logit_offset, void* out_host, int64_t chunk_tokens,
                        void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  return forward_host_impl(x_host, W_r, b, W_gate, W_up, W_down, T, d, N, Z, K, I, logit_offset,
                           out_host, chunk_tokens, stream);
}

int moe_zc_synchronize(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int s = get_ctx(&c);
  if (s != MOE_ZC_OK) return s;
  return sync_impl(*c);
}

int moe_zc_expert_load(int32_t* out_counts) {
  if (!out_counts) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int s = get_ctx(&c);
  if (s != MOE_ZC_OK) return s;
  if ((s = sync_impl(*c)) != MOE_ZC_OK) return s;
  CK(cudaMemcpy(out_counts, c->counts_total ? c->cnt_total.p : c->cnt.p,
                sizeof(int32_t) * (c->N + c->Z), cudaMemcpyDeviceToHost));
  return MOE_ZC_OK;
}

int moe_zc_last_routing(int32_t* idx, float* gate) {
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int s = get_ctx(&c);
  if (s != MOE_ZC_OK) return s;
  if ((s = sync_impl(*c)) != MOE_ZC_OK) return s;
  const size_t n = static_cast<size_t>(c->T) * c->K;
  if (n == 0) return MOE_ZC_OK;
  if (idx) CK(cudaMemcpy(idx, c->idx.p, n * sizeof(int32_t), cudaMemcpyDeviceToHost));
  if (gate) CK(cudaMemcpy(gate, c->gate.p, n * sizeof(float), cudaMemcpyDeviceToHost));
  return MOE_ZC_OK;
}

int moe_zc_last_expert(int32_t e, int32_t max_rows, int32_t* n_rows, int32_t* tokens, void* H,
                       void* Y) {
  if (!n_rows || max_rows < 0) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int s = get_ctx(&c);
  if (s != MOE_ZC_OK) return s;
  if ((s = sync_impl(*c)) != MOE_ZC_OK) return s;
  if (e < 0 || e >= c->N) return MOE_ZC_ERR_INVALID_ARG;
  int cnt = 0, off = 0;
  if (c->T > 0) {
    CK(cudaMemcpy(&cnt, static_cast<int*>(c->cnt.p) + e, sizeof(int), cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(&off, static_cast<int*>(c->grp_off.p) + e, sizeof(int),
                  cudaMemcpyDeviceToHost));
  }
  *n_rows = cnt;
  const int n = cnt < max_rows ? cnt : max_rows;
  if (n == 0) return MOE_ZC_OK;
  if (tokens) {
    const size_t pairs = static_cast<size_t>(c->T) * c->K;
    std::vector<int32_t> sl(pairs);
    CK(cudaMemcpy(sl.data(), c->slot.p, pairs * sizeof(int32_t), cudaMemcpyDeviceToHost));
    for (size_t i = 0; i < pairs; ++i) {
      const int r = sl[i] - off;
      if (sl[i] >= 0 && r >= 0 && r < n) tokens[r] = static_cast<int32_t>(i / c->K);
    }
  }
  if (H)
    CK(cudaMemcpy(H, static_cast<const char*>(c->H.p) + static_cast<size_t>(off) * c->I * 2,
                  static_cast<size_t>(n) * c->I * 2, cudaMemcpyDeviceToHost));
  if (Y)
    CK(cudaMemcpy(Y, static_cast<const char*>(c->Y.p) + static_cast<size_t>(off) * c->d * 2,
                  static_cast<size_t>(n) * c->d * 2, cudaMemcpyDeviceToHost));
  return MOE_ZC_OK;
}

int moe_zc_reserve(int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I) {
  if (T < 0 || d <= 0 || N < 0 || Z < 0 || K < 1 || N + Z < 1 || K > N + Z)
    return MOE_ZC_ERR_INVALID_ARG;
  if (N > 0 && I <= 0) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int s = get_ctx(&c);
  if (s != MOE_ZC_OK) return s;
  return reserve_impl(*c, T, d, N, Z, K, N > 0 ? I : 128);
}

void moe_zc_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int prev = 0;
  cudaGetDevice(&prev);
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    Ctx& c = g_ctx[dev];
    if (!c.init) continue;
    cudaSetDevice(dev);
    cudaDeviceSynchronize();
    Buf* bufs[] = {&c.logits, &c.idx,     &c.gate,    &c.zsum,      &c.slot,
                   &c.cnt,    &c.fill,    &c.grp_off, &c.grp_ttp,   &c.Xp,
                   &c.H,      &c.Y,       &c.err,     &c.xin[0],    &c.xin[1],
                   &c.yout[0], &c.yout[1], &c.cnt_total, &c.Xp8,     &c.sfx,
                   &c.grp_ttp8};
    for (Buf* b : bufs) {
      if (b->p) cudaFree(b->p);
      *b = Buf{};
    }
    if (c.done) cudaEventDestroy(c.done);
    for (int i = 0; i < 2; ++i) {
      if (c.ev_in[i]) cudaEventDestroy(c.ev_in[i]);
      if (c.ev_comp[i]) cudaEventDestroy(c.ev_comp[i]);
      if (c.ev_out[i]) cudaEventDestroy(c.ev_out[i]);
    }
    if (c.ev_start) cudaEventDestroy(c.ev_start);
    if (c.s_in) cudaStreamDestroy(c.s_in);
    if (c.s_out) cudaStreamDestroy(c.s_out);
    c = Ctx{};
  }
  cudaSetDevice(prev);
}

const char* moe_zc_status_string(int status) {
  switch (status) {
    case MOE_ZC_OK: return "ok";
    case MOE_ZC_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ZC_ERR_UNSUPPORTED: return "unsupported size, alignment or device";
    case MOE_ZC_ERR_CUDA: return "CUDA call failed";
    case MOE_ZC_ERR_OOM: return "workspace allocation failed";
    case MOE_ZC_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ZC_ERR_NO_RESULT: return "no forward has run on this device";
    default: return "unknown status";
  }
}

int moe_zc_profile(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ZC_ERR_CUDA;
  if (enable && g_prof.created && g_prof.device != dev) return MOE_ZC_ERR_UNSUPPORTED;
  if (enable && !g_prof.created) {
    for (int r = 0; r < kRing; ++r)
      for (int i = 0; i <= kStages; ++i)
        if (cudaEventCreate(&g_prof.ev[r][i]) != cudaSuccess) return MOE_ZC_ERR_CUDA;
    g_prof.created = true;
    g_prof.device = dev;
  }
  g_prof.on = enable != 0;
  g_prof.n = 0;
  return MOE_ZC_OK;
}

int moe_zc_profile_read(float* stage_ms, int32_t max_stages, int32_t* n_forwards) {
  if (!stage_ms || !n_forwards || max_stages < 0) return MOE_ZC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  *n_forwards = g_prof.n;
  const int ns = max_stages < kStages ? max_stages : kStages;
  for (int i = 0; i < ns; ++i) stage_ms[i] = 0.f;
  if (g_prof.n == 0) return MOE_ZC_OK;
  CK(cudaEventSynchronize(g_prof.ev[g_prof.n - 1][kStages]));
  for (int r = 0; r < g_prof.n; ++r)
    for (int i = 0; i < ns; ++i) {
      float ms = 0.f;
      CK(cudaEventElapsedTime(&ms, g_prof.ev[r][i], g_prof.ev[r][i + 1]));
      stage_ms[i] += ms;
    }
  return MOE_ZC_OK;
}

const char* moe_zc_stage_name(int32_t i) {
  return (i >= 0 && i < kStages) ? kStageNames[i] : nullptr;
}

int moe_zc_plan(int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I, int32_t sms,
                int32_t resident_blocks, moe_zc_launch_plan* plan) {
  if (!plan || sms < 1) return MOE_ZC_ERR_INVALID_ARG;
  const void* f = reinterpret_cast<const void*>(16);   // stand-ins for the device pointers
  const int s = check_args(f, f, static_cast<const float*>(f), f, f, f, T, d, N, Z, K, I,
                           nullptr, f);
  if (s != MOE_ZC_OK) return s;
  Plan pl;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    pl = make_plan(T, d, N, Z, K, N > 0 ? I : 128, sms, resident_blocks);
  }
  plan->kernels = pl.kernels;
  plan->router_grid = static_cast<int32_t>(pl.router_grid);
  plan->router_token_tile = pl.rp.tok_tile;
  plan->router_k_slices = pl.rp.splits;
  plan->expert_gemms_one_grid = pl.one_grid ? 1 : 0;
  plan->expert_grid = static_cast<int32_t>(pl.one_grid ? pl.fused_grid : pl.gateup_grid);
  plan->one_grid_step = pl.step ? 1 : 0;
  return MOE_ZC_OK;
}

void moe_zc_test_one_grid(int32_t mode) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_one_grid_mode = (mode == 1 || mode == 2) ? mode : 0;
}

void moe_zc_test_inject(int32_t fail_allocs, int64_t wait_limit) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_fail_allocs = fail_allocs > 0 ? fail_allocs : 0;
  g_wait_ns_next = wait_limit > 0 ? wait_limit : 0;
}

}  // extern "C"
