// route_noalloc.cu -- routing stage without any device allocation.
//
// Who needs this: a caller that must not let a library call cudaMalloc once
// it is running.  Examples are a serving process that carves all device
// memory into its own pool at start-up (a cudaMalloc later either fails or
// eats into memory the pool has promised elsewhere), and a process running
// under a hard device-memory cap where a surprise allocation can fail at an
// arbitrary step.  cudaMalloc may also synchronise the device, which such
// callers cannot afford in the middle of a step.
//
// moe_zc_route_noalloc runs the same two kernels as the routing part of
// moe_zc_forward (router GEMM on the tensor cores, then softmax + bias +
// top-K + expert-load histogram), but the fp32 logits and per-token
// zero-gate sums they pass between them live in one file-scope device array
// of fixed size (kStaticScratchBytes) instead of the per-device workspace.
// Every GPU that loads this library holds that array until the process exits.
//
// In host code the array's name is only a host-side stand-in for the symbol,
// not a device address: handing it to a kernel would fault or, where the GPU
// can reach host memory, silently use the wrong memory.  So the first call
// on each device (with that device current) looks the real address up with
// cudaGetSymbolAddress and keeps it; make that first call before any stream
// capture.  All calls share the array and it keeps the last call's contents:
// the entry point clears what must start at zero (the caller's counts and
// status word), and calls whose work overlaps on the GPU (two streams, or two
// threads) race on the array -- serialise them.  The status word is the
// caller's (required): a bounded device wait that runs out is reported there
// and nowhere else.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe_zc.h"
#include "kernels.cuh"

namespace {

using namespace moezc;

constexpr size_t kStaticScratchBytes = MOE_ZC_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDev = 16;
constexpr long long kNoallocWaitNs = 2000000000LL;   // bound of every device wait

static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

struct NoallocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch
  int sms = 0;
};
NoallocDevice g_noalloc_dev[kMaxDev];
std::mutex g_noalloc_mu;

// Once per device, with that device current: the array's device address.
int noalloc_setup(NoallocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return MOE_ZC_ERR_CUDA;
  NoallocDevice& s = g_noalloc_dev[dev];
  if (!s.ready) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    if (major != 10) return MOE_ZC_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ZC_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MOE_ZC_ERR_CUDA;
    }
    s.scratch = static_cast<unsigned char*>(p);
    s.ready = true;
  }
  *out = &s;
  return MOE_ZC_OK;
}

// 2-D bf16 tensor map [rows, k], box [box_rows, 64], 128-byte swizzle.
bool noalloc_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t k, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(GEMM_BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" int moe_zc_route_noalloc(const void* x, const void* W_r, const float* b,
                                    const float* logit_offset, int64_t T, int32_t d, int32_t N,
                                    int32_t Z, int32_t K, int32_t* idx, float* gate,
                                    int32_t* counts, int32_t* dev_status, void* stream) {
  if (!W_r || !b || !counts || !dev_status) return MOE_ZC_ERR_INVALID_ARG;
  if (T < 0 || N < 0 || Z < 0 || d <= 0) return MOE_ZC_ERR_INVALID_ARG;
  const int64_t E = static_cast<int64_t>(N) + Z;
  if (E < 1 || K < 1 || K > E) return MOE_ZC_ERR_INVALID_ARG;
  if (T > 0 && (!x || !idx || !gate)) return MOE_ZC_ERR_INVALID_ARG;
  if (K > MOE_ZC_MAX_K || E > MOE_ZC_MAX_E || d % GEMM_BK != 0) return MOE_ZC_ERR_UNSUPPORTED;
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al(x) || !al(W_r) || !al(b) || !al(logit_offset)) return MOE_ZC_ERR_UNSUPPORTED;
  // scratch: logits [T, E] fp32, then zero-gate sums [T] fp32
  const size_t logits_bytes = round256(static_cast<size_t>(T) * E * sizeof(float));
  const size_t zsum_bytes = round256(static_cast<size_t>(T) * sizeof(float));
  if (logits_bytes + zsum_bytes > kStaticScratchBytes) return MOE_ZC_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocDevice* s = nullptr;
  int st = noalloc_setup(&s);
  if (st != MOE_ZC_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  float* logits = reinterpret_cast<float*>(s->scratch);
  float* zsum = reinterpret_cast<float*>(s->scratch + logits_bytes);
  int* err = dev_status;
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, cs) != cudaSuccess ||
      cudaMemsetAsync(err, 0, sizeof(int32_t), cs) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ZC_ERR_CUDA;
  }
  // (the error-path test hook may shorten the waits of this call)
  const long long injected = take_injected_wait_ns();
  if (T == 0) return MOE_ZC_OK;

  CUtensorMap mWr, mX;
  if (!noalloc_map(&mWr, W_r, E, d, GEMM_BM) || !noalloc_map(&mX, x, T, d, GEMM_B_BOX_ROWS))
    return MOE_ZC_ERR_CUDA;
  GemmParams pr{};
  pr.G = 1;
  pr.T = static_cast<int>(T);
  pr.ksteps = d / GEMM_BK;
  pr.mblocks = static_cast<int>((E + 2 * GEMM_BM - 1) / (2 * GEMM_BM));
  pr.a_rows = static_cast<int>(E);
  pr.out = logits;
  pr.out_ld = static_cast<int>(E);
  pr.err = err;
  pr.wait_ns = injected > 0 ? injected : kNoallocWaitNs;
  const int64_t tiles = ((T + GEMM_BN - 1) / GEMM_BN) * pr.mblocks;
  if (launch_gemm(MODE_ROUTER, mWr, mWr, mX, mX, pr, static_cast<int>(tiles < s->sms ? tiles : s->sms),
                  cs) != cudaSuccess ||
      launch_route(logits, b, logit_offset, T, static_cast<int>(E), N, K, idx, gate, zsum, counts,
                   cs) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ZC_ERR_CUDA;
  }
  return MOE_ZC_OK;
}
