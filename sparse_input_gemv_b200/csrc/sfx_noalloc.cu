// sfx_sparse_gemv_noalloc: the input-sparse GEMV for callers that cannot
// allocate device memory.
//
// sfx_sparse_gemv needs a caller-provided workspace for its split-K partial
// sums, arrival counters and status word. Some callers have no way to provide
// one: a plugin behind a fixed C interface that hands over only its inputs and
// outputs, or code inside a host framework that owns every byte of device
// memory through its own pool and forbids side allocations (cudaMalloc also
// synchronises the device, which latency-critical decode loops cannot
// afford). This variant keeps its scratch in a file-scope device array
// instead, so the caller passes inputs and outputs only.
//
// The array is kNoAllocScratchBytes (4 MiB) per GPU, held by every GPU that
// loads this library until the process exits. Calls that need more partial
// sums than fit are rejected with SFX_ERR_UNSUPPORTED before any launch.
#include "sfx_common.cuh"
#include "sfx_internal.h"

#include <mutex>

namespace sfx {

constexpr size_t kNoAllocScratchBytes = 4u << 20;

// Layout: [status word + pad: 256 B][arrival counters: kCounterSlots int32][partials].
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SFX_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SFX_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SFX_OK;
}

}  // namespace
}  // namespace sfx

using namespace sfx;

extern "C" int sfx_sparse_gemv_noalloc(const void* x, int xdt, int B, int K, const void* W,
                                       int wdt, int N, float t, const int32_t* idx,
                                       const int32_t* cnt, void* y, int ydt, int flags,
                                       void* stream) {
  if (!x || !W || !y || B < 1 || B > 16 || K < 1 || N < 8) return SFX_ERR_ARG;
  if (idx && (!cnt || B != 1)) return SFX_ERR_ARG;
  if ((flags & SFX_FLAG_GELU) && (flags & SFX_FLAG_GELU_TANH)) return SFX_ERR_ARG;
  if ((flags & SFX_FLAG_SWIGLU) && (flags & (SFX_FLAG_GELU | SFX_FLAG_GELU_TANH))) return SFX_ERR_ARG;
  if (!(wdt == SFX_F16 || wdt == SFX_BF16) || !(xdt == wdt || xdt == SFX_F32) ||
      !(ydt == SFX_F16 || ydt == SFX_BF16 || ydt == SFX_F32))
    return SFX_ERR_DTYPE;
  if ((flags & SFX_FLAG_SWIGLU) && ydt != SFX_F32) return SFX_ERR_DTYPE;
  if (N % 8 != 0 || (reinterpret_cast<uintptr_t>(W) & 15u) != 0) return SFX_ERR_ALIGN;
  if (kWsHeader + gemv_workspace_bytes(K, N, B) > kNoAllocScratchBytes)
    return SFX_ERR_UNSUPPORTED;  // partial sums would not fit in the fixed scratch
  const GemvPlan plan = plan_gemv(K, N, B, idx != nullptr);

  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != SFX_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the status word and every
  // arrival counter must start at zero, whichever kernel (and so whichever
  // tile count) the previous call or this one launches, so the whole header
  // (16.6 KB) is cleared on the caller's stream.
  if (cudaMemsetAsync(scratch, 0, kWsHeader, s) != cudaSuccess) return SFX_ERR_CUDA;

  GemvArgs a = {};
  a.x = x;
  a.W = W;
  a.y = y;
  a.idx = idx;
  a.cnt = cnt;
  a.bitmap_out = nullptr;
  a.status = reinterpret_cast<unsigned*>(scratch);
  a.counters = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(scratch) + kWsStatusBytes);
  a.partials = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(scratch) + kWsHeader);
  a.K = K;
  a.N = N;
  a.B = B;
  a.ydt = ydt;
  a.epi = (flags & SFX_FLAG_SWIGLU) ? EPI_SWIGLU
        : (flags & SFX_FLAG_GELU)   ? EPI_GELU
        : (flags & SFX_FLAG_GELU_TANH) ? EPI_GELU_TANH
                                       : EPI_NONE;
  a.union_mask = (flags & SFX_FLAG_UNION_MASK) ? 1 : 0;
  a.no_tc = (flags & SFX_FLAG_CUDA_CORES) ? 1 : 0;
  a.t = t;
  a.wait_ns = wait_limit_ns();
  return launch_sparse_gemv(wdt, xdt, plan, a, s, false);
}
