// C ABI of the activation-sparse GEMV / FFN library: argument validation,
// workspace carving and kernel launches. See include/sfx.h for the contract of
// each entry point.
#include "sfx_common.cuh"
#include "sfx_internal.h"

#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

using namespace sfx;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
size_t round256(size_t v) { return (v + 255) / 256 * 256; }
bool valid_dtype(int dt) { return dt == SFX_F16 || dt == SFX_BF16 || dt == SFX_F32; }

// 1-based rank r = ceil(p n); a product within 1e-9 n of an integer counts as
// that integer, so decimal sparsities give their intended rank.
long long calibration_rank(double p, long long n) {
  const double v = p * (double)n;
  const double r = std::nearbyint(v);
  if (std::fabs(v - r) <= 1e-9 * (double)(n > 1 ? n : 1)) return (long long)r;
  return (long long)std::ceil(v);
}

__global__ void pack_gate_up_kernel(const uint16_t* Wg, const uint16_t* Wu, long long d,
                                    long long ffn, uint16_t* Wgu) {
  const long long total = d * ffn;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long i = e / ffn, j = e - i * ffn;
    Wgu[i * 2 * ffn + 2 * j] = Wg[e];
    Wgu[i * 2 * ffn + 2 * j + 1] = Wu[e];
  }
}

size_t ffn_workspace_body(int B, int d, int ffn) {
  const size_t h = round256((size_t)B * ffn * 4);
  const size_t g1 = gemv_workspace_bytes(d, 2LL * ffn, B);
  const size_t g2 = gemv_workspace_bytes(ffn, d, B);
  return h + (g1 > g2 ? g1 : g2);
}

// Split-K counters live in the workspace header; partial sums at `body`.
void carve_gemv(void* ws, unsigned char* body, GemvArgs& a) {
  a.counters = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(ws) + kWsStatusBytes);
  a.partials = reinterpret_cast<float*>(body);
}

}  // namespace

namespace sfx {

static constexpr int kPlanKeys = SFX_PLAN_MOE_CHUNK + 1;
static std::atomic<unsigned long long> g_wait_limit_ns{0};

unsigned long long wait_limit_ns() {
  const unsigned long long v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v ? v : kWaitLimitNs;
}
static std::atomic<int> g_plan_override[kPlanKeys];

int plan_override(int key) {
  return (key >= 0 && key < kPlanKeys) ? g_plan_override[key].load(std::memory_order_relaxed) : 0;
}

int launch_pack_gate_up(const void* W_g, const void* W_u, int, int d, int ffn, void* W_gu,
                        cudaStream_t s) {
  pack_gate_up_kernel<<<sm_count() * 4, 256, 0, s>>>(
      reinterpret_cast<const uint16_t*>(W_g), reinterpret_cast<const uint16_t*>(W_u), d, ffn,
      reinterpret_cast<uint16_t*>(W_gu));
  return cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}
int ensure_dynamic_smem(const void* kern, size_t bytes, size_t* configured) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (bytes <= *configured) return SFX_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return SFX_ERR_CUDA;
  *configured = bytes;
  return SFX_OK;
}

}  // namespace sfx

extern "C" {

const char* sfx_status_string(int st) {
  switch (st) {
    case SFX_OK: return "ok";
    case SFX_ERR_ARG: return "invalid argument";
    case SFX_ERR_DTYPE: return "unsupported dtype";
    case SFX_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case SFX_ERR_WORKSPACE: return "workspace missing or too small";
    case SFX_ERR_CUDA: return "CUDA runtime error";
    case SFX_ERR_DEVICE: return "device status flag raised";
    case SFX_ERR_UNSUPPORTED: return "shape outside the implemented range";
  }
  return "unknown status";
}

int sfx_device_sm_count(void) { return sm_count(); }

const char* sfx_build_info(void) { return "sfx 0.1 sm_100a"; }

int sfx_gemv_plan(int B, long long K, long long N, int flags, int idx_mode, int* out) {
  if (!out || B < 1 || B > 16 || K < 1 || N < 8 || (idx_mode && B != 1)) return SFX_ERR_ARG;
  // the choice launch_sparse_gemv makes: the batch union for union_min_batch()
  // tokens or more in threshold mode unless SFX_FLAG_CUDA_CORES, else CUDA cores
  const bool uni = B >= union_min_batch() && !idx_mode && !(flags & SFX_FLAG_CUDA_CORES);
  const GemvPlan p = uni ? plan_union_tc(K, N) : plan_gemv(K, N, B, idx_mode != 0);
  out[0] = p.kind;
  out[1] = p.NT;
  out[2] = p.S;
  out[3] = p.col_tiles;
  out[4] = p.kind == 2 ? p.chunks : 0;
  out[5] = (p.kind == 0 && idx_mode) ? p.list_cap : p.slice;
  return SFX_OK;
}

int sfx_set_plan_override(int key, int value) {
  bool ok = value == 0;
  switch (key) {
    case SFX_PLAN_UNION_KERNEL: ok = ok || value == 1 || value == 2; break;
    case SFX_PLAN_UNION_MIN_B: ok = ok || (value >= 2 && value <= 16); break;
    case SFX_PLAN_GEMV_NT: ok = ok || value == 256 || value == 512 || value == 1024 || value == 2048; break;
    case SFX_PLAN_GEMV_S:
    case SFX_PLAN_UNION_S: ok = ok || value >= 1; break;
    case SFX_PLAN_MMA_CHUNKS: ok = ok || value == 1 || value == 2 || value == 4 || value == 8; break;
    case SFX_PLAN_DENSE: ok = ok || (value >= 1 && value <= 3); break;
    case SFX_PLAN_TEST_STALL: ok = ok || value == 1; break;
    case SFX_PLAN_MOE_CHUNK: ok = ok || (value >= 16 && value <= 64); break;
    default: return SFX_ERR_ARG;
  }
  if (!ok) return SFX_ERR_ARG;
  g_plan_override[key].store(value, std::memory_order_relaxed);
  return SFX_OK;
}

int sfx_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return SFX_OK;
}

size_t sfx_workspace_bytes(int op, long long a, long long b, long long c, long long d,
                           long long e, long long f) {
  switch (op) {
    case SFX_OP_CALIBRATE:
      if (a < 1 || b < 1 || c < 1) return 0;
      return kWsHeader + calib_workspace_bytes(a, b, (int)c, (int)d);
    case SFX_OP_MASK_COMPACT:
      if (a < 1 || b < 1) return 0;
      return kWsHeader + mask_workspace_bytes((int)a, (int)b, (int)c);
    case SFX_OP_SPARSE_GEMV:
      if (a < 1 || b < 1 || c < 8) return 0;
      return kWsHeader + gemv_workspace_bytes(b, c, (int)a);
    case SFX_OP_FFN_SWIGLU:
      if (a < 1 || b < 8 || c < 4) return 0;
      return kWsHeader + ffn_workspace_body((int)a, (int)b, (int)c);
    case SFX_OP_MOE:
      if (a < 1 || b < 8 || c < 1 || d < 8 || e < 1) return 0;
      return kWsHeader + moe_workspace_bytes((int)a, (int)b, (int)c, (int)d, (int)e, (int)f);
    case SFX_OP_STATIC_FFN:
      if (a < 1 || b < 8 || c < 1) return 0;
      return kWsHeader + static_ffn_workspace_bytes((int)a, (int)b, (int)c);
    case SFX_OP_ERROR_CURVE:
      return error_curve_workspace_bytes(a, b, c, (int)d, (int)e);
  }
  return 0;
}

int sfx_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeader) return SFX_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, ws_bytes, as_stream(stream)) == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

int sfx_check_device_status(void* ws, unsigned int* bits_out, void* stream) {
  if (!ws) return SFX_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  unsigned bits = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SFX_ERR_CUDA;
  if (cudaMemcpy(&bits, ws, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess) return SFX_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  if (bits) {
    if (cudaMemset(ws, 0, sizeof(bits)) != cudaSuccess) return SFX_ERR_CUDA;
    return SFX_ERR_DEVICE;
  }
  return SFX_OK;
}

int sfx_calibrate_thresholds(const void* calib, int dt, long long S, long long K,
                             const double* sparsities, int P, float* thresholds_out, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!calib || !sparsities || !thresholds_out || S < 1 || K < 1 || P < 1 || P > 64)
    return SFX_ERR_ARG;
  if (!valid_dtype(dt)) return SFX_ERR_DTYPE;
  if (!ws || ws_bytes < sfx_workspace_bytes(SFX_OP_CALIBRATE, S, K, P, dt, 0, 0))
    return SFX_ERR_WORKSPACE;
  const long long n = S * K;
  std::vector<long long> ranks;
  std::vector<int> which;
  for (int j = 0; j < P; ++j) {
    const double p = sparsities[j];
    if (!(p == p) || p > 1.0) return SFX_ERR_ARG;  // NaN or above 1
    if (p <= 0.0) {
      thresholds_out[j] = -INFINITY;
      continue;
    }
    long long r = calibration_rank(p, n);
    r = r < 1 ? 1 : (r > n ? n : r);
    ranks.push_back(r);
    which.push_back(j);
  }
  if (ranks.empty()) return SFX_OK;
  std::vector<float> out(ranks.size());
  const int rc = run_calibrate(calib, dt, n, ranks.data(), (int)ranks.size(), out.data(),
                               reinterpret_cast<unsigned char*>(ws) + kWsHeader,
                               as_stream(stream));
  if (rc != SFX_OK) return rc;
  for (size_t q = 0; q < which.size(); ++q) thresholds_out[which[q]] = out[q];
  return SFX_OK;
}

int sfx_mask_compact(const void* x, int dt, int B, int K, int sel, float t, int k,
                     const float* score_l, const float* score_g, double lambda,
                     uint32_t* bitmap, int32_t* idx, int32_t* cnt, int32_t* union_idx,
                     int32_t* union_cnt, void* ws, size_t ws_bytes, void* stream) {
  if (B < 1 || B > 64 || K < 1 || !cnt) return SFX_ERR_ARG;
  if (union_idx && !union_cnt) return SFX_ERR_ARG;
  if (!valid_dtype(dt)) return SFX_ERR_DTYPE;
  if (sel == SFX_SEL_THRESHOLD) {
    if (!x) return SFX_ERR_ARG;
  } else if (sel == SFX_SEL_TOPK_GXO || sel == SFX_SEL_TOPK_CGXO) {
    if (!x || !score_l || k < 0 || k > K) return SFX_ERR_ARG;
    if (K > 32768) return SFX_ERR_UNSUPPORTED;
    if (union_idx) return SFX_ERR_UNSUPPORTED;
  } else if (sel == SFX_SEL_TOPK_GLASS) {
    if (!score_l || !score_g || k < 0 || k > K || !(lambda == lambda)) return SFX_ERR_ARG;
  } else {
    return SFX_ERR_ARG;
  }
  if (!ws || ws_bytes < sfx_workspace_bytes(SFX_OP_MASK_COMPACT, B, K, sel, 0, 0, 0))
    return SFX_ERR_WORKSPACE;
  return launch_mask_compact(x, dt, B, K, sel, t, k, score_l, score_g, lambda, bitmap, idx, cnt,
                             union_idx, union_cnt,
                             reinterpret_cast<unsigned char*>(ws) + kWsHeader,
                             reinterpret_cast<unsigned*>(ws), as_stream(stream));
}

}  // extern "C"

namespace {

// Checks shared by the two sparse GEMV entry points, then the launch arguments
// every mode shares; the caller adds its mask source.
int check_gemv(const void* x, int xdt, int B, int K, const void* W, int wdt, int N, void* y,
               int ydt, int flags, void* ws, size_t ws_bytes) {
  if (!x || !W || !y || B < 1 || B > 16 || K < 1 || N < 8) return SFX_ERR_ARG;
  if ((flags & SFX_FLAG_GELU) && (flags & SFX_FLAG_GELU_TANH)) return SFX_ERR_ARG;
  if ((flags & SFX_FLAG_SWIGLU) && (flags & (SFX_FLAG_GELU | SFX_FLAG_GELU_TANH))) return SFX_ERR_ARG;
  if (!(wdt == SFX_F16 || wdt == SFX_BF16) || !(xdt == wdt || xdt == SFX_F32) || !valid_dtype(ydt))
    return SFX_ERR_DTYPE;
  if ((flags & SFX_FLAG_SWIGLU) && ydt != SFX_F32) return SFX_ERR_DTYPE;
  if (N % 8 != 0 || !aligned16(W)) return SFX_ERR_ALIGN;
  if (!ws || ws_bytes < sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, B, K, N, xdt, 0, 0))
    return SFX_ERR_WORKSPACE;
  return SFX_OK;
}

GemvArgs gemv_args(const void* x, int B, int K, const void* W, int N, void* y, int ydt,
                   int flags, void* ws) {
  GemvArgs a = {};
  a.x = x;
  a.W = W;
  a.y = y;
  a.status = reinterpret_cast<unsigned*>(ws);
  carve_gemv(ws, reinterpret_cast<unsigned char*>(ws) + kWsHeader, a);
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
  a.wait_ns = wait_limit_ns();
  return a;
}

}  // namespace

extern "C" {

int sfx_sparse_gemv(const void* x, int xdt, int B, int K, const void* W, int wdt, int N, float t,
                    const int32_t* idx, const int32_t* cnt, void* y, int ydt, int flags,
                    uint32_t* bitmap_out, void* ws, size_t ws_bytes, void* stream) {
  const int rc = check_gemv(x, xdt, B, K, W, wdt, N, y, ydt, flags, ws, ws_bytes);
  if (rc != SFX_OK) return rc;
  if (idx && (!cnt || B != 1)) return SFX_ERR_ARG;
  GemvArgs a = gemv_args(x, B, K, W, N, y, ydt, flags, ws);
  a.idx = idx;
  a.cnt = cnt;
  a.bitmap_out = idx ? nullptr : bitmap_out;
  a.t = t;
  return launch_sparse_gemv(wdt, xdt, plan_gemv(K, N, B, idx != nullptr), a, as_stream(stream),
                            false);
}

int sfx_sparse_gemv_mask(const void* x, int xdt, int B, int K, const void* W, int wdt, int N,
                         const uint32_t* mask, void* y, int ydt, int flags, void* ws,
                         size_t ws_bytes, void* stream) {
  if (!mask) return SFX_ERR_ARG;
  const int rc = check_gemv(x, xdt, B, K, W, wdt, N, y, ydt, flags, ws, ws_bytes);
  if (rc != SFX_OK) return rc;
  GemvArgs a = gemv_args(x, B, K, W, N, y, ydt, flags, ws);
  a.mask_in = mask;
  a.no_tc = 1;  // the mask comes in: the CUDA-core kernel for every batch
  return launch_sparse_gemv(wdt, xdt, plan_gemv(K, N, B, false), a, as_stream(stream), false);
}

int sfx_sparse_ffn_swiglu(const void* x, int dt, int B, int d, int ffn, const void* W_gu,
                          const void* W_d, float t_in, float t_h, void* y, int ydt, float* h_out,
                          uint32_t* bitmap_x_out, uint32_t* bitmap_h_out, int flags, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!x || !W_gu || !W_d || !y || B < 1 || B > 16 || d < 8 || ffn < 4) return SFX_ERR_ARG;
  if (!(dt == SFX_F16 || dt == SFX_BF16) || !valid_dtype(ydt)) return SFX_ERR_DTYPE;
  if (d % 8 != 0 || ffn % 4 != 0 || !aligned16(W_gu) || !aligned16(W_d)) return SFX_ERR_ALIGN;
  if (!ws || ws_bytes < sfx_workspace_bytes(SFX_OP_FFN_SWIGLU, B, d, ffn, dt, 0, 0))
    return SFX_ERR_WORKSPACE;
  unsigned char* body = reinterpret_cast<unsigned char*>(ws) + kWsHeader;
  float* h = h_out ? h_out : reinterpret_cast<float*>(body);
  unsigned char* gbody = body + round256((size_t)B * ffn * 4);
  cudaStream_t s = as_stream(stream);
  const int umask = (flags & SFX_FLAG_UNION_MASK) ? 1 : 0;

  GemvArgs a = {};
  a.x = x;
  a.W = W_gu;
  a.y = h;
  a.bitmap_out = bitmap_x_out;
  a.status = reinterpret_cast<unsigned*>(ws);
  a.K = d;
  a.N = 2LL * ffn;
  a.B = B;
  a.ydt = SFX_F32;
  a.epi = EPI_SWIGLU;
  a.union_mask = umask;
  a.no_tc = (flags & SFX_FLAG_CUDA_CORES) ? 1 : 0;
  a.t = t_in;
  a.wait_ns = wait_limit_ns();
  carve_gemv(ws, gbody, a);
  int rc = launch_sparse_gemv(dt, dt, plan_gemv(a.K, a.N, B, false), a, s, false);
  if (rc != SFX_OK) return rc;

  GemvArgs b = {};
  b.x = h;
  b.W = W_d;
  b.y = y;
  b.bitmap_out = bitmap_h_out;
  b.status = reinterpret_cast<unsigned*>(ws);
  b.K = ffn;
  b.N = d;
  b.B = B;
  b.ydt = ydt;
  b.epi = EPI_NONE;
  b.union_mask = umask;
  b.no_tc = a.no_tc;
  b.t = t_h;
  b.wait_ns = a.wait_ns;
  carve_gemv(ws, gbody, b);
  return launch_sparse_gemv(dt, SFX_F32, plan_gemv(b.K, b.N, B, false), b, s, true);
}

int sfx_pack_gate_up(const void* W_g, const void* W_u, int dt, int d, int ffn, void* W_gu,
                     void* stream) {
  if (!W_g || !W_u || !W_gu || d < 1 || ffn < 1) return SFX_ERR_ARG;
  if (!(dt == SFX_F16 || dt == SFX_BF16)) return SFX_ERR_DTYPE;
  return launch_pack_gate_up(W_g, W_u, dt, d, ffn, W_gu, as_stream(stream));
}

int sfx_moe_expert_sparse(const void* x, int dt, const float* logits, int B, int d, int E,
                          int ffn, int top_k, const void* W_gT, const void* W_upT,
                          const void* W_d, const float* t_e, const void* Ws_gT,
                          const void* Ws_upT, const void* Ws_d, int ffn_shared, void* y, int ydt,
                          float* a_out, int32_t* sel_out, int flags, void* ws, size_t ws_bytes,
                          void* stream) {
  if (!x || !logits || !W_gT || !W_upT || !W_d || !t_e || !y) return SFX_ERR_ARG;
  if (B < 1 || B > 16 || E < 1 || E > 1024 || top_k < 1 || top_k > E || d < 8 || ffn < 8 ||
      (long long)B * d > 98304)
    return SFX_ERR_ARG;
  const bool shared = Ws_gT != nullptr;
  if ((Ws_upT != nullptr) != shared || (Ws_d != nullptr) != shared || (shared && ffn_shared < 8))
    return SFX_ERR_ARG;
  if (!(dt == SFX_F16 || dt == SFX_BF16) || !valid_dtype(ydt)) return SFX_ERR_DTYPE;
  if (d % 8 != 0 || ffn % 8 != 0 || !aligned16(W_gT) || !aligned16(W_upT) || !aligned16(W_d) ||
      !aligned16(x) ||
      (shared && (!aligned16(Ws_gT) || !aligned16(Ws_upT) || !aligned16(Ws_d) ||
                  ffn_shared % 8 != 0)))
    return SFX_ERR_ALIGN;
  const size_t need = sfx_workspace_bytes(SFX_OP_MOE, B, d, E, ffn, top_k, shared ? ffn_shared : 0);
  if (!ws || ws_bytes < need) return SFX_ERR_WORKSPACE;
  return run_moe(x, dt, logits, B, d, E, ffn, top_k, W_gT, W_upT, W_d, t_e, Ws_gT, Ws_upT, Ws_d,
                 shared ? ffn_shared : 0, y, ydt, a_out, sel_out, flags,
                 reinterpret_cast<unsigned char*>(ws) + kWsHeader, need - kWsHeader,
                 as_stream(stream));
}

int sfx_static_ffn(const void* x, int dt, int B, int d, int ffn, const void* W_aT,
                   const void* W_bT, const void* W_d, const int32_t* idx, const int32_t* cnt,
                   int flags, void* y, int ydt, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !W_aT || !W_d || !idx || !cnt || !y) return SFX_ERR_ARG;
  if (B < 1 || B > 16 || d < 8 || ffn < 1 || (long long)B * d > 98304) return SFX_ERR_ARG;
  if (!(dt == SFX_F16 || dt == SFX_BF16) || !valid_dtype(ydt)) return SFX_ERR_DTYPE;
  if (d % 8 != 0 || !aligned16(x) || !aligned16(W_aT) || !aligned16(W_d) ||
      (W_bT && !aligned16(W_bT)))
    return SFX_ERR_ALIGN;
  const size_t need = sfx_workspace_bytes(SFX_OP_STATIC_FFN, B, d, ffn, 0, 0, 0);
  if (!ws || ws_bytes < need) return SFX_ERR_WORKSPACE;
  const int act = (flags & SFX_FLAG_GELU_TANH) ? EPI_GELU_TANH : EPI_GELU;
  return run_static_ffn(x, dt, B, d, ffn, W_aT, W_bT, W_d, idx, cnt, act, y, ydt,
                        reinterpret_cast<unsigned char*>(ws) + kWsHeader,
                        reinterpret_cast<unsigned*>(ws), as_stream(stream));
}

}  // extern "C"
