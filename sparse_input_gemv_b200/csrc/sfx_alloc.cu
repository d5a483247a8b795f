// Block-wise greedy sparsity allocation ("TEAL: Training-Free Activation
// Sparsity in Large Language Models", slide 10): every block starts dense;
// each round measures, for every block, how much its l2 activation error
// would grow if its sparsity went one step up, and raises the block whose
// error grows least -- per unit of model-wide sparsity the step buys, since
// blocks weigh differently in it -- until the model-wide sparsity reaches
// the target.
//
// sfx_block_error_curve measures a block's error curve on the GPU: for each
// sparsity level, the threshold calibrated on the block's own draws (the exact
// radix selection of sfx_calibrate_thresholds), the block output of those
// draws through the sparse GEMV, and the l2 norm of its change from the dense
// output, summed in fp64 in a fixed order. sfx_greedy_allocate runs the greedy
// rounds on the host.
#include "sfx_common.cuh"
#include "sfx_internal.h"

#include <cmath>
#include <vector>

namespace sfx {

constexpr int kErrBlocks = 148;
constexpr int kErrThreads = 256;
constexpr int kErrChunk = 16;  // draws per GEMV launch

// Sum of (a - b)^2 over n fp32 values: each block writes its fp64 partial
// (the grid size is fixed, so the summation order is too).
__global__ void __launch_bounds__(kErrThreads) sqdiff_partial_kernel(const float* a, const float* b,
                                                                     long long n, double* out) {
  __shared__ double sw[kErrThreads / 32];
  double s = 0.0;
  for (long long i = (long long)blockIdx.x * kErrThreads + threadIdx.x; i < n;
       i += (long long)gridDim.x * kErrThreads) {
    const double d = (double)a[i] - (double)b[i];
    s += d * d;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) sw[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kErrThreads / 32; ++w) t += sw[w];
    out[blockIdx.x] = t;
  }
}

// err2[j] = the sum of the partials of level j, in order (one thread per level).
__global__ void sum_partials_kernel(const double* part, int per_level, int P, double* err2) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= P) return;
  double t = 0.0;
  for (int i = 0; i < per_level; ++i) t += part[(long long)j * per_level + i];
  err2[j] = t;
}

namespace {

size_t r256(size_t v) { return (v + 255) / 256 * 256; }

struct CurveLayout {
  size_t gemv, calib, ydense, yp, part, err, total;
};

CurveLayout curve_layout(long long S, long long K, long long N, int xdt, int P) {
  CurveLayout L;
  const long long chunks = (S + kErrChunk - 1) / kErrChunk;
  L.gemv = 0;
  L.calib = L.gemv + r256(sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, kErrChunk, K, N, xdt, 0, 0));
  L.ydense = L.calib + r256(sfx_workspace_bytes(SFX_OP_CALIBRATE, S, K, P, xdt, 0, 0));
  L.yp = L.ydense + r256((size_t)S * N * 4);
  L.part = L.yp + r256((size_t)kErrChunk * N * 4);
  L.err = L.part + r256((size_t)P * chunks * kErrBlocks * 8);
  L.total = L.err + r256((size_t)P * 8);
  return L;
}

}  // namespace

size_t error_curve_workspace_bytes(long long S, long long K, long long N, int xdt, int P) {
  if (S < 1 || K < 1 || N < 8 || P < 1 || P > 64) return 0;
  return curve_layout(S, K, N, xdt, P).total;
}

}  // namespace sfx

using namespace sfx;

extern "C" {

int sfx_block_error_curve(const void* calib, int xdt, long long S, long long K, const void* W,
                          int wdt, long long N, const double* levels, int P, double* err_out,
                          float* thr_out, void* ws, size_t ws_bytes, void* stream) {
  if (!calib || !W || !levels || !err_out || S < 1 || K < 1 || N < 8 || P < 1 || P > 64 ||
      K > 0x7fffffffLL || N > 0x7fffffffLL)
    return SFX_ERR_ARG;
  if (!(wdt == SFX_F16 || wdt == SFX_BF16) || !(xdt == wdt || xdt == SFX_F32)) return SFX_ERR_DTYPE;
  if (N % 8 != 0 || (reinterpret_cast<uintptr_t>(W) & 15u) != 0) return SFX_ERR_ALIGN;
  const CurveLayout L = curve_layout(S, K, N, xdt, P);
  if (!ws || ws_bytes < L.total) return SFX_ERR_WORKSPACE;
  unsigned char* base = reinterpret_cast<unsigned char*>(ws);
  void* ws_gemv = base + L.gemv;
  void* ws_calib = base + L.calib;
  float* ydense = reinterpret_cast<float*>(base + L.ydense);
  float* yp = reinterpret_cast<float*>(base + L.yp);
  double* part = reinterpret_cast<double*>(base + L.part);
  double* err2 = reinterpret_cast<double*>(base + L.err);
  const size_t gemv_bytes = L.calib - L.gemv, calib_bytes = L.ydense - L.calib;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // thresholds of every level (exact selection; returns on the host)
  std::vector<float> thr(P);
  int rc = sfx_calibrate_thresholds(calib, xdt, S, K, levels, P, thr.data(), ws_calib, calib_bytes,
                                    stream);
  if (rc != SFX_OK) return rc;
  const size_t xrow = (size_t)K * (xdt == SFX_F32 ? 4 : 2);
  const unsigned char* xb = reinterpret_cast<const unsigned char*>(calib);
  const long long chunks = (S + kErrChunk - 1) / kErrChunk;
  // dense outputs of every draw
  for (long long c = 0; c < chunks; ++c) {
    const int B = (int)std::min<long long>(kErrChunk, S - c * kErrChunk);
    rc = sfx_sparse_gemv(xb + (size_t)c * kErrChunk * xrow, xdt, B, (int)K, W, wdt, (int)N,
                         -INFINITY, nullptr, nullptr, ydense + (size_t)c * kErrChunk * N, SFX_F32,
                         0, nullptr, ws_gemv, gemv_bytes, stream);
    if (rc != SFX_OK) return rc;
  }
  // each level: the masked outputs, their squared change, summed per block
  for (int j = 0; j < P; ++j) {
    for (long long c = 0; c < chunks; ++c) {
      const int B = (int)std::min<long long>(kErrChunk, S - c * kErrChunk);
      rc = sfx_sparse_gemv(xb + (size_t)c * kErrChunk * xrow, xdt, B, (int)K, W, wdt, (int)N,
                           thr[j], nullptr, nullptr, yp, SFX_F32, 0, nullptr, ws_gemv, gemv_bytes,
                           stream);
      if (rc != SFX_OK) return rc;
      sqdiff_partial_kernel<<<kErrBlocks, kErrThreads, 0, s>>>(
          yp, ydense + (size_t)c * kErrChunk * N, (long long)B * N,
          part + ((size_t)j * chunks + c) * kErrBlocks);
      if (cudaGetLastError() != cudaSuccess) return SFX_ERR_CUDA;
    }
  }
  sum_partials_kernel<<<(P + 63) / 64, 64, 0, s>>>(part, (int)(chunks * kErrBlocks), P, err2);
  if (cudaGetLastError() != cudaSuccess) return SFX_ERR_CUDA;
  std::vector<double> e2(P);
  if (cudaMemcpyAsync(e2.data(), err2, (size_t)P * 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SFX_ERR_CUDA;
  for (int j = 0; j < P; ++j) {
    err_out[j] = std::sqrt(e2[j]);
    if (thr_out) thr_out[j] = thr[j];
  }
  return SFX_OK;
}

int sfx_greedy_allocate(const double* err, const double* weights, int M, int P, double step,
                        double target, int* level_out) {
  if (!err || !weights || !level_out || M < 1 || P < 1 || !(step > 0.0)) return SFX_ERR_ARG;
  double wsum = 0.0;
  for (int i = 0; i < M; ++i) {
    if (!(weights[i] >= 0.0)) return SFX_ERR_ARG;
    wsum += weights[i];
  }
  if (!(wsum > 0.0)) return SFX_ERR_ARG;
  std::vector<int> lvl(M, 0);
  const auto overall = [&]() {
    double acc = 0.0;
    for (int i = 0; i < M; ++i) acc += weights[i] * (lvl[i] * step);
    return acc / wsum;
  };
  while (overall() < target - 1e-12) {
    int pick = -1;
    double least = INFINITY;
    for (int i = 0; i < M; ++i) {
      if (lvl[i] + 1 >= P || !(weights[i] > 0.0)) continue;  // top level, or buys nothing
      // error growth per unit of model-wide sparsity the step buys
      const double growth =
          (err[(size_t)i * P + lvl[i] + 1] - err[(size_t)i * P + lvl[i]]) / weights[i];
      if (growth < least) {  // strict: equal growths keep the lower block
        least = growth;
        pick = i;
      }
    }
    if (pick < 0) break;
    ++lvl[pick];
  }
  for (int i = 0; i < M; ++i) level_out[i] = lvl[i];
  return SFX_OK;
}

}  // extern "C"
