// Magnitude-threshold calibration ("TEAL: Training-Free Activation Sparsity in
// Large Language Models", slide 8: t_p is chosen on calibration activations so
// that a target fraction p of them is zeroed).
//
// t_p is the r-th smallest pooled magnitude, r = ceil(p n). Non-negative
// floating-point magnitudes order like their bit patterns with the sign bit
// cleared, so the r-th smallest value is found exactly by an MSB-first radix
// selection over those bits:
//  * f16 / bf16: one pass, a 32768-bin histogram of the 15 magnitude bits;
//  * f32: three passes over bits [30:16], [15:8] and [7:0], each later pass
//    histogramming only the values whose higher bits match the bin chosen so
//    far for that p.
// Histograms are privatised in shared memory and merged with global atomics.
#include "sfx_common.cuh"
#include "sfx_internal.h"

#include <vector>

namespace sfx {

constexpr int kCalibThreads = 1024;
constexpr int kMaxP = 64;

template <typename T> __device__ __forceinline__ uint32_t mag_bits(T v);
template <> __device__ __forceinline__ uint32_t mag_bits<__half>(__half v) {
  return (uint32_t)__half_as_ushort(v) & 0x7fffu;
}
template <> __device__ __forceinline__ uint32_t mag_bits<__nv_bfloat16>(__nv_bfloat16 v) {
  return (uint32_t)__bfloat16_as_ushort(v) & 0x7fffu;
}
template <> __device__ __forceinline__ uint32_t mag_bits<float>(float v) {
  return __float_as_uint(v) & 0x7fffffffu;
}

// Pass 1: histogram of (mag >> shift) over 32768 bins (shift 0 for 16-bit
// types, 16 for f32).
template <typename T>
__global__ void __launch_bounds__(kCalibThreads) calib_hist1_kernel(const T* data, long long n,
                                                                    int shift, uint32_t* ghist) {
  extern __shared__ uint32_t sh[];  // 32768 bins
  for (int i = threadIdx.x; i < 32768; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    atomicAdd(&sh[mag_bits<T>(data[e]) >> shift], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < 32768; i += blockDim.x)
    if (sh[i]) atomicAdd(&ghist[i], sh[i]);
}

// Passes 2/3 (f32): per-p 256-bin histogram of ((mag >> shift) & 255) over the
// values with (mag >> (shift + 8)) == prefix[p].
__global__ void __launch_bounds__(kCalibThreads) calib_histp_kernel(const float* data, long long n,
                                                                    int shift, int P,
                                                                    const uint32_t* prefix,
                                                                    uint32_t* ghist) {
  extern __shared__ uint32_t sh[];  // [P * 256] bins, then [P] prefixes
  uint32_t* spre = sh + P * 256;
  for (int i = threadIdx.x; i < P * 256; i += blockDim.x) sh[i] = 0;
  for (int i = threadIdx.x; i < P; i += blockDim.x) spre[i] = prefix[i];
  __syncthreads();
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const uint32_t m = mag_bits<float>(data[e]);
    const uint32_t hi = m >> (shift + 8);
    const uint32_t bin = (m >> shift) & 255u;
    for (int p = 0; p < P; ++p)
      if (hi == spre[p]) atomicAdd(&sh[p * 256 + bin], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < P * 256; i += blockDim.x)
    if (sh[i]) atomicAdd(&ghist[i], sh[i]);
}

// For each p: find the bin c with cum(c-1) < rank_p <= cum(c) in its histogram
// (nbins bins; histogram p at hist + p * hist_stride), append c to prefix[p]
// (prefix = prefix << bits | c) and leave the residual rank in rank[p].
__global__ void __launch_bounds__(kCalibThreads) calib_select_kernel(const uint32_t* hist,
                                                                     int nbins, int hist_stride,
                                                                     int bits, int P,
                                                                     long long* rank,
                                                                     uint32_t* prefix) {
  __shared__ unsigned long long s_wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (nbins + kCalibThreads - 1) / kCalibThreads;
  for (int p = 0; p < P; ++p) {
    const uint32_t* h = hist + (long long)p * hist_stride;
    const long long r = rank[p];
    unsigned long long local = 0;
    const int b0 = tid * per;
    for (int j = 0; j < per && b0 + j < nbins; ++j) local += h[b0 + j];
    // inclusive scan over the block
    unsigned long long v = local;
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned long long o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    if (lane == 31) s_wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      unsigned long long w = s_wsum[lane];
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long o = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += o;
      }
      s_wsum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const unsigned long long incl = v + (warp > 0 ? s_wsum[warp - 1] : 0ull);
    const unsigned long long excl = incl - local;
    if ((long long)excl < r && r <= (long long)incl) {
      unsigned long long c = excl;
      for (int j = 0; j < per && b0 + j < nbins; ++j) {
        const unsigned long long hj = h[b0 + j];
        if ((long long)c < r && r <= (long long)(c + hj)) {
          prefix[p] = (prefix[p] << bits) | (uint32_t)(b0 + j);
          rank[p] = r - (long long)c;
          break;
        }
        c += hj;
      }
    }
    __syncthreads();
  }
}

// Decode the selected magnitude codes to float thresholds.
template <typename T>
__global__ void calib_decode_kernel(const uint32_t* code, int P, float* out) {
  const int p = threadIdx.x;
  if (p >= P) return;
  const uint32_t c = code[p];
  if (DT<T>::id == SFX_F32)
    out[p] = __uint_as_float(c);
  else if (DT<T>::id == SFX_BF16)
    out[p] = __uint_as_float(c << 16);
  else
    out[p] = __half2float(__ushort_as_half((unsigned short)c));
}

size_t calib_workspace_bytes(long long, long long, int P, int) {
  // hist1 [32768] + histp [P*256] + ranks [P] + prefix [P] + out [P]
  return 32768 * 4 + (size_t)kMaxP * 256 * 4 + (size_t)kMaxP * (8 + 4 + 4) + 256;
}

template <typename T>
static int calibrate_t(const T* data, long long n, const long long* ranks, int P, float* out_host,
                       unsigned char* ws, cudaStream_t s) {
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(ws);
  uint32_t* histp = hist1 + 32768;
  long long* rank = reinterpret_cast<long long*>(histp + kMaxP * 256);
  uint32_t* prefix = reinterpret_cast<uint32_t*>(rank + kMaxP);
  float* outd = reinterpret_cast<float*>(prefix + kMaxP);
  const bool f32 = DT<T>::id == SFX_F32;
  if (cudaMemsetAsync(hist1, 0, 32768 * 4, s) != cudaSuccess) return SFX_ERR_CUDA;
  if (cudaMemsetAsync(prefix, 0, kMaxP * 4, s) != cudaSuccess) return SFX_ERR_CUDA;
  if (cudaMemcpyAsync(rank, ranks, sizeof(long long) * P, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SFX_ERR_CUDA;
  auto k1 = calib_hist1_kernel<T>;
  static size_t k1_configured = 0;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(k1), 32768 * 4, &k1_configured) != SFX_OK)
    return SFX_ERR_CUDA;
  const int grid = sm_count();
  k1<<<grid, kCalibThreads, 32768 * 4, s>>>(data, n, f32 ? 16 : 0, hist1);
  calib_select_kernel<<<1, kCalibThreads, 0, s>>>(hist1, 32768, 0, 15, P, rank, prefix);
  if (f32) {
    for (int shift = 8; shift >= 0; shift -= 8) {
      if (cudaMemsetAsync(histp, 0, (size_t)P * 256 * 4, s) != cudaSuccess) return SFX_ERR_CUDA;
      const size_t smem_p = ((size_t)P * 256 + P) * 4;
      static size_t histp_configured = 48 * 1024;  // the default limit
      if (ensure_dynamic_smem(reinterpret_cast<const void*>(calib_histp_kernel), smem_p,
                              &histp_configured) != SFX_OK)
        return SFX_ERR_CUDA;
      calib_histp_kernel<<<grid, kCalibThreads, smem_p, s>>>(reinterpret_cast<const float*>(data), n,
                                                        shift, P, prefix, histp);
      calib_select_kernel<<<1, kCalibThreads, 0, s>>>(histp, 256, 256, 8, P, rank, prefix);
    }
  }
  calib_decode_kernel<T><<<1, kMaxP, 0, s>>>(prefix, P, outd);
  if (cudaGetLastError() != cudaSuccess) return SFX_ERR_CUDA;
  if (cudaMemcpyAsync(out_host, outd, sizeof(float) * P, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SFX_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SFX_ERR_CUDA;
  return SFX_OK;
}

// ranks: 1-based ranks for the P' sparsities that need a device selection.
int run_calibrate(const void* calib, int dt, long long n, const long long* ranks, int P,
                  float* out, unsigned char* ws, cudaStream_t s) {
  if (P <= 0) return SFX_OK;
  if (P > kMaxP) return SFX_ERR_UNSUPPORTED;
  if (dt == SFX_F16) return calibrate_t(reinterpret_cast<const __half*>(calib), n, ranks, P, out, ws, s);
  if (dt == SFX_BF16)
    return calibrate_t(reinterpret_cast<const __nv_bfloat16*>(calib), n, ranks, P, out, ws, s);
  if (dt == SFX_F32) return calibrate_t(reinterpret_cast<const float*>(calib), n, ranks, P, out, ws, s);
  return SFX_ERR_DTYPE;
}

}  // namespace sfx
