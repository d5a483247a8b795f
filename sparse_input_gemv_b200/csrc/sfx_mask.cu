// Mask construction and compaction kernels (sm_100a).
//
//  * threshold:  m_i = 1[|x_i| > t] ("TEAL: Training-Free Activation Sparsity in
//    Large Language Models", slides 8 and 11), per token and for the batch union;
//  * GxO top-k:  keep the k largest s_i = |fl32(x_i g_i)| ("Attribution-based
//    Sparse Activation in Large Language Models", "proposed method" and
//    "implementation"), selected exactly by an MSB-first radix select on the
//    float bits (non-negative floats order like their bit patterns), equal
//    scores resolved toward the lower index;
//  * GLASS:      ranks of two score vectors, F = (1-l) R^l + l R^g in double,
//    top-k of F ("GLASS: Global-Local Aggregation for inference-time
//    Sparsification", section 2.2). Ranks are computed by counting, which is
//    exact and order-independent; the GLASS mask is built once per prompt.
//
// Compaction everywhere: warp ballot -> popc of the lanes below -> prefix over
// the block's warps -> ascending positions; bitmap words are the ballots.
#include "sfx_common.cuh"
#include "sfx_internal.h"

namespace sfx {

constexpr int kMaskThreads = 1024;
constexpr int kMaskWarps = kMaskThreads / 32;

// Block-wide ordered compaction step for one chunk of 1024 candidates.
// Returns the number of set flags in the chunk; writes positions to `out`.
__device__ __forceinline__ int compact_chunk(bool act, int i, int base, int32_t* out,
                                             int* s_tot, unsigned* bal_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned bal = __ballot_sync(0xffffffffu, act);
  if (lane == 0) s_tot[warp] = __popc(bal);
  __syncthreads();
  int woff = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kMaskWarps; ++w) {
    const int c = s_tot[w];
    woff += (w < warp) ? c : 0;
    tot += c;
  }
  if (act && out) out[base + woff + __popc(bal & lanemask_lt())] = i;
  __syncthreads();
  *bal_out = bal;
  return tot;
}

// Source of the per-element decision: threshold on x, or a 0/1 flag array.
template <typename TX>
__global__ void __launch_bounds__(kMaskThreads) mask_compact_kernel(
    const TX* x, const int32_t* flags, int B, int K, float t, uint32_t* bitmap, int32_t* idx,
    int32_t* cnt, int32_t* uidx, int32_t* ucnt) {
  __shared__ int s_tot[kMaskWarps];
  const int b = blockIdx.x;
  const bool is_union = (b == B);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (K + 31) >> 5;
  int32_t* out = is_union ? uidx : (idx ? idx + (long long)b * K : nullptr);
  int base = 0;
  for (int c0 = 0; c0 < K; c0 += kMaskThreads) {
    const int i = c0 + threadIdx.x;
    const bool in = i < K;
    bool act = false;
    if (in) {
      const int b0 = is_union ? 0 : b, b1 = is_union ? B : b + 1;
      for (int bb = b0; bb < b1; ++bb) {
        const long long e = (long long)bb * K + i;
        act |= flags ? (flags[e] != 0) : (fabsf(to_f32(x[e])) > t);
      }
    }
    unsigned bal;
    base += compact_chunk(act, i, base, out, s_tot, &bal);
    const int w0 = c0 + warp * 32;
    if (!is_union && bitmap && lane == 0 && w0 < K) bitmap[(long long)b * words + (w0 >> 5)] = bal;
  }
  if (threadIdx.x == 0) {
    if (is_union)
      *ucnt = base;
    else
      cnt[b] = base;
  }
}

// Exact top-k of s_i = |fl32(x_i * g_i)| for one token per CTA.
template <typename TX>
__global__ void __launch_bounds__(kMaskThreads) topk_gxo_kernel(const TX* x, const float* g,
                                                                int K, int k, uint32_t* bitmap,
                                                                int32_t* idx, int32_t* cnt) {
  extern __shared__ uint32_t keys[];  // [K]
  __shared__ uint32_t hist[256];
  __shared__ int s_tot[kMaskWarps];
  __shared__ int s_tie[kMaskWarps];
  __shared__ uint32_t s_prefix;
  __shared__ uint32_t s_remaining;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TX* xb = x + (long long)b * K;
  const float* gb = g + (long long)b * K;
  for (int i = tid; i < K; i += kMaskThreads)
    keys[i] = __float_as_uint(fabsf(__fmul_rn(to_f32(xb[i]), gb[i])));
  __syncthreads();

  uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
  if (k > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int j = tid; j < 256; j += kMaskThreads) hist[j] = 0;
      __syncthreads();
      // warp-aggregated: the scores share a few leading bytes, so most lanes of a
      // warp hit the same bin; one lane per distinct bin adds its group's count
      for (int i0 = 0; i0 < K; i0 += kMaskThreads) {
        const int i = i0 + tid;
        const uint32_t key = i < K ? keys[i] : 0u;
        const bool cand = i < K && (key & pmask) == prefix;
        const uint32_t bin = cand ? ((key >> shift) & 255u) : 256u;
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (cand && lane == __ffs(same) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(same));
      }
      __syncthreads();
      if (warp == 0) {
        uint32_t h[8], local = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          h[j] = hist[lane * 8 + j];
          local += h[j];
        }
        uint32_t incl = local;  // sum over lanes >= lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t v = __shfl_down_sync(0xffffffffu, incl, off);
          if (lane + off < 32) incl += v;
        }
        uint32_t c = incl - local;  // elements in higher bins
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (c < remaining && remaining <= c + h[j]) {
            s_prefix = prefix | ((uint32_t)(lane * 8 + j) << shift);
            s_remaining = remaining - c;
          }
          c += h[j];
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= 255u << shift;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;  // k-th largest key; `remaining` ties at T are kept
  const int words = (K + 31) >> 5;
  int base = 0, ties_seen = 0;
  for (int c0 = 0; c0 < K; c0 += kMaskThreads) {
    const int i = c0 + tid;
    const bool in = i < K;
    const uint32_t key = in ? keys[i] : 0u;
    const bool gt = in && k > 0 && key > T;
    const bool eq = in && k > 0 && key == T;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_tie[warp] = __popc(beq);
    __syncthreads();
    int toff = 0, ttot = 0;
#pragma unroll
    for (int w = 0; w < kMaskWarps; ++w) {
      const int c = s_tie[w];
      toff += (w < warp) ? c : 0;
      ttot += c;
    }
    const int tie_rank = ties_seen + toff + __popc(beq & lanemask_lt());
    const bool act = gt || (eq && (uint32_t)tie_rank < remaining);
    unsigned bal;
    base += compact_chunk(act, i, base, idx ? idx + (long long)b * K : nullptr, s_tot, &bal);
    ties_seen += ttot;
    const int w0 = c0 + warp * 32;
    if (bitmap && lane == 0 && w0 < K) bitmap[(long long)b * words + (w0 >> 5)] = bal;
  }
  if (tid == 0) cnt[b] = base;
}

// q_j = #{i : key_i > key_j or (key_i == key_j and i < j)} by counting.
// mode 0: out = n - q_j (rank, most important = n); mode 1: out = (q_j < k).
template <typename KT>
__global__ void __launch_bounds__(256) rank_count_kernel(const KT* keys, int n, int mode, int k,
                                                          int32_t* out) {
  __shared__ KT tile[2048];
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const KT* kb = keys + (long long)b * n;
  const KT kj = (j < n) ? kb[j] : KT(0);
  int q = 0;
  for (int t0 = 0; t0 < n; t0 += 2048) {
    const int m = min(2048, n - t0);
    for (int ii = threadIdx.x; ii < m; ii += blockDim.x) tile[ii] = kb[t0 + ii];
    __syncthreads();
    for (int ii = 0; ii < m; ++ii) {
      const KT ki = tile[ii];
      const int i = t0 + ii;
      q += (ki > kj) || (ki == kj && i < j);
    }
    __syncthreads();
  }
  if (j < n) out[(long long)b * n + j] = (mode == 0) ? (n - q) : (q < k ? 1 : 0);
}

// F_j = (1 - lambda) R^l_j + lambda R^g_j with each product and the sum
// rounded once (no fused multiply-add), in double.
__global__ void glass_fuse_kernel(const int32_t* Rl, const int32_t* Rg, long long total,
                                  double lam, double* F) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < total)
    F[e] = __dadd_rn(__dmul_rn(1.0 - lam, (double)Rl[e]), __dmul_rn(lam, (double)Rg[e]));
}

size_t mask_workspace_bytes(int B, int K, int sel) {
  if (sel == SFX_SEL_TOPK_GLASS) return (size_t)B * K * (4 + 4 + 8 + 4) + 256;
  return 0;
}

template <typename TX>
static int launch_threshold(const void* x, int B, int K, float t, uint32_t* bitmap, int32_t* idx,
                            int32_t* cnt, int32_t* uidx, int32_t* ucnt, cudaStream_t s) {
  const int grid = B + (uidx ? 1 : 0);
  mask_compact_kernel<TX><<<grid, kMaskThreads, 0, s>>>(reinterpret_cast<const TX*>(x), nullptr,
                                                        B, K, t, bitmap, idx, cnt, uidx, ucnt);
  return cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

template <typename TX>
static int launch_gxo(const void* x, const float* g, int B, int K, int k, uint32_t* bitmap,
                      int32_t* idx, int32_t* cnt, cudaStream_t s) {
  const size_t smem = (size_t)K * 4;
  auto kern = topk_gxo_kernel<TX>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return SFX_ERR_CUDA;
  kern<<<B, kMaskThreads, smem, s>>>(reinterpret_cast<const TX*>(x), g, K, k, bitmap, idx, cnt);
  return cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

int launch_mask_compact(const void* x, int dt, int B, int K, int sel, float t, int k,
                        const float* score_l, const float* score_g, double lambda,
                        uint32_t* bitmap, int32_t* idx, int32_t* cnt, int32_t* uidx,
                        int32_t* ucnt, unsigned char* ws, unsigned* status, cudaStream_t s) {
  (void)status;
  if (sel == SFX_SEL_THRESHOLD) {
    if (dt == SFX_F16) return launch_threshold<__half>(x, B, K, t, bitmap, idx, cnt, uidx, ucnt, s);
    if (dt == SFX_BF16)
      return launch_threshold<__nv_bfloat16>(x, B, K, t, bitmap, idx, cnt, uidx, ucnt, s);
    return launch_threshold<float>(x, B, K, t, bitmap, idx, cnt, uidx, ucnt, s);
  }
  int rc = SFX_OK;
  if (sel == SFX_SEL_TOPK_GXO) {
    if (dt == SFX_F16) rc = launch_gxo<__half>(x, score_l, B, K, k, bitmap, idx, cnt, s);
    else if (dt == SFX_BF16) rc = launch_gxo<__nv_bfloat16>(x, score_l, B, K, k, bitmap, idx, cnt, s);
    else rc = launch_gxo<float>(x, score_l, B, K, k, bitmap, idx, cnt, s);
  } else {
    // GLASS: ranks of both vectors, fused score, top-k flags, compaction
    const long long total = (long long)B * K;
    int32_t* Rl = reinterpret_cast<int32_t*>(ws);
    int32_t* Rg = Rl + total;
    double* F = reinterpret_cast<double*>(Rg + total);  // 8-byte aligned: 2*total int32 before
    int32_t* flags = reinterpret_cast<int32_t*>(F + total);
    const dim3 grid((K + 255) / 256, B);
    rank_count_kernel<float><<<grid, 256, 0, s>>>(score_l, K, 0, 0, Rl);
    rank_count_kernel<float><<<grid, 256, 0, s>>>(score_g, K, 0, 0, Rg);
    glass_fuse_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(Rl, Rg, total, lambda, F);
    rank_count_kernel<double><<<grid, 256, 0, s>>>(F, K, 1, k, flags);
    mask_compact_kernel<float><<<B + (uidx ? 1 : 0), kMaskThreads, 0, s>>>(
        nullptr, flags, B, K, 0.f, bitmap, idx, cnt, uidx, ucnt);
    rc = cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
    return rc;
  }
  return rc;  // (a union list for GxO top-k is rejected on the host)
}

}  // namespace sfx
