// Mask construction and compaction kernels (sm_100a).
//
//  * threshold:  m_i = 1[|x_i| > t] ("TEAL: Training-Free Activation Sparsity in
//    Large Language Models", slides 8 and 11), per token and for the batch union;
//  * GxO top-k:  keep the k largest s_i = |fl32(x_i g_i)| ("Attribution-based
//    Sparse Activation in Large Language Models", "proposed method" and
//    "implementation"), selected exactly by an MSB-first radix select on the
//    float bits (non-negative floats order like their bit patterns), equal
//    scores resolved toward the lower index;
//  * corrected GxO top-k: the same select on the signed score
//    s_i = x_i g_i + |x_i| ||g||_2 / 2 (same page, "correction term"), mapped to
//    an order-preserving unsigned key (sign bit flipped, negatives inverted);
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

// Block-wide exclusive prefix sum of one int per thread (kMaskThreads threads);
// *total gets the sum. Uses s_w[kMaskWarps + 1]; ends with a barrier.
__device__ __forceinline__ int block_excl_scan(int v, int* s_w, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) s_w[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int wv = s_w[lane];  // kMaskWarps == 32
    int winc = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += n;
    }
    s_w[lane] = winc - wv;  // exclusive over warps
    if (lane == 31) s_w[32] = winc;
  }
  __syncthreads();
  const int r = s_w[warp] + inc - v;
  *total = s_w[32];
  __syncthreads();  // s_w may be reused
  return r;
}

// Exact top-k of s_i = |fl32(x_i * g_i)| (or the corrected GxO score) for one
// token per CTA. Warp w owns the 32 kpt elements from 32 kpt w on, in
// lane-major slots (kpt <= KPT per thread, keys in registers). Up to three
// radix passes over the key bits (11, 11 and 10 bits, most significant first;
// wide digits keep the histogram atomics spread even though the scores share
// their leading bits) find the k-th largest key T on the digits examined and
// how many keys equal to it are kept, stopping early once that bin is kept
// whole. Slot ballots and one scan over the warps then place every kept index,
// so the list comes out ascending with ties resolved toward the lower index.
constexpr int kTopkBins = 2048;  // 2 bins per thread
template <typename TX, int KPT>
__global__ void __launch_bounds__(kMaskThreads) topk_gxo_kernel(const TX* __restrict__ x,
                                                                const float* __restrict__ g,
                                                                int K, int k, int corrected,
                                                                uint32_t* bitmap, int32_t* idx,
                                                                int32_t* cnt) {
  __shared__ uint32_t hist[kTopkBins];
  __shared__ int s_w[kMaskWarps + 1];
  __shared__ uint32_t s_prefix;
  __shared__ uint32_t s_remaining;
  __shared__ int s_whole;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // h comes from the previous kernel (launched as its programmatic dependent);
  // the next kernel may start its CTAs now: it waits for this grid's results
  pdl_wait();
  pdl_launch_dependents();
  // Warp w owns the span of 32 kpt elements starting at 32 kpt w, lane-major:
  // its slot j holds element 32 kpt w + 32 j + lane. Every load is coalesced,
  // and slot j of a warp is one 32-bit word of the bitmap.
  const int kpt = (K + kMaskThreads - 1) / kMaskThreads;
  const int base = 32 * kpt * warp;
  const TX* xb = x + (long long)b * K;
  const float* gb = g + (long long)b * K;
  float xv[KPT], gv[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int e = base + 32 * j + lane;
    const bool ok = j < kpt && e < K;
    xv[j] = ok ? to_f32(xb[e]) : 0.f;
    gv[j] = ok ? gb[e] : 0.f;
  }
  // corrected GxO: n / 2 with n = fl32(sqrt(sum g^2)), the squares exact in
  // double and summed in double (a fixed order: per thread, then warp and
  // block trees)
  float half_n = 0.f;
  if (corrected) {
    __shared__ double s_d[kMaskWarps];
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) ss += (double)gv[j] * (double)gv[j];
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_d[warp] = ss;
    __syncthreads();
    if (tid < 32) {
      double v = s_d[tid];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (tid == 0) s_d[0] = v;
    }
    __syncthreads();
    half_n = __double2float_rn(sqrt(s_d[0])) * 0.5f;  // exact halving
  }
  uint32_t key[KPT];
  unsigned valid = 0;  // slots that hold an element
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (j < kpt && base + 32 * j + lane < K) valid |= 1u << j;
    if (corrected) {
      // signed score -> unsigned key in the same order
      const float sc = __fadd_rn(__fmul_rn(xv[j], gv[j]), __fmul_rn(fabsf(xv[j]), half_n));
      const uint32_t bits = __float_as_uint(sc);
      key[j] = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
    } else {
      key[j] = __float_as_uint(fabsf(__fmul_rn(xv[j], gv[j])));
    }
  }

  uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
  // each thread owns bins 2 tid and 2 tid + 1: it zeroes them, and after a pass
  // reads and re-zeroes them itself
  hist[2 * tid] = 0u;
  hist[2 * tid + 1] = 0u;
  if (k > 0) {
    constexpr int kShift[3] = {21, 10, 0};
    constexpr int kBits[3] = {11, 11, 10};
#pragma unroll
    for (int ps = 0; ps < 3; ++ps) {
      const int shift = kShift[ps];
      const uint32_t dmask = (1u << kBits[ps]) - 1u;
      __syncthreads();  // zeroed bins (or the previous selection) visible
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if (((valid >> j) & 1u) && (key[j] & pmask) == prefix)
          atomicAdd(&hist[(key[j] >> shift) & dmask], 1u);
      __syncthreads();
      // keys in bins above this thread's two: total minus the inclusive prefix
      const uint32_t h0 = hist[2 * tid], h1 = hist[2 * tid + 1];
      hist[2 * tid] = 0u;
      hist[2 * tid + 1] = 0u;
      const int local = (int)(h0 + h1);
      int total;
      const int before = block_excl_scan(local, s_w, &total);
      uint32_t c = (uint32_t)(total - before - local);
      if (c < remaining && remaining <= c + h1) {
        s_prefix = prefix | ((uint32_t)(2 * tid + 1) << shift);
        s_remaining = remaining - c;
        s_whole = remaining - c == h1;
      }
      c += h1;
      if (c < remaining && remaining <= c + h0) {
        s_prefix = prefix | ((uint32_t)(2 * tid) << shift);
        s_remaining = remaining - c;
        s_whole = remaining - c == h0;
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= dmask << shift;
      // the bin holding the k-th key is kept whole: every key above it and
      // every key in it are the top k, so the digits left decide nothing
      if (s_whole) break;
    }
  }
  // T: the k-th largest key on the digits examined (pmask). Kept: every key
  // above T, and the first `remaining` keys equal to T in index order (after
  // k = 0 no pass ran: remaining = 0 and nothing is above T = 0 on no digits).
  const uint32_t T = prefix;
  // per-warp counts of larger and equal keys, then one scan over the warps
  unsigned w_gt = 0, w_eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool v = (valid >> j) & 1u;
    w_gt += __popc(__ballot_sync(0xffffffffu, v && (key[j] & pmask) > T));
    w_eq += __popc(__ballot_sync(0xffffffffu, v && (key[j] & pmask) == T));
  }
  if (lane == 0) s_w[warp] = (int)((w_gt << 16) | w_eq);  // both <= K <= 32768
  __syncthreads();
  if (warp == 0) {
    const int wv = s_w[lane];
    int winc = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += n;
    }
    s_w[lane] = winc - wv;
    if (lane == 31) s_w[32] = winc;
  }
  __syncthreads();
  // larger and equal keys at lower indices, running over the warp's slots
  unsigned gt_run = (unsigned)s_w[warp] >> 16, eq_run = (unsigned)s_w[warp] & 0xffffu;
  const unsigned all_gt = (unsigned)s_w[32] >> 16, all_eq = (unsigned)s_w[32] & 0xffffu;
  int32_t* out = idx ? idx + (long long)b * K : nullptr;
  const int words = (K + 31) >> 5;
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int e = base + 32 * j + lane;
    if (j < kpt && base + 32 * j < K) {  // warp-uniform: the slot's word exists
      const bool v = (valid >> j) & 1u;
      const bool gt = v && (key[j] & pmask) > T, eq = v && (key[j] & pmask) == T;
      const unsigned bg = __ballot_sync(0xffffffffu, gt);
      const unsigned be = __ballot_sync(0xffffffffu, eq);
      const unsigned eq_rank = eq_run + __popc(be & lt);
      const bool keep = gt || (eq && eq_rank < remaining);
      const unsigned bk = __ballot_sync(0xffffffffu, keep);
      if (keep && out) {
        const unsigned gt_rank = gt_run + __popc(bg & lt);
        out[gt_rank + (eq_rank < remaining ? eq_rank : remaining)] = e;
      }
      if (lane == 0 && bitmap) bitmap[(long long)b * words + ((base + 32 * j) >> 5)] = bk;
      gt_run += __popc(bg);
      eq_run += __popc(be);
    }
  }
  if (tid == 0) cnt[b] = (int)(all_gt + (all_eq < remaining ? all_eq : remaining));
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

template <typename TX, int KPT>
static int launch_gxo_k(const void* x, const float* g, int B, int K, int k, int corrected,
                        uint32_t* bitmap, int32_t* idx, int32_t* cnt, cudaStream_t s) {
  // a programmatic dependent launch: the kernel waits for its inputs itself
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B, 1, 1);
  cfg.blockDim = dim3(kMaskThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_gxo_kernel<TX, KPT>, reinterpret_cast<const TX*>(x), g, K,
                            k, corrected, bitmap, idx, cnt) == cudaSuccess
             ? SFX_OK
             : SFX_ERR_CUDA;
}

// keys per thread in registers: K <= 1024 KPT (K <= 32768)
template <typename TX>
static int launch_gxo(const void* x, const float* g, int B, int K, int k, int corrected,
                      uint32_t* bitmap, int32_t* idx, int32_t* cnt, cudaStream_t s) {
  const int kpt = (K + kMaskThreads - 1) / kMaskThreads;
  if (kpt <= 4) return launch_gxo_k<TX, 4>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
  if (kpt <= 8) return launch_gxo_k<TX, 8>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
  // every per-key loop is unrolled over the slots, so spare slots cost issue
  // slots: 10 for n = 8193..10240 (10 keys per thread at n = 10240), 12 up to 12288
  if (kpt <= 10) return launch_gxo_k<TX, 10>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
  if (kpt <= 12) return launch_gxo_k<TX, 12>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
  if (kpt <= 16) return launch_gxo_k<TX, 16>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
  return launch_gxo_k<TX, 32>(x, g, B, K, k, corrected, bitmap, idx, cnt, s);
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
  if (sel == SFX_SEL_TOPK_GXO || sel == SFX_SEL_TOPK_CGXO) {
    const int cor = sel == SFX_SEL_TOPK_CGXO;
    if (dt == SFX_F16) rc = launch_gxo<__half>(x, score_l, B, K, k, cor, bitmap, idx, cnt, s);
    else if (dt == SFX_BF16)
      rc = launch_gxo<__nv_bfloat16>(x, score_l, B, K, k, cor, bitmap, idx, cnt, s);
    else rc = launch_gxo<float>(x, score_l, B, K, k, cor, bitmap, idx, cnt, s);
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
