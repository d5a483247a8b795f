// FFN with a static neuron mask on both projections, on sm_100a.
//
// "GLASS: Global-Local Aggregation for inference-time Sparsification",
// "selection": the set S of kept intermediate neurons is fixed for the prompt,
// so the pruned neurons' up-projection columns are skipped as well as their
// down-projection rows. Every matrix is stored one row per intermediate neuron
// ([ffn x d]), so a kept neuron's weights are contiguous 2d-byte rows:
//   GeLU:    h_j = GeLU(W_aT[j, :] . x_t)                   (erf or tanh form)
//   SwiGLU:  h_j = SiLU(W_aT[j, :] . x_t) (W_bT[j, :] . x_t)
//   y_t = sum_{j in S} h_j W_d[j, :]
//
// Batch 1 (decode) takes two launches: static_up_rows_kernel streams the kept up
// rows (one warp per row, a whole row's loads in flight) into h, then the
// index-list GEMV reads the kept down rows. Larger batches take three:
// the fp32 accumulator is zeroed (cudaMemsetAsync), then
// static_ffn_kernel (persistent CTAs, programmatic dependent launch): each CTA
// takes chunks of S whose size it derives from the device-side count so that
// the chunks spread over all resident CTAs; the dot products run as
// tensor-core tiles, and the down projection adds 16-byte
// float4 atomics into the accumulator (the combine order, hence the last bits
// of y, may vary between runs); then static_ffn_finalize_kernel writes y.
#include "sfx_common.cuh"
#include "sfx_internal.h"
#include "sfx_rowdot.cuh"

namespace sfx {

constexpr int kSfChunkMax = 64;  // kept neurons per work item, at most
constexpr int kSfChunkMin = 16;  // one tensor-core row tile

template <typename TW>
__global__ void __launch_bounds__(kRowThreads, 2)
    static_ffn_kernel(const TW* __restrict__ x, int B, int d, int ffn, const TW* __restrict__ WaT,
                      const TW* __restrict__ WbT, const TW* __restrict__ Wd,
                      const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt_p, int act,
                      float* acc, unsigned* status) {
  extern __shared__ __align__(16) unsigned char s_xraw[];  // [B][d + kXPad] staged x
  __shared__ float s_part[kRowThreads / 32][16][kRowTok];
  __shared__ float s_a[kSfChunkMax][kRowTok];
  __shared__ float s_v[kSfChunkMax][kRowTok];
  __shared__ int s_list[kSfChunkMax];
  __shared__ int s_bad[kSfChunkMax];
  __shared__ int s_tok[kRowTok];

  const int tid = threadIdx.x;
  pdl_wait();  // x, the list and the zeroed accumulator come from earlier work on the stream
  const int cnt = min(max(*cnt_p, 0), ffn);
  // chunk size from the count: the fewest equal rounds of one item per resident
  // CTA with at most 64 neurons per item (at least 16). Rounding 10035 neurons
  // on 148 CTAs to 157 items of 64 left 9 CTAs a second item and doubled the
  // time; 296 items of 34 take two even rounds.
  const int rounds = max(1, (cnt + (int)gridDim.x * kSfChunkMax - 1) / ((int)gridDim.x * kSfChunkMax));
  int ch = (cnt + (int)gridDim.x * rounds - 1) / ((int)gridDim.x * rounds);
  ch = ch < kSfChunkMin ? kSfChunkMin : (ch > kSfChunkMax ? kSfChunkMax : ch);
  const int n_items = (cnt + ch - 1) / ch;
  if ((int)blockIdx.x >= n_items) return;

  // No L2 prefetch of the items' rows: measured on B200 at 4 and 16 tokens
  // (Phi-2 GeLU and 8B-shaped SwiGLU sets, keep 0.3-0.7), bulk-prefetching
  // every row of the next item cost up to 14 % more than letting the
  // row-dot loads stream them.

  const int xstride = d + kXPad;
  TW* xs = reinterpret_cast<TW*>(s_xraw);
  for (int i = tid; i < B * (d / 8); i += kRowThreads) {
    const int b = i / (d / 8), c = i - b * (d / 8);
    *reinterpret_cast<uint4*>(xs + (long long)b * xstride + c * 8) =
        __ldg(reinterpret_cast<const uint4*>(x + (long long)b * d) + c);
  }
  if (tid < B) s_tok[tid] = tid;

  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int j0 = it * ch, nj = min(ch, cnt - j0);
    __syncthreads();  // staged x ready; the previous item is done with the arrays
    if (tid < nj) {
      int r = idx[j0 + tid];
      const int bad = r < 0 || r >= ffn;
      if (bad) {
        raise_status(status, SFX_DEV_BAD_INDEX);
        r = 0;  // read a valid row, contribute nothing
      }
      s_list[tid] = r;
      s_bad[tid] = bad;
    }
    __syncthreads();
    int n_tiles, ksplit;
    auto row_of = [&](int r) { return (long long)s_list[r]; };
    mma_rows(WaT, row_of, nj, d, xs, xstride, B, s_part, &n_tiles, &ksplit);
    __syncthreads();
    if (WbT) {
      for (int i = tid; i < nj * B; i += kRowThreads) {
        const int r = i / B, t = i - r * B;
        s_a[r][t] = sum_parts(s_part, n_tiles, ksplit, r, t);
      }
      __syncthreads();
      mma_rows(WbT, row_of, nj, d, xs, xstride, B, s_part, &n_tiles, &ksplit);
      __syncthreads();
    }
    for (int i = tid; i < nj * B; i += kRowThreads) {
      const int r = i / B, t = i - r * B;
      const float s = sum_parts(s_part, n_tiles, ksplit, r, t);
      float v;
      if (WbT) v = silu_f(s_a[r][t]) * s;
      else v = act == EPI_GELU_TANH ? gelu_tanh_f(s) : gelu_erf_f(s);
      s_v[r][t] = s_bad[r] ? 0.f : v;
    }
    __syncthreads();
    down_all(Wd, s_list, nj, s_v, B, s_tok, d, acc, it);  // all items share the tokens
  }
}

// Batch 1: h[S[k]] = act(W_aT[S[k], :] . x) for every kept neuron, one warp per
// row with the whole row's 16-byte loads in flight (x read through L1). The
// down projection then runs as the index-list GEMV over the kept rows of W_d.
template <typename TW, bool SWI>
__global__ void __launch_bounds__(256, 4) static_up_rows_kernel(const TW* __restrict__ x, int d,
                                                                int ffn, const TW* __restrict__ WaT,
                                                                const TW* __restrict__ WbT,
                                                                const int32_t* __restrict__ idx,
                                                                const int32_t* __restrict__ cnt_p,
                                                                int act, float* h,
                                                                unsigned* status) {
  // 16-byte loads per lane in flight per row (5 KB of one row, a whole Phi-2
  // row, or 2 KB of each of the two SwiGLU rows, per warp); 64 registers keep
  // 32 warps per SM
  constexpr int kLoads = SWI ? 4 : 10;
  pdl_wait();  // x and the list may come from the previous grid
  const int lane = threadIdx.x & 31;
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  const int cnt = min(max(*cnt_p, 0), ffn);
  // one matrix: start every row this warp will read towards L2 (one bulk
  // prefetch per row, spread over the lanes), so the rows stream while the
  // first ones are summed. Measured on B200: with the two SwiGLU rows per
  // neuron the prefetches cost more than they save (8B shape, keep 0.5: 36.8
  // against 41.8 us without / with), with one GeLU row they save 0.7-1 us.
  const uint32_t row_bytes = (uint32_t)((long long)d * sizeof(TW));
  for (int k = gw + lane * nw; !SWI && k < cnt; k += 32 * nw) {
    const int r = idx[k];
    if (r >= 0 && r < ffn) prefetch_l2_bulk(WaT + (long long)r * d, row_bytes);
  }
  for (int k = gw; k < cnt; k += nw) {
    const int r = idx[k];
    if (r < 0 || r >= ffn) {
      if (lane == 0) raise_status(status, SFX_DEV_BAD_INDEX);
      continue;  // the down GEMV skips it too
    }
    float sa = 0.f, sb = 0.f;
    const TW* pa = WaT + (long long)r * d;
    const TW* pb = SWI ? WbT + (long long)r * d : nullptr;
    for (int c0 = lane * 8; c0 < d; c0 += 256 * kLoads) {
      uint4 qa[kLoads], qb[kLoads];
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int c = c0 + u * 256;
        if (c < d) {
          qa[u] = __ldcs(reinterpret_cast<const uint4*>(pa + c));
          if (SWI) qb[u] = __ldcs(reinterpret_cast<const uint4*>(pb + c));
        }
      }
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int c = c0 + u * 256;
        if (c < d) {
          float xv[8], wa[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(x + c)), xv, TW());
          unpack8(qa[u], wa, TW());
#pragma unroll
          for (int e = 0; e < 8; ++e) sa = fmaf(wa[e], xv[e], sa);
          if (SWI) {
            float wb[8];
            unpack8(qb[u], wb, TW());
#pragma unroll
            for (int e = 0; e < 8; ++e) sb = fmaf(wb[e], xv[e], sb);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      sb += __shfl_xor_sync(0xffffffffu, sb, o);
    }
    if (lane == 0)
      h[r] = SWI ? silu_f(sa) * sb : (act == EPI_GELU_TANH ? gelu_tanh_f(sa) : gelu_erf_f(sa));
  }
}

__global__ void static_ffn_finalize_kernel(const float* acc, long long n, void* y, int ydt) {
  pdl_wait();  // the accumulator of the previous grid
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    store_as(y, i, ydt, acc[i]);
}

// batch > 1: the fp32 accumulator [B x d]; batch 1: h [ffn] f32, then the down
// GEMV's split-K partials
static size_t al256s(size_t v) { return (v + 255) / 256 * 256; }
size_t static_ffn_workspace_bytes(int B, int d, int ffn) {
  const size_t fused = (size_t)B * d * 4;
  const size_t one = al256s((size_t)ffn * 4) + gemv_workspace_bytes(ffn, d, 1);
  return B == 1 ? (fused > one ? fused : one) : fused;
}

template <typename TW>
static int launch_static(const void* x, int B, int d, int ffn, const void* WaT, const void* WbT,
                         const void* Wd, const int32_t* idx, const int32_t* cnt, int act, float* acc,
                         unsigned* status, cudaStream_t s) {
  auto kern = static_ffn_kernel<TW>;
  const size_t smem = (size_t)B * (d + kXPad) * sizeof(TW);
  static size_t configured = 0;
  // opt in whenever the size grows: dynamic plus ~17 KB static may pass 48 KB
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem, &configured) != SFX_OK)
    return SFX_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRowThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return SFX_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sm_count() * per_sm), 1, 1);
  cfg.blockDim = dim3(kRowThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const TW*>(x), B, d, ffn,
                            reinterpret_cast<const TW*>(WaT), reinterpret_cast<const TW*>(WbT),
                            reinterpret_cast<const TW*>(Wd), idx, cnt, act, acc, status) ==
                 cudaSuccess
             ? SFX_OK
             : SFX_ERR_CUDA;
}

int run_static_ffn(const void* x, int dt, int B, int d, int ffn, const void* WaT, const void* WbT,
                   const void* Wd, const int32_t* idx, const int32_t* cnt, int act, void* y,
                   int ydt, unsigned char* body, unsigned* status, cudaStream_t s) {
  if (B == 1) {
    // kept up rows streamed one warp per row, then the index-list GEMV for the down rows
    float* h = reinterpret_cast<float*>(body);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sm_count() * 4), 1, 1);  // four resident CTAs per SM
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (dt == SFX_BF16) {
      using T = __nv_bfloat16;
      e = cudaLaunchKernelEx(&cfg, WbT ? static_up_rows_kernel<T, true> : static_up_rows_kernel<T, false>,
                             reinterpret_cast<const T*>(x), d, ffn, reinterpret_cast<const T*>(WaT),
                             reinterpret_cast<const T*>(WbT), idx, cnt, act, h, status);
    } else {
      using T = __half;
      e = cudaLaunchKernelEx(&cfg, WbT ? static_up_rows_kernel<T, true> : static_up_rows_kernel<T, false>,
                             reinterpret_cast<const T*>(x), d, ffn, reinterpret_cast<const T*>(WaT),
                             reinterpret_cast<const T*>(WbT), idx, cnt, act, h, status);
    }
    if (e != cudaSuccess) return SFX_ERR_CUDA;
    GemvArgs g = {};
    g.x = h;
    g.W = Wd;
    g.y = y;
    g.idx = idx;
    g.cnt = cnt;
    g.status = status;
    g.counters = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(status) + kWsStatusBytes);
    g.partials = reinterpret_cast<float*>(body + al256s((size_t)ffn * 4));
    g.K = ffn;
    g.N = d;
    g.B = 1;
    g.ydt = ydt;
    g.epi = EPI_NONE;
    return launch_sparse_gemv(dt, SFX_F32, plan_gemv(ffn, d, 1, true), g, s, true);
  }
  float* acc = reinterpret_cast<float*>(body);
  const long long n = (long long)B * d;
  if (cudaMemsetAsync(acc, 0, (size_t)n * 4, s) != cudaSuccess) return SFX_ERR_CUDA;
  const int rc = dt == SFX_BF16 ? launch_static<__nv_bfloat16>(x, B, d, ffn, WaT, WbT, Wd, idx,
                                                               cnt, act, acc, status, s)
                                : launch_static<__half>(x, B, d, ffn, WaT, WbT, Wd, idx, cnt, act,
                                                        acc, status, s);
  if (rc != SFX_OK) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, static_ffn_finalize_kernel, (const float*)acc, n, y, ydt) ==
                 cudaSuccess
             ? SFX_OK
             : SFX_ERR_CUDA;
}

}  // namespace sfx
