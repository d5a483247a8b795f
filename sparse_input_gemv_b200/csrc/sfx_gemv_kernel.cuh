// Input-sparse GEMV / skinny GEMM on CUDA cores for sm_100a.
//
// y[b, n] = sum_{i active} x[b, i] W[i, n] with W [K x N] row-major, reading
// only the rows of active neurons ("TEAL: Training-Free Activation Sparsity in
// Large Language Models", slide 11: the mask is generated inside the kernel
// and only the needed weights are loaded; "Activation sparsity (LLM)"
// glossary: a zero input skips one weight row).
//
// Grid = (column tiles) x (K splits). Each CTA
//   1. builds the active list of its K-slice in shared memory: |x| > t per
//      token, warp ballots + popc + a block prefix give ascending positions
//      (or it reads its share of a caller list in the top-k modes);
//   2. streams the active rows' segments W[i, n0:n0+NT] into a ring of 16 KB
//      shared-memory stages with 1-D bulk copies (TMA) issued by a producer
//      warp, each stage guarded by a full/empty mbarrier pair, weights marked
//      L2 evict-first;
//   3. eight consumer warps read 128-bit words from the stages and accumulate
//      x * w in fp32 registers;
//   4. reduces across row groups in shared memory, then across K splits: each
//      CTA writes its fp32 partial tile, and the last CTA to arrive at the
//      tile's counter sums the S partials in split order (deterministic) and
//      applies the epilogue (store, GeLU, or SiLU(g) * u for interleaved
//      gate|up columns).
#pragma once

#include "sfx_common.cuh"
#include "sfx_internal.h"

namespace sfx {

constexpr int kConsumerThreads = 256;
constexpr int kProducerWarp = kConsumerThreads / 32;  // warp 8
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kWarps = kThreads / 32;
constexpr int kStageBytes = 16384;

__device__ __forceinline__ float apply_epi(int epi, float v) {
  if (epi == EPI_GELU) return gelu_erf_f(v);
  if (epi == EPI_GELU_TANH) return gelu_tanh_f(v);
  return v;
}

template <typename TW, typename TX, int NT, int BMAX>
__global__ void __launch_bounds__(kThreads, 1) sparse_gemv_kernel(const GemvArgs a) {
  constexpr int TPR = NT / 8;                 // threads per row segment (8 columns each)
  constexpr int RG = kConsumerThreads / TPR;  // row groups working in parallel
  constexpr int SR = kStageBytes / (NT * 2);  // rows per stage
  constexpr int RPT = SR / RG;                // rows per thread per stage
  static_assert(TPR <= kConsumerThreads && SR % RG == 0, "tile shape");

  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* stage_mem = smem;
  int32_t* list_row = reinterpret_cast<int32_t*>(smem + (size_t)a.nstage * kStageBytes);
  float* list_x = reinterpret_cast<float*>(list_row + a.list_cap);
  uint64_t* full = reinterpret_cast<uint64_t*>(list_x + (size_t)a.list_cap * BMAX);
  uint64_t* empty = full + a.nstage;

  __shared__ int s_warp_tot[kWarps];
  __shared__ int s_count;
  __shared__ int s_last;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tile = blockIdx.x;
  const int split = blockIdx.y;
  const long long n0 = (long long)tile * NT;
  const int ncols = (int)min((long long)NT, a.N - n0);

  if (tid == 0) {
    for (int s = 0; s < a.nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerThreads / 32);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  // Inputs (x, caller lists) and the workspace may be written by the
  // previous kernel on the stream when launched as a dependent grid.
  pdl_wait();

  // ---------------------------------------------------------------- 1. active list
  if (a.idx == nullptr) {
    const long long k0 = (long long)split * a.slice;
    const long long k1 = min(a.K, k0 + a.slice);
    const TX* xp = reinterpret_cast<const TX*>(a.x);
    int base = 0;
    for (long long c0 = k0; c0 < k1; c0 += kThreads) {
      const long long i = c0 + tid;
      const bool in = i < k1;
      float xv[BMAX];
      bool act = false;
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        float v = 0.f;
        bool m = false;
        if (b < a.B) {
          if (in) {
            v = to_f32(xp[(long long)b * a.K + i]);
            m = fabsf(v) > a.t;
          }
          if (a.bitmap_out != nullptr && tile == 0) {
            const unsigned bal = __ballot_sync(0xffffffffu, m);
            const long long w0 = c0 + (long long)warp * 32;
            if (lane == 0 && w0 < k1)
              a.bitmap_out[(long long)b * ((a.K + 31) >> 5) + (w0 >> 5)] = bal;
          }
        }
        act |= m;
        xv[b] = m ? v : 0.f;
        if (a.union_mask) xv[b] = v;  // fixed below once the union is known
      }
      if (a.union_mask && !act) {
#pragma unroll
        for (int b = 0; b < BMAX; ++b) xv[b] = 0.f;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, act);
      if (lane == 0) s_warp_tot[warp] = __popc(bal);
      __syncthreads();
      int woff = 0, tot = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int c = s_warp_tot[w];
        woff += (w < warp) ? c : 0;
        tot += c;
      }
      if (act) {
        const int pos = base + woff + __popc(bal & lanemask_lt());
        list_row[pos] = (int32_t)i;
#pragma unroll
        for (int b = 0; b < BMAX; ++b) list_x[pos * BMAX + b] = xv[b];
      }
      base += tot;
      __syncthreads();
    }
    if (tid == 0) s_count = base;
  } else {
    // caller-provided ascending list (B == 1): this split takes an even share
    const long long c = min((long long)max(*a.cnt, 0), a.K);
    const long long p0 = c * split / a.S;
    const long long p1 = c * (split + 1) / a.S;
    const TX* xp = reinterpret_cast<const TX*>(a.x);
    for (long long p = p0 + tid; p < p1; p += kThreads) {
      int i = a.idx[p];
      float v = 0.f;
      if (i < 0 || (long long)i >= a.K) {
        raise_status(a.status, SFX_DEV_BAD_INDEX);
        i = 0;  // read a valid row, contribute nothing
      } else {
        v = to_f32(xp[i]);
      }
      const int q = (int)(p - p0);
      list_row[q] = i;
      list_x[q * BMAX] = v;
#pragma unroll
      for (int b = 1; b < BMAX; ++b) list_x[q * BMAX + b] = 0.f;
    }
    if (tid == 0) s_count = (int)(p1 - p0);
  }
  __syncthreads();

  // ---------------------------------------------------------------- 2/3. stream + FMA
  const int nrows = s_count;
  const int nst = (nrows + SR - 1) / SR;
  const uint32_t seg_bytes = (uint32_t)ncols * (uint32_t)sizeof(TW);
  const int rg = tid / TPR;
  const int tc = tid % TPR;
  float acc[BMAX][8];
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[b][j] = 0.f;

  if (warp == kProducerWarp) {
    const uint64_t pol = l2_evict_first_policy();
    const TW* Wp = reinterpret_cast<const TW*>(a.W);
    for (int st = 0; st < nst; ++st) {
      const int slot = st % a.nstage;
      const int use = st / a.nstage;
      if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, &s_abort)) {
        s_abort = 1;
        raise_status(a.status, SFX_DEV_TIMEOUT);
        break;
      }
      const int r0 = st * SR;
      const int rows = min(SR, nrows - r0);
      if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)rows * seg_bytes);
      __syncwarp();
      unsigned char* dst = stage_mem + (size_t)slot * kStageBytes;
      for (int r = lane; r < rows; r += 32) {
        const TW* src = Wp + (long long)list_row[r0 + r] * a.N + n0;
        bulk_g2s(dst + (size_t)r * NT * sizeof(TW), src, seg_bytes, &full[slot], pol);
      }
    }
  } else {
    const bool col_ok = tc * 8 < ncols;
    for (int st = 0; st < nst; ++st) {
      const int slot = st % a.nstage;
      const int use = st / a.nstage;
      if (!mbar_wait(&full[slot], use & 1, &s_abort)) {
        s_abort = 1;
        raise_status(a.status, SFX_DEV_TIMEOUT);
        break;
      }
      const int r0 = st * SR;
      const int rows = min(SR, nrows - r0);
      const unsigned char* src = stage_mem + (size_t)slot * kStageBytes;
      if (col_ok) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
          const int r = rg + rr * RG;
          if (r < rows) {
            const uint4 q = *reinterpret_cast<const uint4*>(src + (size_t)r * NT * 2 + tc * 16);
            float w[8];
            unpack8(q, w, TW());
            const float* xr = list_x + (size_t)(r0 + r) * BMAX;
#pragma unroll
            for (int b = 0; b < BMAX; ++b) {
              const float xv = xr[b];
#pragma unroll
              for (int j = 0; j < 8; ++j) acc[b][j] = fmaf(xv, w[j], acc[b][j]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  }
  pdl_launch_dependents();
  __syncthreads();
  if (s_abort) {
    // Bounded drain of copies that may still be in flight, then leave.
    if (tid == 0) {
      for (int s = 0; s < a.nstage; ++s) {
        mbar_wait(&full[s], 0, nullptr, kDrainLimitNs);
        mbar_wait(&full[s], 1, nullptr, kDrainLimitNs);
      }
    }
    __syncthreads();
    return;
  }

  // ---------------------------------------------------------------- 4. reductions
  float* red = reinterpret_cast<float*>(stage_mem);  // [RG][NT], stages are drained
  const bool swiglu = a.epi == EPI_SWIGLU;
  const long long N = a.N;
#pragma unroll
  for (int b = 0; b < BMAX; ++b) {
    if (b >= a.B) break;
    if (tid < kConsumerThreads && tc * 8 < ncols) {
      float4* dst = reinterpret_cast<float4*>(red + rg * NT + tc * 8);
      dst[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
      dst[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
    }
    __syncthreads();
    if (a.S == 1) {
      if (swiglu) {
        float* h = reinterpret_cast<float*>(a.y);
        for (int p = tid; p < ncols / 2; p += kThreads) {
          float g = 0.f, u = 0.f;
#pragma unroll
          for (int r = 0; r < RG; ++r) {
            g += red[r * NT + 2 * p];
            u += red[r * NT + 2 * p + 1];
          }
          h[(long long)b * (N / 2) + n0 / 2 + p] = silu_f(g) * u;
        }
      } else {
        for (int c = tid; c < ncols; c += kThreads) {
          float v = 0.f;
#pragma unroll
          for (int r = 0; r < RG; ++r) v += red[r * NT + c];
          store_as(a.y, (long long)b * N + n0 + c, a.ydt, apply_epi(a.epi, v));
        }
      }
    } else {
      float* part = a.partials + ((long long)split * a.B + b) * N + n0;
      for (int c = tid; c < ncols; c += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) v += red[r * NT + c];
        part[c] = v;
      }
    }
    __syncthreads();
  }
  if (a.S == 1) return;

  // last CTA of this column tile sums the S partials in split order
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(&a.counters[tile], 1);
    s_last = (prev == a.S - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int b = 0; b < a.B; ++b) {
    const float* part = a.partials + (long long)b * N + n0;
    const long long sstride = (long long)a.B * N;
    if (swiglu) {
      float* h = reinterpret_cast<float*>(a.y);
      for (int p = tid; p < ncols / 2; p += kThreads) {
        float g = 0.f, u = 0.f;
        for (int s = 0; s < a.S; ++s) {
          const float2 gu = __ldcg(reinterpret_cast<const float2*>(part + s * sstride) + p);
          g += gu.x;
          u += gu.y;
        }
        h[(long long)b * (N / 2) + n0 / 2 + p] = silu_f(g) * u;
      }
    } else {
      for (int c = tid; c < ncols; c += kThreads) {
        float v = 0.f;
        for (int s = 0; s < a.S; ++s) v += __ldcg(part + s * sstride + c);
        store_as(a.y, (long long)b * N + n0 + c, a.ydt, apply_epi(a.epi, v));
      }
    }
  }
  if (tid == 0) a.counters[tile] = 0;  // leave the workspace ready for the next call
}


template <typename TW, typename TX, int NT, int BMAX>
inline int launch_t(const GemvPlan& p, const GemvArgs& a, cudaStream_t stream, bool pdl) {
  auto kern = sparse_gemv_kernel<TW, TX, NT, BMAX>;
  static size_t configured = 0;
  if (p.smem > configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem) !=
        cudaSuccess)
      return SFX_ERR_CUDA;
    configured = p.smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.col_tiles, (unsigned)p.S, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return SFX_ERR_CUDA;
  return SFX_OK;
}

}  // namespace sfx
