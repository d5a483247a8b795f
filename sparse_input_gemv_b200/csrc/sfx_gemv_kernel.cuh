// Input-sparse GEMV / skinny GEMM on CUDA cores for sm_100a.
//
// y[b, n] = sum_{i active} x[b, i] W[i, n] with W [K x N] row-major, reading
// only the rows of active neurons ("TEAL: Training-Free Activation Sparsity in
// Large Language Models", slide 11: the mask is generated inside the kernel
// and only the needed weights are loaded; "Activation sparsity (LLM)"
// glossary: a zero input skips one weight row).
//
// Grid = (column tiles of NT columns) x (K splits), 512 threads; kernels with
// 1 or 2 batch slots run two CTAs per SM, the 4-slot kernel one. Each CTA
//   1. builds the active list of its K-slice in shared memory: |x| > t per
//      token, warp ballots + popc + a block prefix give ascending positions
//      (or it reads its share of a caller-provided list);
//   2. streams the active rows' segments W[i, n0:n0+NT] with 128-bit loads
//      that bypass L1 and carry an L2 evict-first policy: each warp owns one
//      256-column chunk of the tile (32 lanes x 8 bf16/fp16) and keeps four
//      rows in flight (eight in the 4-slot kernel, which runs one CTA per SM),
//      so an SM holds ~64 KB of weight reads in flight,
//      enough to cover HBM latency; products accumulate in fp32 registers;
//   3. reduces the warps of each chunk in shared memory, then across K
//      splits: every CTA writes its fp32 partial tile and the last CTA to
//      arrive at the tile's counter sums the S partials in split order
//      (deterministic; the sum is spread over all threads, four split groups
//      at a time) and applies the epilogue (store, GeLU, or SiLU(g) * u for
//      interleaved gate|up columns).
//
// Why plain loads rather than bulk (TMA) copies into a shared-memory ring: on
// this GPU a CTA issues 1-D bulk copies at a few million per second, so the
// 0.5-4 KB row segments of a sparse GEMV top out at 1-4 TB/s that way,
// while 128-bit loads with enough rows in flight reach the HBM peak.
#pragma once

#include "sfx_common.cuh"
#include "sfx_internal.h"

namespace sfx {

// 512 threads (two CTAs per SM) up to 4 batch slots; 256 threads with the
// register room for 8 x BMAX accumulators above that.
__host__ __device__ constexpr int gemv_threads(int bmax) { return bmax >= 8 ? 256 : 512; }
// independent row loads per warp: 4 for the 1- and 2-slot kernels (two CTAs
// per SM), 8 for the 4-slot kernel (one CTA per SM, with the registers to
// spare), so that an SM keeps ~64 KB of weight reads in flight either way
__host__ __device__ constexpr int rows_in_flight(int bmax) { return bmax == 4 ? 8 : 4; }
// Shared memory of a CTA's active list: one row index plus BMAX fp32 x values
// per active row, so a K-split holds at most list_cap_max rows.
constexpr size_t kListBudget = 48 * 1024;
__host__ __device__ constexpr int list_cap_max(int bmax) {
  return (int)(kListBudget / (4 * (1 + (size_t)bmax))) / 32 * 32;
}
// Rows of the slice one thread tests: each thread owns a contiguous run.
__host__ __device__ constexpr int rows_per_thread_max(int bmax) {
  return (list_cap_max(bmax) + gemv_threads(bmax) - 1) / gemv_threads(bmax);
}

__device__ __forceinline__ float apply_epi(int epi, float v) {
  if (epi == EPI_GELU) return gelu_erf_f(v);
  if (epi == EPI_GELU_TANH) return gelu_tanh_f(v);
  return v;
}

// 16-byte weight load: skip L1, L2 evict-first (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// x[i .. i+3] as floats (0 past `lim`): one 8- or 16-byte load when `vec`
// (the four are 4-element aligned) and all four lie below `lim`.
__device__ __forceinline__ void unpack4(const uint2& q, float (&v)[4], __nv_bfloat16) {
  v[0] = __uint_as_float(q.x << 16);
  v[1] = __uint_as_float(q.x & 0xffff0000u);
  v[2] = __uint_as_float(q.y << 16);
  v[3] = __uint_as_float(q.y & 0xffff0000u);
}
__device__ __forceinline__ void unpack4(const uint2& q, float (&v)[4], __half) {
  const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&q.x));
  const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&q.y));
  v[0] = lo.x;
  v[1] = lo.y;
  v[2] = hi.x;
  v[3] = hi.y;
}
template <typename TX>
__device__ __forceinline__ void load4(const TX* p, long long i, long long lim, bool vec,
                                      float (&v)[4]) {
  if (vec && i + 3 < lim) {
    if constexpr (sizeof(TX) == 4) {
      const float4 q = *reinterpret_cast<const float4*>(p + i);
      v[0] = q.x;
      v[1] = q.y;
      v[2] = q.z;
      v[3] = q.w;
    } else {
      unpack4(*reinterpret_cast<const uint2*>(p + i), v, TX());
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = (i + j < lim) ? to_f32(p[i + j]) : 0.f;
  }
}

template <typename TW, typename TX, int NT, int BMAX>
__global__ void __launch_bounds__(gemv_threads(BMAX), (BMAX <= 2) ? 2 : 1)
    sparse_gemv_kernel(const GemvArgs a) {
  constexpr int kThreads = gemv_threads(BMAX);
  constexpr int kWarps = kThreads / 32;
  constexpr int C = NT / 256;          // 256-column chunks per tile
  constexpr int WPC = kWarps / C;      // warps per chunk
  static_assert(NT % 256 == 0 && kWarps % C == 0, "tile shape");

  // shared memory: [warp-reduction buffer, kWarps x 256 floats][active list:
  // rows, x values]; the split-K tail reuses the front as 4 x NT floats
  extern __shared__ __align__(16) unsigned char smem[];
  float* red = reinterpret_cast<float*>(smem);                       // [WPC][NT] floats
  int32_t* list_row = reinterpret_cast<int32_t*>(smem + (size_t)kWarps * 256 * 4);
  float* list_x = reinterpret_cast<float*>(list_row + a.list_cap);   // [cap][BMAX]

  __shared__ int s_warp_tot[kWarps];
  __shared__ int s_count;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tile = blockIdx.x;
  const int split = blockIdx.y;
  const long long n0 = (long long)tile * NT;
  const int ncols = (int)min((long long)NT, a.N - n0);

  // Inputs (x, caller lists) and the workspace may be written by the
  // previous kernel on the stream when launched as a dependent grid.
  pdl_wait();

  // ---------------------------------------------------------------- 1. active list
  if (a.idx == nullptr) {
    // Every active thread tests a contiguous run of r rows of the slice, r a
    // multiple of 4 and at least 4, in groups of four whose x values come in
    // one vector load; all of a thread's loads are independent, so the CTA
    // pays one L2 round trip for x. Runs of at least four rows keep the
    // number of threads (and instructions) that take part small: on B200 the
    // compaction of a few hundred rows is bound by instruction issue, not by
    // memory. One block scan of the per-thread counts then places the active
    // rows, ascending.
    constexpr int KG = (rows_per_thread_max(BMAX) + 3) / 4;  // groups of 4 per thread
    const long long k0 = (long long)split * a.slice;
    const long long k1 = min(a.K, k0 + a.slice);
    const int n = (int)max(0LL, k1 - k0);
    const int r = 4 * ((n + 4 * kThreads - 1) / (4 * kThreads));  // <= 4 KG
    const long long i0 = k0 + (long long)tid * r;
    const TX* xp = reinterpret_cast<const TX*>(a.x);
    const bool vec = (reinterpret_cast<uintptr_t>(a.x) % (4 * sizeof(TX))) == 0 &&
                     (a.B == 1 || (a.K & 3) == 0);
    // a given mask: the four rows of a group share one word (i % 4 == 0),
    // loaded together with x
    const uint32_t* mk = a.mask_in;
    const long long mwords = (a.K + 31) >> 5;
    float xv[4 * KG][BMAX];
    unsigned act = 0;
#pragma unroll
    for (int g = 0; g < KG; ++g) {
      const long long i = i0 + 4 * g;
      if (4 * g < r && i < k1) {
        unsigned mw[BMAX];
#pragma unroll
        for (int b = 0; b < BMAX; ++b) {
          float v[4] = {0.f, 0.f, 0.f, 0.f};
          mw[b] = 0u;
          if (b < a.B) {
            load4(xp + (long long)b * a.K, i, k1, vec, v);
            if (mk != nullptr) mw[b] = __ldg(mk + (long long)b * mwords + (i >> 5)) >> (i & 31);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) xv[4 * g + j][b] = v[j];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bool any = false;
#pragma unroll
          for (int b = 0; b < BMAX; ++b) {
            const bool m = b < a.B && i + j < k1 &&
                           (mk != nullptr ? ((mw[b] >> j) & 1u) != 0u
                                          : fabsf(xv[4 * g + j][b]) > a.t);
            any |= m;
            if (!m && !a.union_mask) xv[4 * g + j][b] = 0.f;
          }
          if (any) act |= 1u << (4 * g + j);
        }
      }
    }
    // exclusive scan of the counts: warp shuffles, then the warp totals
    const int mine = __popc(act);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp_tot[warp] = incl;
    __syncthreads();
    int pos = incl - mine, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = s_warp_tot[w];
      pos += (w < warp) ? c : 0;
      tot += c;
    }
#pragma unroll
    for (int g = 0; g < KG; ++g) {
      if ((act >> (4 * g)) & 0xFu) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if ((act >> (4 * g + j)) & 1u) {
            list_row[pos] = (int32_t)(i0 + 4 * g + j);
#pragma unroll
            for (int b = 0; b < BMAX; ++b) list_x[pos * BMAX + b] = xv[4 * g + j][b];
            ++pos;
          }
        }
      }
    }
    if (tid == 0) s_count = tot;
    // the fused mask, if asked for: the first column tile's CTAs write their
    // slice's bitmap words (k0 is a multiple of 32, so no word is shared)
    if (a.bitmap_out != nullptr && tile == 0) {
      const long long words = (a.K + 31) >> 5;
      for (long long w0 = k0 + (long long)warp * 32; w0 < k1; w0 += kThreads) {
        const long long i = w0 + lane;
        for (int b = 0; b < a.B; ++b) {
          const bool m = i < k1 && fabsf(to_f32(xp[(long long)b * a.K + i])) > a.t;
          const unsigned bal = __ballot_sync(0xffffffffu, m);
          if (lane == 0) a.bitmap_out[(long long)b * words + (w0 >> 5)] = bal;
        }
      }
    }
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

  // ---------------------------------------------------------------- 2. stream + FMA
  const int nrows = s_count;
  const int chunk = warp % C;      // which 256-column chunk this warp reads
  const int wrow = warp / C;       // row phase of this warp within the chunk
  const int col = chunk * 256 + lane * 8;
  const bool col_ok = col < ncols;
  const uint64_t pol = l2_evict_first_policy();
  const TW* Wc = reinterpret_cast<const TW*>(a.W) + n0 + col;
  float acc[BMAX][8];
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[b][j] = 0.f;

  if (col_ok) {
    // rows wrow, wrow + WPC, wrow + 2 WPC, ... ; kRows of them per step
    constexpr int kRows = rows_in_flight(BMAX);
    for (int r0 = wrow; r0 < nrows; r0 += WPC * kRows) {
      uint4 q[kRows];
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int r = r0 + u * WPC;
        if (r < nrows) q[u] = ldg_stream(Wc + (long long)list_row[r] * a.N, pol);
      }
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int r = r0 + u * WPC;
        if (r < nrows) {
          float w[8];
          unpack8(q[u], w, TW());
          const float* xr = list_x + (size_t)r * BMAX;
#pragma unroll
          for (int b = 0; b < BMAX; ++b) {
            const float xv = xr[b];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[b][j] = fmaf(xv, w[j], acc[b][j]);
          }
        }
      }
    }
  }
  pdl_launch_dependents();

  // ---------------------------------------------------------------- 3. reductions
  const bool swiglu = a.epi == EPI_SWIGLU;
  const long long N = a.N;
#pragma unroll
  for (int b = 0; b < BMAX; ++b) {
    if (b >= a.B) break;
    __syncthreads();  // red is free (previous token done, list reads done)
    if (col_ok) {
      float4* dst = reinterpret_cast<float4*>(red + wrow * NT + col);
      dst[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
      dst[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
    }
    __syncthreads();
    // sum the WPC warps of each chunk: thread handles 4 columns
    for (int v = tid; v < ncols / 4; v += kThreads) {
      float4 s = reinterpret_cast<const float4*>(red)[v];
#pragma unroll
      for (int r = 1; r < WPC; ++r) {
        const float4 t4 = reinterpret_cast<const float4*>(red + r * NT)[v];
        s.x += t4.x; s.y += t4.y; s.z += t4.z; s.w += t4.w;
      }
      if (a.S == 1) {
        if (swiglu) {
          float* h = reinterpret_cast<float*>(a.y) + (long long)b * (N / 2) + n0 / 2;
          *reinterpret_cast<float2*>(h + 2 * v) = make_float2(silu_f(s.x) * s.y, silu_f(s.z) * s.w);
        } else {
          const long long o = (long long)b * N + n0 + 4 * v;
          store_as(a.y, o + 0, a.ydt, apply_epi(a.epi, s.x));
          store_as(a.y, o + 1, a.ydt, apply_epi(a.epi, s.y));
          store_as(a.y, o + 2, a.ydt, apply_epi(a.epi, s.z));
          store_as(a.y, o + 3, a.ydt, apply_epi(a.epi, s.w));
        }
      } else {
        float* part = a.partials + ((long long)split * a.B + b) * N + n0;
        reinterpret_cast<float4*>(part)[v] = s;
      }
    }
  }
  if (a.S == 1) return;

  // last CTA of this column tile sums the S partials in split order
  __syncthreads();
  if (tid == 0) s_last = (arrive_acq_rel(&a.counters[tile]) == a.S - 1);
  __syncthreads();
  if (!s_last) return;
  // thread = (column group of 4, split group g of 4); split group g sums the
  // splits s = g, g + 4, g + 8, ... in order; the four group sums are then
  // added in group order.
  const long long vs = (long long)a.B * N / 4;  // float4 stride between splits
  const int nv = ncols / 4;
  float4* gsum = reinterpret_cast<float4*>(red);  // [4][nv]
  for (int b = 0; b < a.B; ++b) {
    __syncthreads();
    const float4* pb = reinterpret_cast<const float4*>(a.partials + (long long)b * N + n0);
    for (int e = tid; e < 4 * nv; e += kThreads) {
      const int g = e / nv, v = e - g * nv;
      // up to eight of the group's partials are loaded at once, then added
      // in split order
      float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = g; s0 < a.S; s0 += 32) {
        float4 q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int s = s0 + 4 * u;
          q[u] = s < a.S ? __ldcg(pb + (long long)s * vs + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (s0 + 4 * u < a.S) {
            acc4.x += q[u].x; acc4.y += q[u].y; acc4.z += q[u].z; acc4.w += q[u].w;
          }
        }
      }
      gsum[g * nv + v] = acc4;
    }
    __syncthreads();
    for (int v = tid; v < nv; v += kThreads) {
      float4 s4 = gsum[v];
#pragma unroll
      for (int g = 1; g < 4; ++g) {
        const float4 t4 = gsum[g * nv + v];
        s4.x += t4.x; s4.y += t4.y; s4.z += t4.z; s4.w += t4.w;
      }
      if (swiglu) {
        float* h = reinterpret_cast<float*>(a.y) + (long long)b * (N / 2) + n0 / 2;
        *reinterpret_cast<float2*>(h + 2 * v) = make_float2(silu_f(s4.x) * s4.y, silu_f(s4.z) * s4.w);
      } else {
        const long long o = (long long)b * N + n0 + 4 * v;
        store_as(a.y, o + 0, a.ydt, apply_epi(a.epi, s4.x));
        store_as(a.y, o + 1, a.ydt, apply_epi(a.epi, s4.y));
        store_as(a.y, o + 2, a.ydt, apply_epi(a.epi, s4.z));
        store_as(a.y, o + 3, a.ydt, apply_epi(a.epi, s4.w));
      }
    }
  }
  if (tid == 0) a.counters[tile] = 0;  // leave the workspace ready for the next call
}

template <typename TW, typename TX, int NT, int BMAX>
inline int launch_t(const GemvPlan& p, const GemvArgs& a, cudaStream_t stream, bool pdl) {
  auto kern = sparse_gemv_kernel<TW, TX, NT, BMAX>;
  static size_t configured = 0;  // per instantiation; raised under the helper's lock
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), p.smem, &configured) != SFX_OK)
    return SFX_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.col_tiles, (unsigned)p.S, 1);
  cfg.blockDim = dim3(gemv_threads(BMAX), 1, 1);
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
