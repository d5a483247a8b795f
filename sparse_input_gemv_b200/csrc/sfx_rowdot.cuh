// Row-dot building blocks shared by the MoE expert kernel and the static-mask
// FFN kernel (sm_100a): neuron-row dot products on the tensor cores and the
// row-sparse down projection into an fp32 accumulator.
#pragma once

#include "sfx_common.cuh"

namespace sfx {

constexpr int kRowThreads = 256;  // CTA size of the kernels built on these helpers
constexpr int kRowTok = 16;       // tokens per pass: two 8-token MMA tiles
constexpr int kXPad = 32;         // staged x row stride d + 32 elements (bank spread)

// D (16 x 8, f32) += A (16 x 16) B (16 x 8) on the tensor cores, A and B in the
// storage dtype (both bf16 or both f16), one warp.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1, __nv_bfloat16) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1, __half) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// S[r][t] = W[row(r), :] . x_t for r < nrows (<= 64) and the item's ne tokens,
// on the tensor cores: warps take (16-row tile, slice of K) pairs. Lane
// (g = lane / 4, q = lane % 4) loads 16 bytes at k0 + 8q of rows g and g + 8 of
// its tile and of tokens g and g + 8; the contraction runs over physical k, so
// the fragment's logical k order need not match memory (A and B use the same
// assignment). Partial sums go to s_part; the caller reduces them.
template <typename TW, typename RowFn>
__device__ __forceinline__ void mma_rows(const TW* __restrict__ Wm, RowFn row_of, int nrows,
                                         int d, const TW* xs, int xstride, int ne,
                                         float (*s_part)[16][kRowTok], int* n_tiles_out,
                                         int* ksplit_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  constexpr int kWarps = kRowThreads / 32;
  const int n_tiles = (nrows + 15) >> 4;
  const int ksplit = n_tiles > 0 ? kWarps / n_tiles : 0;
  *n_tiles_out = n_tiles;
  *ksplit_out = ksplit;
  const int rt = n_tiles > 0 ? warp % n_tiles : 0, ks = n_tiles > 0 ? warp / n_tiles : kWarps;
  if (ks >= ksplit) return;
  const int nblk = (d + 31) >> 5;
  const int per = (nblk + ksplit - 1) / ksplit;
  const int blk0 = ks * per, blk1 = blk0 + per < nblk ? blk0 + per : nblk;
  const int r0 = rt * 16 + g, r1 = r0 + 8;
  const TW* p0 = r0 < nrows ? Wm + row_of(r0) * (long long)d : nullptr;
  const TW* p1 = r1 < nrows ? Wm + row_of(r1) * (long long)d : nullptr;
  const bool t0 = g < ne, t1 = g + 8 < ne, two = ne > 8;
  const TW* x0 = xs + (long long)g * xstride;
  const TW* x1 = xs + (long long)(g + 8) * xstride;
  float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  constexpr int U = 4;  // 32-element blocks in flight per lane (2 rows x 16 B each)
  for (int b = blk0; b < blk1; b += U) {
    uint4 wa[U], wb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = (b + u) * 32 + 8 * q;
      const bool ok = b + u < blk1 && k < d;
      wa[u] = (ok && p0) ? __ldcs(reinterpret_cast<const uint4*>(p0 + k)) : z;
      wb[u] = (ok && p1) ? __ldcs(reinterpret_cast<const uint4*>(p1 + k)) : z;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = (b + u) * 32 + 8 * q;
      if (b + u < blk1) {
        const bool kin = k < d;
        const uint4 xa = (kin && t0) ? *reinterpret_cast<const uint4*>(x0 + k) : z;
        mma_16816(c0, wa[u].x, wb[u].x, wa[u].y, wb[u].y, xa.x, xa.y, TW());
        mma_16816(c0, wa[u].z, wb[u].z, wa[u].w, wb[u].w, xa.z, xa.w, TW());
        if (two) {
          const uint4 xb = (kin && t1) ? *reinterpret_cast<const uint4*>(x1 + k) : z;
          mma_16816(c1, wa[u].x, wb[u].x, wa[u].y, wb[u].y, xb.x, xb.y, TW());
          mma_16816(c1, wa[u].z, wb[u].z, wa[u].w, wb[u].w, xb.z, xb.w, TW());
        }
      }
    }
  }
  // D fragment: c[0], c[1] = (row g, tokens 2q, 2q+1); c[2], c[3] = (row g+8, same)
  float(*sp)[kRowTok] = s_part[warp];
  sp[g][2 * q] = c0[0];
  sp[g][2 * q + 1] = c0[1];
  sp[g + 8][2 * q] = c0[2];
  sp[g + 8][2 * q + 1] = c0[3];
  sp[g][8 + 2 * q] = c1[0];
  sp[g][8 + 2 * q + 1] = c1[1];
  sp[g + 8][8 + 2 * q] = c1[2];
  sp[g + 8][8 + 2 * q + 1] = c1[3];
}

// Sum of the K-slice partials of row r, token t (after mma_rows and a barrier).
__device__ __forceinline__ float sum_parts(const float (*s_part)[16][kRowTok], int n_tiles,
                                           int ksplit, int r, int t) {
  const int rt = r >> 4, rr = r & 15;
  float s = 0.f;
  for (int ks = 0; ks < ksplit; ++ks) s += s_part[ks * n_tiles + rt][rr][t];
  return s;
}

// acc[tok(t0 + b)] += sum_k v[k][t0 + b] Wd[s_list[k], :] for NTOK tokens, the
// warps taking (256-column chunk, row phase) tasks; 16-byte atomics into acc.
// The chunks start at `rot` (mod the chunk count): callers whose items all add
// into the same token rows at the same time pass the item index, so that their
// atomics land on different columns.
template <typename TW, int NTOK>
__device__ __forceinline__ void down_pass(const TW* __restrict__ Wd, const int* s_list, int na,
                                          const float (*s_v)[kRowTok], int t0, const int* s_tok,
                                          int d, float* acc_out, int rot) {
  constexpr int kWarps = kRowThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = (d + 255) / 256;
  const int nsplit = kWarps >= nch ? kWarps / nch : 1;
  for (int task = warp; task < nch * nsplit; task += kWarps) {
    const int chk = (task + rot) % nch, par = task / nch;
    const int col = chk * 256 + lane * 8;
    if (col >= d) continue;
    float acc[NTOK][8];
#pragma unroll
    for (int b = 0; b < NTOK; ++b)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[b][k] = 0.f;
    constexpr int L = NTOK <= 2 ? 4 : 2;  // rows in flight (registers: acc grows with NTOK)
    for (int k0 = par; k0 < na; k0 += L * nsplit) {
      uint4 wq[L];
#pragma unroll
      for (int u = 0; u < L; ++u) {
        const int k = k0 + u * nsplit;
        if (k < na)
          wq[u] = __ldcs(reinterpret_cast<const uint4*>(Wd + (long long)s_list[k] * d + col));
      }
#pragma unroll
      for (int u = 0; u < L; ++u) {
        const int k = k0 + u * nsplit;
        if (k < na) {
          float wv[8];
          unpack8(wq[u], wv, TW());
#pragma unroll
          for (int b = 0; b < NTOK; ++b) {
            const float vv = s_v[k][t0 + b];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) acc[b][kk] = fmaf(vv, wv[kk], acc[b][kk]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NTOK; ++b) {
      float4* dst = reinterpret_cast<float4*>(acc_out + (long long)s_tok[t0 + b] * d + col);
      atomicAdd(dst, make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]));
      atomicAdd(dst + 1, make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]));
    }
  }
}


// Runs down_pass over ne tokens in passes of at most four.
template <typename TW>
__device__ __forceinline__ void down_all(const TW* __restrict__ Wd, const int* s_list, int na,
                                         const float (*s_v)[kRowTok], int ne, const int* s_tok,
                                         int d, float* acc_out, int rot = 0) {
  for (int t0 = 0; t0 < ne && na > 0; t0 += 4) {
    switch (ne - t0 < 4 ? ne - t0 : 4) {
      case 1: down_pass<TW, 1>(Wd, s_list, na, s_v, t0, s_tok, d, acc_out, rot); break;
      case 2: down_pass<TW, 2>(Wd, s_list, na, s_v, t0, s_tok, d, acc_out, rot); break;
      case 3: down_pass<TW, 3>(Wd, s_list, na, s_v, t0, s_tok, d, acc_out, rot); break;
      default: down_pass<TW, 4>(Wd, s_list, na, s_v, t0, s_tok, d, acc_out, rot); break;
    }
  }
}

}  // namespace sfx
