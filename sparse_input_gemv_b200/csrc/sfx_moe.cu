// MoE layer with intra-expert activation sparsity on sm_100a.
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution", section "method": the routed experts' gate projection is
// computed densely and gives each neuron's activation score, a single O(n)
// threshold pass masks it, and the up and down projections read only the
// weights of active neurons; the router and the always-on shared expert are
// unchanged.
//
// Launches per call:
//  1. moe_route_kernel (one CTA): per token softmax over E logits, top-k by
//     probability (ties to the lower expert index), weights renormalised over
//     the selection (or raw); groups the selected (token, slot) pairs by
//     expert (experts ascending, tokens ascending) and zeroes the fp32 output
//     accumulator.
//  2. moe_expert_kernel, grid (ffn / 32 neuron chunks) x (active experts):
//       gate:  g_tj = W_gT[e][j, :] . x_t for the chunk's 32 neurons (dense,
//              one warp per neuron row, 4 KB contiguous rows), a = SiLU(g);
//       mask:  m_tj = |a_tj| > t_e[e];
//       up:    u_tj = W_upT[e][j, :] . x_t, only for neurons some token keeps;
//       down:  y_t += sum_j (w_te m_tj a_tj u_tj) W_d[e][j, :], reading only
//              those rows; the CTA's contribution is added to the fp32
//              accumulator with atomics (the combine order, hence the last
//              bits of y, may vary between runs).
//  3. the shared expert (if any): dense SwiGLU through the sparse GEMV path
//     with threshold -inf (gate|up with the SiLU epilogue, then down), fp32.
//  4. moe_finalize_kernel: y = accumulator (+ shared) in the output dtype.
#include "sfx_common.cuh"
#include "sfx_internal.h"

namespace sfx {

constexpr int kMoeChunk = 32;        // intermediate neurons per CTA
constexpr int kMaxMoeTokens = 16;    // tokens per call (each expert sees at most this many)

__host__ __device__ constexpr int moe_threads(int be) { return be >= 8 ? 256 : 512; }

// ---------------------------------------------------------------- workspace layout

struct MoeWs {
  int32_t* sel;       // [B x top_k] selected experts, selection order
  float* wsel;        // [B x top_k] routing weights
  int32_t* n_active;  // [1]
  int32_t* active;    // [max_active] active experts, ascending
  int32_t* tok_off;   // [max_active + 1]
  int32_t* tok;       // [B x top_k] token of each grouped pair
  int32_t* slot;      // [B x top_k] selection slot of each grouped pair
  float* tokw;        // [B x top_k] routing weight of each grouped pair
  float* acc;         // [B x d] fp32 output accumulator
  float* hs;          // [B x ffn_shared] shared-expert h
  float* ys;          // [B x d] shared-expert output
  unsigned char* gemv;  // partial sums of the shared-expert GEMVs
};

static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

// Carves the layout from `body`; returns the bytes used before the GEMV area.
static size_t carve_moe(unsigned char* body, int B, int d, int E, int top_k, int ffn_s, MoeWs* w) {
  const int pairs = B * top_k;
  const int max_active = pairs < E ? pairs : E;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += al256(bytes);
    return body ? body + at : nullptr;
  };
  MoeWs v;
  v.sel = reinterpret_cast<int32_t*>(take((size_t)pairs * 4));
  v.wsel = reinterpret_cast<float*>(take((size_t)pairs * 4));
  v.n_active = reinterpret_cast<int32_t*>(take(4));
  v.active = reinterpret_cast<int32_t*>(take((size_t)max_active * 4));
  v.tok_off = reinterpret_cast<int32_t*>(take((size_t)(max_active + 1) * 4));
  v.tok = reinterpret_cast<int32_t*>(take((size_t)pairs * 4));
  v.slot = reinterpret_cast<int32_t*>(take((size_t)pairs * 4));
  v.tokw = reinterpret_cast<float*>(take((size_t)pairs * 4));
  v.acc = reinterpret_cast<float*>(take((size_t)B * d * 4));
  v.hs = reinterpret_cast<float*>(take((size_t)B * (ffn_s > 0 ? ffn_s : 1) * 4));
  v.ys = reinterpret_cast<float*>(take((size_t)B * d * 4));
  v.gemv = body ? body + off : nullptr;
  if (w) *w = v;
  return off;
}

size_t moe_workspace_bytes(int B, int d, int E, int ffn, int top_k, int ffn_shared) {
  (void)ffn;
  const size_t head = carve_moe(nullptr, B, d, E, top_k, ffn_shared, nullptr);
  size_t g = 0;
  if (ffn_shared > 0) {
    const size_t g1 = gemv_workspace_bytes(d, 2LL * ffn_shared, B);
    const size_t g2 = gemv_workspace_bytes(ffn_shared, d, B);
    g = g1 > g2 ? g1 : g2;
  }
  return head + g;
}

// ---------------------------------------------------------------- 1. routing

__global__ void __launch_bounds__(1024) moe_route_kernel(const float* logits, int B, int E,
                                                         int top_k, int renorm, int d, MoeWs w) {
  extern __shared__ float s_z[];  // [E]
  __shared__ float s_red[32];
  __shared__ int s_redi[32];
  __shared__ int s_cnt[1024];     // per-expert pair counts (E <= 1024)
  __shared__ int s_off[1025];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;

  for (int i = tid; i < B * d; i += blockDim.x) w.acc[i] = 0.f;
  for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = 0;

  for (int t = 0; t < B; ++t) {
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) s_z[e] = logits[(long long)t * E + e];
    __syncthreads();
    // max logit and the softmax denominator over all experts
    float m = -INFINITY;
    for (int e = tid; e < E; e += blockDim.x) m = fmaxf(m, s_z[e]);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = s_red[0];
    for (int i = 1; i < nw; ++i) m = fmaxf(m, s_red[i]);
    __syncthreads();
    float den = 0.f;
    for (int e = tid; e < E; e += blockDim.x) den += expf(s_z[e] - m);
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) s_red[warp] = den;
    __syncthreads();
    den = 0.f;
    for (int i = 0; i < nw; ++i) den += s_red[i];
    __syncthreads();
    // top-k by repeated arg-max (largest logit, then lowest index); softmax is
    // monotone in the logit, so this is the top-k by probability
    float selsum = 0.f;
    for (int k = 0; k < top_k; ++k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int e = tid; e < E; e += blockDim.x) {
        const float v = s_z[e];
        if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
      }
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (lane == 0) { s_red[warp] = bv; s_redi[warp] = bi; }
      __syncthreads();
      bv = s_red[0];
      bi = s_redi[0];
      for (int i = 1; i < nw; ++i) {
        if (s_red[i] > bv || (s_red[i] == bv && s_redi[i] < bi)) { bv = s_red[i]; bi = s_redi[i]; }
      }
      const float pe = expf(bv - m);
      selsum += pe;
      if (tid == 0) {
        w.sel[t * top_k + k] = bi;
        w.wsel[t * top_k + k] = pe;  // scaled below
        s_cnt[bi] += 1;
        s_z[bi] = -INFINITY;  // taken
      }
      __syncthreads();
    }
    if (tid < top_k) w.wsel[t * top_k + tid] /= (renorm ? selsum : den);
  }
  __syncthreads();
  // group pairs by expert: ascending experts, tokens ascending within one
  if (tid == 0) {
    int na = 0, off = 0;
    for (int e = 0; e < E; ++e) {
      if (s_cnt[e] > 0) {
        w.active[na] = e;
        w.tok_off[na] = off;
        s_off[e] = off;
        off += s_cnt[e];
        ++na;
      }
    }
    w.tok_off[na] = off;
    *w.n_active = na;
    for (int t = 0; t < B; ++t)
      for (int k = 0; k < top_k; ++k) {
        const int e = w.sel[t * top_k + k];
        const int q = s_off[e]++;
        w.tok[q] = t;
        w.slot[q] = k;
        w.tokw[q] = w.wsel[t * top_k + k];
      }
  }
}

// ---------------------------------------------------------------- 2. experts

template <typename TW>
__device__ __forceinline__ void load_x8(const TW* x, float (&v)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(x));
  unpack8(q, v, TW());
}

template <typename TW, int BE>
__global__ void __launch_bounds__(moe_threads(BE), BE == 1 ? 2 : 1)
    moe_expert_kernel(const TW* __restrict__ x, int d, int ffn, int top_k,
                      const TW* __restrict__ WgT, const TW* __restrict__ WupT,
                      const TW* __restrict__ Wd, const float* __restrict__ t_e, float* a_out,
                      MoeWs w) {
  constexpr int kThreads = moe_threads(BE);
  constexpr int kWarps = kThreads / 32;
  __shared__ int s_tok[BE];
  __shared__ int s_slot[BE];
  __shared__ float s_w[BE];
  __shared__ float s_a[kMoeChunk][BE];
  __shared__ float s_v[kMoeChunk][BE];
  __shared__ int s_list[kMoeChunk];
  __shared__ int s_n;

  const int p = blockIdx.y;
  if (p >= *w.n_active) return;
  const int e = w.active[p];
  const int q0 = w.tok_off[p];
  const int ne = w.tok_off[p + 1] - q0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < ne) {
    s_tok[tid] = w.tok[q0 + tid];
    s_slot[tid] = w.slot[q0 + tid];
    s_w[tid] = w.tokw[q0 + tid];
  }
  __syncthreads();
  const int j0 = blockIdx.x * kMoeChunk;
  const long long erow = (long long)e * ffn;  // first row of expert e in [E x ffn x d]
  const float te = t_e[e];

  // dot products W[j, :] . x_t for the tokens of this expert, one warp per row
  auto dot_rows = [&](const TW* Wm, int j, float (&out)[BE]) {
#pragma unroll
    for (int b = 0; b < BE; ++b) out[b] = 0.f;
    const TW* row = Wm + (erow + j) * d;
    for (int c0 = lane * 8; c0 < d; c0 += 256 * 4) {
      uint4 wq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + u * 256 < d) wq[u] = __ldcs(reinterpret_cast<const uint4*>(row + c0 + u * 256));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 256;
        if (c < d) {
          float wv[8];
          unpack8(wq[u], wv, TW());
#pragma unroll
          for (int b = 0; b < BE; ++b) {
            if (b < ne) {
              float xv[8];
              load_x8(x + (long long)s_tok[b] * d + c, xv);
#pragma unroll
              for (int k = 0; k < 8; ++k) out[b] = fmaf(wv[k], xv[k], out[b]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BE; ++b)
      for (int o = 16; o; o >>= 1) out[b] += __shfl_xor_sync(0xffffffffu, out[b], o);
  };

  // gate (dense) and SiLU
  for (int jl = warp; jl < kMoeChunk; jl += kWarps) {
    const int j = j0 + jl;
    float g[BE];
    if (j < ffn) {
      dot_rows(WgT, j, g);
    } else {
#pragma unroll
      for (int b = 0; b < BE; ++b) g[b] = 0.f;
    }
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < BE; ++b) {
        if (b < ne) {
          const float av = silu_f(g[b]);
          s_a[jl][b] = av;
          if (a_out && j < ffn)
            a_out[((long long)s_tok[b] * top_k + s_slot[b]) * ffn + j] = av;
        }
      }
    }
  }
  __syncthreads();
  // threshold mask; neurons some token keeps, ascending
  if (warp == 0) {
    bool keep = false;
    const int j = j0 + lane;
    if (lane < kMoeChunk && j < ffn)
      for (int b = 0; b < ne; ++b) keep |= fabsf(s_a[lane][b]) > te;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) s_list[__popc(bal & lanemask_lt())] = lane;
    if (lane == 0) s_n = __popc(bal);
  }
  __syncthreads();
  const int na = s_n;
  // up projection for kept neurons; v = w_te * m * a * u
  for (int k = warp; k < na; k += kWarps) {
    const int jl = s_list[k];
    float u[BE];
    dot_rows(WupT, j0 + jl, u);
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < BE; ++b) {
        if (b < ne) {
          const float av = s_a[jl][b];
          s_v[k][b] = (fabsf(av) > te) ? s_w[b] * av * u[b] : 0.f;
        }
      }
    }
  }
  __syncthreads();
  if (na == 0) return;
  // down projection over the kept rows: warps own 256-column chunks
  const int nch = (d + 255) / 256;
  for (int ch0 = 0; ch0 < nch; ch0 += kWarps) {
    // one pass covers kWarps chunks (each warp one chunk, all kept rows)
    const int ch = ch0 + warp;
    const int col = ch * 256 + lane * 8;
    float acc[BE][8];
#pragma unroll
    for (int b = 0; b < BE; ++b)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[b][k] = 0.f;
    if (ch < nch && col < d) {
      for (int k0 = 0; k0 < na; k0 += 4) {
        uint4 wq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (k0 + u < na)
            wq[u] = __ldcs(reinterpret_cast<const uint4*>(Wd + (erow + j0 + s_list[k0 + u]) * d + col));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (k0 + u < na) {
            float wv[8];
            unpack8(wq[u], wv, TW());
#pragma unroll
            for (int b = 0; b < BE; ++b) {
              const float vv = (b < ne) ? s_v[k0 + u][b] : 0.f;
#pragma unroll
              for (int k = 0; k < 8; ++k) acc[b][k] = fmaf(vv, wv[k], acc[b][k]);
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < BE; ++b) {
        if (b < ne) {
          float* dst = w.acc + (long long)s_tok[b] * d + col;
#pragma unroll
          for (int k = 0; k < 8; ++k) atomicAdd(dst + k, acc[b][k]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- 4. finalize

__global__ void moe_finalize_kernel(const float* acc, const float* ys, long long n, void* y, int ydt) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    float v = acc[i];
    if (ys) v += ys[i];
    store_as(y, i, ydt, v);
  }
}

// ---------------------------------------------------------------- host

template <typename TW, int BE>
static int launch_experts(const void* x, int d, int ffn, int top_k, int max_active,
                          const void* WgT, const void* WupT, const void* Wd, const float* t_e,
                          float* a_out, const MoeWs& w, cudaStream_t s) {
  const dim3 grid((ffn + kMoeChunk - 1) / kMoeChunk, max_active);
  moe_expert_kernel<TW, BE><<<grid, moe_threads(BE), 0, s>>>(
      reinterpret_cast<const TW*>(x), d, ffn, top_k, reinterpret_cast<const TW*>(WgT),
      reinterpret_cast<const TW*>(WupT), reinterpret_cast<const TW*>(Wd), t_e, a_out, w);
  return cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

template <typename TW>
static int launch_experts_t(int B, const void* x, int d, int ffn, int top_k, int max_active,
                            const void* WgT, const void* WupT, const void* Wd, const float* t_e,
                            float* a_out, const MoeWs& w, cudaStream_t s) {
  if (B <= 1) return launch_experts<TW, 1>(x, d, ffn, top_k, max_active, WgT, WupT, Wd, t_e, a_out, w, s);
  if (B <= 4) return launch_experts<TW, 4>(x, d, ffn, top_k, max_active, WgT, WupT, Wd, t_e, a_out, w, s);
  if (B <= 8) return launch_experts<TW, 8>(x, d, ffn, top_k, max_active, WgT, WupT, Wd, t_e, a_out, w, s);
  return launch_experts<TW, 16>(x, d, ffn, top_k, max_active, WgT, WupT, Wd, t_e, a_out, w, s);
}

int run_moe(const void* x, int dt, const float* logits, int B, int d, int E, int ffn, int top_k,
            const void* W_gT, const void* W_upT, const void* W_d, const float* t_e,
            const void* Ws_gu, const void* Ws_d, int ffn_shared, void* y, int ydt, float* a_out,
            int32_t* sel_out, int flags, unsigned char* body, size_t body_bytes, unsigned* status,
            cudaStream_t s) {
  (void)body_bytes;
  if (B > kMaxMoeTokens || E > 1024) return SFX_ERR_UNSUPPORTED;
  MoeWs w;
  carve_moe(body, B, d, E, top_k, ffn_shared, &w);
  const int renorm = (flags & SFX_FLAG_NO_RENORM) ? 0 : 1;
  moe_route_kernel<<<1, 1024, (size_t)E * 4, s>>>(logits, B, E, top_k, renorm, d, w);
  if (cudaGetLastError() != cudaSuccess) return SFX_ERR_CUDA;
  if (sel_out &&
      cudaMemcpyAsync(sel_out, w.sel, sizeof(int32_t) * B * top_k, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return SFX_ERR_CUDA;
  const int pairs = B * top_k;
  const int max_active = pairs < E ? pairs : E;
  int rc = (dt == SFX_BF16)
               ? launch_experts_t<__nv_bfloat16>(B, x, d, ffn, top_k, max_active, W_gT, W_upT,
                                                 W_d, t_e, a_out, w, s)
               : launch_experts_t<__half>(B, x, d, ffn, top_k, max_active, W_gT, W_upT, W_d,
                                          t_e, a_out, w, s);
  if (rc != SFX_OK) return rc;
  const float* ys = nullptr;
  if (Ws_gu != nullptr) {
    // dense shared SwiGLU expert through the GEMV path (threshold -inf)
    GemvArgs g = {};
    g.x = x;
    g.W = Ws_gu;
    g.y = w.hs;
    g.status = status;
    g.counters = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(status) + kWsStatusBytes);
    g.partials = reinterpret_cast<float*>(w.gemv);
    g.K = d;
    g.N = 2LL * ffn_shared;
    g.B = B;
    g.ydt = SFX_F32;
    g.epi = EPI_SWIGLU;
    g.t = -INFINITY;
    rc = launch_sparse_gemv(dt, dt, plan_gemv(g.K, g.N, B, false), g, s, true);
    if (rc != SFX_OK) return rc;
    GemvArgs h = g;
    h.x = w.hs;
    h.W = Ws_d;
    h.y = w.ys;
    h.K = ffn_shared;
    h.N = d;
    h.epi = EPI_NONE;
    rc = launch_sparse_gemv(dt, SFX_F32, plan_gemv(h.K, h.N, B, false), h, s, true);
    if (rc != SFX_OK) return rc;
    ys = w.ys;
  }
  const long long n = (long long)B * d;
  moe_finalize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w.acc, ys, n, y, ydt);
  return cudaGetLastError() == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

}  // namespace sfx
