// MoE layer with intra-expert activation sparsity on sm_100a.
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution", section "method": the routed experts' gate projection is
// computed densely and gives each neuron's activation score, a single O(n)
// threshold pass masks it, and the up and down projections read only the
// weights of active neurons; the router and the always-on shared expert are
// unchanged.
//
// Every expert matrix, routed or shared, is stored one row per intermediate
// neuron ([ffn x d]), so a neuron's gate, up and down weights are three
// contiguous 2d-byte rows.
//
// Launches per call (all three programmatic dependent launches):
//  1. moe_route_kernel (one CTA, one warp per token): softmax over E logits,
//     top-k by probability (ties to the lower expert index), weights
//     renormalised over the selection (or raw); the selected (token, slot)
//     pairs grouped by expert (experts ascending, tokens ascending); the fp32
//     output accumulator zeroed.
//  2. moe_expert_kernel, one persistent CTA per SM taking work items (the
//     first by block index, the rest from an atomic counter): a chunk of the
//     shared expert's neurons (all tokens, weight 1, no threshold; these items
//     come first and do their gate and up work while routing still runs), or
//     of one active routed expert's (its tokens, at most 16):
//       gate:  g_tj = W_gT[e][j, :] . x_t for the chunk's neurons (dense; a
//              16-neuron x 8-token tensor-core tile per warp and K slice; the
//              chunk's rows are one contiguous block, prefetched to L2 when
//              the item starts), a = SiLU(g);
//       mask:  m_tj = |a_tj| > t_e[e] (then the kept up/down rows and the
//              next item's gate block are prefetched to L2);
//       up:    u_tj = W_upT[e][j, :] . x_t, only for neurons some token keeps
//              (tensor-core tiles over the kept rows);
//       down:  y_t += sum_j (w_te m_tj a_tj u_tj) W_d[e][j, :], reading only
//              those rows; each warp adds its 256-column partial to the
//              accumulator with 16-byte atomics (the combine order, hence the
//              last bits of y, may vary between runs).
//  3. moe_finalize_kernel (programmatic dependent of 2): y = accumulator in
//     the output dtype.
#include "sfx_common.cuh"
#include "sfx_internal.h"
#include "sfx_rowdot.cuh"

namespace sfx {

constexpr int kMaxMoeTokens = 16;  // tokens per call (each expert sees at most this many)
// the expert kernel stages x of all tokens of an item in shared memory
constexpr long long kMaxMoeTokenElems = 98304;  // B * d (192 KB of bf16)

constexpr int kMoeThreads = kRowThreads;  // expert CTAs: two per SM where shared memory allows
constexpr int kMoeChunkMax = 64;  // intermediate neurons per work item, at most

// ---------------------------------------------------------------- workspace layout

struct MoeWs {
  int32_t* n_active;   // [1]
  int32_t* next_item;  // [1] work-item counter of the expert grid
  int32_t* active;    // [max_active] active experts, ascending
  int32_t* tok_off;   // [max_active + 1]
  int32_t* tok;       // [B x top_k] token of each grouped pair
  int32_t* slot;      // [B x top_k] selection slot of each grouped pair
  float* tokw;        // [B x top_k] routing weight of each grouped pair
  float* acc;         // [B x d] fp32 output accumulator
};

static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

// Carves the layout from `body`; returns the bytes it takes.
static size_t carve_moe(unsigned char* body, int B, int d, int E, int top_k, MoeWs* w) {
  const int pairs = B * top_k;
  const int max_active = pairs < E ? pairs : E;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += al256(bytes);
    return body ? body + at : nullptr;
  };
  MoeWs v;
  v.n_active = reinterpret_cast<int32_t*>(take(4));
  v.next_item = reinterpret_cast<int32_t*>(take(4));
  v.active = reinterpret_cast<int32_t*>(take((size_t)max_active * 4));
  v.tok_off = reinterpret_cast<int32_t*>(take((size_t)(max_active + 1) * 4));
  v.tok = reinterpret_cast<int32_t*>(take((size_t)pairs * 4));
  v.slot = reinterpret_cast<int32_t*>(take((size_t)pairs * 4));
  v.tokw = reinterpret_cast<float*>(take((size_t)pairs * 4));
  v.acc = reinterpret_cast<float*>(take((size_t)B * d * 4));
  if (w) *w = v;
  return off;
}

size_t moe_workspace_bytes(int B, int d, int E, int ffn, int top_k, int ffn_shared) {
  (void)ffn;
  (void)ffn_shared;
  return carve_moe(nullptr, B, d, E, top_k, nullptr);
}

// ---------------------------------------------------------------- 1. routing

// One warp per token keeps the token's logits in shared memory, reduces max and
// softmax denominator with shuffles and takes the top-k by repeated warp
// arg-max (largest logit, then lowest index -- softmax is monotone in the
// logit, so this is the top-k by probability). The grouping by expert then
// runs on shared memory: per-expert counts and token masks, one warp's scan
// over experts, and each pair's rank among the earlier tokens of its expert.
__global__ void __launch_bounds__(512) moe_route_kernel(const float* logits, int B, int E,
                                                        int top_k, int renorm, int d, MoeWs w,
                                                        int32_t* sel_out) {
  extern __shared__ __align__(16) unsigned char s_raw[];
  float* s_z = reinterpret_cast<float*>(s_raw);                  // [B x E] logits
  int* s_sel = reinterpret_cast<int*>(s_z + (size_t)B * E);     // [B x top_k]
  float* s_wsel = reinterpret_cast<float*>(s_sel + B * top_k);  // [B x top_k]
  __shared__ int s_cnt[1024];  // per-expert pair counts (E <= 1024)
  __shared__ int s_off[1024];  // first grouped position of each expert
  __shared__ unsigned s_tokmask[1024];  // tokens (B <= 16) that selected each expert
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x, pairs = B * top_k;
  // launched as a programmatic dependent: the previous kernel's results (the
  // logits, x, this workspace's accumulator) are complete after the wait; only
  // then may the expert grid start (its shared-expert items read x at once and
  // wait for this grid's results where they need them)
  pdl_wait();
  pdl_launch_dependents();

  for (int i = tid; i < B * d; i += nthr) w.acc[i] = 0.f;
  if (tid == 0) *w.next_item = 0;
  for (int e = tid; e < E; e += nthr) {
    s_cnt[e] = 0;
    s_tokmask[e] = 0u;
  }
  if (warp < B) {
    const int t = warp;
    float* z = s_z + (size_t)t * E;
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) {
      z[e] = logits[(size_t)t * E + e];
      m = fmaxf(m, z[e]);
    }
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float den = 0.f;
    for (int e = lane; e < E; e += 32) den += expf(z[e] - m);
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    float selsum = 0.f;
    for (int k = 0; k < top_k; ++k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int e = lane; e < E; e += 32) {
        const float v = z[e];
        if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
      }
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      const float pe = expf(bv - m);
      selsum += pe;
      if (lane == 0) {
        s_sel[t * top_k + k] = bi;
        s_wsel[t * top_k + k] = pe;  // scaled below
        z[bi] = -INFINITY;           // taken
      }
      __syncwarp();
    }
    const float norm = renorm ? selsum : den;
    for (int k = lane; k < top_k; k += 32) {
      s_wsel[t * top_k + k] /= norm;
      if (sel_out) sel_out[t * top_k + k] = s_sel[t * top_k + k];
    }
  }
  __syncthreads();
  for (int q = tid; q < pairs; q += nthr) {
    atomicAdd(&s_cnt[s_sel[q]], 1);
    atomicOr(&s_tokmask[s_sel[q]], 1u << (q / top_k));
  }
  __syncthreads();
  // active experts ascending and their first grouped positions (warp scan)
  if (warp == 0) {
    int na = 0, off = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = (e < E) ? s_cnt[e] : 0;
      const unsigned act = __ballot_sync(0xffffffffu, c > 0);
      int v = c;  // inclusive scan of the counts
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      const int excl = off + v - c;
      if (c > 0) {
        const int ai = na + __popc(act & lanemask_lt());
        w.active[ai] = e;
        w.tok_off[ai] = excl;
      }
      if (e < E) s_off[e] = excl;
      off += __shfl_sync(0xffffffffu, v, 31);
      na += __popc(act);
    }
    if (lane == 0) {
      w.tok_off[na] = off;
      *w.n_active = na;
    }
  }
  __syncthreads();
  // pair q = (token t, slot k) goes after the earlier tokens of its expert (a
  // token selects an expert at most once)
  for (int q = tid; q < pairs; q += nthr) {
    const int e = s_sel[q], t = q / top_k;
    const int pos = s_off[e] + __popc(s_tokmask[e] & ((1u << t) - 1u));
    w.tok[pos] = t;
    w.slot[pos] = q % top_k;
    w.tokw[pos] = s_wsel[q];
  }
}

// ---------------------------------------------------------------- 2. experts

// Pointers of one expert kind: the routed stack [E x ffn x d] or the shared expert.
template <typename TW>
struct ExpertMats {
  const TW* gT;
  const TW* upT;
  const TW* d;
};

// Work items: 0 .. n_shared-1 are the shared expert's chunks of ch_s neurons,
// then (active expert p, chunk c) with ch neurons, in order of p. A routed
// neuron costs its gate row plus, at about half kept, one up and one down row;
// a shared neuron costs all three rows, so shared chunks are 2/3 as long.
struct MoeItems {
  int ch, ch_s;    // neurons per routed / shared item
  int n_chunks;    // items per routed expert
  int n_shared;    // shared-expert items
  int n_total;     // n_shared + max_active * n_chunks
};

struct MoeItem {
  bool shared;
  int p, e, j0, nj;
  int q0, ne;  // routed items: first grouped pair and number of tokens
};

// Decodes item `it`; false for a routed item past the active experts (all
// later items are past them too). Routed items need the routing results.
__device__ __forceinline__ bool decode_item(int it, const MoeItems& I, int ffn, int ffn_s,
                                            const MoeWs& w, MoeItem* out) {
  MoeItem m;
  m.shared = it < I.n_shared;
  if (m.shared) {
    m.p = -1;
    m.e = 0;
    m.q0 = m.ne = 0;  // the shared expert takes every token
    m.j0 = it * I.ch_s;
    m.nj = ffn_s - m.j0 < I.ch_s ? ffn_s - m.j0 : I.ch_s;
  } else {
    const int k = it - I.n_shared;
    m.p = k / I.n_chunks;
    // p < max_active, so the expert and token offsets are in bounds: load them
    // together with the count (one round trip instead of three)
    const int na = *w.n_active;
    const int e = w.active[m.p];
    const int q0 = w.tok_off[m.p], q1 = w.tok_off[m.p + 1];
    if (m.p >= na) return false;
    m.e = e;
    m.q0 = q0;
    m.ne = q1 - q0;
    m.j0 = (k - m.p * I.n_chunks) * I.ch;
    m.nj = ffn - m.j0 < I.ch ? ffn - m.j0 : I.ch;
  }
  *out = m;
  return true;
}

// Persistent CTAs (as many as fit on the SMs): the first item is blockIdx.x, later ones come
// from an atomic counter (gridDim.x + counter), so SMs that finish early take
// more. While an item runs its up and down phases, the next item's gate block
// is already on its way to L2.
template <typename TW>
__global__ void __launch_bounds__(kMoeThreads, 2)
    moe_expert_kernel(const TW* __restrict__ x, int B, int d, int ffn, int ffn_s, MoeItems I,
                      int top_k, ExpertMats<TW> R, ExpertMats<TW> S,
                      const float* __restrict__ t_e, float* a_out, MoeWs w) {
  constexpr int CH = kMoeChunkMax;
  constexpr int kWarps = kMoeThreads / 32;
  extern __shared__ __align__(16) unsigned char s_xraw[];  // [ne][d + kXPad] x of the item's tokens
  __shared__ float s_part[kWarps][16][kRowTok];             // K-slice partial sums
  __shared__ float s_a[CH][kRowTok];
  __shared__ float s_v[CH][kRowTok];
  __shared__ int s_tok[kRowTok];
  __shared__ float s_w[kRowTok];
  __shared__ int s_slot[kRowTok];
  __shared__ int s_list[CH];
  __shared__ int s_wcnt[CH / 32];
  __shared__ int s_next;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long row_bytes = (long long)d * sizeof(TW);
  const int xstride = d + kXPad;
  TW* xs = reinterpret_cast<TW*>(s_xraw);
  // routing results, the zeroed accumulator and the item counter come from the
  // previous grid; every thread takes the same branches, so the wait is CTA-uniform
  bool waited = false;
  auto wait_routing = [&]() {
    if (!waited) {
      pdl_wait();
      waited = true;
    }
  };
  // the item's gate rows are one contiguous block: 16 KB bulk prefetches to L2
  auto prefetch_gate = [&](const MoeItem& m) {
    const TW* gm = m.shared ? S.gT : R.gT;
    const char* base = reinterpret_cast<const char*>(
        gm + ((long long)m.e * (m.shared ? ffn_s : ffn) + m.j0) * d);
    const long long total = m.nj * row_bytes;
    constexpr long long kPiece = 16384;
    for (long long off = (long long)tid * kPiece; off < total; off += kMoeThreads * kPiece)
      prefetch_l2_bulk(base + off, (uint32_t)(total - off < kPiece ? total - off : kPiece));
  };

  int it = blockIdx.x;
  if (it >= I.n_total) return;
  if (it >= I.n_shared) wait_routing();
  MoeItem cur;
  if (!decode_item(it, I, ffn, ffn_s, w, &cur)) return;
  prefetch_gate(cur);

  for (;;) {
    const ExpertMats<TW> M = cur.shared ? S : R;
    const int nf = cur.shared ? ffn_s : ffn;
    const long long erow = (long long)cur.e * nf;  // first row of the expert in its stack
    const int j0 = cur.j0, nj = cur.nj;
    int ne;
    float te;
    __syncthreads();  // the previous item is done with the shared arrays
    if (cur.shared) {
      ne = B;
      te = -INFINITY;
      if (tid < B) {
        s_tok[tid] = tid;
        s_slot[tid] = -1;
        s_w[tid] = 1.f;
      }
    } else {
      const int q0 = cur.q0;
      ne = cur.ne;
      te = t_e[cur.e];
      if (tid < ne) {
        s_tok[tid] = w.tok[q0 + tid];
        s_slot[tid] = w.slot[q0 + tid];
        s_w[tid] = w.tokw[q0 + tid];
      }
    }
    __syncthreads();
    // stage x of the item's tokens (d % 8 == 0: whole 16-byte words)
    for (int i = tid; i < ne * (d / 8); i += kMoeThreads) {
      const int b = i / (d / 8), c = i - b * (d / 8);
      *reinterpret_cast<uint4*>(xs + (long long)b * xstride + c * 8) =
          __ldg(reinterpret_cast<const uint4*>(x + (long long)s_tok[b] * d) + c);
    }
    __syncthreads();

    // gate (dense) on the tensor cores, then SiLU
    int n_tiles, ksplit;
    mma_rows(M.gT, [&](int r) { return erow + j0 + r; }, nj, d, xs, xstride, ne, s_part,
             &n_tiles, &ksplit);
    __syncthreads();
    for (int i = tid; i < nj * ne; i += kMoeThreads) {
      const int r = i / ne, t = i - r * ne;
      const float av = silu_f(sum_parts(s_part, n_tiles, ksplit, r, t));
      s_a[r][t] = av;
      if (a_out && !cur.shared)
        a_out[((long long)s_tok[t] * top_k + s_slot[t]) * ffn + j0 + r] = av;
    }
    __syncthreads();
    // threshold mask; the chunk's neurons some token keeps, ascending
    bool keep = false;
    unsigned bal = 0;
    if (warp < CH / 32) {
      if (tid < nj)
        for (int t = 0; t < ne; ++t) keep |= fabsf(s_a[tid][t]) > te;
      bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) s_wcnt[warp] = __popc(bal);
    }
    __syncthreads();
    int na = 0, woff = 0;
#pragma unroll
    for (int q = 0; q < CH / 32; ++q) {
      woff += (q < warp) ? s_wcnt[q] : 0;
      na += s_wcnt[q];
    }
    if (keep) s_list[woff + __popc(bal & lanemask_lt())] = tid;
    // start the kept up and down rows towards L2, one bulk prefetch per row
    __syncthreads();
    for (int k = tid; k < 2 * na; k += kMoeThreads) {
      const TW* m = (k < na) ? M.upT : M.d;
      const int kk = (k < na) ? k : k - na;
      prefetch_l2_bulk(m + (erow + j0 + s_list[kk]) * d, (uint32_t)row_bytes);
    }
    // the next item: take one from the counter, start its gate block too
    wait_routing();
    if (tid == 0) s_next = (int)gridDim.x + atomicAdd(w.next_item, 1);
    // up projection for the kept neurons on the tensor cores
    mma_rows(M.upT, [&](int r) { return erow + j0 + s_list[r]; }, na, d, xs, xstride, ne, s_part,
             &n_tiles, &ksplit);
    __syncthreads();
    const int nxt_it = s_next;
    MoeItem nxt;
    const bool has_next = nxt_it < I.n_total && decode_item(nxt_it, I, ffn, ffn_s, w, &nxt);
    if (has_next) prefetch_gate(nxt);
    // v = w_te * m * a * u
    for (int i = tid; i < na * ne; i += kMoeThreads) {
      const int k = i / ne, t = i - k * ne;
      const float av = s_a[s_list[k]][t];
      s_v[k][t] = (fabsf(av) > te) ? s_w[t] * av * sum_parts(s_part, n_tiles, ksplit, k, t) : 0.f;
    }
    __syncthreads();
    // down projection over the kept rows, four tokens per pass
    down_all(M.d + (erow + j0) * d, s_list, na, s_v, ne, s_tok, d, w.acc);
    if (!has_next) break;
    cur = nxt;
    it = nxt_it;
  }
}

// ---------------------------------------------------------------- 3. finalize

__global__ void moe_finalize_kernel(const float* acc, long long n, void* y, int ydt) {
  pdl_wait();  // the expert grid's accumulator
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    store_as(y, i, ydt, acc[i]);
}

// ---------------------------------------------------------------- host

// Item sizes: routed chunks of 32 neurons (shared-expert chunks of 21: all three
// of a shared neuron's rows are read). Measured on B200 for the 128 x 768 top-8
// layer with a 2048-neuron shared expert, chunks of 16 / 24 / 32 / 48 / 64
// neurons at 1 / 4 / 8 / 16 tokens: 32 is the fastest or within 0.1 % of it at
// every batch (4 tokens, p = 0.5: 64.6 us against 80.4 with 64). Then 8 warps
// split a chunk as two 16-row tiles x four K slices, and the atomic item counter
// balances the SMs at every batch. SFX_PLAN_MOE_CHUNK overrides it for sweeps.
constexpr int kMoeChunkDefault = 32;
static MoeItems moe_items(int ffn, int ffn_s, int max_active) {
  MoeItems I;
  const int ov = plan_override(SFX_PLAN_MOE_CHUNK);
  const int ch = (ov >= 16 && ov <= kMoeChunkMax) ? ov : kMoeChunkDefault;
  I.ch = ch;
  I.ch_s = (2 * ch + 1) / 3;
  I.n_chunks = (ffn + ch - 1) / ch;
  I.n_shared = ffn_s > 0 ? (ffn_s + I.ch_s - 1) / I.ch_s : 0;
  I.n_total = I.n_shared + max_active * I.n_chunks;
  return I;
}

template <typename TW>
static int launch_experts(int B, const void* x, int d, int ffn, int ffn_s, int top_k,
                          int max_active, const void* W_gT, const void* W_upT, const void* W_d,
                          const void* Ws_gT, const void* Ws_upT, const void* Ws_d,
                          const float* t_e, float* a_out, const MoeWs& w, cudaStream_t s) {
  const ExpertMats<TW> R = {reinterpret_cast<const TW*>(W_gT), reinterpret_cast<const TW*>(W_upT),
                            reinterpret_cast<const TW*>(W_d)};
  const ExpertMats<TW> S = {reinterpret_cast<const TW*>(Ws_gT),
                            reinterpret_cast<const TW*>(Ws_upT), reinterpret_cast<const TW*>(Ws_d)};
  auto kern = moe_expert_kernel<TW>;
  const size_t smem = (size_t)B * (d + kXPad) * sizeof(TW);  // x of an item's tokens (<= B)
  static size_t configured = 0;  // one opt-in per kernel instantiation
  // opt in whenever the size grows: dynamic plus ~17 KB static may pass 48 KB
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem, &configured) != SFX_OK)
    return SFX_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kMoeThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return SFX_ERR_CUDA;
  const int slots = sm_count() * per_sm;
  const MoeItems I = moe_items(ffn, ffn_s, max_active);
  const int grid = I.n_total < slots ? I.n_total : slots;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kMoeThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const TW*>(x), B, d, ffn, ffn_s, I, top_k,
                         R, S, t_e, a_out, w) != cudaSuccess)
    return SFX_ERR_CUDA;
  return SFX_OK;
}

int run_moe(const void* x, int dt, const float* logits, int B, int d, int E, int ffn, int top_k,
            const void* W_gT, const void* W_upT, const void* W_d, const float* t_e,
            const void* Ws_gT, const void* Ws_upT, const void* Ws_d, int ffn_shared, void* y,
            int ydt, float* a_out, int32_t* sel_out, int flags, unsigned char* body,
            size_t body_bytes, cudaStream_t s) {
  (void)body_bytes;
  if (B > kMaxMoeTokens || E > 1024 || (long long)B * d > kMaxMoeTokenElems)
    return SFX_ERR_UNSUPPORTED;
  MoeWs w;
  carve_moe(body, B, d, E, top_k, &w);
  const int renorm = (flags & SFX_FLAG_NO_RENORM) ? 0 : 1;
  const size_t route_smem = (size_t)B * E * 4 + (size_t)B * top_k * 8;
  if (route_smem > 48 * 1024) {
    static size_t route_configured = 0;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(moe_route_kernel), route_smem,
                            &route_configured) != SFX_OK)
      return SFX_ERR_CUDA;
  }
  const int route_threads = 32 * (B > 4 ? B : 4);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3((unsigned)route_threads, 1, 1);
    cfg.dynamicSmemBytes = route_smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, moe_route_kernel, logits, B, E, top_k, renorm, d, w, sel_out) !=
        cudaSuccess)
      return SFX_ERR_CUDA;
  }
  const int pairs = B * top_k;
  const int max_active = pairs < E ? pairs : E;
  const int ffn_s = Ws_gT ? ffn_shared : 0;
  const int rc = (dt == SFX_BF16)
                     ? launch_experts<__nv_bfloat16>(B, x, d, ffn, ffn_s, top_k, max_active,
                                                       W_gT, W_upT, W_d, Ws_gT, Ws_upT, Ws_d,
                                                       t_e, a_out, w, s)
                     : launch_experts<__half>(B, x, d, ffn, ffn_s, top_k, max_active, W_gT,
                                                W_upT, W_d, Ws_gT, Ws_upT, Ws_d, t_e, a_out, w, s);
  if (rc != SFX_OK) return rc;
  // finalize as a programmatic dependent: its launch overlaps the expert grid's tail
  const long long n = (long long)B * d;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_finalize_kernel, (const float*)w.acc, n, y, ydt) ==
                 cudaSuccess
             ? SFX_OK
             : SFX_ERR_CUDA;
}

}  // namespace sfx
