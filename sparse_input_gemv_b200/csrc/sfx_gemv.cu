// Host side of the input-sparse GEMV: launch planning (tile width, K splits,
// ring depth, list capacity) and dispatch to the compiled instantiations.
#include "sfx_gemv_kernel.cuh"

#include <algorithm>

namespace sfx {

// ------------------------------------------------------------------ host side

int sm_count() {
  static int cached = 0;
  if (cached == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached = n;
  }
  return cached;
}

static int bmax_for(int B) {
  if (B <= 1) return 1;
  if (B <= 2) return 2;
  if (B <= 4) return 4;
  if (B <= 8) return 8;
  return 16;
}

static long long round_up(long long v, long long m) { return (v + m - 1) / m * m; }

GemvPlan plan_gemv(long long K, long long N, int B, bool idx_mode) {
  GemvPlan p;
  p.BMAX = bmax_for(B);
  // resident CTAs: two per SM up to 2 batch slots (64 registers per thread), one above
  const int slots = sm_count() * (p.BMAX <= 2 ? 2 : 1);
  // Column tile: the first of 256, 512, 1024, 2048 columns whose tiles times
  // K splits fill at least 90% of the resident slots in one wave; otherwise
  // the best filling one. (Measured on B200 for the Llama-3-8B shapes:
  // 256-column tiles win for N = 4096 / 6144, 512 for N = 28672.)
  int nt = 256;
  double best = -1.0;
  for (int cand : {256, 512, 1024, 2048}) {
    const long long ct = (N + cand - 1) / cand;
    long long S = std::max<long long>(1, slots / ct);
    S = std::min<long long>(S, std::max<long long>(1, (K + 31) / 32));
    const long long ctas = ct * S;
    const long long waves = (ctas + slots - 1) / slots;
    const double util = (double)ctas / (double)(waves * slots);
    if (util >= 0.9) {
      nt = cand;
      break;
    }
    if (util > best) {
      best = util;
      nt = cand;
    }
  }
  if (plan_override(SFX_PLAN_GEMV_NT)) nt = plan_override(SFX_PLAN_GEMV_NT);
  p.NT = nt;
  p.col_tiles = (int)((N + nt - 1) / nt);
  long long S = std::max<long long>(1, slots / p.col_tiles);
  S = std::min<long long>(S, std::max<long long>(1, (K + 31) / 32));
  if (plan_override(SFX_PLAN_GEMV_S)) S = plan_override(SFX_PLAN_GEMV_S);
  const size_t per_row = 4 * (size_t)(1 + p.BMAX);
  const long long cap_max = list_cap_max(p.BMAX);
  long long slice = round_up((K + S - 1) / S, 32);
  if (slice > cap_max) slice = cap_max;
  S = (K + slice - 1) / slice;
  if (!idx_mode) {
    p.slice = (int)slice;
    p.list_cap = (int)slice;
  } else {
    p.slice = 0;
    p.list_cap = (int)round_up((K + S - 1) / S, 32);
  }
  p.S = (int)S;
  // shared memory: warp-reduction buffer (warps x 256 floats) + list; the
  // split-K tail reuses the front as 4 x NT floats
  const size_t main_bytes =
      (size_t)(gemv_threads(p.BMAX) / 32) * 256 * 4 + (size_t)p.list_cap * per_row;
  p.smem = std::max(main_bytes, (size_t)16 * nt);
  return p;
}

size_t gemv_workspace_bytes(long long K, long long N, int B) {
  // partial sums for the larger split count of the two plans (the arrival
  // counters live in the workspace header)
  GemvPlan p = plan_gemv(K, N, B, false);
  GemvPlan q = plan_gemv(K, N, B, true);
  const long long S = std::max(p.S, q.S);
  const size_t cuda_cores = (size_t)(S > 1 ? S : 0) * B * N * 4;
  const size_t tc = B >= union_min_batch() ? union_tc_workspace_bytes(K, N, B) : 0;
  return std::max(cuda_cores, tc);
}

int union_min_batch() {
  const int v = plan_override(SFX_PLAN_UNION_MIN_B);
  return v >= 2 ? v : (union_uses_mma() ? kMmaMinBatch : kTcMinBatch);
}

// Per-(weight, activation, tile) instantiations live in sfx_gemv_inst_*.cu so
// they compile in parallel.
#define SFX_DECL(name) int name(const GemvPlan&, const GemvArgs&, cudaStream_t, bool);
SFX_DECL(gemv_bf16_bf16_small) SFX_DECL(gemv_bf16_bf16_large)
SFX_DECL(gemv_bf16_f32_small) SFX_DECL(gemv_bf16_f32_large)
SFX_DECL(gemv_f16_f16_small) SFX_DECL(gemv_f16_f16_large)
SFX_DECL(gemv_f16_f32_small) SFX_DECL(gemv_f16_f32_large)
#undef SFX_DECL

// Every launch is a programmatic dependent grid: the kernel waits
// (griddepcontrol.wait) before it reads any input or workspace, so it is
// correct after any predecessor, and its CTAs get scheduled while the
// previous kernel finishes its tail.
int launch_sparse_gemv(int wdt, int xdt, const GemvPlan& p, GemvArgs a, cudaStream_t s, bool) {
  const bool pdl = true;
  // a batch of union_min_batch() .. 16 tokens in threshold mode: the union
  // tile on the tensor cores
  if (a.B >= union_min_batch() && a.idx == nullptr && a.mask_in == nullptr && !a.no_tc)
    return launch_union_tc(wdt, xdt, plan_union_tc(a.K, a.N), a, s);
  if (p.col_tiles > kCounterSlots) return SFX_ERR_UNSUPPORTED;
  a.S = p.S;
  a.slice = p.slice;
  a.list_cap = p.list_cap;
  const bool large = p.NT >= 1024;
  if (wdt == SFX_BF16) {
    if (xdt == SFX_BF16) return large ? gemv_bf16_bf16_large(p, a, s, pdl) : gemv_bf16_bf16_small(p, a, s, pdl);
    if (xdt == SFX_F32) return large ? gemv_bf16_f32_large(p, a, s, pdl) : gemv_bf16_f32_small(p, a, s, pdl);
  } else if (wdt == SFX_F16) {
    if (xdt == SFX_F16) return large ? gemv_f16_f16_large(p, a, s, pdl) : gemv_f16_f16_small(p, a, s, pdl);
    if (xdt == SFX_F32) return large ? gemv_f16_f32_large(p, a, s, pdl) : gemv_f16_f32_small(p, a, s, pdl);
  }
  return SFX_ERR_DTYPE;
}

}  // namespace sfx
