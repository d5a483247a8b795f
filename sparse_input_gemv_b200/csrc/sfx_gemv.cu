// Host side of the input-sparse GEMV: launch planning (tile width, K splits,
// ring depth, list capacity) and dispatch to the compiled instantiations.
#include "sfx_gemv_kernel.cuh"

#include <algorithm>
#include <cstdlib>

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
  if (B <= 4) return 4;
  if (B <= 8) return 8;
  return 16;
}

static long long round_up(long long v, long long m) { return (v + m - 1) / m * m; }

static int env_int(const char* name, int dflt) {
  const char* s = std::getenv(name);
  return (s && *s) ? std::atoi(s) : dflt;
}

static constexpr size_t kSmemBudget = 200 * 1024;
static constexpr size_t kListBudget = 48 * 1024;

GemvPlan plan_gemv(long long K, long long N, int B, bool idx_mode) {
  GemvPlan p;
  p.BMAX = bmax_for(B);
  const int sms = sm_count();
  // Column tile: the widest tile that still leaves at least 4 K-splits'
  // worth of CTAs to fill the SMs (wider segments = longer contiguous reads).
  int nt = 256;
  for (int cand : {2048, 1024, 512, 256}) {
    const long long ct = (N + cand - 1) / cand;
    if (ct * 4 <= sms || cand == 256) {
      nt = cand;
      break;
    }
  }
  nt = env_int("SFX_GEMV_NT", nt);
  p.NT = nt;
  p.col_tiles = (int)((N + nt - 1) / nt);
  // K splits: fill the SMs once, with at least 64 rows per split.
  long long S = std::max<long long>(1, sms / p.col_tiles);
  S = std::min<long long>(S, std::max<long long>(1, K / 64));
  S = env_int("SFX_GEMV_S", (int)S);
  const size_t per_row = 4 * (size_t)(1 + p.BMAX);
  const long long cap_max = (long long)(kListBudget / per_row) / 32 * 32;
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
  const size_t list_bytes = (size_t)p.list_cap * per_row;
  const size_t bar_bytes = 2 * 8 * 16;
  int nstage = (int)((kSmemBudget - list_bytes - bar_bytes) / kStageBytes);
  nstage = std::max(2, std::min(nstage, 8));
  nstage = env_int("SFX_GEMV_STAGES", nstage);
  p.nstage = nstage;
  p.smem = (size_t)nstage * kStageBytes + list_bytes + 2 * 8 * (size_t)nstage;
  return p;
}

size_t gemv_workspace_bytes(long long K, long long N, int B) {
  // partial sums for the larger split count of the two plans (the arrival
  // counters live in the workspace header)
  GemvPlan p = plan_gemv(K, N, B, false);
  GemvPlan q = plan_gemv(K, N, B, true);
  const long long S = std::max(p.S, q.S);
  return (size_t)(S > 1 ? S : 0) * B * N * 4;
}

// Per-(weight, activation, tile) instantiations live in sfx_gemv_inst_*.cu so
// they compile in parallel.
#define SFX_DECL(name) int name(const GemvPlan&, const GemvArgs&, cudaStream_t, bool);
SFX_DECL(gemv_bf16_bf16_small) SFX_DECL(gemv_bf16_bf16_large)
SFX_DECL(gemv_bf16_f32_small) SFX_DECL(gemv_bf16_f32_large)
SFX_DECL(gemv_f16_f16_small) SFX_DECL(gemv_f16_f16_large)
SFX_DECL(gemv_f16_f32_small) SFX_DECL(gemv_f16_f32_large)
#undef SFX_DECL

int launch_sparse_gemv(int wdt, int xdt, const GemvPlan& p, GemvArgs a, cudaStream_t s,
                       bool pdl) {
  if (p.col_tiles > kCounterSlots) return SFX_ERR_UNSUPPORTED;
  a.S = p.S;
  a.slice = p.slice;
  a.list_cap = p.list_cap;
  a.nstage = p.nstage;
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
