// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sfx.h"

namespace sfx {

// Every workspace starts with a header: the device status word (bytes 0..3),
// then, at byte 256, the split-K arrival counters. The counters are used by
// the GEMV kernels only and are always left at zero, so no other operation may
// use the header as scratch; operation-specific scratch starts after it.
constexpr size_t kWsStatusBytes = 256;
constexpr int kCounterSlots = 4096;  // max column tiles of one GEMV launch
constexpr size_t kWsHeader = kWsStatusBytes + kCounterSlots * 4;

enum Epi { EPI_NONE = 0, EPI_GELU = 1, EPI_GELU_TANH = 2, EPI_SWIGLU = 3 };

// Arguments of one input-sparse GEMV launch (device pointers).
struct GemvArgs {
  const void* x;          // [B x K] activations, dtype xdt
  const void* W;          // [K x N] weights, dtype wdt
  void* y;                // [B x N] (or [B x N/2] fp32 h for EPI_SWIGLU)
  const int32_t* idx;     // optional active list (B == 1)
  const uint32_t* mask_in;  // optional mask bitmap [B x ceil(K/32)] instead of |x| > t
  const int32_t* cnt;     // device count of idx
  uint32_t* bitmap_out;   // optional fused-mask output [B x ceil(K/32)]
  float* partials;        // [S x B x N] split-K partial sums (workspace)
  int32_t* counters;      // [col_tiles] arrival counters (workspace, zero between calls)
  unsigned* status;       // device status word (workspace)
  long long K, N;
  int B;
  int S;                  // number of K splits
  int slice;              // rows of K per split (threshold mode), multiple of 32
  int list_cap;           // capacity of the per-CTA active list
  int ydt;                // output dtype (ignored for EPI_SWIGLU: fp32)
  int epi;                // Epi
  int union_mask;         // every token uses the batch-union mask
  int no_tc;              // keep B >= 4 on the CUDA-core kernel
  float t;                // magnitude threshold (threshold mode)
  unsigned long long wait_ns;  // limit of every bounded wait in the kernel
};

struct GemvPlan {
  int NT = 0;        // columns per CTA tile
  int BMAX = 1;      // batch slots compiled into the kernel
  int S = 1;         // K splits
  int slice = 0;     // rows per split
  int list_cap = 0;
  int col_tiles = 0;
  size_t smem = 0;
  int kind = 0;      // 0 CUDA-core GEMV, 1 union on tcgen05, 2 union on mma.sync
  int chunks = 0;    // kind 2: 64-column chunks per CTA
};

int sm_count();

// Limit of the kernels' bounded waits (sfx_set_wait_limit_ns; 2 s by default).
unsigned long long wait_limit_ns();

// Plan override for `key` (sfx_plan_key) set through sfx_set_plan_override,
// 0 when the planner chooses.
int plan_override(int key);

// Raises the kernel's dynamic shared-memory limit to at least `bytes` (never
// lowers it). *configured remembers the limit set so far; calls from several
// host threads are serialised, so the remembered limit is never above the one
// in force. Returns SFX_OK or SFX_ERR_CUDA.
int ensure_dynamic_smem(const void* kern, size_t bytes, size_t* configured);
GemvPlan plan_gemv(long long K, long long N, int B, bool idx_mode);
size_t gemv_workspace_bytes(long long K, long long N, int B);  // excludes the header
int launch_sparse_gemv(int wdt, int xdt, const GemvPlan& plan, GemvArgs a, cudaStream_t stream,
                       bool pdl);

// batch-union GEMM (sfx_union_tc.cu), used for B >= union_min_batch()
// Smallest batch that takes the union path (measured on B200: the CUDA-core
// kernel wins at 2 tokens; the mma.sync union kernel from 3 or 4 tokens on,
// the tcgen05 one from 5)
constexpr int kMmaMinBatch = 3;
constexpr int kTcMinBatch = 5;
int union_min_batch();          // by union kernel, unless overridden for a sweep
GemvPlan plan_union_tc(long long K, long long N);
// The union product runs on mma.sync with register-direct weight loads
// (union_gemm_mma_kernel) instead of tcgen05 (union_gemm_tc_kernel).
constexpr bool kUnionMmaDefault = true;
bool union_uses_mma();
// Batch-union products: 0 the union kernels only, 1 the device chooses between
// the union kernels and the dense kernel by the union's row count, 2 the dense
// kernel only (plan override SFX_PLAN_DENSE).
int dense_mode();
size_t union_tc_workspace_bytes(long long K, long long N, int B);
int launch_union_tc(int wdt, int xdt, const GemvPlan& plan, const GemvArgs& a, cudaStream_t stream);

// mask / selection kernels (sfx_mask.cu)
size_t mask_workspace_bytes(int B, int K, int sel);
int launch_mask_compact(const void* x, int dt, int B, int K, int sel, float t, int k,
                        const float* score_l, const float* score_g, double lambda,
                        uint32_t* bitmap, int32_t* idx, int32_t* cnt, int32_t* union_idx,
                        int32_t* union_cnt, unsigned char* ws_body, unsigned* status,
                        cudaStream_t stream);

// calibration (sfx_calib.cu)
size_t calib_workspace_bytes(long long S, long long K, int P, int dt);
int run_calibrate(const void* calib, int dt, long long n, const long long* ranks, int P,
                  float* thresholds_out_host, unsigned char* ws_body, cudaStream_t stream);

// MoE (sfx_moe.cu)
size_t moe_workspace_bytes(int B, int d, int E, int ffn, int top_k, int ffn_shared);
int run_moe(const void* x, int dt, const float* logits, int B, int d, int E, int ffn, int top_k,
            const void* W_gT, const void* W_upT, const void* W_d, const float* t_e,
            const void* Ws_gT, const void* Ws_upT, const void* Ws_d, int ffn_shared, void* y,
            int ydt, float* a_out, int32_t* sel_out, int flags, unsigned char* ws_body,
            size_t body_bytes, cudaStream_t stream);

// FFN with a static neuron mask (sfx_static_ffn.cu)
size_t static_ffn_workspace_bytes(int B, int d, int ffn);
int run_static_ffn(const void* x, int dt, int B, int d, int ffn, const void* WaT, const void* WbT,
                   const void* Wd, const int32_t* idx, const int32_t* cnt, int act, void* y,
                   int ydt, unsigned char* ws_body, unsigned* status, cudaStream_t stream);

// block error curves for the greedy allocation (sfx_alloc.cu); the whole
// workspace, headers of its sub-workspaces included
size_t error_curve_workspace_bytes(long long S, long long K, long long N, int xdt, int P);

// gate/up interleave (sfx_api.cu)
int launch_pack_gate_up(const void* W_g, const void* W_u, int dt, int d, int ffn, void* W_gu,
                        cudaStream_t stream);

}  // namespace sfx
