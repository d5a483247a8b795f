// Batch-union skinny GEMM on the tensor cores.
//
// For a batch of B <= 16 tokens with per-token magnitude masks ("TEAL:
// Training-Free Activation Sparsity in Large Language Models", slide 8),
// y[b, n] = sum_i (x[b, i] m[b, i]) W[i, n]. The rows any token keeps (the
// union) are fetched once and multiplied as a dense tile: with B tokens the
// product has B FLOPs per weight byte, more than CUDA cores issue at HBM speed
// once B grows.
//
//  1. union_count_kernel and union_pack_kernel, one CTA per 256-row chunk of
//     K: compact each K-split's union rows (warp ballots, ascending) into a row
//     list in the workspace and write the x operand for them as 16 x 16
//     bf16/f16 tiles per 16-row K-step (x * m per token, zero rows past the
//     list up to whole 64-row stages), plus a "lo" copy holding x - hi when x
//     is fp32 (two MMAs per K-step keep ~16 bits). The tile layout is the
//     register order of an mma.sync A fragment for kernel 2a, or the
//     canonical K-major no-swizzle layout of tcgen05 (8 x 8 core matrices,
//     SBO = 128 B between token groups, LBO = 256 B between row halves) for 2b.
//  2a. union_gemm_mma_kernel (the default; section 3 below): every warp loads
//     its weight rows straight into registers, transposes them with movmatrix
//     into B fragments and runs m16n8k16 MMAs; no shared-memory staging.
//  2b. union_gemm_tc_kernel (SFX_UNION_KERNEL=tc), tcgen05.mma with
//     D[m, b] (TMEM, fp32) += A[m, k] * B[k, b], A = W[union rows, n0 : n0+128]
//     (M = 128 output columns, MN-major), B = the packed x tiles (N = 16).
//     Grid (128-column tiles) x (K-splits), warp specialised: 8 producer warps
//     copy A (64 rows x 256 B per stage, 16-byte cp.async straight into the
//     canonical MN-major layout: SBO = 128 B between column groups, LBO = 2 KB
//     between row halves; L2 evict-first) and B into a 4-stage ring and signal
//     each stage's "full" mbarrier with cp.async.mbarrier.arrive.noinc; one
//     MMA warp waits on it, issues the stage's four K-steps into a TMEM
//     accumulator and commits them to the stage's "empty" mbarrier, on which
//     the producers wait before refilling. Epilogue: tcgen05.ld (warps 0-3 own
//     TMEM lanes 32w..32w+31), then the deterministic split-K reduction.
//     Every mbarrier wait is bounded; on timeout the kernel raises
//     SFX_DEV_TIMEOUT, drains its copies, frees its TMEM and returns.
// Measured on B200 at 16 tokens, 2a streams 4.3-5.4 TB/s and 2b 2.3-3.5
// TB/s: 2b is limited by its producers' cp.async gather of 256-byte row pieces
// into shared memory, not by the MMAs.
#include "sfx_common.cuh"
#include "sfx_internal.h"
#include "sfx_rowdot.cuh"

#include <cuda.h>  // CUtensorMap (the encoder is fetched at run time; no driver library link)
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

namespace sfx {

namespace {

constexpr int kTcM = 128;          // output columns per CTA (MMA M)
constexpr int kTcN = 16;           // padded tokens (MMA N)
constexpr int kTcK = 16;           // rows per MMA K-step (16-bit inputs)
constexpr int kSub = 4;            // K-steps per stage
constexpr int kRowsPerStage = kSub * kTcK;  // 64
constexpr int kStages = 4;
constexpr int kProducers = 256;    // warps 0-7
constexpr int kTcThreads = kProducers + 32;  // + the MMA warp
constexpr int kABytes = kTcM * kTcK * 2;    // 4 KB per K-step
constexpr int kBBytes = kTcN * kTcK * 2;    // 512 B per K-step (hi or lo)
constexpr int kSubBytes = kABytes + 2 * kBBytes;
constexpr int kStageBytes = kSub * kSubBytes;  // 20 KB
constexpr int kTmemCols = 64;         // four 16-column accumulators (one per K-step of a stage)
constexpr int kPackThreads = 256;

// Which product a batch-union launch runs: the union kernels (the rows any
// token keeps, gathered) or the dense kernel (every row, streamed as 2-D
// tiles). With DENSE_AUTO both are launched and the one not chosen returns at
// once; the choice is made on the device from the union's row count.
enum DenseMode { DENSE_NEVER = 0, DENSE_AUTO = 1, DENSE_ALWAYS = 2 };

struct TcArgs {
  GemvArgs g;
  int32_t* rows;      // [S x slice] union rows per split
  int32_t* counts;    // [S] union rows per split
  int32_t* chunk_counts;  // [ceil(K / 256)] union rows per 256-row chunk
  uint16_t* pack;     // [S x slice/16 x (hi, lo) x 256] B tiles per split
  int split_b;        // 1 if x is fp32 (hi + lo tiles)
  int frag;           // 1: x tiles in mma.sync A-fragment order (union_gemm_mma_kernel)
  int chunks;         // union_gemm_mma_kernel: 64-column chunks per CTA (1, 2, 4 or 8)
  int dense_mode;     // DenseMode
  int switch_rows;    // DENSE_AUTO: the dense kernel runs when the union has more rows
  int dense_frag;     // the dense kernel's x tiles in A-fragment order (mma.sync warps)
  int stall_test;     // test hook: the dense kernels' second TMA lane skips stage 0, so
                      // that stage's barrier never completes and every wait on it runs out
};

// Union rows of the whole batch, from the count kernel's per-chunk counts
// (every lane of the calling warp gets the sum).
__device__ __forceinline__ long long union_total(const TcArgs& t, int lane) {
  const int chunks = (int)((t.g.K + kPackThreads - 1) / kPackThreads);
  long long sum = 0;
  for (int c = lane; c < chunks; c += 32) sum += t.chunk_counts[c];
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  return sum;
}

__device__ __forceinline__ bool dense_chosen(int mode, int switch_rows, long long total) {
  return mode == DENSE_ALWAYS || (mode == DENSE_AUTO && total > switch_rows);
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid,
                                                 uint64_t pol) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst),
               "l"(src), "r"(n), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, no swizzle (version 1 for this architecture).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor for kind::f16: fp32 accumulate, A and B of the same
// 16-bit type, A MN-major, B K-major, N = 16, M = 128.
__host__ __device__ constexpr uint32_t instr_desc(bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | (1u << 15) |
         (0u << 16) | ((uint32_t)(kTcN >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

template <typename T> __device__ __forceinline__ uint16_t to_bits16(float v);
template <> __device__ __forceinline__ uint16_t to_bits16<__nv_bfloat16>(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
template <> __device__ __forceinline__ uint16_t to_bits16<__half>(float v) {
  return __half_as_ushort(__float2half_rn(v));
}
template <typename T> __device__ __forceinline__ float from_bits16(uint16_t b);
template <> __device__ __forceinline__ float from_bits16<__nv_bfloat16>(uint16_t b) {
  return __bfloat162float(__ushort_as_bfloat16(b));
}
template <> __device__ __forceinline__ float from_bits16<__half>(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// offset (in elements) of (token b, row kk) inside one 16 x 16 K-major B tile
__device__ __forceinline__ int btile_off(int b, int kk) {
  return ((b & 7) * 16 + (b >> 3) * 128 + (kk & 7) * 2 + (kk >> 3) * 256) / 2;
}

// offset (in elements) of (token b, row kk) inside one 16 x 16 tile stored in
// the register order of an m16n8k16 A fragment (A[m = token][k = row]): lane
// 4g + q holds A[g][2q, 2q+1], A[g+8][2q, 2q+1], A[g][2q+8, 2q+9],
// A[g+8][2q+8, 2q+9] as 16 contiguous bytes
__device__ __forceinline__ int frag_off(int b, int kk) {
  return (((b & 7) << 2) | ((kk & 7) >> 1)) * 8 + (kk & 1) + ((b >> 3) << 1) + ((kk >> 3) << 2);
}

__device__ __forceinline__ int xtile_off(bool frag, int b, int kk) {
  return frag ? frag_off(b, kk) : btile_off(b, kk);
}

}  // namespace

// ---------------------------------------------------------------- 1. union + pack

// Token bits of row i: bit b set iff |x[b, i]| > t (xv receives the values).
template <typename TX>
__device__ __forceinline__ uint32_t row_bits(const GemvArgs& a, long long i, bool in, float (&xv)[kTcN]) {
  const TX* xp = reinterpret_cast<const TX*>(a.x);
  uint32_t bits = 0;
#pragma unroll
  for (int b = 0; b < kTcN; ++b) {
    xv[b] = (in && b < a.B) ? to_f32(xp[(long long)b * a.K + i]) : 0.f;
    bits |= ((in && b < a.B && fabsf(xv[b]) > a.t) ? 1u : 0u) << b;
  }
  return bits;
}

// Pass 1, one CTA per 256-row chunk of K: the number of union rows in the
// chunk (and the fused-mask bitmap words, if requested).
template <typename TX>
__global__ void __launch_bounds__(kPackThreads) union_count_kernel(const TcArgs t) {
  const GemvArgs& a = t.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long i = (long long)blockIdx.x * kPackThreads + tid;
  const bool in = i < a.K;
  pdl_wait();
  float xv[kTcN];
  const uint32_t bits = row_bits<TX>(a, i, in, xv);
  if (a.bitmap_out != nullptr) {
    const long long w0 = (long long)blockIdx.x * kPackThreads + warp * 32;
    for (int b = 0; b < a.B; ++b) {
      const unsigned bal = __ballot_sync(0xffffffffu, (bits >> b) & 1u);
      if (lane == 0 && w0 < a.K) a.bitmap_out[(long long)b * ((a.K + 31) >> 5) + (w0 >> 5)] = bal;
    }
  }
  const int n = __syncthreads_count(bits != 0);
  if (tid == 0) t.chunk_counts[blockIdx.x] = n;
  pdl_launch_dependents();
}

// Pass 2, one CTA per 256-row chunk: the chunk's union rows go to positions
// base + (rank within the chunk) of its split's list, base = union rows of the
// split's earlier chunks; the matching B operand values go into the packed
// K-major tiles. The split's last chunk records the split's count and zeroes
// the B rows up to the end of the last 64-row stage.
template <typename TW, typename TX>
__global__ void __launch_bounds__(kPackThreads) union_pack_kernel(const TcArgs t) {
  const GemvArgs& a = t.g;
  __shared__ int s_warp_tot[kPackThreads / 32];
  __shared__ int s_base;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;
  const long long i = (long long)chunk * kPackThreads + tid;
  const bool in = i < a.K;
  const int per_split = a.slice / kPackThreads;
  const int split = chunk / per_split;
  const int first = split * per_split;
  const int last = min((int)((a.K + kPackThreads - 1) / kPackThreads), first + per_split) - 1;
  int32_t* rows = t.rows + (long long)split * a.slice;
  const int tile_elems = 256 * (t.split_b ? 2 : 1);  // per 16-row K-step
  uint16_t* pack = t.pack + (long long)split * (a.slice / kTcK) * tile_elems;
  __shared__ int s_dense;
  pdl_wait();  // chunk counts of pass 1
  if (warp == 0) {
    int s = 0;
    for (int c = first + lane; c < chunk; c += 32) s += t.chunk_counts[c];
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) s_base = s;
    const bool dense = t.dense_mode != DENSE_NEVER &&
                       dense_chosen(t.dense_mode, t.switch_rows, union_total(t, lane));
    if (lane == 0) s_dense = dense ? 1 : 0;
  }
  float xv[kTcN];
  uint32_t bits = row_bits<TX>(a, i, in, xv);
  const bool act = bits != 0;
  const unsigned bal = __ballot_sync(0xffffffffu, act);
  if (lane == 0) s_warp_tot[warp] = __popc(bal);
  __syncthreads();
  if (s_dense) {
    // the dense kernel's x operand: every row at its own position (tile
    // i / 16 overall, in the layout its consumers read), zero where no token
    // keeps the row and past K
    const long long pos = i - (long long)split * a.slice;
    uint16_t* tl = pack + (pos / kTcK) * tile_elems;
    const int kk = (int)(pos % kTcK);
    if (a.union_mask && bits) bits = (1u << a.B) - 1u;
#pragma unroll
    for (int b = 0; b < kTcN; ++b) {
      const float v = ((bits >> b) & 1u) ? xv[b] : 0.f;
      const uint16_t hi = to_bits16<TW>(v);
      const int off = xtile_off(t.dense_frag != 0, b, kk);
      tl[off] = hi;
      if (t.split_b) tl[256 + off] = to_bits16<TW>(v - from_bits16<TW>(hi));
    }
    pdl_launch_dependents();
    return;
  }
  int woff = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kPackThreads / 32; ++w) {
    const int c = s_warp_tot[w];
    woff += (w < warp) ? c : 0;
    tot += c;
  }
  const int base = s_base;
  if (act) {
    const int pos = base + woff + __popc(bal & lanemask_lt());
    rows[pos] = (int32_t)i;
    uint16_t* tl = pack + (long long)(pos / kTcK) * tile_elems;
    const int kk = pos % kTcK;
    if (a.union_mask) bits = (1u << a.B) - 1u;
#pragma unroll
    for (int b = 0; b < kTcN; ++b) {
      const float v = ((bits >> b) & 1u) ? xv[b] : 0.f;
      const uint16_t hi = to_bits16<TW>(v);
      const int off = xtile_off(t.frag, b, kk);
      tl[off] = hi;
      if (t.split_b) tl[256 + off] = to_bits16<TW>(v - from_bits16<TW>(hi));
    }
  }
  if (chunk == last) {
    const int n = base + tot;
    if (tid == 0) t.counts[split] = n;
    const int padded = (n + kRowsPerStage - 1) / kRowsPerStage * kRowsPerStage;
    for (int e = n * kTcN + tid; e < padded * kTcN; e += kPackThreads) {
      const int pos = e / kTcN, b = e % kTcN;
      uint16_t* tl = pack + (long long)(pos / kTcK) * tile_elems;
      const int off = xtile_off(t.frag, b, pos % kTcK);
      tl[off] = 0;
      if (t.split_b) tl[256 + off] = 0;
    }
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------- 2. tcgen05 GEMM

template <typename TW>
__global__ void __launch_bounds__(kTcThreads, 2) union_gemm_tc_kernel(const TcArgs t) {
  const GemvArgs& a = t.g;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* stages = smem;
  int32_t* list_row = reinterpret_cast<int32_t*>(smem + (size_t)kStages * kStageBytes);
  __shared__ __align__(8) uint64_t s_full[kStages];
  __shared__ __align__(8) uint64_t s_empty[kStages];
  __shared__ uint32_t s_tmem;
  __shared__ int s_last;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const long long n0 = (long long)tile * kTcM;
  const int ncols = (int)min((long long)kTcM, a.N - n0);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&s_full[s], kProducers);
      mbar_init(&s_empty[s], 1);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 8) {  // TMEM: four fp32 accumulators of 128 lanes x 16 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();  // the pack kernel's rows, counts and B tiles
  const int nrows = min(max(t.counts[split], 0), a.slice);
  for (int r = tid; r < nrows; r += kTcThreads) list_row[r] = t.rows[(long long)split * a.slice + r];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int nit = (nrows + kRowsPerStage - 1) / kRowsPerStage;
  const uint32_t sbase = smem_u32(stages);
  const int tile_elems = 256 * (t.split_b ? 2 : 1);
  const uint16_t* pack = t.pack + (long long)split * (a.slice / kTcK) * tile_elems;

  if (warp < 8) {
    // ------------------------------------------------ producers
    const uint64_t pol = l2_evict_first_policy();
    const TW* Wp = reinterpret_cast<const TW*>(a.W);
    for (int c = 0; c < nit; ++c) {
      const int s = c % kStages, use = c / kStages;
      if (use > 0 && !mbar_wait(&s_empty[s], (use - 1) & 1, &s_abort, a.wait_ns)) {
        s_abort = 1;
        raise_status(a.status, SFX_DEV_TIMEOUT);
        break;
      }
      const uint32_t sa = sbase + s * kStageBytes;
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // A: 64 rows x 16 groups of 16 bytes
        // a warp takes 8 consecutive rows x 4 column groups: its 16-byte pieces
        // land in four contiguous 128-byte runs of the stage (no bank conflicts;
        // rows-fastest would put a row's 16 groups 128 bytes apart, 16-way)
        const int idx = tid + q * kProducers;
        const int r = ((idx >> 7) << 3) | (idx & 7), g = (idx >> 3) & 15;
        const int row = c * kRowsPerStage + r;
        const bool valid = row < nrows && g * 8 < ncols;
        const TW* src = Wp + (valid ? (long long)list_row[row] * a.N + n0 + g * 8 : 0);
        const int sub = r >> 4, rr = r & 15;
        cp_async16_zfill(sa + sub * kSubBytes + (rr >> 3) * 2048 + g * 128 + (rr & 7) * 16, src,
                         valid, pol);
      }
      {  // B: the packed tiles of the stage's 4 K-steps (hi [, lo])
        const int per_sub = t.split_b ? 64 : 32;  // 16-byte chunks per K-step
        if (tid < kSub * per_sub) {
          const int sub = tid / per_sub, ch = tid % per_sub;
          const uint16_t* src = pack + (long long)(c * kSub + sub) * tile_elems + ch * 8;
          cp_async16(sa + sub * kSubBytes + kABytes + ch * 16, src);
        }
      }
      cp_async_arrive_noinc(&s_full[s]);
    }
  } else if (lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(DT<TW>::id == SFX_BF16);
    int last_commit = -1;
    for (int c = 0; c < nit; ++c) {
      const int s = c % kStages;
      if (!mbar_wait(&s_full[s], (c / kStages) & 1, &s_abort, a.wait_ns)) {
        s_abort = 1;
        raise_status(a.status, SFX_DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t sa = sbase + s * kStageBytes;
#pragma unroll
      for (int q = 0; q < kSub; ++q) {
        const uint32_t st = sa + q * kSubBytes;
        const uint64_t adesc = smem_desc(st, 2048, 128);
        // K-step q accumulates into its own 16 columns: four independent
        // accumulation chains instead of one serial chain of MMAs
        const uint32_t dq = tmem + (uint32_t)(q * kTcN);
        mma_f16(dq, adesc, smem_desc(st + kABytes, 256, 128), idesc, c > 0 ? 1u : 0u);
        if (t.split_b) mma_f16(dq, adesc, smem_desc(st + kABytes + kBBytes, 256, 128), idesc, 1u);
      }
      mma_commit(&s_empty[s]);
      last_commit = c;
    }
    // bounded, also after a timeout: the MMAs issued so far have finished
    // before TMEM can be freed
    if (last_commit >= 0)
      mbar_wait(&s_empty[last_commit % kStages], (last_commit / kStages) & 1, nullptr,
                kDrainLimitNs);
  }
  // all MMAs done: the last commit covers every earlier MMA
  if (nit > 0 && !s_abort) {
    const int c = nit - 1;
    if (!mbar_wait(&s_empty[c % kStages], (c / kStages) & 1, &s_abort, a.wait_ns)) {
      s_abort = 1;
      raise_status(a.status, SFX_DEV_TIMEOUT);
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();

  // ---------------------------------------------------------------- epilogue
  float d[kTcN];
#pragma unroll
  for (int b = 0; b < kTcN; ++b) d[b] = 0.f;
  if (warp < 4 && nit > 0 && !s_abort) {
    // sum the four accumulators in K-step order
#pragma unroll
    for (int q = 0; q < kSub; ++q) {
      uint32_t r[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
          "%14,%15}, [%16];"
          : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
            "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
            "=r"(r[14]), "=r"(r[15])
          : "r"(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(q * kTcN)));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int b = 0; b < kTcN; ++b) d[b] += __uint_as_float(r[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
  if (s_abort) return;

  const long long N = a.N;
  const bool swiglu = a.epi == EPI_SWIGLU;
  const int m = tid;  // output column within the tile (threads 0..127)
  if (a.S == 1) {
    if (warp < 4) {
#pragma unroll
      for (int b = 0; b < kTcN; ++b) {
        if (b >= a.B) break;
        if (swiglu) {
          const float up = __shfl_down_sync(0xffffffffu, d[b], 1);
          if ((m & 1) == 0 && m < ncols)
            reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + (n0 + m) / 2] = silu_f(d[b]) * up;
        } else if (m < ncols) {
          float v = d[b];
          if (a.epi == EPI_GELU) v = gelu_erf_f(v);
          else if (a.epi == EPI_GELU_TANH) v = gelu_tanh_f(v);
          store_as(a.y, (long long)b * N + n0 + m, a.ydt, v);
        }
      }
    }
    return;
  }
  if (warp < 4 && m < ncols) {
#pragma unroll
    for (int b = 0; b < kTcN; ++b)
      if (b < a.B) a.partials[((long long)split * a.B + b) * N + n0 + m] = d[b];
  }
  __syncthreads();
  if (tid == 0) s_last = (arrive_acq_rel(&a.counters[tile]) == a.S - 1);
  __syncthreads();
  if (!s_last) return;
  const long long vs = (long long)a.B * N;
  // pairs of columns so the SwiGLU epilogue sees (gate, up) together
  for (int e = tid; e < a.B * (kTcM / 2); e += kTcThreads) {
    const int b = e / (kTcM / 2), c2 = 2 * (e % (kTcM / 2));
    if (c2 >= ncols) continue;
    const float* pb = a.partials + (long long)b * N + n0 + c2;
    float s0 = 0.f, s1 = 0.f;
    for (int s = 0; s < a.S; ++s) {
      const float2 q = __ldcg(reinterpret_cast<const float2*>(pb + s * vs));
      s0 += q.x;
      s1 += q.y;
    }
    if (swiglu) {
      reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + (n0 + c2) / 2] = silu_f(s0) * s1;
    } else {
      if (a.epi == EPI_GELU) { s0 = gelu_erf_f(s0); s1 = gelu_erf_f(s1); }
      else if (a.epi == EPI_GELU_TANH) { s0 = gelu_tanh_f(s0); s1 = gelu_tanh_f(s1); }
      store_as(a.y, (long long)b * N + n0 + c2, a.ydt, s0);
      store_as(a.y, (long long)b * N + n0 + c2 + 1, a.ydt, s1);
    }
  }
  if (tid == 0) a.counters[tile] = 0;
}


// ---------------------------------------------------------------- 3. mma.sync GEMM

// The same union product with the weights loaded straight into registers:
// y[b, n0 + c] = sum over union rows r of x'[b, r] W[r, n0 + c], per warp a
// 64-column chunk and 16 union rows (a K-block) at a time. A CTA of 8 warps
// covers C = 1, 2, 4 or 8 chunks; the 8 / C warps of a chunk take its K-blocks
// in turn and are summed in a fixed order through shared memory (narrow
// matrices get more column tiles instead of more K splits). Lane 4p + c loads 16 bytes of row p (and of row p + 8) at columns
// 8c .. 8c + 7 and 32 + 8c .. 32 + 8c + 7 of the slice (64 contiguous bytes per
// row and load). Each 32-bit register j of such a load is one element pair of
// an 8 x 8 matrix M[p][2c + e] = W[row p][col 8c + 2j + e]; movmatrix.trans
// hands lane 4g + q the pair M[2q][g], M[2q + 1][g]: rows 2q, 2q + 1 at one
// column, which is the B fragment of m16n8k16 (k = union row, n = column).
// The A fragment (m = token, k = union row) is one 16-byte load from the
// packed tiles. Lane 4g + q ends with tokens g and g + 8 at the 8 consecutive
// columns 8q .. 8q + 7 of each 32-column half. No shared-memory staging of
// weights and no CTA barrier inside the loop: every warp streams on its own,
// with 16-bit x through a rolling pipeline of kMmaPipe K-blocks (two, 4 KB,
// in flight while one is multiplied), with fp32 x in groups of kMmaDepth.
constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMmaWarpCols = 64;
constexpr int kMmaDepth = 1;  // fp32 x: K-blocks loaded per group (1 measured best of 1-3)
constexpr int kMmaPipe = 3;   // 16-bit x: register slots of the rolling pipeline
// token row stride of the reduction buffer: 2 (mod 32) words, so that the
// float2 stores of a half-warp (tokens g = 0..3, column groups q = 0..3) hit
// 16 distinct bank pairs
constexpr int kRedStride = kMmaWarpCols + 2;
constexpr size_t kRedBytes = (size_t)kMmaWarps * 16 * kRedStride * 4;

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t v) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(v));
  return d;
}

__device__ __forceinline__ uint4 ld_frag(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// 16-byte weight load: skip L1, L2 evict-first (weights are read once)
__device__ __forceinline__ uint4 ld_weight16(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ float epi_f(int epi, float v) {
  if (epi == EPI_GELU) return gelu_erf_f(v);
  if (epi == EPI_GELU_TANH) return gelu_tanh_f(v);
  return v;
}

template <typename TW, bool SPLIT>
__global__ void __launch_bounds__(kMmaThreads, 2) union_gemm_mma_kernel(const TcArgs t) {
  const GemvArgs& a = t.g;
  // [row list] during the loop, then [8 warps][16 tokens][kRedStride] fp32 sums
  extern __shared__ __align__(16) unsigned char smem[];
  int32_t* list_row = reinterpret_cast<int32_t*>(smem);
  float* red = reinterpret_cast<float*>(smem);
  __shared__ int s_last;

  const int C = t.chunks, WPC = kMmaWarps / C;  // 64-column chunks, warps per chunk
  const int NT = kMmaWarpCols * C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = warp % C, wrow = warp / C;
  const int tile = blockIdx.x, split = blockIdx.y;
  const long long n0 = (long long)tile * NT;
  const long long N = a.N;
  const int p = lane >> 2, c = lane & 3;  // load role: row p (and p + 8), column group c
  const int g = lane >> 2, q = lane & 3;  // fragment role

  pdl_wait();  // the pack kernel's rows, counts and x tiles
  if (t.dense_mode != DENSE_NEVER) {  // the dense kernel may run this product instead
    __shared__ int s_skip;
    if (warp == 0) {
      const bool dense = dense_chosen(t.dense_mode, t.switch_rows, union_total(t, lane));
      if (lane == 0) s_skip = dense ? 1 : 0;
    }
    __syncthreads();
    if (s_skip) {
      pdl_launch_dependents();
      return;
    }
  }
  const int nrows = min(max(t.counts[split], 0), a.slice);
  for (int r = tid; r < nrows; r += kMmaThreads) list_row[r] = t.rows[(long long)split * a.slice + r];
  __syncthreads();

  const int tile_elems = 256 * (SPLIT ? 2 : 1);
  const uint16_t* pack = t.pack + (long long)split * (a.slice / kTcK) * tile_elems;
  const long long nw = n0 + chunk * kMmaWarpCols;  // first column of this warp
  // the two 16-byte column groups of this lane (N is a multiple of 8)
  const bool col0 = nw + 8 * c < N, col1 = nw + 32 + 8 * c < N;
  const TW* Wb = reinterpret_cast<const TW*>(a.W) + nw + 8 * c;
  const uint64_t pol = l2_evict_first_policy();
  const int nblk = (nrows + kTcK - 1) / kTcK;

  float acc[2][4][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][j][e] = 0.f;

  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  // one K-block: the weight pieces of its 16 rows and the x fragment(s)
  auto load = [&](int kb, bool kv, uint4 (&ws)[2][2], uint4& xas, uint4& xls) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = kb * kTcK + h * 8 + p;
      const bool rv = kv && r < nrows;
      const TW* src = Wb + (rv ? (long long)list_row[r] * N : 0);
      ws[h][0] = (rv && col0) ? ld_weight16(src, pol) : z;
      ws[h][1] = (rv && col1) ? ld_weight16(src + 32, pol) : z;
    }
    xas = kv ? ld_frag(pack + (long long)kb * tile_elems + lane * 8) : z;
    if (SPLIT) xls = kv ? ld_frag(pack + (long long)kb * tile_elems + 256 + lane * 8) : z;
  };
  auto compute = [&](const uint4 (&ws)[2][2], const uint4& xas, const uint4& xls) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const uint32_t r0[4] = {ws[0][m].x, ws[0][m].y, ws[0][m].z, ws[0][m].w};
      const uint32_t r1[4] = {ws[1][m].x, ws[1][m].y, ws[1][m].z, ws[1][m].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t b0 = movmatrix_trans(r0[j]);
        const uint32_t b1 = movmatrix_trans(r1[j]);
        mma_16816(acc[m][j], xas.x, xas.y, xas.z, xas.w, b0, b1, TW());
        if (SPLIT) mma_16816(acc[m][j], xls.x, xls.y, xls.z, xls.w, b0, b1, TW());
      }
    }
  };
  if constexpr (!SPLIT) {
    // this warp's K-blocks wrow, wrow + WPC, ... through a rolling pipeline of
    // kMmaPipe register slots: kMmaPipe - 1 K-blocks stay in flight while one
    // is multiplied
    const int nmine = nblk > wrow ? (nblk - wrow + WPC - 1) / WPC : 0;
    uint4 w[kMmaPipe][2][2];
    uint4 xa[kMmaPipe], xl[kMmaPipe];
#pragma unroll
    for (int u = 0; u < kMmaPipe - 1; ++u) load(wrow + u * WPC, u < nmine, w[u], xa[u], xl[u]);
    for (int i0 = 0; i0 < nmine; i0 += kMmaPipe) {
#pragma unroll
      for (int u = 0; u < kMmaPipe; ++u) {
        const int i = i0 + u;
        if (i >= nmine) break;
        constexpr int kAhead = kMmaPipe - 1;
        const int ls = (u + kAhead) % kMmaPipe;
        load(wrow + (i + kAhead) * WPC, i + kAhead < nmine, w[ls], xa[ls], xl[ls]);
        compute(w[u], xa[u], xl[u]);
      }
    }
  } else {
    // fp32 x (hi + lo fragments, two MMAs per tile): the WPC warps of a chunk
    // take groups of kMmaDepth K-blocks in turn, loaded together, then
    // multiplied (a rolling pipeline costs this variant more than it saves;
    // on the 70B down, groups of one K-block were 2-3.5 % faster than two)
    for (int kb0 = wrow * kMmaDepth; kb0 < nblk; kb0 += WPC * kMmaDepth) {
      uint4 w[kMmaDepth][2][2];
      uint4 xa[kMmaDepth], xl[kMmaDepth];
#pragma unroll
      for (int u = 0; u < kMmaDepth; ++u) load(kb0 + u, kb0 + u < nblk, w[u], xa[u], xl[u]);
#pragma unroll
      for (int u = 0; u < kMmaDepth; ++u) {
        if (kb0 + u >= nblk) break;
        compute(w[u], xa[u], xl[u]);
      }
    }
  }
  pdl_launch_dependents();

  // lane (g, q): acc[m][j][e] = token g, acc[m][j][2 + e] = token g + 8, at
  // chunk column 32m + 8q + 2j + e. Through shared memory: red[warp][token][col]
  __syncthreads();  // every warp is done with the row list
  {
    float* rw = red + warp * (16 * kRedStride);
#pragma unroll
    for (int hi = 0; hi < 2; ++hi)
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float2*>(rw + (g + 8 * hi) * kRedStride + 32 * m + 8 * q + 2 * j) =
              make_float2(acc[m][j][2 * hi], acc[m][j][2 * hi + 1]);
  }
  __syncthreads();

  // (chunk, token, column pair): the chunk's WPC warps summed in order, then
  // the epilogue (S == 1) or this split's partial tile
  const bool swiglu = a.epi == EPI_SWIGLU;
  const int ncols = (int)min((long long)NT, N - n0);
  const int items = C * a.B * (kMmaWarpCols / 2);
  for (int e = tid; e < items; e += kMmaThreads) {
    const int ch = e / (a.B * (kMmaWarpCols / 2));
    const int rem = e - ch * (a.B * (kMmaWarpCols / 2));
    const int b = rem / (kMmaWarpCols / 2), cp = rem - b * (kMmaWarpCols / 2);
    const int col = ch * kMmaWarpCols + 2 * cp;  // within the tile
    if (col >= ncols) continue;
    float s0 = 0.f, s1 = 0.f;
    for (int w = 0; w < WPC; ++w) {
      const float2 v =
          *reinterpret_cast<const float2*>(red + ((w * C + ch) * 16 + b) * kRedStride + 2 * cp);
      s0 += v.x;
      s1 += v.y;
    }
    const long long n = n0 + col;
    if (a.S == 1) {
      if (swiglu) {
        reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + n / 2] = silu_f(s0) * s1;
      } else {
        store_as(a.y, (long long)b * N + n, a.ydt, epi_f(a.epi, s0));
        store_as(a.y, (long long)b * N + n + 1, a.ydt, epi_f(a.epi, s1));
      }
    } else {
      *reinterpret_cast<float2*>(a.partials + ((long long)split * a.B + b) * N + n) =
          make_float2(s0, s1);
    }
  }
  if (a.S == 1) return;

  __syncthreads();
  if (tid == 0) s_last = (arrive_acq_rel(&a.counters[tile]) == a.S - 1);
  __syncthreads();
  if (!s_last) return;
  // the last CTA of the tile sums the S partials in split order, column pairs
  // so that the SwiGLU epilogue sees (gate, up) together
  const long long vs = (long long)a.B * N;
  for (int e = tid; e < a.B * (NT / 2); e += kMmaThreads) {
    const int b = e / (NT / 2), c2 = 2 * (e % (NT / 2));
    if (c2 >= ncols) continue;
    const float* pb = a.partials + (long long)b * N + n0 + c2;
    float s0 = 0.f, s1 = 0.f;
    for (int s = 0; s < a.S; ++s) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(pb + s * vs));
      s0 += v.x;
      s1 += v.y;
    }
    if (swiglu) {
      reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + (n0 + c2) / 2] = silu_f(s0) * s1;
    } else {
      store_as(a.y, (long long)b * N + n0 + c2, a.ydt, epi_f(a.epi, s0));
      store_as(a.y, (long long)b * N + n0 + c2 + 1, a.ydt, epi_f(a.epi, s1));
    }
  }
  if (tid == 0) a.counters[tile] = 0;
}

// ---------------------------------------------------------------- 4. dense TMA + tcgen05 GEMM

// When the union keeps most rows, reading every row as a dense tile is cheaper
// than gathering the union: the rows of a 128-column tile arrive as two 2-D
// TMA boxes of 64 columns x 128 rows (16 KB each, 128-byte swizzle), and a
// 16-byte-gather cannot move bytes as fast (measured on B200: 16 KB 2-D boxes
// from two issuing lanes stream 6.9 TB/s; 16-byte gathers into shared memory
// 3.5 TB/s). The x operand for all K rows comes from the pack kernel as the
// same 16 x 16 K-major tiles, with the rows no token keeps holding zeros, so
// the product is the same masked one as the union kernels compute.
//
// One persistent CTA per SM; CTA c streams stages [W c / G, W (c + 1) / G) of
// the (column tile, 128-row stage) sequence, so every CTA moves the same
// number of bytes. Warp 4 lanes 0 and 1 issue the two boxes of a stage (lane
// 0 also the stage's x tiles, a 1-D bulk copy) into a 4-stage ring; warp 5
// lane 0 issues tcgen05.mma, M = 128 columns (A: the stage, MN-major, 128-byte
// swizzle), N = 16 tokens (B: the x tiles, K-major), K = 16, one accumulator
// per K-step of the stage, into one of two TMEM accumulator sets per run of
// stages on one tile (a "segment"); warps 0-3 read a finished segment's
// accumulators (TMEM lane = column), sum them in K-step order and either
// write the tile (a segment that covers all of K) or its partial, after
// which the last segment of the tile to arrive adds the partials in segment
// order (deterministic). Every wait is bounded; on timeout the kernel raises
// SFX_DEV_TIMEOUT, waits (bounded) for its copies and MMAs, frees its TMEM and
// returns.
constexpr int kDM = 128;                          // output columns per tile
constexpr int kDRows = 128;                       // rows of W per stage
constexpr int kDSteps = kDRows / kTcK;            // 8 K-steps per stage
constexpr int kDStages = 4;
constexpr int kDBoxBytes = 64 * kDRows * 2;       // one 64-column box: 16 KB
constexpr int kDABytes = 2 * kDBoxBytes;          // 32 KB of W per stage
constexpr int kDThreads = 192;                    // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int kDTmemCols = 256;                   // two sets of 8 accumulators x 16 columns
__host__ __device__ constexpr int dense_b_bytes(bool split) { return kDSteps * kBBytes * (split ? 2 : 1); }
__host__ __device__ constexpr int dense_stage_bytes(bool split) { return kDABytes + dense_b_bytes(split); }
__host__ __device__ constexpr size_t dense_smem_bytes(bool split) {
  return (size_t)kDStages * dense_stage_bytes(split) + 1024;  // + alignment slack
}

struct DenseArgs {
  TcArgs t;
  long long T;          // column tiles of kDM columns
  long long SPT;        // stages per tile (ceil(K / kDRows))
  long long W;          // T * SPT
  int max_seg;          // partial slots per tile
};

// Barrier 1 over the four epilogue warps (128 threads), returning the OR of
// `pred` over them.
__device__ __forceinline__ bool named_barrier_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&d)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return smem_desc(addr, lbo, sbo) | (2ull << 61);  // layout: 128-byte swizzle
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// CTA holding stage-iteration w of the stream-K split over G CTAs:
// CTA c covers [W c / G, W (c + 1) / G).
__device__ __forceinline__ long long dense_cta_of(long long w, long long W, long long G) {
  return ((w + 1) * G - 1) / W;
}

template <typename TW, bool SPLIT>
__global__ void __launch_bounds__(kDThreads, 1)
    dense_gemm_tma_kernel(const __grid_constant__ CUtensorMap wmap, const DenseArgs d) {
  const TcArgs& t = d.t;
  const GemvArgs& a = t.g;
  constexpr int SB = dense_stage_bytes(SPLIT);
  constexpr int BB = dense_b_bytes(SPLIT);
  constexpr int kTileElems = 256 * (SPLIT ? 2 : 1);
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_full[kDStages];
  __shared__ __align__(8) uint64_t s_empty[kDStages];
  __shared__ __align__(8) uint64_t s_acc_full[2];
  __shared__ __align__(8) uint64_t s_acc_empty[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_last;
  __shared__ int s_skip;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // 128-byte swizzle atoms
  const long long G = gridDim.x, c = blockIdx.x;
  const long long w0 = d.W * c / G, w1 = d.W * (c + 1) / G;
  const long long n = w1 - w0;

  pdl_wait();  // the count and pack kernels' results
  if (warp == 0) {
    const long long total = union_total(t, lane);
    if (lane == 0) s_skip = dense_chosen(t.dense_mode, t.switch_rows, total) ? 0 : 1;
  }
  if (tid == 0) {
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&s_full[s], 2);  // the two issuing lanes
      mbar_init(&s_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_acc_full[i], 1);
      mbar_init(&s_acc_empty[i], 128);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  __syncthreads();
  if (s_skip) {  // the union kernels run this product
    pdl_launch_dependents();
    return;
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kDTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint16_t* pack = t.pack;  // all K rows, split-major = row-major tiles

  if (warp == 4) {
    // ------------------------------------------------ TMA producers
    if (lane < 2) {
      const uint64_t pol = l2_evict_first_policy();
      long long j = 0;
      for (; j < n; ++j) {
        const int s = (int)(j % kDStages);
        const uint32_t use = (uint32_t)(j / kDStages);
        if (use > 0 && !mbar_wait(&s_empty[s], (use - 1) & 1, &s_abort, a.wait_ns)) {
          s_abort = 1;
          raise_status(a.status, SFX_DEV_TIMEOUT);
          break;
        }
        if (t.stall_test && lane == 1 && j == 0) continue;
        const long long w = w0 + j, tile = w / d.SPT, ks = w - tile * d.SPT;
        const uint32_t st = base + (uint32_t)(s * SB);
        const int col = (int)(tile * kDM) + 64 * lane;  // a multiple of 64 elements
        const int row = (int)(ks * kDRows);
        mbar_arrive_expect_tx(&s_full[s], kDBoxBytes + (lane == 0 ? BB : 0));
        tma_load_2d(st + (uint32_t)(lane * kDBoxBytes), &wmap, col, row, &s_full[s], pol);
        if (lane == 0)
          bulk_load(st + kDABytes, pack + ks * kDSteps * kTileElems, (uint32_t)BB, &s_full[s]);
      }
      // bounded drain: every copy this lane issued has landed before the CTA
      // may leave (normally the MMAs have consumed them already)
      for (long long q = (j > kDStages ? j - kDStages : 0); q < j; ++q)
        mbar_wait(&s_full[q % kDStages], (uint32_t)((q / kDStages) & 1), nullptr, kDrainLimitNs);
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(DT<TW>::id == SFX_BF16);
      long long seg = -1, cur_tile = -1, last_commit = -1;
      int set = 0;
      for (long long j = 0; j < n && !*reinterpret_cast<volatile int*>(&s_abort); ++j) {
        const int s = (int)(j % kDStages);
        const long long w = w0 + j, tile = w / d.SPT;
        const bool seg_start = tile != cur_tile;
        if (seg_start) {
          ++seg;
          set = (int)(seg & 1);
          cur_tile = tile;
          if (seg >= 2 &&
              !mbar_wait(&s_acc_empty[set], (uint32_t)(((seg - 2) >> 1) & 1), &s_abort,
                         a.wait_ns)) {
            s_abort = 1;
            raise_status(a.status, SFX_DEV_TIMEOUT);
            break;
          }
        }
        if (!mbar_wait(&s_full[s], (uint32_t)((j / kDStages) & 1), &s_abort, a.wait_ns)) {
          s_abort = 1;
          raise_status(a.status, SFX_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t st = base + (uint32_t)(s * SB);
#pragma unroll
        for (int kk = 0; kk < kDSteps; ++kk) {
          // A: 16 rows x 128 columns; two 64-column atoms 16 KB apart (LBO),
          // 8-row groups 1 KB apart (SBO)
          const uint64_t adesc = smem_desc_sw128(st + (uint32_t)(kk * kTcK * 128), kDBoxBytes, 1024);
          const uint32_t bst = st + kDABytes + (uint32_t)(kk * kTileElems * 2);
          const uint32_t dq = tmem + (uint32_t)(set * 128 + kk * kTcN);
          mma_f16(dq, adesc, smem_desc(bst, 256, 128), idesc, seg_start ? 0u : 1u);
          if (SPLIT) mma_f16(dq, adesc, smem_desc(bst + kBBytes, 256, 128), idesc, 1u);
        }
        mma_commit(&s_empty[s]);
        last_commit = j;
        const bool seg_end = (j == n - 1) || ((w + 1) / d.SPT != tile);
        if (seg_end) mma_commit(&s_acc_full[set]);
      }
      // bounded: the last committed MMAs have finished before TMEM is freed
      if (last_commit >= 0)
        mbar_wait(&s_empty[last_commit % kDStages], (uint32_t)((last_commit / kDStages) & 1),
                  nullptr, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-3)
    const long long N = a.N;
    const bool swiglu = a.epi == EPI_SWIGLU;
    const int m = tid;  // column within the tile = TMEM lane
    long long seg = -1;
    for (long long w = w0; w < w1;) {
      const long long tile = w / d.SPT;
      const long long we = min(w1, (tile + 1) * d.SPT);
      const bool whole = (w == tile * d.SPT) && (we == (tile + 1) * d.SPT);
      ++seg;
      const int set = (int)(seg & 1);
      w = we;
      bool bad = !mbar_wait(&s_acc_full[set], (uint32_t)((seg >> 1) & 1), &s_abort, a.wait_ns);
      if (bad) {
        s_abort = 1;
        raise_status(a.status, SFX_DEV_TIMEOUT);
      }
      // one decision for all four warps (a thread may have seen the abort
      // flag while another saw the accumulators complete)
      if (named_barrier_or(bad)) break;
      tc_fence_after();
      float acc[kTcN];
#pragma unroll
      for (int b = 0; b < kTcN; ++b) acc[b] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kDSteps; ++kk) {
        uint32_t r[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(set * 128 + kk * kTcN)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int b = 0; b < kTcN; ++b) acc[b] += __uint_as_float(r[b]);
      }
      tc_fence_before();
      mbar_arrive(&s_acc_empty[set]);  // the MMA issuer may reuse the set
      const long long col = tile * kDM + m;
      if (whole) {
        // the segment is the whole tile: write it
#pragma unroll
        for (int b = 0; b < kTcN; ++b) {
          if (b >= a.B) break;
          if (swiglu) {
            const float up = __shfl_down_sync(0xffffffffu, acc[b], 1);
            if ((m & 1) == 0 && col < N)
              reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + col / 2] = silu_f(acc[b]) * up;
          } else if (col < N) {
            store_as(a.y, (long long)b * N + col, a.ydt, epi_f(a.epi, acc[b]));
          }
        }
        continue;
      }
      // a part of the tile: its partial, then the tile's last segment adds them up
      const long long c_first = dense_cta_of(tile * d.SPT, d.W, G);
      const long long c_last = dense_cta_of((tile + 1) * d.SPT - 1, d.W, G);
      const int nseg = (int)(c_last - c_first + 1);
      float* part = a.partials + (tile * d.max_seg) * (long long)a.B * kDM;
#pragma unroll
      for (int b = 0; b < kTcN; ++b)
        if (b < a.B) part[((c - c_first) * a.B + b) * kDM + m] = acc[b];
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) s_last = (arrive_acq_rel(&a.counters[tile]) == nseg - 1);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!s_last) continue;
      for (int b = 0; b < a.B; ++b) {
        float v = 0.f;
        for (int q = 0; q < nseg; ++q) v += __ldcg(part + ((long long)q * a.B + b) * kDM + m);
        if (swiglu) {
          const float up = __shfl_down_sync(0xffffffffu, v, 1);
          if ((m & 1) == 0 && col < N)
            reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + col / 2] = silu_f(v) * up;
        } else if (col < N) {
          store_as(a.y, (long long)b * N + col, a.ydt, epi_f(a.epi, v));
        }
      }
      if (tid == 0) a.counters[tile] = 0;
    }
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kDTmemCols)
                 : "memory");
  }
}

// The dense product with mma.sync consumers (the default dense kernel): the
// same TMA-fed ring and stream-K split as dense_gemm_tma_kernel, but eight
// consumer warps multiply each stage, warp w owning columns 16w .. 16w + 15 of
// the tile for all eight K-blocks: ldmatrix.x4.trans reads the two 8-column
// blocks of a K-block straight out of the 128-byte-swizzled box (the B
// fragments of m16n8k16), the x fragment is one 16-byte shared load of the
// K-block's tile (A-fragment order), and the warp keeps its 16 x 16 partial in
// eight registers per lane, so no warp-to-warp reduction is needed. Measured
// on B200 at 16 tokens: tcgen05.mma with N = 16 tokens and an MN-major A took
// ~0.12 us per 4 KB of A, which held the tcgen05 version of this kernel to
// 5.2 TB/s; the mma.sync warps keep pace with the TMA stream.
constexpr int kDMWarps = 8;                        // consumer warps
constexpr int kDMThreads = (kDMWarps + 1) * 32;    // + the TMA warp

template <typename TW, bool SPLIT>
__global__ void __launch_bounds__(kDMThreads, 1)
    dense_gemm_mma_kernel(const __grid_constant__ CUtensorMap wmap, const DenseArgs d) {
  const TcArgs& t = d.t;
  const GemvArgs& a = t.g;
  constexpr int SB = dense_stage_bytes(SPLIT);
  constexpr int BB = dense_b_bytes(SPLIT);
  constexpr int kTileElems = 256 * (SPLIT ? 2 : 1);
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_full[kDStages];
  __shared__ __align__(8) uint64_t s_empty[kDStages];
  __shared__ int s_abort;
  __shared__ int s_last;
  __shared__ int s_skip;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // 128-byte swizzle atoms
  const long long G = gridDim.x, c = blockIdx.x;
  const long long w0 = d.W * c / G, w1 = d.W * (c + 1) / G;
  const long long n = w1 - w0;

  pdl_wait();  // the count and pack kernels' results
  if (warp == 0) {
    const long long total = union_total(t, lane);
    if (lane == 0) s_skip = dense_chosen(t.dense_mode, t.switch_rows, total) ? 0 : 1;
  }
  if (tid == 0) {
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&s_full[s], 2);         // the two issuing lanes
      mbar_init(&s_empty[s], kDMWarps);  // one arrival per consumer warp
    }
    fence_barrier_init();
    s_abort = 0;
  }
  __syncthreads();
  if (s_skip) {  // the union kernels run this product
    pdl_launch_dependents();
    return;
  }
  const uint16_t* pack = t.pack;  // all K rows, split-major = row-major tiles

  if (warp == kDMWarps) {
    // ------------------------------------------------ TMA producers
    if (lane < 2) {
      const uint64_t pol = l2_evict_first_policy();
      long long j = 0;
      for (; j < n; ++j) {
        const int s = (int)(j % kDStages);
        const uint32_t use = (uint32_t)(j / kDStages);
        if (use > 0 && !mbar_wait(&s_empty[s], (use - 1) & 1, &s_abort, a.wait_ns)) {
          s_abort = 1;
          raise_status(a.status, SFX_DEV_TIMEOUT);
          break;
        }
        if (t.stall_test && lane == 1 && j == 0) continue;
        const long long w = w0 + j, tile = w / d.SPT, ks = w - tile * d.SPT;
        const uint32_t st = base + (uint32_t)(s * SB);
        const int col = (int)(tile * kDM) + 64 * lane;  // a multiple of 64 elements
        const int row = (int)(ks * kDRows);
        mbar_arrive_expect_tx(&s_full[s], kDBoxBytes + (lane == 0 ? BB : 0));
        tma_load_2d(st + (uint32_t)(lane * kDBoxBytes), &wmap, col, row, &s_full[s], pol);
        if (lane == 0)
          bulk_load(st + kDABytes, pack + ks * kDSteps * kTileElems, (uint32_t)BB, &s_full[s]);
      }
      // bounded drain: every copy this lane issued has landed before the CTA leaves
      for (long long q = (j > kDStages ? j - kDStages : 0); q < j; ++q)
        mbar_wait(&s_full[q % kDStages], (uint32_t)((q / kDStages) & 1), nullptr, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------ consumers (warps 0-7)
    const long long N = a.N;
    const bool swiglu = a.epi == EPI_SWIGLU;
    const int g = lane >> 2, q = lane & 3;
    const int box = warp >> 2;                 // columns 0-63: box 0, 64-127: box 1
    const int nb0 = (2 * warp) & 7;            // the warp's two 8-column blocks in its box
    const int lm = lane >> 3, li = lane & 7;
    const int chunk = nb0 + (lm >> 1);         // 16-byte column this lane addresses
    // A split x's lo halves go to a second accumulator pair, added in at the
    // segment's end: each MMA chain is then as long as with a 16-bit x
    // (measured on B200 at 8 and 16 tokens: the 70B down with fp32 h 92.0 ->
    // 88.6 us; alternating pairs by K-block for a 16-bit x was slower)
    float acc[2][4], acc2[2][4];
    long long cur_tile = -1, seg_first = 0;
    for (long long j = 0; j < n; ++j) {
      const int s = (int)(j % kDStages);
      const long long w = w0 + j, tile = w / d.SPT;
      if (tile != cur_tile) {
        cur_tile = tile;
        seg_first = w;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] = acc2[h][e] = 0.f;
      }
      bool bad = !mbar_wait(&s_full[s], (uint32_t)((j / kDStages) & 1), &s_abort, a.wait_ns);
      bad = __any_sync(0xffffffffu, bad);
      if (bad) {
        if (lane == 0) {
          s_abort = 1;
          raise_status(a.status, SFX_DEV_TIMEOUT);
        }
        break;
      }
      const uint32_t st = base + (uint32_t)(s * SB);
      const uint32_t bx = st + (uint32_t)(box * kDBoxBytes);
#pragma unroll
      for (int kb = 0; kb < kDSteps; ++kb) {
        const int r = kb * kTcK + (lm & 1) * 8 + li;
        uint32_t b[4];
        ldmatrix_x4_trans(bx + (uint32_t)(r * 128 + ((chunk ^ li) << 4)), b);
        const uint32_t xs = st + kDABytes + (uint32_t)(kb * kTileElems * 2 + lane * 16);
        const uint4 xa = lds128(xs);
        mma_16816(acc[0], xa.x, xa.y, xa.z, xa.w, b[0], b[1], TW());
        mma_16816(acc[1], xa.x, xa.y, xa.z, xa.w, b[2], b[3], TW());
        if (SPLIT) {
          const uint4 xl = lds128(xs + 512);
          mma_16816(acc2[0], xl.x, xl.y, xl.z, xl.w, b[0], b[1], TW());
          mma_16816(acc2[1], xl.x, xl.y, xl.z, xl.w, b[2], b[3], TW());
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);  // the stage may be refilled
      const bool seg_end = (j == n - 1) || ((w + 1) / d.SPT != tile);
      if (!seg_end) continue;
      if (SPLIT) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] += acc2[h][e];
      }
      // lane (g, q): acc[h][e] = token g (e < 2) or g + 8 (e >= 2) at tile
      // column 16 warp + 8 h + 2q + (e & 1)
      const bool whole = seg_first == tile * d.SPT && w + 1 == (tile + 1) * d.SPT;
      if (whole) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const long long col = tile * kDM + 16 * warp + 8 * h + 2 * q;
          if (col >= N) continue;
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int b = g + 8 * hi;
            if (b >= a.B) continue;
            const float v0 = acc[h][2 * hi], v1 = acc[h][2 * hi + 1];
            if (swiglu) {
              reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + col / 2] = silu_f(v0) * v1;
            } else {
              store_as(a.y, (long long)b * N + col, a.ydt, epi_f(a.epi, v0));
              store_as(a.y, (long long)b * N + col + 1, a.ydt, epi_f(a.epi, v1));
            }
          }
        }
        continue;
      }
      // a part of the tile: the warp writes its 16 columns of the segment's
      // partial and arrives on the counter of (tile, warp); the last of the
      // tile's segments to arrive there adds up those 16 columns in segment
      // order. No barrier between warps: a warp that gives up on a wait cannot
      // stall the others.
      const long long c_first = dense_cta_of(tile * d.SPT, d.W, G);
      const long long c_last = dense_cta_of((tile + 1) * d.SPT - 1, d.W, G);
      const int nseg = (int)(c_last - c_first + 1);
      float* part = a.partials + (tile * d.max_seg) * (long long)a.B * kDM;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int b = g + 8 * hi;
          if (b < a.B)
            *reinterpret_cast<float2*>(part + ((c - c_first) * a.B + b) * kDM + 16 * warp + 8 * h +
                                       2 * q) = make_float2(acc[h][2 * hi], acc[h][2 * hi + 1]);
        }
      __syncwarp();
      int32_t* counter = a.counters + tile * kDMWarps + warp;
      int last = 0;
      if (lane == 0) last = arrive_acq_rel(counter) == nseg - 1;
      last = __shfl_sync(0xffffffffu, last, 0);
      __syncwarp();
      if (!last) continue;
      for (int e = lane; e < a.B * 8; e += 32) {  // 8 column pairs per token
        const int b = e >> 3, c2 = 16 * warp + 2 * (e & 7);
        const long long col = tile * kDM + c2;
        if (col >= N) continue;
        float v0 = 0.f, v1 = 0.f;
        for (int sg = 0; sg < nseg; ++sg) {
          const float2 v =
              __ldcg(reinterpret_cast<const float2*>(part + ((long long)sg * a.B + b) * kDM + c2));
          v0 += v.x;
          v1 += v.y;
        }
        if (swiglu) {
          reinterpret_cast<float*>(a.y)[(long long)b * (N / 2) + col / 2] = silu_f(v0) * v1;
        } else {
          store_as(a.y, (long long)b * N + col, a.ydt, epi_f(a.epi, v0));
          store_as(a.y, (long long)b * N + col + 1, a.ydt, epi_f(a.epi, v1));
        }
      }
      if (lane == 0) *counter = 0;
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host

static long long rup(long long v, long long m) { return (v + m - 1) / m * m; }
static constexpr long long kMaxSlice = 6144;       // tcgen05: 24 KB row list in shared memory
static constexpr long long kMmaMaxSlice = 16384;   // mma.sync: 64 KB row list

bool union_uses_mma() {
  const int v = plan_override(SFX_PLAN_UNION_KERNEL);  // 1 tcgen05, 2 mma.sync
  return v ? v == 2 : kUnionMmaDefault;
}

// Splits of K for `tiles` column tiles: one wave of resident CTAs (two per
// SM), K splits only to fill it (at least 256 rows each) or to keep a split's
// list within kMaxSlice rows.
static void plan_splits(GemvPlan& p, long long K, long long max_slice) {
  const long long slots = 2LL * sm_count();
  long long S = std::max<long long>(1, slots / p.col_tiles);
  S = std::min<long long>(S, std::max<long long>(1, K / 256));
  if (plan_override(SFX_PLAN_UNION_S)) S = plan_override(SFX_PLAN_UNION_S);
  long long slice = rup((K + S - 1) / S, kPackThreads);  // whole 256-row pack chunks
  if (slice > max_slice) slice = max_slice;
  p.S = (int)((K + slice - 1) / slice);
  p.slice = (int)slice;
  p.list_cap = (int)slice;
}

GemvPlan plan_union_tc(long long K, long long N) {
  GemvPlan p;
  p.BMAX = kTcN;
  if (!union_uses_mma()) {
    p.kind = 1;
    p.NT = kTcM;
    p.col_tiles = (int)((N + kTcM - 1) / kTcM);
    plan_splits(p, K, kMaxSlice);
    p.smem = (size_t)kStages * kStageBytes + (size_t)p.slice * 4;
    return p;
  }
  // mma.sync: among the CTA tiles (1, 2, 4 or 8 chunks of 64 columns) that
  // need the fewest K splits, the widest that still gives at least 1.5 CTAs
  // per SM, else the narrowest. Measured on B200 at 4-16 tokens: the serial sum
  // of many split partials by the last CTA of a tile costs more than narrow
  // tiles do, and among tiles without extra splits wider ones win down to
  // ~1.5 CTAs per SM (70B gate|up: 256 columns 4-6 % faster than 128; 8B
  // gate|up: 128 columns, 224 CTAs, fastest; 70B down: 64 columns, 2 splits).
  p.kind = 2;
  int C = 1;
  if (plan_override(SFX_PLAN_MMA_CHUNKS)) {
    C = plan_override(SFX_PLAN_MMA_CHUNKS);
  } else {
    int best_S = 1 << 30;
    for (int cand = 1; cand <= 8; cand *= 2) {
      GemvPlan q;
      q.col_tiles = (int)((N + 64LL * cand - 1) / (64LL * cand));
      plan_splits(q, K, kMmaMaxSlice);
      best_S = std::min(best_S, q.S);
    }
    const long long min_ctas = (3LL * sm_count() + 1) / 2;
    for (int cand = 1; cand <= 8; cand *= 2) {
      GemvPlan q;
      q.col_tiles = (int)((N + 64LL * cand - 1) / (64LL * cand));
      plan_splits(q, K, kMmaMaxSlice);
      if (q.S == best_S && (cand == 1 || (long long)q.col_tiles * q.S >= min_ctas)) C = cand;
    }
  }
  p.chunks = C;
  p.NT = 64 * C;
  p.col_tiles = (int)((N + p.NT - 1) / p.NT);
  plan_splits(p, K, kMmaMaxSlice);
  p.smem = std::max((size_t)p.slice * 4, kRedBytes);
  return p;
}

// workspace after the header: [partials S x B x N f32] then, 256-aligned,
// [rows S x slice][split counts][chunk counts][B tiles S x slice/16 x (hi, lo)]
struct TcAux {
  size_t rows, counts, chunk_counts, pack, total;
};
static TcAux tc_aux(const GemvPlan& p, long long K) {
  TcAux x;
  x.rows = 0;
  x.counts = x.rows + (size_t)p.S * p.slice * 4;
  x.chunk_counts = x.counts + rup((long long)p.S * 4, 256);
  x.pack = x.chunk_counts + rup((K + kPackThreads - 1) / kPackThreads * 4, 256);
  x.total = x.pack + (size_t)p.S * (p.slice / kTcK) * 256 * 2 * 2;  // hi + lo, bytes
  return x;
}

// The dense kernel's stream-K split: T column tiles of kDM columns, SPT
// stages of kDRows rows per tile, W = T SPT stages over G CTAs (one per SM),
// and the most CTAs that share one tile (partial slots per tile).
struct DensePlan {
  long long T, SPT, W, G;
  int max_seg;
};
static DensePlan plan_dense(long long K, long long N) {
  DensePlan d;
  d.T = (N + kDM - 1) / kDM;
  d.SPT = (K + kDRows - 1) / kDRows;
  d.W = d.T * d.SPT;
  d.G = std::min<long long>(sm_count(), d.W);
  int mx = 1;
  for (long long tile = 0; tile < d.T; ++tile) {
    const long long c0 = ((tile * d.SPT + 1) * d.G - 1) / d.W;
    const long long c1 = (((tile + 1) * d.SPT) * d.G - 1) / d.W;
    mx = std::max<int>(mx, (int)(c1 - c0 + 1));
  }
  d.max_seg = mx;
  return d;
}

// The union (sparse) and dense products never both run, so they share the
// partial-sum area at the front of the workspace body.
static size_t union_partials_bytes(const GemvPlan& p, long long K, long long N, int B) {
  const size_t sparse = (size_t)(p.S > 1 ? p.S : 0) * B * N * 4;
  if (p.kind != 2) return sparse;
  const DensePlan d = plan_dense(K, N);
  const size_t dense = (size_t)d.T * d.max_seg * B * kDM * 4;
  return std::max(sparse, dense);
}

size_t union_tc_workspace_bytes(long long K, long long N, int B) {
  const GemvPlan p = plan_union_tc(K, N);
  return union_partials_bytes(p, K, N, B) + 256 /* alignment */ + tc_aux(p, K).total;
}

// ------------------------------------------------------------------ tensor maps

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library). Maps are cached per (matrix, shape, dtype):
// encoding one costs host time, and a call captured in a CUDA graph keeps its
// map by value.
using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

static EncodeFn tensor_map_encoder() {
  static EncodeFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeFn) nullptr;
    return reinterpret_cast<EncodeFn>(f);
  }();
  return fn;
}

struct MapKey {
  const void* W;
  long long K, N;
  int dt;
  bool operator==(const MapKey& o) const { return W == o.W && K == o.K && N == o.N && dt == o.dt; }
};

// The weight matrix W [K x N] (16-bit) as a 2-D tensor, boxes of 64 columns x
// kDRows rows with the 128-byte swizzle; reads past N or K fill zeros.
static int weight_tensor_map(const void* W, long long K, long long N, int dt, CUtensorMap* out) {
  static std::mutex mu;
  static MapKey keys[64];
  static CUtensorMap maps[64];
  static int used = 0, next = 0;
  const MapKey key{W, K, N, dt};
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (keys[i] == key) {
      *out = maps[i];
      return SFX_OK;
    }
  EncodeFn enc = tensor_map_encoder();
  if (!enc) return SFX_ERR_CUDA;
  CUtensorMap m;
  const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)K};
  const cuuint64_t strides[1] = {(cuuint64_t)N * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kDRows};
  const cuuint32_t es[2] = {1, 1};
  if (enc(&m, dt == SFX_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
          const_cast<void*>(W), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return SFX_ERR_CUDA;
  keys[next] = key;
  maps[next] = m;
  next = (next + 1) % 64;
  used = std::min(used + 1, 64);
  *out = m;
  return SFX_OK;
}

// The union row fraction above which the dense kernel runs. Measured on B200
// at 4-16 tokens, forcing each side on the 70B FFN: with 16-bit x the union
// kernel streams gathered rows at ~0.85 of the dense kernel's rate, and the
// gate|up product crosses over at 82-86 % of the rows; with fp32 x the dense
// kernel's split operand (two MMAs per K-step) slows it down, and the down
// product's union still wins at 90 % (87.0 against 88.4 us) and loses only
// near the full union (95.4 against 89.4 us at 99.9 %).
static constexpr double kDenseSwitchFraction = 0.85;
static constexpr double kDenseSwitchFractionSplit = 0.93;

int dense_mode() {
  // 1 union kernels only, 2 dense kernel only, 3 the tcgen05 dense kernel only
  const int v = plan_override(SFX_PLAN_DENSE);
  return v == 1 ? DENSE_NEVER : v >= 2 ? DENSE_ALWAYS : DENSE_AUTO;
}
static bool dense_on_tcgen05() { return plan_override(SFX_PLAN_DENSE) == 3; }

// One opt-in per kernel (shared by the bf16/f16 and fp32 activation paths):
// the largest dynamic shared memory any plan asks for.
template <typename TW>
static int configure_tc_kernel() {
  static int rc = cudaFuncSetAttribute(union_gemm_tc_kernel<TW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)((size_t)kStages * kStageBytes + kMaxSlice * 4)) ==
                          cudaSuccess
                      ? SFX_OK
                      : SFX_ERR_CUDA;
  return rc;
}

template <typename TW>
static int configure_mma_kernel() {
  const int bytes = (int)std::max((size_t)kMmaMaxSlice * 4, kRedBytes);
  static int rc =
      (cudaFuncSetAttribute(union_gemm_mma_kernel<TW, false>,
                            cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
       cudaFuncSetAttribute(union_gemm_mma_kernel<TW, true>,
                            cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess)
          ? SFX_OK
          : SFX_ERR_CUDA;
  return rc;
}

template <typename TW>
static int configure_dense_kernels() {
  const auto set = [](const void* k, bool split) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)dense_smem_bytes(split)) == cudaSuccess;
  };
  static int rc = (set((const void*)dense_gemm_mma_kernel<TW, false>, false) &&
                   set((const void*)dense_gemm_mma_kernel<TW, true>, true) &&
                   set((const void*)dense_gemm_tma_kernel<TW, false>, false) &&
                   set((const void*)dense_gemm_tma_kernel<TW, true>, true))
                      ? SFX_OK
                      : SFX_ERR_CUDA;
  return rc;
}

template <typename TW, typename TX>
static int launch_tc(const GemvPlan& p, TcArgs t, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((t.g.K + kPackThreads - 1) / kPackThreads), 1, 1);
  cfg.blockDim = dim3(kPackThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, union_count_kernel<TX>, t) != cudaSuccess) return SFX_ERR_CUDA;
  if (cudaLaunchKernelEx(&cfg, union_pack_kernel<TW, TX>, t) != cudaSuccess) return SFX_ERR_CUDA;

  cfg.gridDim = dim3((unsigned)p.col_tiles, (unsigned)p.S, 1);
  cfg.dynamicSmemBytes = p.smem;
  if (t.frag) {  // p.smem = the row list (up to 64 KB) or the reduction buffer
    cfg.blockDim = dim3(kMmaThreads, 1, 1);
    auto kern = t.split_b ? union_gemm_mma_kernel<TW, true> : union_gemm_mma_kernel<TW, false>;
    if (configure_mma_kernel<TW>() != SFX_OK) return SFX_ERR_CUDA;
    if (t.dense_mode != DENSE_ALWAYS && cudaLaunchKernelEx(&cfg, kern, t) != cudaSuccess)
      return SFX_ERR_CUDA;
    if (t.dense_mode == DENSE_NEVER) return SFX_OK;
    // the dense product: one CTA per SM over the stream-K split
    DenseArgs d;
    d.t = t;
    const DensePlan dp = plan_dense(t.g.K, t.g.N);
    d.T = dp.T;
    d.SPT = dp.SPT;
    d.W = dp.W;
    d.max_seg = dp.max_seg;
    CUtensorMap wmap;
    if (weight_tensor_map(t.g.W, t.g.K, t.g.N, DT<TW>::id, &wmap) != SFX_OK) return SFX_ERR_CUDA;
    if (configure_dense_kernels<TW>() != SFX_OK) return SFX_ERR_CUDA;
    cfg.gridDim = dim3((unsigned)dp.G, 1, 1);
    cfg.dynamicSmemBytes = dense_smem_bytes(t.split_b != 0);
    if (dense_on_tcgen05()) {
      cfg.blockDim = dim3(kDThreads, 1, 1);
      auto dk = t.split_b ? dense_gemm_tma_kernel<TW, true> : dense_gemm_tma_kernel<TW, false>;
      return cudaLaunchKernelEx(&cfg, dk, wmap, d) == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
    }
    cfg.blockDim = dim3(kDMThreads, 1, 1);
    auto dk = t.split_b ? dense_gemm_mma_kernel<TW, true> : dense_gemm_mma_kernel<TW, false>;
    return cudaLaunchKernelEx(&cfg, dk, wmap, d) == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
  }
  auto kern = union_gemm_tc_kernel<TW>;
  if (configure_tc_kernel<TW>() != SFX_OK) return SFX_ERR_CUDA;
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, t) == cudaSuccess ? SFX_OK : SFX_ERR_CUDA;
}

int launch_union_tc(int wdt, int xdt, const GemvPlan& p, const GemvArgs& a, cudaStream_t s) {
  if (p.col_tiles > kCounterSlots) return SFX_ERR_UNSUPPORTED;
  TcArgs t;
  t.g = a;
  t.g.S = p.S;
  t.g.slice = p.slice;
  t.g.list_cap = p.list_cap;
  // auxiliary buffers follow the partial sums in the workspace
  unsigned char* aux = reinterpret_cast<unsigned char*>(a.partials) +
                       union_partials_bytes(p, a.K, a.N, a.B);
  aux = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(aux) + 255) & ~uintptr_t(255));
  const TcAux lay = tc_aux(p, a.K);
  t.rows = reinterpret_cast<int32_t*>(aux + lay.rows);
  t.counts = reinterpret_cast<int32_t*>(aux + lay.counts);
  t.chunk_counts = reinterpret_cast<int32_t*>(aux + lay.chunk_counts);
  t.pack = reinterpret_cast<uint16_t*>(aux + lay.pack);
  t.split_b = xdt == SFX_F32 ? 1 : 0;
  t.frag = p.kind == 2 ? 1 : 0;
  // the sparse/dense switch: with the mma.sync union kernel, the dense kernel
  // takes the product when the union keeps more than kDenseSwitchFraction of
  // the rows (decided on the device from the union count)
  t.dense_mode = p.kind == 2 ? dense_mode() : DENSE_NEVER;
  t.switch_rows = (int)std::min<long long>(
      a.K, (long long)((xdt == SFX_F32 ? kDenseSwitchFractionSplit : kDenseSwitchFraction) *
                       (double)a.K));
  t.dense_frag = dense_on_tcgen05() ? 0 : 1;
  t.stall_test = plan_override(SFX_PLAN_TEST_STALL) ? 1 : 0;
  // counters: one per tile (tcgen05 kernel) or per tile and consumer warp
  if (t.dense_mode != DENSE_NEVER && plan_dense(a.K, a.N).T * kDMWarps > kCounterSlots)
    t.dense_mode = DENSE_NEVER;
  t.chunks = p.chunks;
  if (wdt == SFX_BF16) {
    if (xdt == SFX_BF16) return launch_tc<__nv_bfloat16, __nv_bfloat16>(p, t, s);
    if (xdt == SFX_F32) return launch_tc<__nv_bfloat16, float>(p, t, s);
  } else if (wdt == SFX_F16) {
    if (xdt == SFX_F16) return launch_tc<__half, __half>(p, t, s);
    if (xdt == SFX_F32) return launch_tc<__half, float>(p, t, s);
  }
  return SFX_ERR_DTYPE;
}

}  // namespace sfx
