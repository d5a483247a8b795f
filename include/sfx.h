/*
 * sfx.h -- C ABI of the B200 (sm_100a) activation-sparse GEMV / FFN library.
 *
 * The library computes input-activation-sparse products for decoding at batch
 * 1..16: input activations are masked by magnitude (|x| > t) or by top-k of a
 * per-neuron score, the active neurons are compacted, and only the weight rows
 * of active neurons are read from HBM.
 *
 * Sources (by page title and section):
 *  [TEAL]  "TEAL: Training-Free Activation Sparsity in Large Language Models"
 *          (reading-group slides), slide 8 (threshold t_p from calibration
 *          data for a target sparsity), slide 11 ("Hardware-Aware
 *          Acceleration": mask generation fused into the sparse GEMV so only
 *          the needed weights are read).
 *  [ATTR]  "Attribution-based Sparse Activation in Large Language Models",
 *          sections "proposed method" (GxO score) and "implementation" (top
 *          fraction per layer).
 *  [GLASS] "GLASS: Global-Local Aggregation for inference-time
 *          Sparsification", section 2.2 (rank aggregation, top-k selection).
 *  [GLOSS] "Activation sparsity (LLM)" glossary, "why sparsity reduces
 *          computation" (a zero intermediate skips one row of W2).
 *  [MOE]   "Uncovering Intra-expert Activation Sparsity for Efficient
 *          Mixture-of-Expert Model Execution", section "method".
 *
 * Conventions for every entry point
 *  - Pointers marked (dev) are CUDA device pointers, (host) are host pointers.
 *    The caller allocates and owns every buffer, including the workspace;
 *    the library never allocates or frees memory.
 *  - Weights are stored row-per-input-neuron: W is [K x N] row-major, so
 *    y = x W and dropping input neuron i skips the contiguous row i ([GLOSS]).
 *    Activations are [B x K] row-major, outputs [B x N] row-major.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream) unless stated otherwise.
 *  - Return value: SFX_OK (0) or a negative sfx_status. Arguments are checked
 *    on the host before any launch; a rejected call launches nothing.
 *  - Device-side checks (an index outside [0, K) in a caller-provided list)
 *    never trap: the offending row is skipped and a bit is OR-ed into the
 *    status word at the start of the workspace. sfx_check_device_status()
 *    reads (and clears) it.
 *  - Alignment: weight matrices must be 16-byte aligned and their row length
 *    a multiple of 8 elements, because weight rows are moved with 16-byte
 *    bulk copies and read with 128-bit loads; otherwise SFX_ERR_ALIGN.
 *  - Workspace: size it with sfx_workspace_bytes() and zero it once with
 *    sfx_workspace_init() before first use; the library leaves it in a
 *    reusable state after every successful call. Calls that share a workspace
 *    must not run concurrently.
 */
#ifndef SFX_H_
#define SFX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SFX_F16 = 0, SFX_BF16 = 1, SFX_F32 = 2 } sfx_dtype;

typedef enum {
  SFX_SEL_THRESHOLD = 0,   /* m_i = 1[|x_i| > t]                         [TEAL] */
  SFX_SEL_TOPK_GXO = 1,    /* top-k of s_i = |fl32(x_i * g_i)|            [ATTR] */
  SFX_SEL_TOPK_GLASS = 2,  /* top-k of (1-l) R^l_i + l R^g_i             [GLASS] */
  SFX_SEL_TOPK_CGXO = 3    /* top-k of x_i g_i + |x_i| ||g||_2 / 2        [ATTR] */
} sfx_select;

typedef enum {
  SFX_OK = 0,
  SFX_ERR_ARG = -1,          /* null pointer, bad size, k > n, ...          */
  SFX_ERR_DTYPE = -2,        /* dtype not supported by this entry point     */
  SFX_ERR_ALIGN = -3,        /* pointer or row stride not 16-byte aligned   */
  SFX_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required  */
  SFX_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed        */
  SFX_ERR_DEVICE = -6,       /* device status word has a bit set            */
  SFX_ERR_UNSUPPORTED = -7   /* shape outside the implemented range         */
} sfx_status;

/* Device status bits (OR-ed into the first word of the workspace). */
#define SFX_DEV_BAD_INDEX   0x1u   /* caller index list held an index >= K   */
#define SFX_DEV_TIMEOUT     0x2u   /* a bounded wait gave up                 */

/* Flags for sfx_sparse_gemv / sfx_sparse_ffn_swiglu / sfx_moe_expert_sparse. */
#define SFX_FLAG_GELU        0x1   /* epilogue y = GeLU(acc), erf form        */
#define SFX_FLAG_GELU_TANH   0x2   /* epilogue y = GeLU(acc), tanh form       */
#define SFX_FLAG_UNION_MASK  0x4   /* B>1: every token uses the batch union   */
#define SFX_FLAG_NO_RENORM   0x8   /* MoE: keep raw top-k softmax weights     */
#define SFX_FLAG_CUDA_CORES  0x10  /* B>1: force the CUDA-core kernel         */
#define SFX_FLAG_SWIGLU      0x20  /* gemv: W columns interleave gate|up;
                                      y = SiLU(g) * u as fp32 [B x N/2]       */

/* Operation ids for sfx_workspace_bytes(). */
typedef enum {
  SFX_OP_CALIBRATE = 0,
  SFX_OP_MASK_COMPACT = 1,
  SFX_OP_SPARSE_GEMV = 2,
  SFX_OP_FFN_SWIGLU = 3,
  SFX_OP_MOE = 4,
  SFX_OP_STATIC_FFN = 5,
  SFX_OP_ERROR_CURVE = 6
} sfx_op;

/* Bytes of workspace an operation needs (>= 256: the status header).
 *  CALIBRATE:     a = S (draws), b = K, c = P (number of sparsities), d = dtype
 *  MASK_COMPACT:  a = B, b = K (n), c = sfx_select,   d = unused
 *  SPARSE_GEMV:   a = B, b = K,     c = N,            d = dtype of x
 *  FFN_SWIGLU:    a = B, b = d,     c = ffn,          d = unused
 *  MOE:           a = B, b = d,     c = E,            d = ffn (expert), e = top_k,
 *                 f = ffn_shared
 *  STATIC_FFN:    a = B, b = d,     c = ffn
 *  ERROR_CURVE:   a = S (draws), b = K, c = N,       d = dtype of the draws,
 *                 e = P (number of levels)
 * Returns 0 for an unknown op or invalid sizes. */
size_t sfx_workspace_bytes(int op, long long a, long long b, long long c, long long d,
                           long long e, long long f);

/* Zero `ws_bytes` bytes of a workspace (cudaMemsetAsync on `stream`). */
int sfx_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Human-readable name of a status code (static string). */
const char* sfx_status_string(int status);

/* Synchronise `stream`, read and clear the device status word of `ws`.
 * Returns SFX_OK if it was 0, SFX_ERR_DEVICE otherwise (*bits_out, if not
 * NULL, receives the bits). */
int sfx_check_device_status(void* ws, unsigned int* bits_out, void* stream);

/* Number of SMs of the current device and the library's build target. */
int sfx_device_sm_count(void);
const char* sfx_build_info(void);

/* The launch plan sfx_sparse_gemv takes for a B x K input and a [K x N]
 * matrix (host only: no GPU work, no allocation; the plan depends on the
 * device's SM count, 148 when no device is visible). flags as for
 * sfx_sparse_gemv (SFX_FLAG_CUDA_CORES changes the plan); idx_mode != 0 for
 * a caller index list (B must be 1). out (host int[6]):
 *   out[0] kernel: 0 CUDA-core GEMV, 1 batch union on tcgen05, 2 batch union
 *          on mma.sync
 *   out[1] columns per CTA tile      out[2] K splits     out[3] column tiles
 *   out[4] 64-column chunks per CTA (kernel 2, else 0)
 *   out[5] rows of K per split (threshold mode; kernel 0 with a caller list:
 *          the list capacity of a split)
 * Returns SFX_OK or SFX_ERR_ARG. */
int sfx_gemv_plan(int B, long long K, long long N, int flags, int idx_mode, int* out);

/* Plan overrides for tuning sweeps and tests (host only, process-wide).
 * The library reads no environment variable: a launch plan is the planner's
 * choice unless a caller overrides one of these knobs. Value 0 restores the
 * planner's choice for that knob. Overrides apply to calls planned after
 * this one returns; setting them while other host threads launch is a race
 * on which plan those launches take (each launch still sees valid values).
 *  SFX_PLAN_UNION_KERNEL  batch-union kernel: 1 tcgen05, 2 mma.sync
 *  SFX_PLAN_UNION_MIN_B   smallest batch on the union path (2..16)
 *  SFX_PLAN_GEMV_NT       CUDA-core GEMV column tile: 256, 512, 1024, 2048
 *  SFX_PLAN_GEMV_S        CUDA-core GEMV K splits (>= 1; the list capacity
 *                         may still raise it)
 *  SFX_PLAN_UNION_S       batch-union K splits (>= 1, same caveat)
 *  SFX_PLAN_MMA_CHUNKS    mma.sync union tile in 64-column chunks: 1, 2, 4, 8
 *  SFX_PLAN_DENSE         batches of 3-16 tokens: 1 always the union kernels
 *                         (gathered union rows), 2 always the dense kernel
 *                         (every row; rows no token keeps multiply zeros),
 *                         3 the dense kernel on tcgen05 (kept for comparison);
 *                         0 lets the device choose by the union's row count
 *  SFX_PLAN_TEST_STALL    tests only: 1 makes the dense kernels leave their
 *                         first ring stage incomplete, so every wait on it
 *                         runs out (see sfx_set_wait_limit_ns)
 *  SFX_PLAN_MOE_CHUNK     MoE expert kernel: intermediate neurons per routed
 *                         work item, 16..64 (the shared expert's items take
 *                         2/3 as many)
 * Returns SFX_OK, or SFX_ERR_ARG for an unknown key or a value out of range. */
typedef enum {
  SFX_PLAN_UNION_KERNEL = 0,
  SFX_PLAN_UNION_MIN_B = 1,
  SFX_PLAN_GEMV_NT = 2,
  SFX_PLAN_GEMV_S = 3,
  SFX_PLAN_UNION_S = 4,
  SFX_PLAN_MMA_CHUNKS = 5,
  SFX_PLAN_DENSE = 6,
  SFX_PLAN_TEST_STALL = 7,
  SFX_PLAN_MOE_CHUNK = 8
} sfx_plan_key;
int sfx_set_plan_override(int key, int value);

/* Limit of the kernels' bounded waits, in nanoseconds, for calls made after
 * this one returns (host only, process-wide). Kernels that hand data between
 * warps through mbarriers (the batch-union tcgen05 kernel and the dense
 * kernels of the batch path) never wait longer than this: a wait that runs
 * out raises SFX_DEV_TIMEOUT in the workspace status word, waits (at most
 * 20 ms) for the copies and MMAs it started, releases its tensor memory and
 * returns, so the context stays usable; the output is then incomplete.
 * After a timeout the workspace's arrival counters may be left mid-count:
 * re-initialise it (sfx_workspace_init) before its next use.
 * 0 restores the default of 2 s. Returns SFX_OK. */
int sfx_set_wait_limit_ns(unsigned long long ns);

/* ------------------------------------------------------------------------
 * a1. Threshold calibration                                 [TEAL] slide 8
 *
 * For each target sparsity p_j, t_j is the lower empirical p_j-quantile of the
 * pooled magnitudes |calib| (S draws x K activations): with the sorted
 * magnitudes a_(1) <= ... <= a_(S K), t_j = a_(r) where r = ceil(p_j S K)
 * (a product within 1e-9 S K of an integer counts as that integer); p_j <= 0
 * gives t_j = -INFINITY (keep all). t_j is therefore a value of the input
 * dtype and the strict mask |x| > t_j zeroes at least p_j of the calibration
 * activations. Selection is exact (radix histogram of the magnitude bits).
 *
 *  calib          (dev)  [S x K] values of dtype dt (f16, bf16 or f32)
 *  sparsities     (host) [P] in [0, 1], double
 *  thresholds_out (host) [P] float
 *  ws             (dev)  sfx_workspace_bytes(SFX_OP_CALIBRATE, S, K, P, dt)
 * Synchronises `stream` (the thresholds are returned on the host).
 * ---------------------------------------------------------------------- */
int sfx_calibrate_thresholds(const void* calib, int dt, long long S, long long K,
                             const double* sparsities, int P, float* thresholds_out,
                             void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * a2-a4. Mask and compaction         [TEAL] slide 11, [ATTR], [GLASS] 2.2
 *
 * Per token b (row of x), builds the mask m_b over n = K neurons and its
 * ascending index list:
 *  THRESHOLD:   m_bi = 1[|x_bi| > t]                         (uses x, t)
 *  TOPK_GXO:    keep the k largest s_bi = |fl32(x_bi * g_bi)|, x of dtype dt,
 *               g = score_l (f32 [B x K]); equal scores go to the lower index
 *  TOPK_GLASS:  R^l, R^g = ranks of score_l / score_g (f32 [B x K]) with the
 *               most important neuron ranked n (score descending, then index
 *               ascending); F = (1-lambda) R^l + lambda R^g in double; keep
 *               the k largest F, ties to the lower index. x is unused.
 *  TOPK_CGXO:   corrected GxO ([ATTR] "correction term"): keep the k largest
 *               signed s_bi = fl32(fl32(x_bi g_bi) + fl32(|x_bi| n_b / 2)) with
 *               n_b = fl32(sqrt(sum_i g_bi^2)), the sum of squares in double over
 *               all K neurons of the row; g = score_l (f32 [B x K]); ties to the
 *               lower index.
 *
 *  x          (dev)  [B x K] of dtype dt (f16, bf16, f32); may be NULL for GLASS
 *  bitmap     (dev)  [B x ceil(K/32)] uint32, bit (i % 32) of word i/32 = m_bi;
 *                    may be NULL
 *  idx        (dev)  [B x K] int32: row b holds cnt[b] ascending indices,
 *                    the rest is left untouched; may be NULL
 *  cnt        (dev)  [B] int32 active counts (required)
 *  union_idx  (dev)  [K] int32 ascending indices of OR_b m_b; may be NULL
 *  union_cnt  (dev)  [1] int32; required when union_idx is given
 * Limits: 1 <= B <= 64; K <= 32768 for the top-k modes; 0 <= k <= K.
 * ---------------------------------------------------------------------- */
int sfx_mask_compact(const void* x, int dt, int B, int K, int sel, float t, int k,
                     const float* score_l, const float* score_g, double lambda,
                     uint32_t* bitmap, int32_t* idx, int32_t* cnt,
                     int32_t* union_idx, int32_t* union_cnt,
                     void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * a5/a7. Input-sparse GEMV / skinny GEMM       [TEAL] slide 11, [GLOSS]
 *
 * y[b, n] = sum_{i active for b} x[b, i] * W[i, n], accumulated in fp32,
 * reading only rows of W that some token of the batch needs.
 *  - idx == NULL: the mask is built inside the kernel (fused, never stored):
 *    token b keeps row i iff |x[b, i]| > t (t = -INFINITY: dense). Rows are
 *    fetched once for the batch (the union) and each token applies its own
 *    mask, unless SFX_FLAG_UNION_MASK makes every token use the union.
 *  - idx != NULL (B must be 1): the active rows are idx[0 .. *cnt-1]
 *    (device count), e.g. from sfx_mask_compact's top-k modes.
 * Kernels: B <= 2, or an idx list: CUDA cores (fp32 FMAs). B >= 3 with a
 * threshold: the union rows are fetched once into registers and multiplied on
 * the tensor cores (mma.sync, fp32 accumulation; fp32 x enters as two 16-bit
 * halves, hi + lo); SFX_FLAG_CUDA_CORES keeps such a batch on CUDA cores.
 * Either way the K-split sums are added in a fixed order (same bits per call).
 * Epilogue: SFX_FLAG_GELU / SFX_FLAG_GELU_TANH apply GeLU to y;
 * SFX_FLAG_SWIGLU treats columns (2j, 2j+1) as (gate_j, up_j) and writes
 * h_j = SiLU(gate_j) * up_j to y as fp32 [B x N/2] (ydt must be SFX_F32) --
 * the first stage of sfx_sparse_ffn_swiglu on its own.
 *
 *  x        (dev)  [B x K] of dtype xdt (f16, bf16, f32); xdt == wdt or f32
 *  W        (dev)  [K x N] of dtype wdt (f16, bf16), row-major, 16-byte aligned
 *  y        (dev)  [B x N] of dtype ydt (f16, bf16, f32)
 *  bitmap_out (dev, optional) [B x ceil(K/32)] receives the fused mask
 *  ws       (dev)  sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, B, K, N, xdt)
 * Limits: 1 <= B <= 16, K >= 1, N >= 8 and N % 8 == 0.
 * ---------------------------------------------------------------------- */
int sfx_sparse_gemv(const void* x, int xdt, int B, int K, const void* W, int wdt, int N,
                    float t, const int32_t* idx, const int32_t* cnt,
                    void* y, int ydt, int flags, uint32_t* bitmap_out,
                    void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * a5. Input-sparse GEMV on a given mask       [TEAL] slide 11, [ATTR]
 *
 * y[b, n] = sum_{i : m_bi} x[b, i] * W[i, n], accumulated in fp32, with the
 * mask given as a bitmap in the layout sfx_mask_compact and the fused mask
 * outputs write (bit i % 32 of word i / 32 of row b; bits at or past K are
 * ignored). Every CTA reads the mask words of its K-slice in the same round
 * trip as x and builds its active list itself, so a selection such as the
 * GxO top-k reaches the product as a bitmap, with no index list in between.
 * Rows are fetched once for the batch and each token keeps its own rows,
 * unless SFX_FLAG_UNION_MASK makes every token keep the rows any token keeps
 * (each with its own x). Every B runs on the CUDA-core kernel; the K-split
 * sums are added in a fixed order (same bits per call). Epilogue flags, dtypes,
 * workspace and limits as sfx_sparse_gemv.
 *
 *  x     (dev) [B x K] of dtype xdt (f16, bf16, f32); xdt == wdt or f32
 *  W     (dev) [K x N] of dtype wdt (f16, bf16), row-major, 16-byte aligned
 *  mask  (dev) [B x ceil(K/32)] uint32
 *  y     (dev) [B x N] of dtype ydt ([B x N/2] fp32 with SFX_FLAG_SWIGLU)
 *  ws    (dev) sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, B, K, N, xdt)
 * Returns SFX_ERR_ARG for a NULL mask or the arguments sfx_sparse_gemv
 * rejects.
 * ---------------------------------------------------------------------- */
int sfx_sparse_gemv_mask(const void* x, int xdt, int B, int K, const void* W, int wdt, int N,
                         const uint32_t* mask, void* y, int ydt, int flags,
                         void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * sfx_sparse_gemv without a workspace. The source pages have no counterpart:
 * this entry point exists for callers, not for the method.
 *
 * Same computation, arguments and limits as sfx_sparse_gemv, minus the fused
 * mask output and the workspace. It is for callers that cannot allocate
 * device memory: a plugin behind a fixed C interface that is handed only its
 * inputs and outputs, or code inside a framework that owns all device memory
 * through its own pool and forbids side allocations (cudaMalloc would also
 * synchronise the device in the middle of a latency-critical decode loop).
 * The call's scratch (status word, split-K arrival counters, partial sums)
 * lives in a 4 MiB file-scope device array inside the library instead; every
 * GPU that loads the library holds that array until the process exits. The
 * call allocates and frees nothing.
 *  - Shapes whose partial sums do not fit in the array are rejected with
 *    SFX_ERR_UNSUPPORTED before any launch.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current: make that first call
 *    before any stream capture.
 *  - Each call clears the status word and the arrival counters it uses on
 *    `stream`, then launches. All calls share the one array and it keeps the
 *    last call's contents, so calls that overlap on the GPU (other streams,
 *    other host threads) race with each other; issue them one after another.
 *  - The device status word lives in the array too and no call reads it
 *    back: an out-of-range list index (skipped, as in sfx_sparse_gemv) and a
 *    bounded wait that gave up (SFX_DEV_TIMEOUT: y is then left partly
 *    unwritten) both go unreported, and the next call clears the word.
 *    Callers that need those checks use sfx_sparse_gemv with a workspace.
 * ---------------------------------------------------------------------- */
int sfx_sparse_gemv_noalloc(const void* x, int xdt, int B, int K, const void* W, int wdt, int N,
                            float t, const int32_t* idx, const int32_t* cnt,
                            void* y, int ydt, int flags, void* stream);

/* ------------------------------------------------------------------------
 * a6. Activation-sparse SwiGLU FFN            [TEAL] slides 6 and 8
 *
 * m_x = |x| > t_in; [g | u] = (x m_x) [W_g | W_u]; h = SiLU(g) * u (fp32,
 * never rounded to the weight dtype); m_h = |h| > t_h; y = (h m_h) W_d.
 * Both products read only the rows of active neurons.
 *
 *  x      (dev) [B x d] of dtype dt (f16 or bf16)
 *  W_gu   (dev) [d x 2 ffn] of dtype dt: row i interleaves gate and up,
 *               W_gu[i, 2j] = W_g[i, j], W_gu[i, 2j+1] = W_u[i, j]
 *               (build it once with sfx_pack_gate_up)
 *  W_d    (dev) [ffn x d] of dtype dt
 *  y      (dev) [B x d] of dtype ydt
 *  h_out  (dev, optional) [B x ffn] fp32 receives h (before the m_h mask)
 *  bitmap_x_out (dev, optional) [B x ceil(d/32)], bitmap_h_out (dev,
 *               optional) [B x ceil(ffn/32)] receive the two fused masks
 *  ws     (dev) sfx_workspace_bytes(SFX_OP_FFN_SWIGLU, B, d, ffn, dt)
 * Limits: 1 <= B <= 16; d % 8 == 0; ffn % 4 == 0.
 * ---------------------------------------------------------------------- */
int sfx_sparse_ffn_swiglu(const void* x, int dt, int B, int d, int ffn,
                          const void* W_gu, const void* W_d, float t_in, float t_h,
                          void* y, int ydt, float* h_out, uint32_t* bitmap_x_out,
                          uint32_t* bitmap_h_out, int flags,
                          void* ws, size_t ws_bytes, void* stream);

/* Interleave W_g [d x ffn] and W_u [d x ffn] (dtype dt) into W_gu [d x 2 ffn]
 * (layout preparation, done once per weight set). */
int sfx_pack_gate_up(const void* W_g, const void* W_u, int dt, int d, int ffn,
                     void* W_gu, void* stream);

/* ------------------------------------------------------------------------
 * a8. MoE layer with intra-expert activation sparsity             [MOE]
 *
 * Per token t: p = softmax(logits[t]) over E experts; the top_k experts by p
 * (ties to the lower index) with weights w = p / sum(p_selected)
 * (SFX_FLAG_NO_RENORM: raw p). For each selected expert e:
 *   a_j = SiLU(W_gT[e][j, :] . x_t)  (dense gate projection)
 *   m_j = |a_j| > t_e[e]             (one threshold pass)
 *   y_t += w_e * sum_{j: m_j} a_j (W_upT[e][j, :] . x_t) W_d[e][j, :]
 * reading only rows j of W_upT[e] and W_d[e] with m_j = 1. If Ws_gT is not
 * NULL, a dense shared SwiGLU expert (always on, weight 1) is added:
 * y_t += sum_j SiLU(Ws_gT[j, :] . x_t) (Ws_upT[j, :] . x_t) Ws_d[j, :].
 * Every expert matrix, routed or shared, is stored one row per intermediate
 * neuron ([ffn x d] per expert), so each neuron's gate, up and down weights
 * are contiguous 2d-byte rows. Experts are combined into an fp32 accumulator
 * with atomics, so the last bits of y may differ between runs.
 *
 *  x       (dev) [B x d] dtype dt (bf16 or f16), 16-byte aligned
 *  logits  (dev) [B x E] f32
 *  W_gT    (dev) [E x ffn x d]   W_upT (dev) [E x ffn x d]   W_d (dev) [E x ffn x d]
 *  t_e     (dev) [E] f32 per-expert thresholds (-INFINITY: dense expert)
 *  Ws_gT, Ws_upT, Ws_d (dev, optional, all or none) [ffn_shared x d] dtype dt
 *  y       (dev) [B x d] dtype ydt
 *  a_out   (dev, optional) [B x top_k x ffn] f32 gate activations a, in each
 *          token's selection order; sel_out (dev, optional) [B x top_k] int32
 *          selected experts
 *  ws      (dev) sfx_workspace_bytes(SFX_OP_MOE, B, d, E, ffn, top_k, ffn_shared)
 * Limits: 1 <= B <= 16, 1 <= top_k <= E <= 1024, d % 8 == 0, ffn % 8 == 0,
 * ffn_shared % 8 == 0,
 * B * d <= 98304 (the expert kernel holds x of the batch in shared memory);
 * violations return SFX_ERR_ARG / SFX_ERR_ALIGN before any launch.
 * ---------------------------------------------------------------------- */
int sfx_moe_expert_sparse(const void* x, int dt, const float* logits, int B, int d, int E,
                          int ffn, int top_k, const void* W_gT, const void* W_upT,
                          const void* W_d, const float* t_e, const void* Ws_gT,
                          const void* Ws_upT, const void* Ws_d, int ffn_shared, void* y, int ydt,
                          float* a_out, int32_t* sel_out, int flags,
                          void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * a9. FFN with a static neuron mask on both projections          [GLASS]
 *
 * "GLASS: Global-Local Aggregation for inference-time Sparsification",
 * "selection": with the kept neuron set S fixed for the prompt (for example
 * the SFX_SEL_TOPK_GLASS list of sfx_mask_compact), the pruned neurons' up
 * columns are skipped as well as their down rows. For every token t:
 *   GeLU (W_bT == NULL):  h_j = GeLU(W_aT[j, :] . x_t)   (SFX_FLAG_GELU_TANH:
 *                         the tanh form, else the erf form)
 *   SwiGLU (W_bT given):  h_j = SiLU(W_aT[j, :] . x_t) (W_bT[j, :] . x_t)
 *   y_t = sum_{j in S} h_j W_d[j, :]
 * reading only the rows j in S of every matrix. For B > 1 neurons are combined
 * in an fp32 accumulator with atomics, so the last bits of y may differ
 * between runs; B = 1 runs the kept up rows, then the deterministic
 * index-list GEMV over the kept down rows.
 *
 *  x       (dev) [B x d] dtype dt (bf16 or f16), 16-byte aligned
 *  W_aT, W_bT (optional), W_d (dev) [ffn x d] dtype dt, one row per neuron
 *  idx     (dev) [>= *cnt] int32 distinct kept neurons in [0, ffn) (any order;
 *          an entry outside sets SFX_DEV_BAD_INDEX in the workspace status and
 *          adds 0)
 *  cnt     (dev) [1] int32 number of kept neurons (clamped to [0, ffn])
 *  y       (dev) [B x d] dtype ydt
 *  ws      (dev) sfx_workspace_bytes(SFX_OP_STATIC_FFN, B, d, ffn)
 * Limits: 1 <= B <= 16, d % 8 == 0, B * d <= 98304, ffn >= 1; violations
 * return SFX_ERR_ARG / SFX_ERR_DTYPE / SFX_ERR_ALIGN before any launch.
 * ---------------------------------------------------------------------- */
int sfx_static_ffn(const void* x, int dt, int B, int d, int ffn, const void* W_aT,
                   const void* W_bT, const void* W_d, const int32_t* idx, const int32_t* cnt,
                   int flags, void* y, int ydt, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Block-wise greedy sparsity allocation        [TEAL] slide 10
 *
 * "TEAL: Training-Free Activation Sparsity in Large Language Models",
 * slide 10 ("block-wise greedy optimization"): the sparsity of each block is
 * chosen to minimise the blocks' l2 activation error under a model-wide
 * sparsity target. Every block starts dense; each round raises by one step
 * the block whose error would grow least (per unit of model-wide sparsity);
 * rounds repeat until the target.
 *
 * sfx_block_error_curve: one block's error curve. The block is an input site
 * with its weight matrix W [K x N]; calib [S x K] are the site's calibration
 * draws. For each level p_j the threshold t_j is calibrated on calib exactly
 * as sfx_calibrate_thresholds does, and
 *   err_out[j] = || (calib * m_j) W - calib W ||   (Frobenius, over the S draws)
 * with m_j = 1[|calib| > t_j]; the products run through sfx_sparse_gemv (fp32
 * outputs) and the squared changes are summed in fp64 in a fixed order.
 *  calib  (dev)  [S x K] dtype xdt (f16, bf16 or f32); W (dev) [K x N] wdt
 *  levels (host) [P] sparsities in [0, 1], 1 <= P <= 64
 *  err_out (host) [P] double; thr_out (host, optional) [P] float thresholds
 *  ws     (dev)  sfx_workspace_bytes(SFX_OP_ERROR_CURVE, S, K, N, xdt, P),
 *                zeroed once (sfx_workspace_init)
 * Synchronises `stream` (the curve is returned on the host).
 * ---------------------------------------------------------------------- */
int sfx_block_error_curve(const void* calib, int xdt, long long S, long long K, const void* W,
                          int wdt, long long N, const double* levels, int P, double* err_out,
                          float* thr_out, void* ws, size_t ws_bytes, void* stream);

/* sfx_greedy_allocate (host only): the greedy rounds on given error curves.
 *  err     (host) [M x P] block i's error at level j, levels 0, step, 2 step,
 *          ... (err[i * P] is the dense block)
 *  weights (host) [M] the blocks' weights in the model-wide sparsity
 *          sum_i w_i p_i / sum_i w_i (their parameter counts: the weight rows a
 *          block's sparsity skips)
 * Each round raises by one level the block with the smallest error growth per
 * unit of model-wide sparsity, (err[i][l_i + 1] - err[i][l_i]) / w_i (equal
 * values: the lower block index), among the blocks below level P - 1 with
 * w_i > 0, until the model-wide sparsity reaches `target` or no block can go
 * further. With equal weights this is the slide's rule: the smallest growth.
 * level_out (host) [M] receives l_i (block sparsity = l_i * step). Returns
 * SFX_OK or SFX_ERR_ARG. */
int sfx_greedy_allocate(const double* err, const double* weights, int M, int P, double step,
                        double target, int* level_out);

#ifdef __cplusplus
}
#endif

#endif /* SFX_H_ */
