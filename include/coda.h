/*
 * coda.h — C ABI of the B200 (sm_100a) GEMM-epilogue library for the CODA
 * GEMM-Residual-RMSNorm-GEMM(+SwiGLU) block and the SwiGLU MLP.
 *
 * The method (toolin.ai, "CODA：LLMと初心者が光速のGPUカーネルを書けるようにする",
 * section 核心の洞察; kucoin.com (ru) "CODA: ...", section
 * «В «Финале» спрятаны сокровища»): memory-bound Transformer operations are
 * rewritten so they run in the epilogue of a GEMM while the GEMM's output is
 * still on chip.  In GEMM -> RMSNorm -> GEMM the RMSNorm row scale r commutes
 * with the second GEMM, so GEMM1's epilogue only adds the residual and emits
 * per-tile partial sums of squares, a light reduction turns them into r, and
 * GEMM2's epilogue applies r (and here SwiGLU).  The same structure carries to
 * the backward pass (kucoin (ru), same section: a block-local forward epilogue
 * gives a backward of the same form) and to SwiGLU.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or synchronises in these calls; all work is
 *    enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *    default stream) and runs asynchronously.
 *  - "bf16" arrays hold IEEE bfloat16 values (uint16 bit patterns), row-major,
 *    densely packed (leading dimension = number of columns).  fp32 arrays are
 *    IEEE float, also densely packed.
 *  - Weights use the [out_features, in_features] layout, so the pages'
 *    "X * W1" is X[M,K] times W1[d,K]^T.
 *  - Gate/up weights stack the F gate rows first and the F up rows after them
 *    ([2F, d]); saved pre-activations AB[M, 2F] hold a in columns [0, F) and
 *    b in columns [F, 2F).
 *  - Alignment: every pointer must be 16-byte aligned.  Shape requirements are
 *    stated per call; violations return an error code and launch nothing.
 *  - `ws` is a caller-owned device workspace of at least the size returned by
 *    the matching *_workspace_bytes() query.  Its first 256 bytes hold a
 *    device status word: kernels record bounded-wait timeouts there.  Zero it
 *    once (coda_status_clear) before first use; it is sticky until cleared.
 *  - The return value reports host-detectable errors only (arguments, shapes,
 *    alignment, device capability, launch failures).  Device-side errors are
 *    read with coda_status_query().  No call aborts or throws.
 *  - Requires an sm_100 device (B200); otherwise CODA_ERR_NO_SM100.
 *  - An empty batch (M = 0 tokens) is valid everywhere: the other sizes are
 *    still checked, no kernel runs, and row-sized pointers may be NULL.  A
 *    forward call then writes nothing; a backward call writes its weight
 *    gradients (dW1, dW2, dg, dWgu, dWdown, dW) as zeros, the sum over no rows,
 *    on `stream`.  coda_gemm with M = 0 or N = 0 does nothing; with K = 0 it
 *    writes C = 0.  Negative sizes return CODA_ERR_INVALID_ARG.
 */
#ifndef CODA_H_
#define CODA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CODA_OK = 0,
  CODA_ERR_INVALID_ARG = 1,         /* null pointer, negative or zero weight size, eps <= 0 */
  CODA_ERR_UNSUPPORTED_SHAPE = 2,   /* a dimension violates the stated multiple */
  CODA_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  CODA_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the *_workspace_bytes() size */
  CODA_ERR_NO_SM100 = 5,            /* current device is not compute capability 10.x */
  CODA_ERR_CUDA = 6,                /* a CUDA runtime call or kernel launch failed */
  CODA_ERR_DEVICE_TIMEOUT = 7       /* (status word) a device-side wait gave up */
} coda_status;

/* Static human-readable name of a status code. */
const char* coda_status_string(int status);

/* Library version as an integer (major*10000 + minor*100 + patch). */
int coda_version(void);

/* ---------------------------------------------------------------- status word */

/* Enqueue a zeroing of the workspace's status word on `stream`. */
coda_status coda_status_clear(void* ws, void* stream);

/* Synchronise `stream`, then read the workspace's status word.  Returns
 * CODA_OK, or the device-side error recorded by a kernel (for a timeout,
 * CODA_ERR_DEVICE_TIMEOUT).  If `detail` is non-null it receives the raw
 * 32-bit detail word (kernel id << 16 | role << 8 | reason). */
coda_status coda_status_query(const void* ws, void* stream, uint32_t* detail);

/* Set the per-wait limit of device-side bounded waits, in nanoseconds, for
 * launches issued after this call from any host thread (default 4e9 = 4 s).
 * Values are clamped to [1e3, 6e10]. */
void coda_set_wait_limit_ns(uint64_t ns);

/* Self-test of the device-side failure path: a one-warp kernel waits, with
 * the bounded wait every pipeline barrier uses, on a barrier that nothing
 * arrives on.  After limit_ns (clamped as above) it records
 * CODA_ERR_DEVICE_TIMEOUT and the detail word (kernel id 0x3F, role 0,
 * reason 1) in the workspace's status word and returns; nothing faults and
 * the context stays usable.  Read the result with coda_status_query and clear
 * it with coda_status_clear. */
coda_status coda_selftest_wait_timeout(void* ws, uint64_t limit_ns, void* stream);

/* Kernel timing hook.  Arms a one-shot pair of CUDA events around the next
 * launch, from the calling host thread, of the kernel `kernel` names, whichever
 * entry point makes it: a GEMM by its epilogue (CODA_EPI_*) or a light pass
 * (CODA_KERNEL_*).  ev_start is recorded on that launch's stream immediately
 * before the kernel and ev_stop immediately after; then that pair disarms.
 * Up to 16 pairs may be armed at once; several pairs armed for the same kernel
 * fire on its successive launches, in arming order (e.g. the three plain-store
 * GEMMs of the block's backward).  ev_start and ev_stop are cudaEvent_t handles
 * created and owned by the caller (timing enabled); the library only records
 * them.  Both NULL disarms every pair of this thread.  Returns
 * CODA_ERR_INVALID_ARG for an unknown kernel id, a single NULL event or a full
 * table.  Recording the events takes the place of the programmatic (PDL)
 * overlap at that kernel's two boundaries, so an armed launch can start a few
 * microseconds later. */
#define CODA_EPI_STORE 0      /* plain store (optional column scale) */
#define CODA_EPI_RESID_RMS 1  /* + residual, H, partial sums of squares */
#define CODA_EPI_SWIGLU 2     /* r scaling + SwiGLU (the gate/up GEMM) */
#define CODA_EPI_DN 3         /* RMSNorm correction + dg partials (backward) */
#define CODA_EPI_SWIGLU_BWD 4 /* SwiGLU backward (the down GEMM's backward) */
#define CODA_EPI_XENT 5       /* online max / sum-exp (the logits GEMM) */
#define CODA_EPI_XENT_BWD 6   /* softmax - one-hot, dlogits */
#define CODA_EPI_ROPE 7       /* rotary embedding (the QKV GEMM) */
#define CODA_KERNEL_FOLD_GAIN 16          /* W2g = W2 diag(g) */
#define CODA_KERNEL_RMS_ROWREDUCE 17      /* reserved: r is now formed in the gate/up GEMM's epilogue,
                                             so no launch carries this id */
#define CODA_KERNEL_SWIGLU_BWD_ROWSTAT 18 /* dA' = r [da | db] and the row coefficient c */
#define CODA_KERNEL_COL_REDUCE 19         /* dg from its column partials */
#define CODA_KERNEL_ROWCOEF_REDUCE 20     /* c from its row partials (MLP block backward) */
#define CODA_KERNEL_XENT_REDUCE 21        /* loss and log-sum-exp from the tile partials */
#define CODA_KERNEL_ROPE_UNROTATE 22      /* inverse rotation of dQ, dK (RoPE backward) */
coda_status coda_profile_arm(int kernel, void* ev_start, void* ev_stop);

/* ---------------------------------------------------------------- building block */

/* C[M,N] (bf16) = op(A) * op(B)^T with fp32 accumulation on tcgen05 tensor cores.
 *   a_mn_major = 0: A stored [M, K] (K contiguous);  1: A stored [K, M].
 *   b_mn_major = 0: B stored [N, K];                1: B stored [K, N].
 * Requires M, N >= 1, K >= 1; N % 32 == 0; the contiguous dimension of every
 * operand a multiple of 8 (16-byte rows).  Rows/columns beyond the extents are
 * zero-filled on load and masked on store.  ws: coda_gemm_workspace_bytes(). */
size_t coda_gemm_workspace_bytes(void);
coda_status coda_gemm(const void* A, const void* B, void* C, int M, int N, int K,
                      int a_mn_major, int b_mn_major, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- gain fold */

/* W2g[n, j] = bf16(g[j] * W2[n, j]) for the [N, d] gate/up weight: the RMSNorm
 * gain folded into the second GEMM's weight, diag(g) * W2 in the pages'
 * column-vector notation.  Requires d % 8 == 0. */
coda_status coda_fold_gain(const void* W2, const void* g, void* W2g, int d, int N, void* stream);

/* ---------------------------------------------------------------- GEMM + SwiGLU epilogue */

/* The gate/up GEMM-epilogue program on its own (toolin.ai §核心の洞察: r applied
 * in the second GEMM's epilogue; five-primitive table: activation as an
 * elementwise transform, a/b saved by the matrix-tile store):
 *   acc = A Wgu^T (fp32);  a = s_i acc[:, :F], b = s_i acc[:, F:] with
 *   s_i = r[i] (or 1 when r_or_null is null);  Y = silu(a) * b;  AB = [a | b].
 * Inputs A [M,K] bf16, Wgu [2F,K] bf16 (gate rows first), r_or_null [M] fp32.
 * Outputs Y [M,F] bf16, AB_or_null [M,2F] bf16.  Requires K % 64 == 0,
 * F % 64 == 0.  ws: coda_gemm_workspace_bytes(). */
coda_status coda_gemm_swiglu(const void* A, const void* Wgu, const float* r_or_null, void* Y, void* AB_or_null,
                             int M, int K, int F, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- GRG forward */

/* Workspace for coda_grg_fwd: status word, per-tile partial sums of squares
 * P[M, d/256] fp32, and (when the caller passes no pre-folded weight) W2g. */
size_t coda_grg_fwd_workspace_bytes(int M, int K, int d, int N, int prefolded);

/* Forward of GEMM -> residual -> partial RMS -> GEMM -> SwiGLU
 * (toolin.ai §核心の洞察; kucoin (ru) §«В «Финале» спрятаны сокровища»):
 *   GEMM1 epilogue:  H = X W1^T + R (fp32 accumulate + fp32(R), stored bf16),
 *                    P[i, t] = sum_{j in tile t} bf16(H_ij)^2 (tiles of 256 columns)
 *   GEMM2 epilogue:  r_i = 1 / sqrt(sum_t P[i,t] / d + eps) (the light row
 *                    reduction, fp32 [M], stored once per row);
 *                    acc = H W2g^T with W2g = W2 diag(g);  a = r_i acc_gate,
 *                    b = r_i acc_up;  Y = silu(a) * b  (bf16 [M, F]);
 *                    AB = [a | b] (bf16 [M, 2F]) saved for the backward.
 * Inputs:  X [M,K], W1 [d,K], R [M,d], g [d], W2 [N=2F, d] (all bf16).
 *          W2g_or_null: optional caller-folded diag(g)-scaled W2 [N, d]; when
 *          null the fold runs inside this call into the workspace.
 * Outputs: H [M,d] bf16, r [M] fp32, Y [M,F] bf16, AB_or_null [M,N] bf16.
 * Requires M >= 0, K % 64 == 0, d % 64 == 0, N % 128 == 0 (F % 64 == 0), eps > 0.
 * Rows, the last partial-RMS tile and the last F tile may be ragged. */
coda_status coda_grg_fwd(const void* X, const void* W1, const void* R, const void* g,
                         const void* W2, const void* W2g_or_null,
                         void* H, float* r, void* Y, void* AB_or_null,
                         int M, int K, int d, int N, float eps,
                         void* ws, size_t ws_bytes, void* stream);

/* Workspace for coda_grg_fwd_hg: status word, P, and Hg [M, d] bf16 when the
 * caller passes no Hg buffer. */
size_t coda_grg_fwd_hg_workspace_bytes(int M, int K, int d, int N, int hg_given);

/* The same forward with the RMSNorm gain applied on the activation side
 * instead of being folded into W2: GEMM1's epilogue also stores
 * Hg = bf16(H * g) (the elementwise-transform and tile-store primitives of
 * the five-primitive table), and GEMM2 reads Hg with the unmodified W2:
 *   acc = Hg W2^T;  a = r_i acc_gate, b = r_i acc_up;  Y = silu(a) * b.
 * diag(r) (H diag(g)) W2^T equals the folded form exactly, so the results are
 * the forward's up to bf16 rounding; the 4*N*d bytes of the gain fold are
 * replaced by M*d*2 bytes of Hg.  Hg_or_null: optional output [M, d] bf16
 * (placed in the workspace when null).  Other arguments and the shape rules
 * as coda_grg_fwd; the backward is coda_grg_bwd unchanged. */
coda_status coda_grg_fwd_hg(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                            void* H, void* Hg_or_null, float* r, void* Y, void* AB_or_null,
                            int M, int K, int d, int N, float eps,
                            void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- GRG backward */

/* Workspace for coda_grg_bwd: status word, dA' [M, N] bf16, c [M] fp32 and
 * column partials Pg [ceil(M/32), d] fp32. */
size_t coda_grg_bwd_workspace_bytes(int M, int K, int d, int N);

/* Backward of the block for the loss <dY, Y> + <dH_in, H> (toolin.ai §実験結果,
 * GEMM-Residual-PartialRMS-GEMM backward).  Steps, each a GEMM + epilogue or a
 * light pass:
 *   SwiGLU bwd + row stat:  da, db from dY, a, b;  dA' = bf16(r_i [da | db]);
 *                           c_i = (r_i^2 / d) sum_c dA_ic A_ic
 *   dn GEMM + epilogue:     dR = dH = g_j (dA' W2)_ij - c_i H_ij (+ dH_in)
 *                           with column partials of (dA' W2)_ij H_ij for dg
 *   column reduce:          dg_j = sum_i (dA' W2)_ij H_ij
 *   dW2 GEMM + epilogue:    dW2 = g_j (dA'^T H)_cj
 *   plain GEMMs:            dX = dH W1,  dW1 = dH^T X
 * Inputs:  dY [M,F], dH_in_or_null [M,d], X [M,K], W1 [d,K], H [M,d] and
 *          r [M] fp32 and AB [M,N] from coda_grg_fwd, g [d], W2 [N,d].
 * Outputs: dX [M,K], dR [M,d] (= dH), dW1 [d,K], dW2 [N,d] (bf16), dg [d] fp32.
 * Requires the same shape rules as coda_grg_fwd. */
coda_status coda_grg_bwd(const void* dY, const void* dH_in_or_null,
                         const void* X, const void* W1, const void* H, const float* r,
                         const void* AB, const void* g, const void* W2,
                         void* dX, void* dR, void* dW1, void* dW2, float* dg,
                         int M, int K, int d, int N,
                         void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- SwiGLU MLP */

/* Workspace for coda_swiglu_fwd (status word only). */
size_t coda_swiglu_fwd_workspace_bytes(int M, int d, int F);

/* SwiGLU MLP forward (toolin.ai five-primitive table: activation as an
 * elementwise epilogue transform):
 *   gate/up GEMM + epilogue: A = X Wgu^T;  Y = silu(a) * b;  AB = [a | b]
 *   down GEMM:               Out = Y Wdown^T
 * Inputs X [M,d], Wgu [2F,d], Wdown [d,F].  Outputs Y [M,F], AB_or_null
 * [M,2F], Out [M,d] (bf16).  Requires M >= 0, d % 64 == 0, F % 64 == 0. */
coda_status coda_swiglu_fwd(const void* X, const void* Wgu, const void* Wdown,
                            void* Y, void* AB_or_null, void* Out,
                            int M, int d, int F, void* ws, size_t ws_bytes, void* stream);

/* Workspace for coda_swiglu_bwd: status word and dA [M, 2F] bf16. */
size_t coda_swiglu_bwd_workspace_bytes(int M, int d, int F);

/* SwiGLU MLP backward for the loss <dOut, Out> (toolin.ai §実験結果, SwiGLU backward):
 *   down dgrad GEMM + SwiGLU-bwd epilogue:  dY = dOut Wdown, then
 *       da = dY b sigmoid(a) (1 + a (1 - sigmoid(a))), db = dY silu(a);
 *       dA = [da | db] (bf16, workspace)
 *   plain GEMMs:  dWdown = dOut^T Y,  dWgu = dA^T X,  dX = dA Wgu
 * Inputs dOut [M,d], X [M,d], Wgu [2F,d], Wdown [d,F], Y [M,F], AB [M,2F].
 * Outputs dX [M,d], dWgu [2F,d], dWdown [d,F] (bf16).  Same shape rules as
 * coda_swiglu_fwd. */
coda_status coda_swiglu_bwd(const void* dOut, const void* X, const void* Wgu, const void* Wdown,
                            const void* Y, const void* AB,
                            void* dX, void* dWgu, void* dWdown,
                            int M, int d, int F, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- full MLP block */

/* Workspace for coda_mlp_block_fwd (that of coda_grg_fwd without a pre-folded weight). */
size_t coda_mlp_block_fwd_workspace_bytes(int M, int K, int d, int F);

/* The block followed by the down projection, whose epilogue adds the residual
 * for the next block (residual add as an elementwise epilogue transform,
 * toolin.ai five-primitive table):
 *   coda_grg_fwd (H, r, Y, AB);  Out = Y Wdown^T + H  (bf16 [M, d]).
 * Inputs as coda_grg_fwd (N = 2F) plus Wdown [d, F] bf16; AB is required. */
coda_status coda_mlp_block_fwd(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                               const void* Wdown, void* H, float* r, void* Y, void* AB, void* Out,
                               int M, int K, int d, int F, float eps, void* ws, size_t ws_bytes, void* stream);

/* Workspace for coda_mlp_block_bwd: that of coda_grg_bwd plus the row
 * partials of c [M, ceil(F/256)] fp32. */
size_t coda_mlp_block_bwd_workspace_bytes(int M, int K, int d, int F);

/* Backward of <dOut, Out> for coda_mlp_block_fwd.  The down projection's
 * dgrad GEMM carries the SwiGLU backward in its epilogue, so dY never reaches
 * HBM: dY = dOut Wdown (fp32 accumulator); da, db from the saved a, b; the
 * stored operand dA' = bf16(r_i [da | db]) and the row partials of
 * c_i = (r_i^2/d) sum_c (da a + db b) come out of the same epilogue (the
 * block-local backward of kucoin (ru) «В «Финале» спрятаны сокровища»).  Then
 * dWdown = dOut^T Y, and the block's dn GEMM (with dH_in = dOut from the
 * residual), dg, dW2, dX, dW1 as in coda_grg_bwd.
 * Inputs dOut [M,d], and X, W1, H, r, AB, Y, g, W2, Wdown as saved by the
 * forward.  Outputs dX [M,K], dR [M,d], dW1 [d,K], dW2 [2F,d], dg [d] fp32,
 * dWdown [d,F] (bf16 unless stated).  Shape rules of coda_grg_fwd. */
coda_status coda_mlp_block_bwd(const void* dOut, const void* X, const void* W1, const void* H, const float* r,
                               const void* AB, const void* Y, const void* g, const void* W2, const void* Wdown,
                               void* dX, void* dR, void* dW1, void* dW2, float* dg, void* dWdown,
                               int M, int K, int d, int F, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- cross-entropy on the LM head */

/* Workspace for coda_xent_fwd: status word, per-tile (max, sum exp) partials
 * [M, ceil(V/256)] float2 and the target logits [M] fp32. */
size_t coda_xent_fwd_workspace_bytes(int M, int d, int V);

/* Cross-entropy of logits = X W^T without writing the logits to HBM: the
 * LM-head GEMM's epilogue keeps, per row and 256-column tile, the online
 * maximum and sum of exponentials (the stateful transform and tile-wise
 * log-sum-exp of the toolin.ai five-primitive table) and picks out the target
 * logit; a warp-per-row reduce merges the tiles:
 *   lse_i = log sum_j exp(logits_ij),  loss_i = lse_i - logits_i,t_i.
 * Inputs X [M,d] bf16, W [V,d] bf16, targets [M] int32 in [0, V).
 * Outputs loss [M] and lse [M] fp32 (loss is NaN for an out-of-range target).
 * Requires M >= 0, d % 64 == 0, V % 64 == 0.  Logits are fp32 accumulators. */
coda_status coda_xent_fwd(const void* X, const void* W, const int32_t* targets, float* loss, float* lse,
                          int M, int d, int V, void* ws, size_t ws_bytes, void* stream);

/* Workspace for coda_xent_bwd: status word and dlogits [M, V] bf16. */
size_t coda_xent_bwd_workspace_bytes(int M, int d, int V);

/* Backward of sum_i dloss_i loss_i.  The GEMM is recomputed and its epilogue
 * writes dlogits_ij = dloss_i (exp(logits_ij - lse_i) - [j == t_i]) (bf16);
 * then dX = dlogits W and dW = dlogits^T X (plain GEMMs).
 * Inputs X, W, targets as coda_xent_fwd, lse [M] from it, dloss [M] fp32.
 * Outputs dX [M,d], dW [V,d] bf16.  Same shape rules. */
coda_status coda_xent_bwd(const void* X, const void* W, const int32_t* targets, const float* lse,
                          const float* dloss, void* dX, void* dW, int M, int d, int V,
                          void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- QKV projection with RoPE */

/* QKV = X Wqkv^T with rotary position embedding applied in the GEMM's
 * epilogue (RoPE as an elementwise transform: toolin.ai five-primitive
 * table).  Columns are [q heads | k heads | v heads] (n_q, n_kv, n_kv heads of
 * head_dim each); in every q and k head the pair (j, j + head_dim/2) turns by
 * pos * base^(-2j/head_dim), pos = token row mod seq_len; v passes through.
 * Inputs X [M,d] bf16, Wqkv [(n_q + 2 n_kv) head_dim, d] bf16.  Output QKV
 * [M, (n_q + 2 n_kv) head_dim] bf16.  Requires d % 64 == 0, head_dim in
 * {64, 128, 256}, seq_len >= 1, base > 1.  ws: coda_gemm_workspace_bytes(). */
coda_status coda_qkv_rope_fwd(const void* X, const void* Wqkv, void* QKV, int M, int d, int n_q, int n_kv,
                              int head_dim, int seq_len, float base, void* ws, size_t ws_bytes, void* stream);

/* Workspace for coda_qkv_rope_bwd: status word and dPre [M, (n_q + 2 n_kv) head_dim] bf16. */
size_t coda_qkv_rope_bwd_workspace_bytes(int M, int d, int n_q, int n_kv, int head_dim);

/* Backward for the loss <dQKV, QKV>: dPre = inverse rotation of the q/k
 * gradient (v copied), then dX = dPre Wqkv and dW = dPre^T X.
 * Outputs dX [M,d], dW [(n_q + 2 n_kv) head_dim, d] bf16.  Same rules. */
coda_status coda_qkv_rope_bwd(const void* dQKV, const void* X, const void* Wqkv, void* dX, void* dW, int M, int d,
                              int n_q, int n_kv, int head_dim, int seq_len, float base,
                              void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- unfused comparison sequence */

/* The same block run operator by operator, the way a framework without
 * epilogue fusion runs it (the operator boundaries that the pages identify as
 * the source of the memory traffic: toolin.ai §課題; kucoin (ru) «Налог на
 * лень»).  Every intermediate goes to HBM and back; the GEMMs are this
 * library's plain-store tcgen05 GEMMs, so comparing these calls with
 * coda_grg_fwd / coda_grg_bwd isolates what the fusion saves.  For
 * measurement and error comparison; results agree with the fused path to
 * bf16 storage precision.
 *
 * Forward: T = X W1^T;  H = T + R;  r, U = bf16(RMSNorm(H) * g);
 *          AB = U W2^T (the pre-activations [a | b]);  Y = silu(a) * b.
 * Outputs as coda_grg_fwd plus U [M, d] bf16 (the normalised activations an
 * unfused backward keeps).  AB is required.
 * Backward: dA = SwiGLU'(dY, AB);  du = dA W2;  dW2 = dA^T U;
 *          dg_j = sum_i du_ij H_ij r_i;  dR = dH = RMSNorm'(du, H, g, r) (+dH_in);
 *          dX = dH W1;  dW1 = dH^T X.
 * Shape rules as coda_grg_fwd.  Workspaces from the *_workspace_bytes calls. */
size_t coda_grg_fwd_unfused_workspace_bytes(int M, int K, int d, int N);
coda_status coda_grg_fwd_unfused(const void* X, const void* W1, const void* R, const void* g, const void* W2,
                                 void* H, float* r, void* Y, void* AB, void* U,
                                 int M, int K, int d, int N, float eps,
                                 void* ws, size_t ws_bytes, void* stream);
size_t coda_grg_bwd_unfused_workspace_bytes(int M, int K, int d, int N);
coda_status coda_grg_bwd_unfused(const void* dY, const void* dH_in_or_null,
                                 const void* X, const void* W1, const void* H, const float* r,
                                 const void* AB, const void* U, const void* g, const void* W2,
                                 void* dX, void* dR, void* dW1, void* dW2, float* dg,
                                 int M, int K, int d, int N,
                                 void* ws, size_t ws_bytes, void* stream);

/* The SwiGLU MLP run operator by operator (measurement and error comparison
 * only): A = X Wgu^T (plain GEMM, stored as AB);  Y = silu(a) * b;
 * Out = Y Wdown^T;  backward: dY = dOut Wdown (stored);  dA = SwiGLU'(dY, AB);
 * dWdown = dOut^T Y;  dWgu = dA^T X;  dX = dA Wgu.  Same arguments and shape
 * rules as coda_swiglu_fwd / coda_swiglu_bwd (AB required). */
size_t coda_swiglu_bwd_unfused_workspace_bytes(int M, int d, int F);
coda_status coda_swiglu_fwd_unfused(const void* X, const void* Wgu, const void* Wdown,
                                    void* Y, void* AB, void* Out,
                                    int M, int d, int F, void* ws, size_t ws_bytes, void* stream);
coda_status coda_swiglu_bwd_unfused(const void* dOut, const void* X, const void* Wgu, const void* Wdown,
                                    const void* Y, const void* AB, void* dX, void* dWgu, void* dWdown,
                                    int M, int d, int F, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- forward without any allocation */

/* Upper bound on M * ceil(d / 256) for coda_grg_fwd_prefolded_static: the
 * partial sums of squares it keeps in the library's own static scratch
 * (4 MiB of fp32, e.g. M = 32768 tokens at d = 8192). */
#define CODA_STATIC_PARTIALS_MAX (1u << 20)

/* The GRG forward for callers that cannot allocate device memory: code that
 * runs where cudaMalloc is not allowed or not wanted (inside a framework that
 * owns every device byte through its own arena, a plugin interface that
 * hands over inputs and outputs but no workspace, a serving loop that must
 * not allocate on the request path).  The pages describe no such entry point;
 * it exists for those callers only.
 *
 * Computes exactly what coda_grg_fwd computes when given a pre-folded weight
 * (same kernels, same results): GEMM1 + residual + partial sums of squares,
 * then GEMM2 forming r from them + SwiGLU.  The caller passes every input and
 * output (X [M,K], W1 [d,K], R [M,d], W2g = bf16(W2 diag(g)) [N,d] from
 * coda_fold_gain, H [M,d], r [M] fp32, Y [M,F], AB_or_null [M,N]); there is no
 * ws argument.  Its only scratch, the partial sums P[M, ceil(d/256)] and a
 * device status word, lives in a file-scope __device__ array of the library
 * (4 MiB + 256 bytes), which every GPU that loads the library keeps until the
 * process exits.  No cudaMalloc, cudaFree or other allocating call is made.
 *
 * Limits and behaviour:
 *  - M * ceil(d/256) above CODA_STATIC_PARTIALS_MAX returns
 *    CODA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued ("the static
 *    scratch is too small for this shape"); the other shape rules are those of
 *    coda_grg_fwd.
 *  - The first call on a device (with that device current) looks up the
 *    array's device address with cudaGetSymbolAddress and caches it; make
 *    that first call before any stream capture.  A failed lookup returns
 *    CODA_ERR_CUDA.
 *  - Every call on a device shares the one array, and the array keeps the
 *    last call's contents.  Each call zeroes the status word first (the
 *    partial sums are fully overwritten); calls whose work overlaps on the GPU
 *    (different streams, or host threads without ordering) race on the array,
 *    so callers must serialise them.
 *  - A device-side wait timeout is recorded in that internal status word;
 *    coda_static_status_query reads it back. */
coda_status coda_grg_fwd_prefolded_static(const void* X, const void* W1, const void* R, const void* W2g,
                                          void* H, float* r, void* Y, void* AB_or_null,
                                          int M, int K, int d, int N, float eps, void* stream);

/* Status of the last coda_grg_fwd_prefolded_static call on the current
 * device: synchronises `stream`, copies the static scratch's status word to
 * the host and returns it (CODA_OK, or CODA_ERR_DEVICE_TIMEOUT with the
 * kernel / role / reason word in *detail when detail is not NULL).  The word
 * is zeroed at the start of every such call.  Allocates nothing; like the
 * first forward call it looks the array's address up on first use.  Returns
 * CODA_ERR_CUDA when the stream cannot be synchronised or the copy fails. */
coda_status coda_static_status_query(void* stream, uint32_t* detail);

#ifdef __cplusplus
}
#endif

#endif /* CODA_H_ */
