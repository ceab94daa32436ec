/*
 * rs.h -- C ABI of librs.so: the pruned-MLP block of Representation Shift on
 * NVIDIA B200 (sm_100a), and the attention sublayer and encoder layers around it.
 *
 * Method: "Representation Shift: Unifying Token Compression with
 * FlashAttention" (arXiv 2508.00367v1, ICCV 2025).
 *   - Block, §3.3 Eq. (6):      y = x-hat = MLP(LN(x')) + x'
 *   - Score, §3.2 Eq. (4) with F = MLP (§3.3 "Operation choice" (ii)) and
 *     D = L2 (§3.3 "Distance metrics" (i)):   s = || MLP(LN(x')) - x' ||_2
 *   - Pruning, §3.1 / §3.2: drop the lowest-s tokens, keep x-tilde in
 *     R^{(N-r) x C} for the attention layer that follows.
 *   - Attention sublayer, §3.1 Eq. (1) and §3.3 Eq. (5): x' = SA(LN(x)) + x
 *     (rs_attn_*), and layers of both with pruning between them
 *     (rs_encoder_forward; the §4.2 DeiT schedule is one choice of keep[]).
 *
 * Conventions shared by every entry point:
 *   - Every tensor argument is a DEVICE pointer owned by the caller, contiguous,
 *     row-major, 16-byte aligned unless stated otherwise. "bf16" is IEEE
 *     bfloat16 (torch.bfloat16). Nothing here frees or keeps caller memory.
 *   - Weights use the nn.Linear layout: W1 is [H, C], W2 is [C, H].
 *   - Token rows are [B, L, C] with r = b*L + t; t = 0 is the CLS token and
 *     t = 1..L-1 are patch tokens.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Every call is asynchronous on that stream and never synchronises,
 *     except rs_get_last_device_error and rs_release_workspace.
 *   - Return value: an rs_status. Argument errors are detected on the host and
 *     returned before anything is launched; outputs are then left untouched.
 *     RS_ERR_CUDA reports a launch or allocation failure from the CUDA runtime.
 *   - Device-side failures (a pipeline wait that ran past its time limit) do
 *     not trap: the kernel records RS_ERR_DEVICE_TIMEOUT in a device flag,
 *     drains its own work and returns; rs_get_last_device_error reports it.
 *   - Shape limits: 1 <= L <= RS_MAX_L; C and H multiples of 64 with
 *     64 <= C <= RS_MAX_C and 64 <= H <= RS_MAX_H; 0 <= keep_k <= L-1;
 *     B*L*max(C,H) < 2^31. B = 0 is an empty batch: RS_OK, nothing launched.
 *   - Library workspace: rs_block_forward, the fc steps, the attention entry
 *     points and rs_encoder_forward use a per-device workspace owned by the
 *     library (grown on demand, reused across calls; rs_encoder_forward also
 *     keeps a second buffer for its activations). Growth is stream-ordered on
 *     the call's stream (cudaFreeAsync of the old buffer, cudaMallocAsync of the
 *     new one from the device's default memory pool) and synchronises nothing.
 *     Calls that share a device must be ordered on one stream, or by the
 *     caller's events (they share the buffers, and a buffer released by growth
 *     on one stream may still be in use by work queued on another). A call on a
 *     stream that is being captured into a CUDA graph cannot grow a buffer: it
 *     returns RS_ERR_NO_MEM before launching anything. Once the buffers have
 *     grown to a call's sizes, repeating the call allocates nothing, so it can
 *     be captured. The first call on a device also allocates, once, the
 *     device's status flag (cudaMalloc + cudaMemset): make it before capturing.
 */
#ifndef RS_H_
#define RS_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RS_MAX_L 16384
#define RS_MAX_C 2048
#define RS_MAX_H 16384

/* Shift distances D of §3.3 "Distance metrics", for the extended (_ex) entry
 * points; the others use RS_DIST_L2, the paper's default:
 *   RS_DIST_L2      s = || h - x' ||_2                               (case (i))
 *   RS_DIST_L1      s = || h - x' ||_1                               (case (ii))
 *   RS_DIST_COSINE  s = 1 - h.x' / max(||h|| ||x'||, 1e-8), floored  (case (iii))
 *                   at 0 in fp32 (the pages give neither floor)
 * with h = MLP(LN(x')) in fp32, before rounding. */
#define RS_DIST_L2 0
#define RS_DIST_L1 1
#define RS_DIST_COSINE 2
/* Flags of the extended entry points. RS_NO_CLS: t = 0 is an ordinary token
 * (a video sequence of patch tokens, as UMT's, §4.1): all L tokens are ranked,
 * 0 <= keep_k <= L, and kept_idx / y_kept hold keep_k entries per sample
 * instead of 1 + keep_k with the CLS token first. */
#define RS_NO_CLS 1

typedef enum rs_status {
  RS_OK = 0,
  RS_ERR_NULL = 1,            /* a required pointer is NULL */
  RS_ERR_SHAPE = 2,           /* B, L, C or H outside the limits above, or an unknown
                                 distance / flag */
  RS_ERR_KEEP_K = 3,          /* keep_k outside 0..L-1 */
  RS_ERR_ALIGN = 4,           /* a pointer is not 16-byte (tensors) / 4-byte (int, float) aligned */
  RS_ERR_CUDA = 5,            /* the CUDA runtime or driver reported an error */
  RS_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up waiting on its pipeline (device flag) */
  RS_ERR_NO_MEM = 7           /* the workspace could not be allocated, or would have to
                                 grow on a stream that is being captured */
} rs_status;

/*
 * rs_block_forward -- the whole hot path for one block (Eq. (6) + Eq. (4) +
 * pruning), on `stream`:
 *   u   = LN(x')            per row: (x'-mean)/sqrt(var+1e-6)*gamma+beta,
 *                           biased variance
 *   h   = W2 GELU(W1 u + b1) + b2   (exact erf GELU; fp32 accumulation of bf16
 *                                    operands; the hidden activation is
 *                                    rounded to bf16 between fc1 and fc2)
 *   y   = x' + h            (rounded to bf16)
 *   s_t = || h_t - x'_t ||_2 (h in fp32, before rounding)
 *   kept_idx[b] = [0] ++ ascending(the keep_k patch tokens of largest s;
 *                 equal s -> lower t first)
 *   y_kept[b, j, :] = y[b, kept_idx[b, j], :]
 *
 *   x        [B, L, C] bf16   input x' (the attention sublayer's output)
 *   W1 [H, C], b1 [H], W2 [C, H], b2 [C], gamma [C], beta [C]: bf16
 *   keep_k   patch tokens kept per sample (CLS is kept in addition)
 *   y_kept   [B, 1+keep_k, C] bf16   output
 *   kept_idx [B, 1+keep_k] int32     output (4-byte aligned)
 *   scores   [B, L] fp32             output, every token incl. CLS (4-byte aligned)
 */
int rs_block_forward(const void* x, int B, int L, int C, int H,
                     const void* W1, const void* b1, const void* W2, const void* b2,
                     const void* gamma, const void* beta, int keep_k,
                     void* y_kept, int32_t* kept_idx, float* scores, void* stream);

/* rs_block_forward with a choice of shift distance (RS_DIST_*) and flags
 * (RS_NO_CLS). With RS_NO_CLS, 0 <= keep_k <= L and y_kept [B, keep_k, C],
 * kept_idx [B, keep_k] (may be NULL when keep_k = 0). rs_block_forward is
 * rs_block_forward_ex(..., RS_DIST_L2, 0, ...). Unknown distance or flags:
 * RS_ERR_SHAPE. */
int rs_block_forward_ex(const void* x, int B, int L, int C, int H, const void* W1,
                        const void* b1, const void* W2, const void* b2, const void* gamma,
                        const void* beta, int keep_k, int distance, int flags, void* y_kept,
                        int32_t* kept_idx, float* scores, void* stream);

/* The MLP sublayer without pruning, y = x + MLP(LN(x)) (Eq. (6)), as the layers
 * of a pruning schedule that do not prune run it: the same three launches as the
 * first three of rs_block_forward (LN statistics + fold, fc1, fc2), y written to
 * the caller's buffer. x, y [M, C] bf16; weights as for rs_block_forward. */
int rs_mlp_forward(const void* x, int M, int C, int H, const void* W1, const void* b1,
                   const void* W2, const void* b2, const void* gamma, const void* beta, void* y,
                   void* stream);

/*
 * The attention sublayer that feeds the block (Eq. (5): x' = SA(LN(x)) + x) and
 * that consumes its pruned output in the next layer. SA is Eq. (1),
 * Softmax(Q K^T / sqrt(d)) V, in the multi-head form of the ViT models the paper
 * runs: [Q, K, V] = LN(x) Wqkv^T + bqkv with Q, K, V at columns [0, C), [C, 2C),
 * [2C, 3C) of the projection, heads of width d = 64 (head h at columns
 * 64h .. 64h+63 of each), the heads' outputs concatenated, then the output
 * projection Wo, bo. C = 64 * heads. The LayerNorm is the block's (biased
 * variance, eps = 1e-6).
 *   x     [B, L, C] bf16       the sublayer input
 *   Wqkv  [3C, C], bqkv [3C]   bf16, nn.Linear layout
 *   Wo    [C, C],  bo [C]      bf16
 *   gamma, beta [C]            bf16, the sublayer's LayerNorm
 * All device pointers, 16-byte aligned unless stated; workspace and error
 * behaviour as for rs_block_forward (argument errors return before any launch).
 */

/* x_out [B, L, C] bf16 = x + SA(LN(x)). Four launches: LN statistics + weight
 * fold, the QKV projection (the folded-LN tcgen05 GEMM without activation),
 * rs_attn_core, the output projection with the residual (the fc2 GEMM, K = C). */
int rs_attn_sublayer(const void* x, int B, int L, int C, int heads, const void* Wqkv,
                     const void* bqkv, const void* Wo, const void* bo, const void* gamma,
                     const void* beta, void* x_out, void* stream);

/* rs_attn_sublayer followed by pruning on the representation shift through the
 * attention, D(SA(LN(x)), x) (§3.3 "Operation choice" case (i)), with the
 * distance and flags of rs_block_forward_ex: x_kept [B, n, C] bf16 holds the
 * kept rows of x' (n = 1 + keep_k with a CLS token, keep_k with RS_NO_CLS),
 * kept_idx [B, n] int32, scores [B, L] fp32 (4-byte aligned). */
int rs_attn_forward_ex(const void* x, int B, int L, int C, int heads, const void* Wqkv,
                       const void* bqkv, const void* Wo, const void* bo, const void* gamma,
                       const void* beta, int keep_k, int distance, int flags, void* x_kept,
                       int32_t* kept_idx, float* scores, void* stream);

/* A ViT encoder of `depth` layers, each the attention sublayer (Eq. (5)) then the
 * MLP sublayer (Eq. (6)), with representation-shift pruning (L2 shift through the
 * MLP, CLS kept) after the MLP of the layers that keep[l] >= 0 names: those keep
 * keep[l] patch tokens (0 <= keep[l] <= tokens entering layer l - 1); keep[l] < 0
 * runs the MLP without pruning (rs_mlp_forward). The pruning schedule of the
 * paper's DeiT runs (§4.2) keeps 80% of the tokens after layers 1, 4 and 7.
 *   x        [B, L, C] bf16, the first layer's input
 *   weights  12 * depth device pointers, per layer: Wqkv, bqkv, Wo, bo, gamma1,
 *            beta1 (attention sublayer), W1, b1, W2, b2, gamma2, beta2 (MLP), all
 *            bf16, 16-byte aligned, shapes as for rs_attn_sublayer and
 *            rs_block_forward (H = hidden width)
 *   keep     depth ints (host memory)
 *   out      [B, L_out, C] bf16, L_out = 1 + the last keep[l] >= 0, else L
 * The library holds the activations between layers (three [B, L, C] buffers and
 * one layer's kept indices and scores) in a cached device buffer beside the
 * workspace; rs_release_workspace frees both. Argument errors (any layer's)
 * return before the first launch. */
int rs_encoder_forward(const void* x, int B, int L, int C, int H, int heads, int depth,
                       const void* const* weights, const int* keep, void* out, void* stream);

/* Test hook of the attention core's failure path: rs_attn_core in which the CTA of
 * query tile 0, head 0, sample 0 withholds the loads of key block `skip_block`
 * (blocks of 64 keys, 0 <= skip_block < ceil(L / 64)) and of every later block,
 * with every pipeline wait limited to timeout_us microseconds (1 .. 1e7). The
 * waits for the withheld tiles run out: the CTA records RS_ERR_DEVICE_TIMEOUT in
 * the device flag, drains its MMAs, frees its TMEM and returns; no fault, no hang.
 * Other arguments as for rs_attn_core. */
int rs_debug_attn_skip_load(const void* qkv, int B, int L, int heads, void* out, int skip_block,
                            int timeout_us, void* stream);

/* The attention core alone: out [B, L, 64 heads] bf16 = per sample and head,
 * Softmax(Q K^T / 8) V from qkv [B, L, 3 * 64 heads] bf16 laid out as above (a
 * tcgen05 kernel: scores and P V in TMEM, online softmax, one CTA per 128
 * queries of a (sample, head)). 1 <= L <= RS_MAX_L, 64 heads <= RS_MAX_C. */
int rs_attn_core(const void* qkv, int B, int L, int heads, void* out, void* stream);

/* rs_block_forward_ex with the representation shift through the entire attention
 * block (§3.3 "Operation choice" case (iii)): the score is D(x-hat, x_in), with
 * x-hat = y = x' + MLP(LN(x')) in fp32 (before its bf16 store) and x_in [B, L, C]
 * bf16 the block input that the attention sublayer (Eq. (5)) started from, instead
 * of D(MLP(LN(x')), x'). Same launches (fc2's epilogue also reads x_in), outputs,
 * distances, flags and errors as rs_block_forward_ex; x_in 16-byte aligned. */
int rs_block_forward_block_shift_ex(const void* x_in, const void* x, int B, int L, int C, int H,
                                    const void* W1, const void* b1, const void* W2,
                                    const void* b2, const void* gamma, const void* beta,
                                    int keep_k, int distance, int flags, void* y_kept,
                                    int32_t* kept_idx, float* scores, void* stream);

/*
 * Step-level entry points. rs_block_forward launches exactly these kernels in
 * this order; they are exported so that each step can be checked on its own.
 */

/* LayerNorm row statistics (Eq. (6)'s LN, the reduction half):
 * stats[2r] = mean of x'[r, :], stats[2r+1] = 1/sqrt(biased var + 1e-6).
 * x [M, C] bf16; stats [M, 2] fp32 (8-byte aligned). */
int rs_ln_stats(const void* x, int M, int C, float* stats, void* stream);

/* a = GELU(LN(x') W1^T + b1) as bf16 [M, H] (Eq. (6)'s LN and fc1 with the
 * exact GELU). LN is fused into fc1 by folding: with Wg = bf16(W1 * gamma),
 * G[j] = sum_c Wg[j, c] and cb[j] = sum_c W1[j, c] beta[c] + b1[j],
 *   LN(x') W1^T + b1 = rstd * (x' Wg^T - mean * G) + cb,
 * so the GEMM reads x' as stored and the epilogue applies mean, rstd, G, cb.
 * Uses rs_ln_stats internally; the statistics and the folded weights live in
 * the library workspace. x [M, C]; hidden [M, H] bf16 output. */
int rs_ln_fc1_gelu(const void* x, int M, int C, int H, const void* W1, const void* b1,
                   const void* gamma, const void* beta, void* hidden, void* stream);

/* The two launches that rs_ln_fc1_gelu makes after rs_ln_stats, exported on
 * their own. rs_ln_fold: Wg [H, C] bf16, colG [H] and colC [H] fp32 as above
 * (the fold of the LayerNorm's gamma, beta into fc1; W1 [H, C], b1 [H],
 * gamma [C], beta [C] bf16). rs_fc1_gelu_folded: the tcgen05 GEMM with the
 * folded-LN + GELU epilogue; stats [M, 2] from rs_ln_stats (8-byte aligned),
 * colG and colC 16-byte aligned; hidden [M, H] bf16 output. */
int rs_ln_fold(const void* W1, const void* b1, const void* gamma, const void* beta, int C, int H,
               void* Wg, float* colG, float* colC, void* stream);
int rs_fc1_gelu_folded(const void* x, const float* stats, const void* Wg, const float* colG,
                       const float* colC, int M, int C, int H, void* hidden, void* stream);

/* The same result with the LayerNorm applied while staging fc1's A operand:
 * LN warps normalise each x' tile in shared memory (fp32 math, bf16 out)
 * before the tensor cores read it. Same arguments and workspace use. */
int rs_ln_fc1_gelu_staged(const void* x, int M, int C, int H, const void* W1, const void* b1,
                          const void* gamma, const void* beta, void* hidden, void* stream);

/* The exact GELU, z * Phi(z), elementwise in fp32 with the arithmetic of the
 * fc1 epilogue (|error| <= 1.2e-6). z, out: [n] fp32 (4-byte aligned). */
int rs_gelu_apply(const float* z, float* out, int n, void* stream);

/* fc2 with the residual and the shift partials (Eq. (6) and Eq. (4)):
 *   h = hidden W2^T + b2 (fp32), y = bf16(x' + h) [M, C],
 *   partials[r, j] = sum over column group j of (h[r,c] - x'[r,c])^2 (fp32).
 * partials is [M, rs_num_partials(C)] fp32; summing a row's partials left to
 * right gives s_t^2. */
int rs_fc2_residual_shift(const void* hidden, const void* x, int M, int C, int H,
                          const void* W2, const void* b2, void* y, float* partials,
                          void* stream);
/* The same with the partials of another distance: RS_DIST_L1 sums |h - x'|,
 * RS_DIST_COSINE writes per column group the triple (sum h x', sum h^2,
 * sum x'^2); partials is [M, rs_num_partials_ex(C, distance)] fp32. */
int rs_fc2_residual_shift_ex(const void* hidden, const void* x, int M, int C, int H,
                             const void* W2, const void* b2, int distance, void* y,
                             float* partials, void* stream);

/* Number of per-row partial sums rs_fc2_residual_shift writes for width C
 * (0 if C is unsupported); rs_num_partials_ex: for a distance (three per column
 * group for RS_DIST_COSINE, one otherwise; 0 for an unknown distance). */
int rs_num_partials(int C);
int rs_num_partials_ex(int C, int distance);

/* Score finalisation and per-sample top-k (§3.2 drop the lowest-k scores):
 *   scores[b, t] = sqrt(sum_{j=0..P-1} partials[b*L+t, j])  (fp32, left to right)
 *   kept_idx[b]  = [0] ++ ascending(top keep_k of t = 1..L-1 by score; ties to
 *                  the lower t). Selection compares the fp32 score bits.
 * partials [B*L, P] fp32 with 1 <= P <= 64; scores [B, L]; kept_idx [B, 1+keep_k]. */
int rs_select_topk(const float* partials, int num_partials, int B, int L, int keep_k,
                   float* scores, int32_t* kept_idx, void* stream);
/* rs_select_topk for another distance and flags: scores are sum_j P (L1) or
 * max(0, 1 - HX / max(sqrt(HH) sqrt(XX), 1e-8)) from per-group triples summed
 * component-wise left to right (cosine; num_partials a multiple of 3); with
 * RS_NO_CLS all L tokens are ranked and kept_idx is [B, keep_k]. */
int rs_select_topk_ex(const float* partials, int num_partials, int B, int L, int keep_k,
                      int distance, int flags, float* scores, int32_t* kept_idx, void* stream);

/* rs_select_topk followed by rs_gather_rows (same outputs), as rs_block_forward
 * runs them: for L <= 256 one fused kernel in which every CTA ranks its
 * sample's scores and copies a share of its kept rows. partials [B*L, P] fp32
 * (1 <= P <= 64), y [B, L, C] bf16; outputs as for the two calls. */
int rs_select_gather(const float* partials, int num_partials, const void* y, int B, int L, int C,
                     int keep_k, float* scores, int32_t* kept_idx, void* y_kept, void* stream);
/* rs_select_gather for another distance and flags (as rs_select_topk_ex);
 * y_kept is [B, keep_k + (flags & RS_NO_CLS ? 0 : 1), C]. */
int rs_select_gather_ex(const float* partials, int num_partials, const void* y, int B, int L,
                        int C, int keep_k, int distance, int flags, float* scores,
                        int32_t* kept_idx, void* y_kept, void* stream);

/* The MLP sublayer (§3.3 Eq. (6)) with the shift partials (Eq. (4)) in one
 * kernel, for narrow blocks: fc1 with the folded LayerNorm and GELU, fc2 with
 * b2 and the residual, the hidden activation kept on chip (TMEM, then shared
 * memory as fc2's A operand, one 128-column chunk at a time) and never stored.
 * Inputs as for rs_fc1_gelu_folded (stats from rs_ln_stats; Wg, colG, colC
 * from rs_ln_fold) plus W2 [C, H] and b2 [C] bf16:
 *   a = bf16(GELU(rstd*(x' Wg^T - mean*G) + cb)), h = a W2^T + b2 (fp32),
 *   y = bf16(x' + h)  [M, C] bf16 output,
 *   partials[r, j] = sum over column quarter j (columns jC/4 .. (j+1)C/4-1) of
 *                    (h[r,c] - x'[r,c])^2, [M, RS_FUSED_PARTIALS] fp32 output
 *                    (4-byte aligned); summed left to right they give s_t^2
 *                    (rs_select_topk / rs_select_gather with num_partials = 4).
 * rs_mlp_fused_supported(C, H) is 1 when 64 <= C <= 384 (C a multiple of 64)
 * and H is a multiple of 128, else 0; rs_mlp_fused returns RS_ERR_SHAPE outside
 * that range. It uses no workspace. rs_block_forward does not take this path:
 * one CTA owns a 128-row tile for the whole hidden loop, so the tensor cores
 * wait on each chunk's GELU and a short M leaves most SMs idle; the two GEMMs
 * measured faster on a B200 at every size tried (M = 394, C = 192, H = 768:
 * 25 against 36 us; M = 50432, C = 384, H = 1536: 150 against 221 us). */
#define RS_FUSED_PARTIALS 4
int rs_mlp_fused_supported(int C, int H);
int rs_mlp_fused(const void* x, const float* stats, const void* Wg, const float* colG,
                 const float* colC, int M, int C, int H, const void* W2, const void* b2, void* y,
                 float* partials, void* stream);

/* Row gather, the pruned set x-tilde (§3.1):
 * y_kept[b, j, :] = y[b, kept_idx[b, j], :]. y [B, L, C] bf16; kept_idx
 * [B, 1+keep_k] int32 with entries in 0..L-1 (not checked on the device);
 * y_kept [B, 1+keep_k, C] bf16. */
int rs_gather_rows(const void* y, int B, int L, int C, const int32_t* kept_idx, int keep_k,
                   void* y_kept, void* stream);

/* rs_ln_fc1_gelu without any allocation, for callers that cannot allocate
 * device memory when they call: a framework that owns every byte of device
 * memory through its own pool and allows no other allocation, or latency-bound
 * code that cannot afford cudaMalloc or cudaFree, which may synchronise the
 * whole device. The paper has no counterpart; this is a library convenience.
 *   Same arguments and result as rs_ln_fc1_gelu. Its scratch (LN statistics,
 *   folded fc1 weights, a status slot) is one static device array of about
 *   8.6 MiB that every GPU loading the library holds until exit; the call
 *   itself makes no cudaMalloc, cudaFree or other allocating call.
 *   Limits: M <= 65536 and H * C <= 4194304, beyond which it returns
 *   RS_ERR_SHAPE without launching (as for any other shape error).
 *   The first call on a device resolves the array's device address for that
 *   device (cudaGetSymbolAddress) and keeps it.
 *   Every call on a device shares the one array and leaves its contents behind;
 *   each call writes every scratch byte it reads before reading it. The status
 *   slot starts at zero (the array is zero-initialised when the library loads)
 *   and goes back to zero when it is read. Calls whose executions overlap on
 *   the GPU (different streams, no ordering between them) race on the array:
 *   order them.
 *   A pipeline timeout on this path is recorded in the status slot, which
 *   rs_get_last_device_error reads and clears. */
int rs_ln_fc1_gelu_noalloc(const void* x, int M, int C, int H, const void* W1, const void* b1,
                           const void* gamma, const void* beta, void* hidden, void* stream);

/* Test hook for failure detection (no counterpart in the paper): runs
 * rs_ln_fc1_gelu except that CTA 0's producer leaves k-block `skip_kblock`
 * (0 <= skip_kblock < C/64) of its first tile unloaded, so the MMA warp's wait
 * on that stage cannot complete. Every pipeline wait is limited to `timeout_us`
 * (1 .. 10^7). The kernel then records RS_ERR_DEVICE_TIMEOUT in the device
 * flag, drains its own in-flight copies and MMAs, frees its tensor memory and
 * returns; rs_get_last_device_error reports the status and the CUDA context
 * stays usable. `hidden` is left partly unwritten. */
int rs_debug_fc1_skip_load(const void* x, int M, int C, int H, const void* W1, const void* b1,
                           const void* gamma, const void* beta, void* hidden, int skip_kblock,
                           int timeout_us, void* stream);

/* Human-readable name of a status code (static storage). */
const char* rs_status_string(int status);

/* Synchronises `stream`, returns and clears the current device's flag
 * (RS_OK or RS_ERR_DEVICE_TIMEOUT) together with rs_ln_fc1_gelu_noalloc's
 * status slot on that device (either one set gives RS_ERR_DEVICE_TIMEOUT), or
 * RS_ERR_CUDA if the synchronisation or a read failed. */
int rs_get_last_device_error(void* stream);

/* Frees the library workspace of every device (synchronises each device that
 * has one). The next call that needs it allocates it again. */
void rs_release_workspace(void);

/* Bytes of workspace rs_block_forward needs for these sizes (0 if invalid). */
uint64_t rs_workspace_bytes(int B, int L, int C, int H);

#ifdef __cplusplus
}
#endif

#endif /* RS_H_ */
