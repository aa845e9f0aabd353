/*
 * sparge.h - C ABI of the pooled block-sparse attention library (sm_100a).
 *
 * Each operation is one stream-ordered launch sequence on the caller's CUDA
 * stream. The three of the hot path:
 *
 *   sparge_mask      block mask: mean-pool Q and K per block, score the
 *                    pooled blocks with softmax(qbar . kbar / sqrt(d)) along
 *                    each query-block row, keep the union of the Top-k and
 *                    Top-p selections. SpargeAttention2 article ("Tsinghua
 *                    invents an AI attention-slimming technique",
 *                    arXiv:2602.13515), section 1 (Top-k, Top-p and their
 *                    merge) and section 4 (pooling pre-filter, block-level
 *                    mask, blocks computed whole or skipped whole).
 *   sparge_attn_fwd  block-sparse attention over the kept blocks only, softmax
 *                    renormalised over the kept keys. Same article, section 4;
 *                    SLA2 article (arXiv:2602.12675), section 2 (the sparse
 *                    branch is renormalised over the kept region).
 *   sla2_attn_fwd    O = alpha_h * O_sparse + (1 - alpha_h) * O_linear, the
 *                    linear branch being phi-feature attention,
 *                    phi(x) = elu(x) + 1, over the keys of the blocks NOT kept.
 *                    SLA2 article, section 1 (sparse attention for important
 *                    regions, linear attention for the rest) and section 2
 *                    (learnable mixing ratio alpha).
 *
 * and three variants of them: sparge_mask_router (the mask scored through
 * learnt projections of the pooled blocks, SLA2 article section 2),
 * sparge_attn_fwd_q8 (the sparse branch on int8 / fp8 operand codes, SLA2
 * article section 3) and sparge_mask_noalloc (the mask with a static scratch).
 *
 * Conventions shared by every entry point
 *   - Q, K, V, O: bf16, [B, H, N, d] contiguous (d fastest), device memory,
 *     16-byte aligned. d is 64 or 128 (sla2_attn_fwd: 128).
 *   - Blocks: bq query rows and bk keys per block, each 64 or 128.
 *     Nqb = ceil(N / bq), Nkb = ceil(N / bk); a ragged last block holds the
 *     remaining rows only. No causal masking.
 *   - Block mask: kv_idx int32 [B, H, Nqb, Nkb] and kv_cnt int32 [B, H, Nqb].
 *     Row (b, h, I) keeps the kv_cnt[b,h,I] blocks kv_idx[b,h,I,0..cnt), which
 *     are strictly ascending and lie in [0, Nkb). Entries past cnt are not
 *     read and not written. The attention entry points trust these lists
 *     (they are not validated on the device).
 *   - Ownership: the caller owns every buffer. The library allocates no
 *     memory and keeps no state between calls, except the device error word
 *     read by sparge_device_status.
 *   - Workspace: scratch device memory of at least
 *     sparge_workspace_bytes(op, shape) bytes, 256-byte aligned, owned by the
 *     caller, not used across calls. May be NULL when that size is 0.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued on it; the calls return without synchronising.
 *   - Errors: arguments are checked on the host before anything is launched;
 *     a failed check returns a status and launches nothing. A failed launch
 *     returns SPARGE_ERR_CUDA. Device-side waits are bounded: a kernel that
 *     gives up records a code that sparge_device_status returns. Nothing
 *     crosses the ABI as an exception.
 *   - Determinism: identical inputs give bit-identical outputs.
 *   - Host threads: any thread may call any entry point, on any stream and
 *     device, concurrently with other threads; the host state the library
 *     keeps (kernel attributes raised once per device, the tensor-map
 *     encoder's address) is initialised under locks. The device error word
 *     is one per device and shared by every caller: the first
 *     sparge_device_status call after a kernel gave up returns the code and
 *     clears it. sparge_mask_noalloc calls share one static scratch array
 *     per device, so two of them must not overlap in time on the device.
 */
#ifndef SPARGE_H_
#define SPARGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARGE_OK = 0,
  SPARGE_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, bad fraction, misaligned buffer */
  SPARGE_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement (d, bq, bk, Nkb) */
  SPARGE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than sparge_workspace_bytes */
  SPARGE_ERR_CUDA = 4,         /* a CUDA call or launch failed */
  SPARGE_ERR_DEVICE_TIMEOUT = 5 /* a kernel gave up a bounded wait (from sparge_device_status) */
} sparge_status;

typedef struct {
  int32_t B, H, N, d; /* batch, heads, tokens, head dim */
  int32_t bq, bk;     /* query rows per block, keys per block */
} sparge_shape;

enum {
  SPARGE_OP_MASK = 0,
  SPARGE_OP_ATTN = 1,
  SPARGE_OP_SLA2 = 2,
  SPARGE_OP_ATTN_Q8 = 3,
  SPARGE_OP_MASK_ROUTER = 4,
  SPARGE_OP_ATTN_BWD = 5,
  SPARGE_OP_SLA2_BWD = 6
};

/* Workspace bytes the operation needs for this shape (0 if none, or if the
 * shape is invalid). */
size_t sparge_workspace_bytes(int op, const sparge_shape* shape);

/* Block mask (SpargeAttention2 article, sections 1 and 4).
 *   Q, K        bf16 [B,H,N,d], device.
 *   topk_frac   in [0,1]: Top-k keeps kc = ceil(topk_frac * Nkb) blocks
 *               (computed as ceil(topk_frac*Nkb - 1e-9)); 0 disables Top-k.
 *   topp        in [0,1]: Top-p keeps the shortest prefix of the blocks
 *               ordered by probability (descending; ties to the lower index)
 *               whose summed probability is >= topp; 0 disables Top-p.
 *   kv_idx, kv_cnt  outputs (see conventions). Each row keeps
 *               max(kc, pc, 1) blocks: the union of two prefixes of one order.
 *   row_thresh  optional output, float [B,H,Nqb]: probability of the last
 *               kept block of each row, rounded to float (NULL to skip).
 *   probs       optional output, float [B,H,Nqb,Nkb]: the pooled block
 *               probabilities rounded to float (NULL to skip).
 * Precision of the decision: double throughout (exact pooled sums, double
 * scores and softmax, running sums in 2^-62 fixed point), so the kept set is
 * the exact definition's except where two probabilities, or a running sum
 * and topp, agree to within a few double rounding units.
 * Workspace: sparge_workspace_bytes(SPARGE_OP_MASK, shape) (pooled Q and K
 * and the score rows, in double), 256-byte aligned.
 * Limits: Nkb <= 4096. */
sparge_status sparge_mask(const void* Q, const void* K, const sparge_shape* shape, double topk_frac,
                          double topp, int32_t* kv_idx, int32_t* kv_cnt, float* row_thresh, float* probs,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Block mask through a learnt router (SLA2 article, arXiv:2602.12675,
 * section 2: two learnable projections map the pooled query and key block
 * features before they are scored). Same steps and outputs as sparge_mask,
 * with one step added between pooling and scoring:
 *   q^_I = q-bar_I . Wq_h,   k^_J = k-bar_J . Wk_h       (h = head of the row)
 *   P[I, :] = softmax_J(q^_I . k^_J / sqrt(dr))
 *   Wq, Wk      fp32 [H, d, dr] row-major, device, 4-byte aligned, read only;
 *               the caller owns them (no copy is kept).
 *   dr          router width: 64 or 128 (else SPARGE_ERR_UNSUPPORTED).
 * Precision: the projections in double (the fp32 weights widened exactly);
 * the rest as in sparge_mask.
 * Workspace: sparge_workspace_bytes(SPARGE_OP_MASK_ROUTER, shape) (pooled
 * and projected blocks, probability rows), 256-byte aligned. */
sparge_status sparge_mask_router(const void* Q, const void* K, const sparge_shape* shape, const float* Wq,
                                 const float* Wk, int dr, double topk_frac, double topp, int32_t* kv_idx,
                                 int32_t* kv_cnt, float* row_thresh, float* probs, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* The same block mask as sparge_mask, for callers that cannot allocate
 * device memory: code hosted inside a framework or runtime that owns every
 * device allocation (a plug-in may not call cudaMalloc behind its host's
 * allocator), or code that must not risk an allocation failure or pay
 * allocation latency in the middle of its work. The articles have no
 * counterpart; this is an interface convenience, not part of the method.
 *
 * Arguments and results are those of sparge_mask; the caller still passes
 * Q, K and every output. The scratch (pooled Q and K and the score rows) is
 * a fixed 16 MiB array inside the library's device code, so nothing is
 * allocated: not by this call, not by the library, not through any
 * allocating library routine.
 *   - Limit: sparge_workspace_bytes(SPARGE_OP_MASK, shape) must not exceed
 *     16 MiB: 8*B*H*d*(Nqb + Nkb) + 8*B*H*Nqb*Nkb bytes, each part rounded
 *     up to 256 (for example B*H = 4 heads at N = 32760, d = 128, bq = 128,
 *     bk = 64 take 7.3 MB). Larger shapes return SPARGE_ERR_WORKSPACE before
 *     anything is launched.
 *   - The first call on a device looks up the array's device address on
 *     that device (cudaGetSymbolAddress, with the device current) and
 *     caches it; make that first call before any stream capture.
 *   - Every call, on any stream, uses the same array, and it keeps the last
 *     call's contents. Calls whose kernels overlap on the GPU race on it;
 *     order them (one stream, or events). Nothing in it needs to start at
 *     zero: each call overwrites what it reads.
 *   - Every device that loads the library holds the 16 MiB until exit. */
sparge_status sparge_mask_noalloc(const void* Q, const void* K, const sparge_shape* shape, double topk_frac,
                                  double topp, int32_t* kv_idx, int32_t* kv_cnt, float* row_thresh, float* probs,
                                  void* stream);

/* Block-sparse attention forward (SpargeAttention2 article, section 4).
 *   O[b,h,i] = sum over the keys j of the kept blocks of i's query block of
 *              softmax_j(q_i . k_j / sqrt(d)) v_j, in fp32, stored as bf16.
 *   lse         optional output, float [B,H,N]: natural-log log-sum-exp of the
 *               scaled scores over the kept keys; -inf where nothing is kept.
 * A row whose block keeps nothing gets O = 0.
 * Workspace: sparge_workspace_bytes(SPARGE_OP_ATTN, shape) (4 bytes per query
 * tile: the launch order of the tiles, heavier kept lists first within groups
 * of heads whose K and V fit in 64 MB of L2; the result does not depend on
 * it). Two launches (one when not even two heads fit: head-major order). */
sparge_status sparge_attn_fwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                              const int32_t* kv_idx, const int32_t* kv_cnt, void* O, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Block-sparse attention backward: gradients of sparge_attn_fwd for a loss L
 * with dL/dO = dO (SpargeAttention2 article, section 1: the sparse attention
 * is trainable; section 4: blocks computed whole or skipped whole, so the
 * gradients flow through the kept blocks only).
 *   D_i = dO_i . O_i,  P_ij = exp(q_i . k_j / sqrt(d) - lse_i),
 *   dS_ij = P_ij (dO_i . v_j - D_i) over the kept keys of i's block,
 *   dQ_i = sum_j dS_ij k_j / sqrt(d),  dK_j = sum_i dS_ij q_i / sqrt(d),
 *   dV_j = sum_i P_ij dO_i.
 *   O, lse      the forward's output and log-sum-exp (sparge_attn_fwd with
 *               lse requested) for the same Q, K, V and mask.
 *   dO          bf16 [B,H,N,d], device. dQ, dK, dV: bf16 [B,H,N,d] outputs;
 *               keys no query block keeps get dK = dV = 0, rows whose block
 *               keeps nothing get dQ = 0.
 * Precision: fp32 scores, P and dS rounded to bf16 as MMA operands, fp32
 * accumulation; D_i from the bf16 O and dO in fp32.
 * d must be 128 (else SPARGE_ERR_UNSUPPORTED), and Nqb * 32 bytes must not
 * exceed 200 KiB (the transposed-mask bit matrix of one CTA).
 * Workspace: sparge_workspace_bytes(SPARGE_OP_ATTN_BWD, shape) (D_i, for
 * every key block the ascending list of query blocks that keep it, and the
 * query tiles' launch order as in sparge_attn_fwd). */
sparge_status sparge_attn_bwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                              const int32_t* kv_idx, const int32_t* kv_cnt, const void* O, const float* lse,
                              const void* dO, void* dQ, void* dK, void* dV, void* workspace,
                              size_t workspace_bytes, void* stream);

/* SLA2 backward: gradients of sla2_attn_fwd for a loss L with dL/dO = dO
 * (SLA2 article, sections 1 and 2: O = alpha_h O_sparse + (1 - alpha_h) O_linear,
 * both branches and alpha trainable).
 *   sparse branch with alpha_h dO (as sparge_attn_bwd);
 *   linear branch, over the keys outside i's kept blocks, w_ij = phi(q_i).phi(k_j),
 *   den_i = sum_j w_ij, O_l,i = sum_j w_ij v_j / den_i, h_i = (1 - alpha_h) dO_i:
 *     dV_j += (w_ij / den_i) h_i,  dw_ij = h_i . (v_j - O_l,i) / den_i,
 *     dQ_i += (sum_j dw_ij phi(k_j)) * phi'(q_i),  dK_j += (sum_i dw_ij phi(q_i)) * phi'(k_j);
 *   dalpha_h = sum over the rows of head h (every batch) of dO_i . (O_s,i - O_l,i).
 *   alpha       float [H], device.  dO: bf16 [B,H,N,d].
 *   dQ, dK, dV  bf16 [B,H,N,d] outputs; dalpha float [H] output, device.
 * The call recomputes what it needs of the forward (the linear summaries,
 * O_linear and its denominators, the sparse branch and its log-sum-exp), so
 * it takes no forward outputs. Precision: as sparge_attn_bwd for the sparse
 * part; the linear part's products take bf16 operands (each query block's
 * complement S_c, each key tile's complement of G_all, phi(Q), c_i dO_i,
 * phi(K), V) with fp32 accumulation; row scalars in fp32.
 * d must be 128 and Nqb * 32 bytes must not exceed 200 KiB.
 * Workspace: sparge_workspace_bytes(SPARGE_OP_SLA2_BWD, shape). */
sparge_status sla2_attn_bwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                            const int32_t* kv_idx, const int32_t* kv_cnt, const float* alpha, const void* dO, void* dQ,
                            void* dK, void* dV, float* dalpha, void* workspace, size_t workspace_bytes, void* stream);

/* Low-bit block-sparse attention forward (SLA2 article, section 3: the
 * sparse branch computes with Q, K, the attention probabilities P and V in
 * a low-bit format, scaled into its range and back). Same mask and output
 * conventions as sparge_attn_fwd; d must be 128.
 * Formats and scales (the article fixes neither; these are this library's):
 *   Q, K  int8 codes, symmetric, one scale per (batch, head, block of bq / bk
 *         rows): s = 127 / max|x| (fp32), code = rint(x * s) clamped to +-127.
 *   V     fp8 e4m3 codes, one scale per (batch, head, channel): s = 448 / max|v|.
 *   S     exact int32 products of the codes; x = float(S) * c with
 *         c = (log2(e)/sqrt(d)) / (s_q * s_k) in fp32.
 *   P     e4m3 codes of e = 2^(x - (m - 8)), m = ceil of the row's max of x
 *         over its kept keys, so the row's largest code lies in (2^7, 2^8];
 *         the normaliser sums e. The kernel tracks the reference while it
 *         walks the key tiles (codes 2^(x - (m_run - 6)), m_run moved by an
 *         exact power-of-two rescale when the max passes it by more than 2),
 *         which changes only the codes of keys more than 12 binades below
 *         the row's max.
 *   O     = sum(P * v_codes) / (sum(e) * s_v), stored as bf16.
 * Workspace: sparge_workspace_bytes(SPARGE_OP_ATTN_Q8, shape) (codes and
 * scales, the tiles' launch order). Three or four launches: Q/K codes with V channel maxima,
 * V codes, the launch order of the query tiles (as sparge_attn_fwd), attention. */
sparge_status sparge_attn_fwd_q8(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, void* O, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Sparse + linear mix (SLA2 article, sections 1 and 2).
 *   O = alpha[h] * O_sparse + (1 - alpha[h]) * O_linear, with O_sparse as in
 *   sparge_attn_fwd and, over the keys j of the blocks NOT kept,
 *   O_linear[i] = sum_j (phi(q_i) . phi(k_j)) v_j / sum_j phi(q_i) . phi(k_j),
 *   phi(x) = elu(x) + 1; O_linear = 0 when every block is kept.
 *   alpha       float [H], device.
 * d must be 128. Workspace: sparge_workspace_bytes(SPARGE_OP_SLA2, shape).
 * Four or five launches: the launch order of the query tiles (as sparge_attn_fwd);
 * phi(K) and per-CTA partial sums of phi(K)^T [V | 1]; their fixed-order
 * reduction to the per-head totals; the linear branch of every
 * query block, written into O as (1 - alpha[h]) O_linear (bf16); the sparse
 * branch, which reads that tile back and adds alpha[h] O_sparse. O is
 * therefore also scratch between the last two launches. */
sparge_status sla2_attn_fwd(const void* Q, const void* K, const void* V, const sparge_shape* shape,
                            const int32_t* kv_idx, const int32_t* kv_cnt, const float* alpha, void* O,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Reads and clears the device error word after synchronising the stream.
 * *code receives 0 if no kernel gave up a wait since the last call, else the
 * site code of the first one. Returns SPARGE_ERR_DEVICE_TIMEOUT in that
 * case, SPARGE_ERR_CUDA if the synchronisation or the read fails. */
sparge_status sparge_device_status(void* stream, int32_t* code);

/* Self-test of the bounded device waits (the articles have no counterpart:
 * this checks the library's failure handling). Launches one small kernel that
 * allocates tensor memory, waits on a barrier that nothing arrives on through
 * the same bounded wait every kernel of the library uses, gives up after
 * limit_us microseconds (1 .. 1e6), frees its tensor memory and returns.
 * Afterwards sparge_device_status returns SPARGE_ERR_DEVICE_TIMEOUT with the
 * code SPARGE_SITE_SELFTEST, and the context stays usable.
 *   gave_up     optional device int32: 1 if every thread of the kernel gave
 *               up its wait, else 0 (NULL to skip). */
#define SPARGE_SITE_SELFTEST 0xF00
sparge_status sparge_selftest_wait(int32_t limit_us, int32_t* gave_up, void* stream);

/* Static, human-readable name of a status. */
const char* sparge_status_string(sparge_status status);

#ifdef __cplusplus
}
#endif

#endif /* SPARGE_H_ */
