/*
 * lighthouse.h -- C ABI of a B200 (sm_100a) library for the data-parallel hot
 * path of one Lighthouse Attention layer, forward and backward.
 *
 * The method, as two pages describe it:
 *   [ES] gist.science/es, "Resumen Técnico: Pre-entrenamiento con Contexto Largo
 *        mediante Atención Lighthouse", §2 Metodología (mirrored on gist.science/ja §2);
 *   [PT] bitsgeniais.com.br, "Adeus Custo Quadrático! Como a Lighthouse Attention
 *        Vai TURBINAR o Treinamento de LLMs!", section "A Grande Sacada: Lighthouse
 *        Attention em Quatro Fases!" (phases 1-4):
 *   (a) an L-level average-pooling pyramid over Q, K and V with pool factor p;
 *   (b) a parameter-free score per entry from the l2 norms of Q and K, coarse
 *       levels inheriting the max of their children;
 *   (c) one top-S selection across all levels;
 *   (d) a gather of the selected (Q, K, V) triplets into a dense,
 *       position-sorted sub-sequence of length S;
 *   (e) causal attention on that sub-sequence;
 *   (f) a deterministic scatter-back of its outputs to the original positions;
 *   and the backward through (f), (e) and (d) (no gradient through (c)).
 *
 * Notation, per unit u = (b, h): n_l = N / p^l, off_l = sum_{m<l} n_m,
 * M = off_L entries; entry (l, j) has gid = off_l + j, covers tokens
 * [j p^l, (j+1) p^l - 1] and is placed at pos = (j+1) p^l - 1.
 *
 * Readings of the pages fixed by this library (the pages leave them open):
 *   score      = ||Q[t]|| + ||K[t]|| at level 0 (fp32, one fixed summation
 *                order), coarse score = max over the p children;
 *   ranking    = score descending, ties to the lower level then lower index
 *                (lower gid), so the selected set is unique;
 *   order      = (pos ascending, level ascending): children before the parent
 *                that ends on the same token;
 *   attention  = causal on the slot index, scale 1/sqrt(d) unless given;
 *   scatter    = each token t gets the mean of the outputs of the selected
 *                entries covering it (its "contributors"), summed in ascending
 *                level; 0 when there is none.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless a parameter says otherwise, to
 *     contiguous row-major arrays with d innermost, 16-byte aligned.
 *   - Q, K, V, O, dO, dQ, dK, dV are [B, H, N, d] in the call's lh_dtype.
 *     The gathered sub-sequence (qs, ks, vs, os, dos) is fp16 (IEEE binary16)
 *     [B, H, S, d]: the tensor-core operands of the attention, 3 more mantissa
 *     bits than bf16.  Finite values beyond +-65504 are clipped to it and
 *     reported (LH_STATUS_FP16_SATURATED, lh_read_device_status).  Pyramid
 *     levels are fp32; gradients of the sub-sequence are fp32.
 *   - The caller allocates and frees every buffer; the library allocates no
 *     device memory and never synchronises the stream (except
 *     lh_read_device_status).  All work is enqueued on `stream` (NULL = the
 *     legacy default stream), in stream order: the stage kernels are
 *     programmatic dependent launches, each waiting at its start until the
 *     work before it on the stream has completed, so the GPU can stage a
 *     kernel while the previous one drains.
 *   - Arguments are checked on the host before any launch; a call that
 *     returns an error has enqueued nothing.  A launch failure returns
 *     LH_ERR_CUDA.  No call traps, asserts or exits.
 *   - Results are bitwise deterministic for identical inputs, shape and device.
 *   - Non-finite inputs give unspecified values, never a crash or a hang.
 *   - Shape limits: B, H >= 1; d in {64, 128}; 2 <= p; 1 <= L <= 8;
 *     N % p^(L-1) == 0; 1 <= S <= M; M < 2^31 and B*H*M < 2^40.
 */
#ifndef LIGHTHOUSE_H
#define LIGHTHOUSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lh_stream_t;

typedef enum {
  LH_OK = 0,
  LH_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, bad enum */
  LH_ERR_SHAPE = 2,         /* shape outside the limits above */
  LH_ERR_UNSUPPORTED = 3,   /* no kernel for this device or configuration */
  LH_ERR_WORKSPACE = 4,     /* workspace smaller than the *_bytes query */
  LH_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  LH_ERR_DEVICE_STATUS = 6  /* a kernel set a status bit (lh_read_device_status) */
} lh_status;

typedef enum { LH_F32 = 0, LH_BF16 = 1 } lh_dtype; /* dtype of Q,K,V,O,dO,dQ,dK,dV */

typedef struct {
  int64_t B, H, N;
  int32_t d, p, L, S;
} lh_shape;

/* Human-readable name of a status code (static string). */
const char* lh_status_string(lh_status s);

/* Host-only check of a shape and dtype against the limits above; no CUDA call. */
lh_status lh_validate(const lh_shape* shape, lh_dtype dtype);

/* Number of pyramid entries M per unit, or -1 for an invalid shape. */
int64_t lh_num_entries(const lh_shape* shape);

/* Bytes of caller workspace that lh_forward (with_backward = 0) or both
 * lh_forward and lh_backward (with_backward = 1) need; 0 for an invalid shape. */
size_t lh_workspace_bytes(const lh_shape* shape, lh_dtype dtype, int with_backward);

/* Bytes of the forward-to-backward state that lh_forward writes and
 * lh_backward reads: selection (idx, pos, slot), gathered qs/ks/vs, os, lse. */
size_t lh_saved_bytes(const lh_shape* shape);

/* Byte offsets inside the saved buffer, for callers that want to look at it:
 * which = 0 idx, 1 pos, 2 slot, 3 qs, 4 ks, 5 vs, 6 os, 7 lse, 8 inverse
 * contributor count (fp32 [B,H,N], 1/c_t or 0).  -1 for a bad argument. */
int64_t lh_saved_offset(const lh_shape* shape, int which);

/* ---------------------------------------------------------------- stages */

/* (a) Pyramid, [ES] §2.A / [PT] phase 1: for l = 1..L-1,
 *   X^(l)[j] = (sum_{i<p} X^(l-1)[p j + i]) / p  (fp32, children in order),
 * for X in {Q, K, V}.  q, k, v: [B,H,N,d] dtype.  pq, pk, pv: fp32
 * [B,H,M-N,d], levels 1..L-1 concatenated (level 0 is the input itself).    */
lh_status lh_build_pyramid(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                           const void* v, float* pq, float* pk, float* pv, lh_stream_t stream);

/* (a)+(b) in one pass over Q, K and V: the pyramid levels and all M scores,
 * exactly as the two calls above compute them (this is what lh_forward runs).
 * pq, pk, pv may be NULL when L == 1.                                        */
lh_status lh_build_pyramid_score(const lh_shape* shape, lh_dtype dtype, const void* q,
                                 const void* k, const void* v, float* pq, float* pk, float* pv,
                                 float* score, lh_stream_t stream);

/* (b) Score, [ES] §2.B / [PT] phase 2: score[t] = ||Q[t]||_2 + ||K[t]||_2 for
 * level 0 (fp32: eight-element fmaf chains, then a pairwise tree, IEEE sqrt),
 * and score^(l)[j] = max_{i<p} score^(l-1)[p j + i].  score: fp32 [B,H,M]. */
lh_status lh_score(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                   float* score, lh_stream_t stream);

/* (c) Joint top-S over all levels, [ES] §2.B: the S entries with the largest
 * (score, -gid), then ordered by (pos, level), [ES] §2.C.
 * idx, pos: int32 [B,H,S] (gid and position of slot k); slot: int32 [B,H,M]
 * (slot of each entry, -1 if not selected).  Scores must be >= 0 (they are
 * sums of norms).  Two implementations, the same bits: with ws = NULL one
 * thread-block cluster per unit keeps all its state in distributed shared
 * memory; with a workspace of lh_topk_workspace_bytes() (16-byte aligned,
 * owned by the caller, overwritten) the selection runs as device-wide passes
 * over every SM (what lh_forward uses); a smaller one is LH_ERR_WORKSPACE.   */
size_t lh_topk_workspace_bytes(const lh_shape* shape);
lh_status lh_topk_select(const lh_shape* shape, const float* score, int32_t* idx, int32_t* pos,
                         int32_t* slot, void* ws, size_t ws_bytes, lh_stream_t stream);

/* (d) Gather, [ES] §2.C: xs[k] = fp16_rne(X^(l_k)[j_k]) (saturating), level 0
 * read from the input, coarser levels from the pyramid.  qs, ks, vs: fp16
 * [B,H,S,d].                                                                 */
lh_status lh_gather(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                    const void* v, const float* pq, const float* pk, const float* pv,
                    const int32_t* idx, void* qs, void* ks, void* vs, lh_stream_t stream);

/* (a)+(d) for the selected entries only: the same rows as lh_gather on a
 * pyramid from lh_build_pyramid (bit for bit: a coarse row is pooled from its
 * span of level-0 rows with the pyramid's own order of fp32 additions and
 * divisions), but no pyramid level is written; only the rows of selected spans
 * are read: cheaper than the pyramid when the selected spans are few, dearer
 * when they cover most of the sequence.                                     */
lh_status lh_gather_pooled(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                           const void* v, const int32_t* idx, void* qs, void* ks, void* vs,
                           lh_stream_t stream);

/* (e) Causal attention on the sub-sequence, [ES] §2.C (stock SDPA on a dense
 * sequence): os[k] = sum_{k'<=k} softmax_k'(scale <qs[k], ks[k']>) vs[k'],
 * lse[k] = natural log of the softmax denominator (with the max folded in).
 * scale <= 0 selects 1/sqrt(d).  qs, ks, vs, os: fp16 [B,H,S,d]; lse: fp32
 * [B,H,S].  Products run on the tensor cores in fp16 with fp32 accumulation;
 * the softmax weights P are rounded to fp16 before the product with vs.     */
lh_status lh_subseq_attn_fwd(const lh_shape* shape, const void* qs, const void* ks,
                             const void* vs, float scale, void* os, float* lse,
                             lh_stream_t stream);

/* (e') Backward of (e): textbook softmax adjoint, D = rowsum(dos * os),
 * dS = P * (dos vs^T - D); dqs = scale dS ks, dks = scale dS^T qs,
 * dvs = P^T dos.  dqs, dks, dvs: fp32 [B,H,S,d].  ws: lh_attn_bwd_workspace_bytes. */
size_t lh_attn_bwd_workspace_bytes(const lh_shape* shape);
lh_status lh_subseq_attn_bwd(const lh_shape* shape, const void* qs, const void* ks,
                             const void* vs, const void* os, const float* lse, const void* dos,
                             float scale, float* dqs, float* dks, float* dvs, void* ws,
                             size_t ws_bytes, lh_stream_t stream);

/* (e'') The same backward as lh_subseq_attn_bwd, for callers that cannot
 * allocate device memory or hand over a workspace -- for example code that runs
 * under a memory planner which has already reserved every byte of the GPU, or
 * a runtime where calling cudaMalloc mid-step is not allowed because it can
 * synchronise the device.  The paper has no counterpart: this is a library
 * convenience, not part of the method.  It allocates nothing: its scratch (two
 * fp32 per row, the softmax statistics, rows padded to whole 128-row tiles) is
 * a fixed 8 MiB array inside the library that every GPU loading the library
 * holds until the process exits.
 *   - At most 1,048,576 padded rows (B * H * ceil(S / 128) * 128); larger
 *     shapes return LH_ERR_WORKSPACE before anything is enqueued.
 *   - All calls on one device share that array: calls whose kernels overlap on
 *     the GPU (unordered streams) race; calls ordered on one stream are safe.
 *   - The first call in each CUDA context of a device (normally one per
 *     device, and a new one after cudaDeviceReset) looks up the array's device
 *     address and caches it under that context's id; make that first call
 *     before any stream capture.
 *   - It runs the same kernels as lh_subseq_attn_bwd: the results are bitwise
 *     equal to that call's.
 * Arguments and results as for lh_subseq_attn_bwd, without ws / ws_bytes.  */
lh_status lh_subseq_attn_bwd_noalloc(const lh_shape* shape, const void* qs, const void* ks,
                                     const void* vs, const void* os, const float* lse,
                                     const void* dos, float scale, float* dqs, float* dks,
                                     float* dvs, lh_stream_t stream);

/* (f) Scatter-back, [ES] §2.C / [PT] phase 4: c_t = number of selected
 * entries covering t; O[t] = (sum over them, ascending level, of os[slot]) / c_t,
 * 0 when c_t = 0.  o: [B,H,N,d] dtype.  inv_count (optional, may be NULL):
 * fp32 [B,H,N] receives 1/c_t (0 when c_t = 0).                              */
lh_status lh_scatter_back(const lh_shape* shape, lh_dtype dtype, const void* os,
                          const int32_t* slot, void* o, float* inv_count, lh_stream_t stream);

/* (f') Adjoint of (f): dos[k] = sum_{t in span(k)} dO[t] / c_t.  dos: fp16
 * [B,H,S,d].  inv_count may be NULL (then c_t is recounted from slot).     */
lh_status lh_scatter_back_bwd(const lh_shape* shape, lh_dtype dtype, const void* dO,
                              const int32_t* slot, const float* inv_count, void* dos,
                              lh_stream_t stream);

/* (d') Adjoint of (a)+(d): dX[t] = sum_{l ascending, selected} dxs[slot_l(t)] / p^l
 * with slot_l(t) = slot[off_l + t / p^l], for X in {Q, K, V}.  dqs, dks, dvs:
 * fp32 [B,H,S,d]; dq, dk, dv: [B,H,N,d] dtype.                               */
lh_status lh_gather_bwd(const lh_shape* shape, lh_dtype dtype, const float* dqs,
                        const float* dks, const float* dvs, const int32_t* slot, void* dq,
                        void* dk, void* dv, lh_stream_t stream);

/* ------------------------------------------------------- fused entry points */

/* Whole forward: (a)+(b) in one pass, (c), (d), (e), (f).  o: [B,H,N,d] dtype.
 * saved: lh_saved_bytes, kept by the caller for lh_backward.
 * ws: lh_workspace_bytes(shape, dtype, 0 or 1). */
lh_status lh_forward(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                     const void* v, float scale, void* o, void* saved, void* ws,
                     size_t ws_bytes, lh_stream_t stream);

/* How lh_forward gathers the sub-sequence for this shape: 0 through the fp32
 * pyramid levels (lh_build_pyramid_score + lh_gather), 1 pooled from the input
 * rows of each selected span (lh_score + lh_gather_pooled, no level written:
 * chosen when even S entries all at the coarsest level read fewer bytes, with a
 * margin of 4, than the levels take to write); -1 for an invalid shape or
 * dtype.  Both give the same bits.  Host-only. */
int lh_forward_gather_path(const lh_shape* shape, lh_dtype dtype);

/* How lh_forward runs the selection for this shape: 0 one thread-block cluster
 * per unit (lh_topk_select without a workspace), 1 device-wide passes (with
 * one; every valid shape at present); -1 for an invalid shape.  Both give the
 * same bits.  Host-only. */
int lh_forward_topk_path(const lh_shape* shape);

/* Whole backward with the saved selection: (f'), (e'), (d').  dO: [B,H,N,d]
 * dtype; dq, dk, dv: [B,H,N,d] dtype.  ws: lh_workspace_bytes(shape, dtype, 1). */
lh_status lh_backward(const lh_shape* shape, lh_dtype dtype, const void* saved, const void* dO,
                      float scale, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                      lh_stream_t stream);

/* ---------------------------------------------------- context parallelism
 * [PT] bitsgeniais.com.br, section "Escalando para o Céu (ou 1 Milhão de
 * Tokens!): Paralelismo de Contexto": the sequence is split into P contiguous
 * shards, one per GPU.  Each GPU runs the pyramid, the scores, the selection,
 * the gather and the scatter-back on its own shard with no communication (the
 * stage calls above, with the shard's N and S/P); the dense sub-sequence -- the
 * shards' sub-sequences in shard order, which is (pos, level) order again --
 * is attended with standard ring attention.  The calls below are one GPU's
 * steps of that ring (long_context_lh_b200/cp.py drives it over NCCL).  A
 * block has shape->S rows; shape->N must equal shape->S (p and L are only
 * validated: pass p = 2, L = 1).  Blocks are fp16 [B,H,S,d] like qs/ks/vs.  */

/* Attention of a query block against one key block of the same length.
 * causal = 1: the diagonal block (row k sees keys k' <= k, as
 * lh_subseq_attn_fwd); causal = 0: an earlier block, every key (rows and keys
 * past S excluded).  os: fp16 [B,H,S,d], the normalised block output; lse: fp32
 * [B,H,S].  causal = 0 needs the tcgen05 kernels (LH_ERR_UNSUPPORTED otherwise). */
lh_status lh_block_attn_fwd(const lh_shape* shape, int causal, const void* qs, const void* ks,
                            const void* vs, float scale, void* os, float* lse, lh_stream_t stream);

/* Online merge of a block result into the running one, `rows` rows of d in
 * {64, 128}: first = 1 copies (o_part, lse_part) into (o_acc, lse_acc);
 * otherwise both become the softmax-weighted combination, weights
 * exp(lse - lse_new), lse_new = log(exp(lse_acc) + exp(lse_part)).  o_acc,
 * lse_acc fp32; o_part fp16; lse_part fp32.  Merging the blocks in a fixed
 * order makes the result deterministic. */
lh_status lh_block_attn_merge(int64_t rows, int32_t d, float* o_acc, float* lse_acc,
                              const void* o_part, const float* lse_part, int first,
                              lh_stream_t stream);

/* os (fp16) = o_acc (fp32) rounded to nearest, `rows` rows of d. */
lh_status lh_block_attn_finish(int64_t rows, int32_t d, const float* o_acc, void* os,
                               lh_stream_t stream);

/* Backward of one (query block, key block) pair, given the query block's final
 * os, lse (after every merge) and dos: the pair's gradients dqs (for the query
 * rows) and dks, dvs (for the key rows), fp32 [B,H,S,d], overwritten.
 * causal as in lh_block_attn_fwd.  ws: lh_attn_bwd_workspace_bytes(shape). */
lh_status lh_block_attn_bwd(const lh_shape* shape, int causal, const void* qs, const void* ks,
                            const void* vs, const void* os, const float* lse, const void* dos,
                            float scale, float* dqs, float* dks, float* dvs, void* ws,
                            size_t ws_bytes, lh_stream_t stream);

/* acc[i] += x[i] for n fp32 values (n a multiple of 4): one fp32 add per
 * element, so gradients summed in a fixed order of calls are deterministic. */
lh_status lh_accumulate(int64_t n, float* acc, const float* x, lh_stream_t stream);

/* Reads and clears the device status words (synchronises `stream`).  LH_OK or
 * LH_ERR_DEVICE_STATUS; *code (may be NULL) receives the OR of the words, 0
 * for none, else LH_STATUS_* bits:
 *   LH_STATUS_ATTN_FWD_TIMEOUT / LH_STATUS_ATTN_BWD_TIMEOUT: a bounded wait in
 *     an attention kernel gave up (the low bits say which); that call's
 *     outputs are incomplete;
 *   LH_STATUS_FP16_SATURATED: a finite value written into the fp16 sub-sequence
 *     (qs, ks, vs by the gather; dos by the scatter-back adjoint) lay beyond
 *     +-65504 and was clipped to it.  The selection is unaffected (it is
 *     computed in fp32 from the inputs); the attention then ran on the clipped
 *     rows.  Inputs whose pooled rows stay within +-65504 never set it;
 *   LH_STATUS_BOUNDS (liblighthouse_debug.so only, the same library built with
 *     -DLH_DEBUG=1): an index computed in a kernel from data (idx, pos, slot)
 *     or from unit, tile or level coordinates fell outside its array; the
 *     access was skipped.  Bits 16-24 name the kernel: pyramid, selection,
 *     gather, scatter-back, its adjoint, gather adjoint, attention forward,
 *     attention backward, softmax statistics. */
#define LH_STATUS_ATTN_FWD_TIMEOUT 0x100u
#define LH_STATUS_ATTN_BWD_TIMEOUT 0x200u
#define LH_STATUS_FP16_SATURATED 0x400u
#define LH_STATUS_BOUNDS 0x800u
lh_status lh_read_device_status(lh_stream_t stream, uint32_t* code);

/* Selects the attention implementation for subsequent calls on this process:
 * 0 = tcgen05/TMEM (default on sm_100), 1 = warp-level mma.sync kernels (kept
 * as the comparison baseline).  Returns the previous value. */
int lh_set_attention_impl(int impl);

/* The attention implementations the next calls would use: 0 tcgen05 for the
 * forward and the backward, 1 mma.sync for both, 2 tcgen05 forward with the
 * mma.sync backward. */
int lh_attention_impl_in_use(void);

/* Number of kernel launches lh_forward (backward = 0) or lh_backward
 * (backward = 1) enqueues for this shape and input dtype with the current
 * implementation; -1 for an invalid shape or dtype. */
int lh_kernel_launches(const lh_shape* shape, lh_dtype dtype, int backward);

/* -------------------------------------------------------------- variants */

/* How the two level-0 norms of an entry combine into its score.  The pages fix
 * that each entry is scored, without parameters, by the l2 norms of its
 * projected Q and K vectors ([ES] §2.B; [PT] phase 2: two scores per entry),
 * not how the two combine: the sum is the default reading, the product and the
 * norm of the concatenation are ablations of that reading.  All in fp32 from the
 * two squared norms ss(q), ss(k) of lh_score:
 *   SUM     sqrt(ss(q)) + sqrt(ss(k))
 *   PRODUCT sqrt(ss(q)) * sqrt(ss(k))
 *   CONCAT  sqrt(ss(q) + ss(k))        (IEEE sqrt, one rounding per operation) */
typedef enum { LH_SCORE_SUM = 0, LH_SCORE_PRODUCT = 1, LH_SCORE_CONCAT = 2 } lh_score_mode;

/* How a selected entry's output spreads back over the original positions.  The
 * pages fix a deterministic scatter-back to a fully dense output with "at least
 * one contributor" per position ([ES] §2.C; [PT] phases 1 and 4), not the
 * weights: the mean over the contributors covering a token is the default
 * reading; the ablations are
 *   SUM   the contributors' outputs added, no division;
 *   LAST  an entry reaches only the last token of its span (its position), the
 *         strictly causal reading of "the output does not see the future"; a
 *         token takes the mean of what reaches it.
 * inv_count (lh_scatter_back) then holds each token's weight in the adjoint:
 * 1/c_t (MEAN, LAST), 1 (SUM), 0 where nothing reaches the token.             */
typedef enum { LH_SCATTER_MEAN = 0, LH_SCATTER_SUM = 1, LH_SCATTER_LAST = 2 } lh_scatter_mode;

/* Variants of the layer.  A NULL pointer, or all fields 0, is the default layer
 * the entry points above compute.
 *   keep_coarsest: 1 = every entry of the coarsest level L-1 is selected, which
 *     gives every original position at least one contributor ([PT] phase 1);
 *     the coarsest entries rank above every score (key bits of +inf; among
 *     themselves by gid), the other S - N/p^(L-1) slots go to the largest keys
 *     as usual.  Needs N / p^(L-1) <= S, else LH_ERR_SHAPE.
 *   score_mode: an lh_score_mode.
 *   scatter_mode: an lh_scatter_mode (the backward must be given the same).
 *   reserved: must be 0 (LH_ERR_INVALID_ARG otherwise).                      */
typedef struct {
  int32_t keep_coarsest;
  int32_t score_mode;
  int32_t scatter_mode;
  int32_t reserved;
} lh_options;

/* Host-only check of a shape and options (NULL allowed); no CUDA call. */
lh_status lh_validate_options(const lh_shape* shape, const lh_options* opt);

/* The stage and fused calls that the options change, with the options; the
 * calls without _ex above are these with opt = NULL.  The backward reads the
 * selection that lh_forward_ex saved; of the options only scatter_mode changes
 * it, so lh_backward_ex must get the options lh_forward_ex got.              */
lh_status lh_build_pyramid_score_ex(const lh_shape* shape, lh_dtype dtype, const void* q,
                                    const void* k, const void* v, float* pq, float* pk, float* pv,
                                    float* score, const lh_options* opt, lh_stream_t stream);
lh_status lh_score_ex(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                      float* score, const lh_options* opt, lh_stream_t stream);
lh_status lh_topk_select_ex(const lh_shape* shape, const float* score, int32_t* idx,
                            int32_t* pos, int32_t* slot, void* ws, size_t ws_bytes,
                            const lh_options* opt, lh_stream_t stream);
lh_status lh_forward_ex(const lh_shape* shape, lh_dtype dtype, const void* q, const void* k,
                        const void* v, float scale, void* o, void* saved, void* ws,
                        size_t ws_bytes, const lh_options* opt, lh_stream_t stream);
lh_status lh_scatter_back_ex(const lh_shape* shape, lh_dtype dtype, const void* os,
                             const int32_t* slot, void* o, float* inv_count, const lh_options* opt,
                             lh_stream_t stream);
lh_status lh_scatter_back_bwd_ex(const lh_shape* shape, lh_dtype dtype, const void* dO,
                                 const int32_t* slot, const float* inv_count, void* dos,
                                 const lh_options* opt, lh_stream_t stream);
lh_status lh_backward_ex(const lh_shape* shape, lh_dtype dtype, const void* saved, const void* dO,
                         float scale, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                         const lh_options* opt, lh_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* LIGHTHOUSE_H */
