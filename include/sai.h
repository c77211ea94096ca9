/*
 * libsai: DeepSeek-V4 CSA lightning-indexer distillation loss on NVIDIA B200
 * (sm_100a). C ABI.
 *
 * The loss is split in three calls, as on the Primus page "perf(deepseek-v4):
 * fuse and enable the indexer distillation loss" (file table:
 * indexer_distill_window_lse, indexer_distill_target, indexer_distill_kl):
 *
 *   sai_window_lse      Q, Kw            -> window_lse [B,S,H]
 *   sai_distill_target  Q, pool, idx, window_lse, sink -> p [B,S,K]
 *   sai_distill_kl      p, scores, valid -> loss (device scalar), dscores [B,S,K]
 *
 * Around them: sai_distill_target_ex (the per-branch target, or the target
 * from the attention forward's own LSE), sai_distill_target_ws (the target
 * with a spill workspace, so long selections are gathered and multiplied
 * once), sai_distill_target_window (window and target in one kernel, Q read
 * once), sai_distill_target_kl (target and
 * KL in one call), sai_distill_kl_noalloc (no workspace argument),
 * sai_indexer_topk, the block selection that produces idx, scores and valid
 * from the indexer's scores, and the calls for splitting sequences across
 * GPUs by token range: sai_window_lse_range, sai_distill_target_range,
 * sai_distill_target_window_range, sai_count_valid_rows and
 * sai_distill_kl_ex (a batch-wide N).
 *
 * Conventions for every call
 *   - Tensor arguments are DEVICE pointers to dense row-major (C-contiguous)
 *     arrays, owned by the caller. The library never allocates device memory
 *     and never synchronises the stream.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All work
 *     is enqueued on it; results are ready when the stream reaches that point.
 *   - Host-detectable errors (NULL pointers, bad sizes, unsupported shapes,
 *     misaligned pointers, a short workspace) return an error status before
 *     anything is enqueued. A failed launch returns SAI_ERR_CUDA.
 *   - Outputs are fully overwritten; masked slots are written as exact 0.
 *   - There is no fallback to another implementation: a shape the kernels do
 *     not cover returns SAI_ERR_UNSUPPORTED.
 *   - Calls on the same stream are ordered; calls on different streams that
 *     share output buffers race.
 */
#ifndef SAI_H
#define SAI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sai_status {
    SAI_OK = 0,
    SAI_ERR_NULL = 1,        /* a required pointer is NULL                          */
    SAI_ERR_SHAPE = 2,       /* a size is non-positive or sizes are inconsistent     */
    SAI_ERR_UNSUPPORTED = 3, /* the shape is outside what the kernels cover          */
    SAI_ERR_CUDA = 4,        /* a CUDA runtime/driver call or a launch failed        */
    SAI_ERR_INDEX = 5,       /* device error word: an idx entry outside {-1}U[0,P)   */
    SAI_ERR_WORKSPACE = 6,   /* workspace NULL, too small or not 16-byte aligned     */
    SAI_ERR_ALIGN = 7,       /* a tensor pointer is misaligned for its call (16 B for
                                bf16 matrices and 16-byte-vector arrays, else 4 B)   */
    SAI_ERR_TIMEOUT = 8      /* device error word: a kernel gave up a bounded wait   */
} sai_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *sai_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int sai_version(void);

/*
 * sai_window_lse -- sliding-window log-mass per (token, head).
 *
 * Source: Primus page, second commit message (the joint target needs each
 * head's log-mass over its window keys; indexer_distill_window_lse computes it
 * without writing the window logits to memory, reading for each block of
 * queries only the keys that block can see).
 *
 *   window_lse[b,t,h] = log sum_{s=lo}^{t} exp(scale * <Q[b,t,h,:], Kw[b,s,:]>)
 *   lo = max(d0, t - W + 1),  d0 = clamp(doc_start[b,t], 0, t) or 0 if NULL.
 *
 * The window holds W single-latent keys (one Kw row per token, shared by all
 * heads) ending at the token itself and clipped at its document start. The
 * per-head sink is not included (sai_distill_target adds it).
 *
 *   Q          [B,S,H,D] bf16, 16-byte aligned
 *   Kw         [B,S,D]   bf16, 16-byte aligned
 *   doc_start  [B,S] int32 or NULL (one document per row)
 *   scale      logit scale > 0, e.g. 1/sqrt(D)
 *   window_lse [B,S,H] fp32, written, 4-byte aligned
 *
 * Sizes: B,S,H,D,W >= 1 and D % 8 == 0. Errors: SAI_ERR_NULL, SAI_ERR_SHAPE,
 * SAI_ERR_ALIGN, SAI_ERR_UNSUPPORTED, SAI_ERR_CUDA.
 */
sai_status sai_window_lse(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start,
                          int B, int S, int H, int D, int W, float scale,
                          float *window_lse, void *stream);

/*
 * sai_window_lse_range -- sai_window_lse over a token range of longer sequences.
 *
 * For splitting each sequence across GPUs by token range (the MaxText page
 * "Add Indexer Loss [Deepseek v4]" speaks of context parallelism only in its
 * configuration checks; the arithmetic is exactly sai_window_lse's). The call
 * covers sequence positions t_begin .. t_begin+S-1 of every sequence:
 *
 *   window_lse[b,i,h] = log sum_{s=lo}^{t} exp(scale * <Q[b,i,h,:], Kw[b, s - t_begin + kw_lead, :]>)
 *   t = t_begin + i,  lo = max(d0, t - W + 1),  d0 = clamp(doc_start[b,i], 0, t)
 *
 *   Q          [B,S,H,D] bf16: the range's own query rows
 *   Kw         [B,S+kw_lead,D] bf16: the keys of positions
 *              t_begin-kw_lead .. t_begin+S-1 (the range plus its halo)
 *   doc_start  [B,S] int32 sequence positions, or NULL
 *   t_begin    >= 0; kw_lead in [min(W-1, t_begin), t_begin] (the halo must
 *              hold every key the range's first window reaches)
 *
 * sai_window_lse is this call with t_begin = kw_lead = 0. Errors as for
 * sai_window_lse (SAI_ERR_SHAPE for a short halo).
 */
sai_status sai_window_lse_range(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start,
                                int B, int S, int H, int D, int W, int t_begin, int kw_lead, float scale,
                                float *window_lse, void *stream);

/*
 * sai_distill_target -- the indexer's teacher target p[b,t,:].
 *
 * Source: Primus page, first commit message (indexer_distill_target reads
 * pool rows by index inside the kernel, so no gathered copy is written, and
 * keeps the softmax and the sum over heads on chip) and second commit message
 * / "Why the target was wrong" (each head normalises jointly over window keys,
 * chosen pool rows and its sink; the pool rows' share of head h is
 * exp(clse - lse_full); the L1 floor is the smallest normal float32).
 * Causal block rule: MaxText page "Add Indexer Loss [Deepseek v4]", commit
 * messages (block j is visible to token t iff (j+1)*cr - 1 <= t;
 * cross-document blocks masked).
 *
 *   slot k selected iff 0 <= idx[b,t,k] < P (P = S/cr), (idx+1)*cr - 1 <= t
 *                       and idx*cr >= d0 (d0 as in sai_window_lse)
 *   z[h,k]      = scale * <Q[b,t,h,:], pool[b,idx[b,t,k],:]>
 *   clse[h]     = log sum_{selected k} exp z[h,k]
 *   lse_full[h] = logsumexp(window_lse[b,t,h], clse[h], sink[h])
 *   u[k]        = sum_h exp(z[h,k] - lse_full[h]);   m = sum_k u[k]
 *   p[b,t,k]    = u[k] / max(m, FLT_MIN) on selected slots, 0 elsewhere
 *
 *   Q          [B,S,H,D] bf16, 16-byte aligned
 *   pool       [B,P,D]   bf16 compressed entries, 16-byte aligned
 *   idx        [B,S,K]   int32 top-k rows, -1 = empty slot; or NULL for the
 *              dense warm-up stage (MaxText page "Add Indexer Loss
 *              [Deepseek v4]": teacher over all causal blocks before sparse
 *              training), where slot k is compressed block k (idx[b,t,k] = k
 *              implicitly; with K = S/cr every block; the causal and document
 *              rules still mask the slots a token cannot see)
 *   window_lse [B,S,H]   fp32 (from sai_window_lse)
 *   sink       [H] fp32 per-head sink logits, or NULL for no sink
 *   doc_start  [B,S] int32 or NULL
 *   p          [B,S,K] fp32, written
 *   d_err      device int32 or NULL. Data errors found on the device (an idx
 *              entry outside {-1} U [0,P)) mask the slot and store
 *              SAI_ERR_INDEX here; the caller zeroes it and reads it back.
 *   The 32-bit arrays (idx, window_lse, sink, doc_start, p, d_err) must be
 *   4-byte aligned.
 *
 * Sizes: S % cr == 0, 1 <= K <= S/cr (the MaxText page's topk <= length/4
 * check), D % 8 == 0, scale > 0. Errors: SAI_ERR_NULL, SAI_ERR_SHAPE, SAI_ERR_ALIGN,
 * SAI_ERR_UNSUPPORTED, SAI_ERR_CUDA.
 */
sai_status sai_distill_target(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                              const float *window_lse, const float *sink, const int32_t *doc_start,
                              int B, int S, int H, int D, int K, int cr, float scale,
                              float *p, int32_t *d_err, void *stream);

/* Flags of sai_distill_target_ex (at most one of the two). */
#define SAI_TARGET_PER_BRANCH 1u
#define SAI_TARGET_FULL_LSE 2u

/*
 * sai_distill_target_ex -- sai_distill_target with a flags word.
 *
 * flags == 0 is exactly sai_distill_target. SAI_TARGET_PER_BRANCH selects
 * the earlier per-branch target, which the Primus page keeps as an A/B
 * switch (second commit message: PRIMUS_V4_DISTILL_NONCOMP_LSE=0) and the
 * MaxText page "Add Indexer Loss [Deepseek v4]" prints in its commit
 * messages: every head is normalised over the selected compressed entries
 * alone and the L1 floor is the earlier 1e-10,
 *
 *   lse_full[h] = clse[h],   p[b,t,k] = u[k] / max(m, 1e-10),
 *
 * i.e. p is the head mean of the per-head softmaxes over the selected slots.
 * window_lse and sink are not read in that mode and may be NULL.
 *
 * SAI_TARGET_FULL_LSE: window_lse [B,S,H] fp32 holds lse_full itself, each
 * head's natural-log normaliser over the whole attention row (window keys,
 * selected compressed entries and sink), as a CSA attention forward that
 * returns its LSE has computed it (Primus page "perf(deepseek-v4): fuse and
 * enable the indexer distillation loss", first commit message: the
 * compressed share of a head is exp(compressed_lse - full_lse); Primus page
 * "Docker Build for DeepSeek-v4", gluon_v3 "Optimization Notes": the CSA
 * forward route returns its LSE). Then
 *
 *   u[k] = sum_h exp(z[h,k] - window_lse[b,t,h]),  p[b,t,k] = u[k] / max(m, FLT_MIN),
 *
 * no window pass is needed, and sink is not read (it is inside the LSE).
 *
 * Unknown flag bits, or both flags at once, return SAI_ERR_UNSUPPORTED;
 * everything else (layouts, sizes, errors, ownership) is as for
 * sai_distill_target.
 */
sai_status sai_distill_target_ex(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start,
                                 int B, int S, int H, int D, int K, int cr, float scale, unsigned flags,
                                 float *p, int32_t *d_err, void *stream);

/*
 * sai_distill_target_range -- sai_distill_target_ex over a token range.
 *
 * The S tokens of each sequence passed here are positions t_begin ..
 * t_begin+S-1 of sequences of S_seq tokens (for splitting a sequence across
 * GPUs, as sai_window_lse_range). Positions, not row numbers, decide the
 * causal and document rules, and the pool is the whole sequence's:
 *
 *   Q          [B,S,H,D] bf16: the range's own query rows
 *   pool       [B,S_seq/cr,D] bf16: every compressed entry of the sequence
 *   idx, window_lse, doc_start, p: [B,S,...] rows of the range; idx holds
 *              pool row numbers, doc_start sequence positions
 *   slot k of local token i selected iff 0 <= idx < S_seq/cr,
 *              (idx+1)*cr - 1 <= t_begin + i and idx*cr >= d0
 *
 * Sizes: S_seq % cr == 0, 0 <= t_begin, t_begin + S <= S_seq,
 * 1 <= K <= S_seq/cr. sai_distill_target_ex is this call with S_seq = S and
 * t_begin = 0. Flags, errors and ownership as for sai_distill_target_ex.
 */
sai_status sai_distill_target_range(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                    const float *window_lse, const float *sink, const int32_t *doc_start,
                                    int B, int S, int S_seq, int t_begin, int H, int D, int K, int cr,
                                    float scale, unsigned flags, float *p, int32_t *d_err, void *stream);

/*
 * sai_distill_target_workspace_bytes / sai_distill_target_ws -- the target
 * with a spill workspace for long selections.
 *
 * The tensor-core kernel keeps a token's scores in tensor memory, at most
 * 256/H tiles of 128 slots at a time (K <= 512 at H = 64). A token with more
 * selected slots is taken in groups: the per-head log-sum-exp needs every
 * group before any u can be formed (Primus page "perf(deepseek-v4): fuse and
 * enable the indexer distillation loss", second commit message: the target
 * normalises each head over the whole row). Without a workspace the groups
 * are gathered and multiplied a second time for u. With one, the first sweep
 * also stores each group's raw fp32 scores there, and u is formed from them:
 * every pool row is gathered and every product formed once.
 *
 *   sai_distill_target_workspace_bytes(B, S, H, D, K): bytes needed on the
 *     current device (one part per CTA of the kernel: groups x 256/H tiles x
 *     H x 128 floats); 0 when no token can need a second group (K <= 256/H
 *     tiles, H < 64, or a shape the tensor-core kernel does not take).
 *   sai_distill_target_ws(...): sai_distill_target_range plus the workspace.
 *     workspace: device memory, 16-byte aligned, owned by the caller, read
 *     and written by the kernel, no contents required or kept between calls;
 *     calls that overlap on the GPU must not share it. With it the last
 *     group's scores also stay in tensor memory for their u pass. NULL, or
 *     ws_bytes below the size above: the second sweep is used; the results
 *     agree up to float32 rounding (the order and form of the exponentials
 *     differ). Errors as for sai_distill_target_range, and SAI_ERR_ALIGN for
 *     a misaligned workspace.
 */
size_t sai_distill_target_workspace_bytes(int B, int S, int H, int D, int K);
sai_status sai_distill_target_ws(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start,
                                 int B, int S, int S_seq, int t_begin, int H, int D, int K, int cr, float scale,
                                 unsigned flags, float *p, int32_t *d_err, void *workspace, size_t ws_bytes,
                                 void *stream);

/*
 * sai_distill_target_window -- sai_window_lse and sai_distill_target in one
 * kernel, so Q is read from device memory once.
 *
 * The pages' V4 CSA attention treats each token's keys as one list, the 128
 * window entries followed by the pool's top-k entries (Primus page "Docker
 * Build for DeepSeek-v4", gluon_v3 commit, "Optimization Notes" / Forward).
 * Here the window band is one more 128-row operand tile of the target's
 * tensor-core contraction: its rows are the Kw rows of positions t-127 .. t,
 * its product with Q[b,t] gives the window logits, and each head's
 * log-sum-exp over the rows in [lo, t] takes the place of the window_lse
 * input. The result is what sai_window_lse followed by sai_distill_target
 * computes (the joint target, Primus page "perf(deepseek-v4): fuse and
 * enable the indexer distillation loss", second commit message):
 *
 *   window_lse[b,t,h] = log sum_{s=lo}^{t} exp(scale * <Q[b,t,h,:], Kw[b,s,:]>),
 *   lo = max(d0, t - W + 1), d0 = clamp(doc_start[b,t], 0, t) or 0;
 *   p[b,t,:] as sai_distill_target with that window_lse.
 *
 *   Q, pool, idx, sink, doc_start, scale, p, d_err: as sai_distill_target
 *   Kw          [B,S,D] bf16, 16-byte aligned
 *   W           window length, 1 <= W <= 128 (the band is one 128-row tile;
 *               a longer window returns SAI_ERR_UNSUPPORTED)
 *   window_lse  [B,S,H] fp32, 4-byte aligned: the window log-mass written
 *               out, or NULL (not written)
 *   workspace   as sai_distill_target_ws: the raw-score spill for tokens of
 *               more than one TMEM group, or NULL (second sweep)
 *
 * Only the tensor-core target kernel does this (H in {16,32,64,128},
 * D % 64 == 0): other shapes return SAI_ERR_UNSUPPORTED, with no fallback;
 * the three-call route covers them. Errors otherwise as sai_distill_target_ws
 * and sai_window_lse.
 */
sai_status sai_distill_target_window(const uint16_t *Q, const uint16_t *Kw, const uint16_t *pool,
                                     const int32_t *idx, const float *sink, const int32_t *doc_start,
                                     int B, int S, int H, int D, int K, int cr, int W, float scale,
                                     float *p, float *window_lse, int32_t *d_err,
                                     void *workspace, size_t ws_bytes, void *stream);

/*
 * sai_distill_target_window_range -- sai_distill_target_window over a token
 * range of longer sequences (a sequence split across GPUs by position, as
 * sai_window_lse_range and sai_distill_target_range).
 *
 *   Q, idx, doc_start, p, window_lse: the range's own rows [B,S,...]
 *   Kw          [B,S+kw_lead,D] bf16: the keys of positions
 *               t_begin-kw_lead .. t_begin+S-1 (the range and its halo)
 *   pool        [B,S_seq/cr,D]: every compressed entry of the sequence
 *   t_begin     >= 0, t_begin + S <= S_seq; kw_lead in
 *               [min(W-1, t_begin), t_begin]
 *
 * Positions, not row numbers, decide the window, causal and document rules.
 * sai_distill_target_window is this call with S_seq = S and t_begin =
 * kw_lead = 0. Errors as for sai_distill_target_window (SAI_ERR_SHAPE for a
 * short halo or a range outside the sequence).
 */
sai_status sai_distill_target_window_range(const uint16_t *Q, const uint16_t *Kw, const uint16_t *pool,
                                           const int32_t *idx, const float *sink, const int32_t *doc_start,
                                           int B, int S, int S_seq, int t_begin, int kw_lead, int H, int D,
                                           int K, int cr, int W, float scale, float *p, float *window_lse,
                                           int32_t *d_err, void *workspace, size_t ws_bytes, void *stream);

/* Bytes of device workspace sai_distill_target_kl needs for these sizes. */
size_t sai_distill_target_kl_workspace_bytes(int B, int S, int K);

/*
 * sai_distill_target_kl -- the target and the KL stage in one call.
 *
 * Computes what sai_distill_target_ex followed by sai_distill_kl computes.
 * Where the tensor-core target kernel runs and K <= 512, the KL row, its
 * gradient and the per-block KL sums come from the target kernel's epilogue
 * while the row is still in shared memory, so p need not be written to or
 * read back from device memory. This is the KL half of the single fused pass
 * the Primus page describes (first commit message: the KL tail is fused and
 * keeps no state between forward and backward). Before it, a small kernel
 * counts the rows with a valid slot (N).
 *
 *   arguments as in sai_distill_target_ex and sai_distill_kl;
 *   p          [B,S,K] fp32 target, written if not NULL. It may be NULL only
 *              where the fused route applies (else SAI_ERR_UNSUPPORTED);
 *   workspace  device scratch of sai_distill_target_kl_workspace_bytes(B,S,K)
 *              bytes, 16-byte aligned, owned by the caller; no initialisation
 *              needed; calls that share it must not overlap.
 *
 * Errors: as sai_distill_target_ex and sai_distill_kl (SAI_ERR_WORKSPACE for
 * a short or misaligned workspace). The loss is deterministic run to run.
 */
sai_status sai_distill_target_kl(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start,
                                 int B, int S, int H, int D, int K, int cr, float scale, unsigned flags,
                                 const float *scores, const uint8_t *valid, float coeff,
                                 float *p, float *loss, float *dscores,
                                 void *workspace, size_t ws_bytes, int32_t *d_err, void *stream);

/* Bytes of device workspace sai_distill_kl needs for these sizes. */
size_t sai_distill_kl_workspace_bytes(int B, int S, int K);

/*
 * sai_distill_kl -- KL(attention || indexer) and its gradient in one pass.
 *
 * Source: Primus page, first commit message (indexer_distill_kl computes the
 * KL and its closed-form gradient together and keeps no state between them);
 * MaxText page review (the gradient of a log-softmax KL is q - p; the indexer's
 * own mask is part of the valid mask).
 *
 * Per token row over its valid slots (valid[b,t,k] != 0):
 *   log q[k]  = scores[k] - log sum_{valid k'} exp scores[k']
 *   KL_t      = sum_{valid k, p[k] > 0} p[k] (log p[k] - log q[k])
 *   N         = number of rows with at least one valid slot
 *   *loss     = coeff * sum_t KL_t / max(N, 1)
 *   dscores[k]= coeff / max(N,1) * (q[k] * sum_{valid} p - p[k]) on valid
 *               slots of valid rows, 0 elsewhere
 *
 *   p, scores  [B,S,K] fp32; valid [B,S,K] uint8; all 16-byte aligned
 *   loss       device fp32 scalar, written (4-byte aligned)
 *   dscores    [B,S,K] fp32, written, 16-byte aligned; NULL = forward only
 *   workspace  device scratch of ws_bytes >= sai_distill_kl_workspace_bytes(),
 *              16-byte aligned; no initialisation needed; must not be shared
 *              by calls that overlap on the device.
 *
 * The loss is reduced in a fixed order (deterministic). The work is one
 * cooperative launch (all blocks resident; N is formed across them behind a
 * bounded grid barrier) after a 16-byte cudaMemsetAsync of the workspace on
 * the stream. Should that barrier ever time out, *loss is NaN and dscores is
 * left unwritten. Errors: SAI_ERR_NULL, SAI_ERR_SHAPE, SAI_ERR_ALIGN,
 * SAI_ERR_WORKSPACE, SAI_ERR_CUDA.
 */
sai_status sai_distill_kl(const float *p, const float *scores, const uint8_t *valid,
                          int B, int S, int K, float coeff,
                          float *loss, float *dscores, void *workspace, size_t ws_bytes,
                          void *stream);

/*
 * sai_count_valid_rows -- N, the rows of `valid` that hold a valid slot.
 *
 *   valid    [B,S,K] uint8 device, 16-byte aligned
 *   n_rows   device int32, written (zeroed, then counted, on the stream)
 *
 * The count sai_distill_kl normalises by. A caller that splits the batch
 * across GPUs sums the ranks' counts (an all-reduce of one integer) and hands
 * the sum to sai_distill_kl_ex, so every rank's dscores carry the batch-wide
 * 1/N and the ranks' losses add up to the batch loss. Errors: SAI_ERR_NULL,
 * SAI_ERR_SHAPE, SAI_ERR_ALIGN, SAI_ERR_CUDA.
 */
sai_status sai_count_valid_rows(const uint8_t *valid, int B, int S, int K, int32_t *n_rows, void *stream);

/*
 * sai_distill_kl_ex -- sai_distill_kl with a caller-given N.
 *
 * n_rows NULL: exactly sai_distill_kl. Otherwise a device int32 (4-byte
 * aligned) holding N, read by the kernels when they run (so it may be written
 * earlier on the same stream, e.g. by an all-reduce of the ranks'
 * sai_count_valid_rows). Then
 *
 *   *loss      = coeff * sum_{rows here} KL_t / max(N, 1)
 *   dscores[k] = coeff / max(N, 1) * (q[k] * sum_{valid} p - p[k])
 *
 * i.e. this call's share of the batch-wide loss (summing the shares over
 * ranks gives the batch loss) and the batch-wide gradient. Everything else as
 * for sai_distill_kl.
 */
sai_status sai_distill_kl_ex(const float *p, const float *scores, const uint8_t *valid,
                             int B, int S, int K, float coeff, const int32_t *n_rows,
                             float *loss, float *dscores, void *workspace, size_t ws_bytes,
                             void *stream);

/*
 * sai_distill_kl_noalloc -- sai_distill_kl for callers that cannot allocate.
 *
 * The source pages have no counterpart to this call; it is a library
 * convenience. Same inputs, outputs, arithmetic and errors as sai_distill_kl,
 * but there is no workspace argument: the scratch words live in a fixed device
 * array inside the library (sai_distill_kl_noalloc_max_scratch_bytes() bytes,
 * held by every GPU that loads the library until the process exits). It calls
 * no cudaMalloc/cudaFree and no allocating library routine, so it suits a
 * caller whose framework owns all device memory, or one that must avoid the
 * device-wide synchronisation an allocation can bring.
 *
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins. The address is kept for the life of
 *     the process: after cudaDeviceReset (or anything else that tears down
 *     and re-creates the device's primary context) it is stale, so do not
 *     call this entry point again after such a reset.
 *   - Every call on a device shares the one array: calls that overlap on the
 *     GPU (other streams, other host threads) race and can corrupt each
 *     other's loss. Nothing needs clearing between calls.
 *   - Sizes whose scratch would exceed the array return SAI_ERR_WORKSPACE.
 */
size_t sai_distill_kl_noalloc_max_scratch_bytes(void);
sai_status sai_distill_kl_noalloc(const float *p, const float *scores, const uint8_t *valid,
                                  int B, int S, int K, float coeff,
                                  float *loss, float *dscores, void *stream);

/*
 * sai_indexer_topk -- which compressed blocks each token selects, from the
 * lightning indexer's scores.
 *
 * Source: MaxText page "Add Indexer Loss [Deepseek v4]": the indexer keeps its
 * top-k block indices, writes -1 wherever the choice is invalid, and returns
 * the index scores with them; its commit messages give the causal block mask
 * and the packing mask. The indexer's own score formula is not on the pages:
 * index_scores is the caller's. Rule, per token (b,t) with document start d0
 * (clamped to [0, t]):
 *
 *   block j (0 <= j < P = S/cr) is a candidate iff (j+1)*cr - 1 <= t,
 *   j*cr >= d0, and index_scores[b,t,j] is neither NaN nor -inf;
 *   the K candidates with the largest scores are selected, an equal score
 *   going to the lower block (+0 and -0 are equal);
 *   idx[b,t,k] = the k-th selected block in ascending block order, and -1
 *   for k >= the number selected (fewer than K candidates).
 *
 * The outputs are the inputs the loss calls take: idx for
 * sai_distill_target, and sel_scores / valid for sai_distill_kl.
 *
 *   index_scores [B,S,P] fp32 device, 4-byte aligned (entries of blocks that
 *                are not candidates are not read)
 *   doc_start    [B,S] int32 or NULL (one document per sequence)
 *   idx          [B,S,K] int32, written
 *   sel_scores   [B,S,K] fp32 or NULL: index_scores[b,t,idx] on selected
 *                slots, 0 on -1 slots
 *   valid        [B,S,K] uint8 or NULL: 1 on selected slots, 0 elsewhere
 *
 * Sizes: S % cr == 0, 1 <= K <= P, P <= 32768. All buffers caller-owned; no
 * allocation, no synchronisation; deterministic. Errors: SAI_ERR_NULL,
 * SAI_ERR_SHAPE, SAI_ERR_ALIGN, SAI_ERR_UNSUPPORTED (P too large),
 * SAI_ERR_CUDA.
 */
sai_status sai_indexer_topk(const float *index_scores, const int32_t *doc_start, int B, int S, int cr, int K,
                            int32_t *idx, float *sel_scores, uint8_t *valid, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SAI_H */
