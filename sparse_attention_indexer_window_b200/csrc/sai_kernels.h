// Internal launch interface between the C-ABI entry points (sai_api.cu) and
// the kernels. Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sai {

// ---------------------------------------------------------------- window_lse
struct WinTcArgs {
    int B, S, H, D, W;
    int t_begin;          // sequence position of local token 0 (token-range calls; else 0)
    int kw_lead;          // Kw rows per sequence before local token 0 (Kw holds S + kw_lead rows)
    int TQ;               // tokens per 128-row tile (128 / H)
    int NB;               // band rows = roundup16(W + TQ - 1), <= 256
    int n_tiles;          // B*S / TQ
    uint32_t b_stage_bytes;
    float scale;
    const int32_t *doc_start;
    float *out;
};
size_t window_tc_smem_bytes(int NB);
cudaError_t launch_window_lse_tc(const CUtensorMap &mapQ, const CUtensorMap &mapK, const WinTcArgs &a,
                                 int grid, cudaStream_t stream);

// ------------------------------------------------------------ distill_target
// How the target forms each head's log-normaliser lse_full.
enum : int {
    kLseJoint = 0,      // LSE(window log-mass, compressed LSE, sink); floor FLT_MIN
    kLsePerBranch = 1,  // the compressed LSE alone; floor 1e-10; wl and sink unused
    kLseGiven = 2,      // wl holds lse_full itself; floor FLT_MIN; sink unused
};
struct TgtTcArgs {
    int B, S, H, D, K, cr, P;   // P = pool rows per sequence (sequence length / cr)
    int t_begin;          // sequence position of local token 0 (token-range calls; else 0)
    int n_tok;            // B*S
    int tiles_per_group;  // 128-slot tiles per TMEM accumulator (256 / H)
    int idx_bulk;         // idx rows are 16-byte aligned (K % 4 == 0): read 16 bytes at a time
    int idx_stage;        // idx rows staged in shared memory two tokens ahead (needs idx_bulk)
    int n_meta;           // compaction ring depth: 4, or 2 where shared memory is short (large K)
    int n_astages;        // depth of the gathered-row stage ring (divides 8)
    int cps;              // 64-column chunks of D per stage (1 or 2; D/64 % cps == 0)
    int pool_box_rows;    // rows of the pool's TMA box (min(128, B*P))
    int lse_mode;         // how lse_full is formed: kLseJoint, kLsePerBranch or kLseGiven
    float scale;
    const uint16_t *pool;
    const int32_t *idx;
    const float *wl;
    const float *sink;
    const int32_t *doc_start;
    float *p;             // may be NULL when the KL is fused (kl_scores set)
    int32_t *err;
    // Raw scores of every TMEM group of a token with more than one group
    // (H >= 64 only): [grid][spill_stride] fp32, each CTA its own part. Set:
    // one sweep of gathers and MMAs per token, the u pass reads the scores
    // back. NULL: the groups are gathered and multiplied a second time.
    float *spill;
    int spill_stride;     // floats per CTA: groups x tiles per group x H x 128
    // Window band in the same kernel (win > 0; sai_distill_target_window):
    // the per-head log-sum-exp over each token's window keys is formed from
    // Kw (the mapK tensor map, rows [B * kw_rows, D]) instead of read from wl.
    int win;              // window length W (1..128); 0: wl is an input
    int kw_rows;          // Kw rows per sequence (local tokens + kw_lead)
    int kw_lead;          // Kw rows before local token 0 (token-range calls; else 0)
    int kw_box_rows;      // rows of the Kw TMA box: min(128, B * kw_rows)
    float *wl_out;        // [n_tok, H] the window log-mass written out, or NULL
    // KL fused into the epilogue (kl_scores NULL: not fused). N comes from the
    // per-block valid-row counts of kl_count_kernel, run before on the stream.
    const float *kl_scores;     // [n_tok, K]
    const uint8_t *kl_valid;    // [n_tok, K]
    float *kl_dscores;          // [n_tok, K]
    float *kl_loss;             // device scalar
    float kl_coeff;
    const int32_t *kl_count_part;
    int kl_count_blocks;
    double *kl_part;            // [grid] per-CTA KL sums
    uint32_t *kl_done;          // completion counter, zeroed by kl_count_kernel
};
// Deepest gathered-row stage ring of `cps`-chunk stages that fits
// `smem_limit` bytes beside a compaction ring of n_meta tokens, with or
// without the staged idx rows, with (win = 1) or without the window-fused
// kernel's TMEM ring barriers (0: none).
int target_tc_stages(int H, int K, int cps, int n_meta, int idx_stage, int win, int smem_limit);
// mapK: the Kw tensor map when a.win > 0 (any valid map otherwise; unused)
cudaError_t launch_target_tc(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                             const TgtTcArgs &a, int grid, cudaStream_t stream);

// ------------------------------------------- generic CUDA-core kernels
// For shapes the tensor-core kernels do not take (small H or D).
size_t window_simt_smem_bytes(int H, int D, int W);
cudaError_t launch_window_lse_simt(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start, int B, int S,
                                   int H, int D, int W, int t_begin, int kw_lead, float scale, float *out,
                                   cudaStream_t stream);
size_t target_simt_smem_bytes(int H, int D, int K);
cudaError_t launch_target_simt(const uint16_t *Q, const uint16_t *pool, const int32_t *idx, const float *wl,
                               const float *sink, const int32_t *doc_start, int B, int S, int P, int t_begin,
                               int H, int D, int K, int cr, float scale, int lse_mode, float *p, int32_t *err,
                               cudaStream_t stream);

// ---------------------------------------------------------------- distill_kl
struct KlPlan {
    int rows, K;
    int count_blocks;   // blocks of the valid-row count kernel
    int row_blocks;     // blocks of the row kernel
    size_t ws_bytes;
};
KlPlan kl_plan(int B, int S, int K);
// Per-block counts of rows with a valid slot into the KL workspace (its
// layout: completion counter at byte 0, which this resets, counts at byte 16).
cudaError_t launch_kl_count(const KlPlan &pl, const uint8_t *valid, void *ws, cudaStream_t stream);
// n_given: device int32 holding N (rows with a valid slot over the whole
// batch, e.g. summed over ranks); NULL: counted here from `valid`.
cudaError_t launch_distill_kl(const KlPlan &pl, const float *p, const float *scores, const uint8_t *valid,
                              float coeff, float *loss, float *dscores, void *ws, cudaStream_t stream,
                              const int32_t *n_given = nullptr);
// *n = rows of `valid` [rows, K] with a valid slot (the stream zeroes *n first).
cudaError_t launch_count_rows(const uint8_t *valid, int rows, int K, int32_t *n, cudaStream_t stream);

}  // namespace sai
