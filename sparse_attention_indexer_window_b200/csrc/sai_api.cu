// C-ABI entry points of libsai (declared in include/sai.h): argument
// validation, kernel selection by shape, TMA descriptor encoding and launch.
// Nothing here allocates device memory or synchronises the stream.
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "sai.h"
#include "indexer_topk.h"
#include "sai_kernels.h"

namespace {

using sai::KlPlan;

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

int max_smem_optin()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bf16 matrix [rows, cols] (row-major), box = box_rows x 64 columns, 128-byte
// swizzle (the layout the tcgen05 descriptors expect).
bool make_map_bf16(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool tc_heads(int H) { return H == 16 || H == 32 || H == 64 || H == 128; }

sai_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SAI_OK : SAI_ERR_CUDA; }

}  // namespace

extern "C" {

const char *sai_status_string(int status)
{
    switch (status) {
    case SAI_OK: return "SAI_OK";
    case SAI_ERR_NULL: return "SAI_ERR_NULL: a required pointer is NULL";
    case SAI_ERR_SHAPE: return "SAI_ERR_SHAPE: a size is out of range or sizes are inconsistent";
    case SAI_ERR_UNSUPPORTED: return "SAI_ERR_UNSUPPORTED: shape outside what the kernels cover";
    case SAI_ERR_CUDA: return "SAI_ERR_CUDA: a CUDA call or kernel launch failed";
    case SAI_ERR_INDEX: return "SAI_ERR_INDEX: an idx entry lies outside {-1} U [0, S/cr)";
    case SAI_ERR_WORKSPACE: return "SAI_ERR_WORKSPACE: workspace missing, too small or misaligned";
    case SAI_ERR_ALIGN: return "SAI_ERR_ALIGN: a tensor pointer is not suitably aligned";
    case SAI_ERR_TIMEOUT: return "SAI_ERR_TIMEOUT: a kernel gave up a bounded wait";
    default: return "unknown sai_status";
    }
}

int sai_version(void) { return 200; }

namespace {

sai_status window_impl(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start, int B, int S, int H, int D,
                       int W, int t_begin, int kw_lead, float scale, float *window_lse, cudaStream_t st)
{
    if (!Q || !Kw || !window_lse)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || H < 1 || D < 1 || W < 1 || (D % 8) != 0 || !isfinite(scale) || scale <= 0.f)
        return SAI_ERR_SHAPE;
    // a range needs every key its first token's window can reach
    if (t_begin < 0 || kw_lead < 0 || kw_lead > t_begin || kw_lead < std::min(W - 1, t_begin))
        return SAI_ERR_SHAPE;
    if ((int64_t)B * S * H * D > INT32_MAX || (int64_t)B * S * H > INT32_MAX ||
        (int64_t)t_begin + S > INT32_MAX || (int64_t)B * (S + kw_lead) * D > INT32_MAX)
        return SAI_ERR_SHAPE;
    if (!al16(Q) || !al16(Kw) || !al4(window_lse) || (doc_start && !al4(doc_start)))
        return SAI_ERR_ALIGN;
    const int smem_cap = max_smem_optin();

    if (tc_heads(H) && (D % 64) == 0 && S % (128 / H) == 0 && W + 128 / H - 1 <= 256) {
        sai::WinTcArgs a;
        a.B = B;
        a.S = S;
        a.H = H;
        a.D = D;
        a.W = W;
        a.t_begin = t_begin;
        a.kw_lead = kw_lead;
        a.TQ = 128 / H;
        a.NB = ((W + a.TQ - 1) + 15) / 16 * 16;
        a.n_tiles = B * S / a.TQ;
        a.b_stage_bytes = (uint32_t)(((size_t)a.NB * 128 + 1023) & ~size_t(1023));
        a.scale = scale;
        a.doc_start = doc_start;
        a.out = window_lse;
        if ((int)sai::window_tc_smem_bytes(a.NB) > smem_cap)
            return SAI_ERR_UNSUPPORTED;
        CUtensorMap mq, mk;
        if (!make_map_bf16(&mq, Q, (uint64_t)B * S * H, D, 128) ||
            !make_map_bf16(&mk, Kw, (uint64_t)B * (S + kw_lead), D, (uint32_t)a.NB))
            return SAI_ERR_CUDA;
        int grid = sm_count();
        if (grid <= 0)
            return SAI_ERR_CUDA;
        if (grid > a.n_tiles)
            grid = a.n_tiles;
        return cuda_status(sai::launch_window_lse_tc(mq, mk, a, grid, st));
    }
    if ((int)sai::window_simt_smem_bytes(H, D, W) <= smem_cap)
        return cuda_status(sai::launch_window_lse_simt(Q, Kw, doc_start, B, S, H, D, W, t_begin, kw_lead, scale,
                                                       window_lse, st));
    return SAI_ERR_UNSUPPORTED;
}

}  // namespace

sai_status sai_window_lse(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start, int B, int S, int H,
                          int D, int W, float scale, float *window_lse, void *stream)
{
    return window_impl(Q, Kw, doc_start, B, S, H, D, W, 0, 0, scale, window_lse,
                       reinterpret_cast<cudaStream_t>(stream));
}

sai_status sai_window_lse_range(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start, int B, int S,
                                int H, int D, int W, int t_begin, int kw_lead, float scale, float *window_lse,
                                void *stream)
{
    return window_impl(Q, Kw, doc_start, B, S, H, D, W, t_begin, kw_lead, scale, window_lse,
                       reinterpret_cast<cudaStream_t>(stream));
}

sai_status sai_distill_target(const uint16_t *Q, const uint16_t *pool, const int32_t *idx, const float *window_lse,
                              const float *sink, const int32_t *doc_start, int B, int S, int H, int D, int K,
                              int cr, float scale, float *p, int32_t *d_err, void *stream)
{
    return sai_distill_target_ex(Q, pool, idx, window_lse, sink, doc_start, B, S, H, D, K, cr, scale, 0u, p, d_err,
                                 stream);
}

namespace {

// Fused KL arguments of sai_distill_target_kl (NULL: target only).
struct KlFuse {
    const float *scores;
    const uint8_t *valid;
    float coeff;
    float *loss;
    float *dscores;
    void *ws;
    sai::KlPlan plan;
};

// Workspace of sai_distill_target_kl: the KL workspace (completion counter,
// per-block valid-row counts, per-block KL sums) with room for one KL sum per
// CTA of the target kernel (at most kMaxTargetCtas).
constexpr int kMaxTargetCtas = 1024;
size_t fused_ws_bytes(const sai::KlPlan &pl)
{
    const size_t a = 16 + (((size_t)pl.count_blocks * 4 + 15) & ~size_t(15));
    const size_t parts = (size_t)(pl.row_blocks > kMaxTargetCtas ? pl.row_blocks : kMaxTargetCtas) * 8;
    return a + parts;
}

// Floats of raw-score spill per CTA of the target kernel: every TMEM group of
// a token whose K slots need more than one (H >= 64; 0 otherwise).
size_t spill_floats_per_cta(int H, int K)
{
    if (!tc_heads(H) || H < 64)
        return 0;
    const int tb = 256 / H;
    const int tiles = (K + 127) / 128;
    const int groups = (tiles + tb - 1) / tb;
    return groups > 1 ? (size_t)groups * tb * H * 128 : 0;
}

// The window band computed inside the target kernel
// (sai_distill_target_window); NULL: window_lse is an input.
struct WinFuse {
    const uint16_t *Kw;   // [B, S + kw_lead, D]
    int W;
    int kw_lead;          // Kw rows before local token 0
    float *wl_out;        // [B, S, H] the window log-mass written out, or NULL
};

// CTAs of the target kernel for n_tok tokens.
int target_grid(int64_t n_tok)
{
    int grid = sm_count();
    if (grid <= 0)
        return 0;
    if (grid > n_tok)
        grid = (int)n_tok;
    return grid > kMaxTargetCtas ? kMaxTargetCtas : grid;
}

// S local tokens per sequence starting at position t_begin of sequences of
// S_seq tokens (the whole sequence: S_seq == S, t_begin == 0). ws: the
// optional raw-score spill (NULL: tokens of more than one TMEM group are
// gathered and multiplied twice).
sai_status target_impl(const uint16_t *Q, const uint16_t *pool, const int32_t *idx, const float *window_lse,
                       const float *sink, const int32_t *doc_start, int B, int S, int S_seq, int t_begin, int H,
                       int D, int K, int cr, float scale, unsigned flags, float *p, int32_t *d_err,
                       cudaStream_t st, const KlFuse *kf, void *ws = nullptr, size_t ws_bytes = 0,
                       const WinFuse *wf = nullptr)
{
    if ((flags & ~(SAI_TARGET_PER_BRANCH | SAI_TARGET_FULL_LSE)) ||
        (flags & (SAI_TARGET_PER_BRANCH | SAI_TARGET_FULL_LSE)) == (SAI_TARGET_PER_BRANCH | SAI_TARGET_FULL_LSE))
        return SAI_ERR_UNSUPPORTED;
    const bool per_branch = (flags & SAI_TARGET_PER_BRANCH) != 0;
    const int lse_mode = per_branch ? sai::kLsePerBranch
                                    : ((flags & SAI_TARGET_FULL_LSE) ? sai::kLseGiven : sai::kLseJoint);
    if (per_branch)
        window_lse = nullptr;   // not read in this mode
    if (lse_mode != sai::kLseJoint)
        sink = nullptr;         // per-branch: no sink; given LSE: the sink is inside it
    if (wf) {
        // the window from Kw: the joint target only, never with the KL fused
        if (lse_mode != sai::kLseJoint || kf)
            return SAI_ERR_UNSUPPORTED;
        if (!wf->Kw)
            return SAI_ERR_NULL;
        window_lse = nullptr;
    }
    // idx NULL: dense over all blocks; p may be NULL only when the KL is fused
    if (!Q || !pool || (!window_lse && !per_branch && !wf) || (!p && !kf))
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || H < 1 || D < 1 || K < 1 || cr < 1 || (D % 8) != 0 || S_seq < 1 || (S_seq % cr) != 0 ||
        !isfinite(scale) || scale <= 0.f)
        return SAI_ERR_SHAPE;
    if (t_begin < 0 || (int64_t)t_begin + S > S_seq)
        return SAI_ERR_SHAPE;
    const int P = S_seq / cr;
    if (K > P)
        return SAI_ERR_SHAPE;
    if ((int64_t)B * S * H * D > INT32_MAX || (int64_t)B * S * K > INT32_MAX)
        return SAI_ERR_SHAPE;
    if (wf) {
        if (wf->W < 1 || wf->kw_lead < 0 || wf->kw_lead > t_begin || wf->kw_lead < std::min(wf->W - 1, t_begin) ||
            (int64_t)B * (S + wf->kw_lead) * D > INT32_MAX)
            return SAI_ERR_SHAPE;
        if (wf->W > 128)
            return SAI_ERR_UNSUPPORTED;   // the window band is one 128-row tile
        if (!al16(wf->Kw) || (wf->wl_out && !al4(wf->wl_out)))
            return SAI_ERR_ALIGN;
    }
    if (!al16(Q) || !al16(pool) || (idx && !al4(idx)) || (window_lse && !al4(window_lse)) || (p && !al4(p)) ||
        (sink && !al4(sink)) || (doc_start && !al4(doc_start)) || (d_err && !al4(d_err)))
        return SAI_ERR_ALIGN;
    const int smem_cap = max_smem_optin();

    // the tensor-core kernel addresses pool rows with 32-bit byte offsets
    const bool pool_fits = (uint64_t)B * P * D * 2 < 0xffffffffull;
    // Shared-memory layout, the first that fits: two 64-column chunks of D
    // per pipeline stage (half the per-stage synchronisation) with a
    // four-token compaction ring and staged idx rows; the same with a
    // two-token ring and idx read from global memory (large K); then one
    // chunk per stage, in the same two forms.
    const bool idx_vec = idx && (K % 4) == 0 && al16(idx);
    const bool tc_ok = tc_heads(H) && (D % 64) == 0 && pool_fits;
    int cps = 1, n_meta = 4, idx_stage = 0, n_astages = 0;
    for (int c = 0; c < 4 && tc_ok && n_astages == 0; ++c) {
        cps = (c < 2 && (D % 128) == 0) ? 2 : 1;
        if (c < 2 && cps == 1)
            continue;
        n_meta = (c % 2 == 0) ? 4 : 2;
        idx_stage = (c % 2 == 0 && idx_vec) ? 1 : 0;
        n_astages = sai::target_tc_stages(H, K, cps, n_meta, idx_stage, wf ? 1 : 0, smem_cap);
    }
    if (wf && n_astages == 0)
        return SAI_ERR_UNSUPPORTED;   // the window band needs the tensor-core kernel
    // the epilogue computes the KL from two slots per thread (K <= 512)
    const bool fuse_here = kf && n_astages > 0 && K <= 512;
    if (kf && !fuse_here && !p)
        return SAI_ERR_UNSUPPORTED;   // the unfused route needs p to pass the target on
    if (n_astages > 0) {
        sai::TgtTcArgs a;
        a.B = B;
        a.S = S;
        a.H = H;
        a.D = D;
        a.K = K;
        a.cr = cr;
        a.P = P;
        a.t_begin = t_begin;
        a.n_tok = B * S;
        a.tiles_per_group = 256 / H;
        a.idx_bulk = idx_vec ? 1 : 0;
        a.idx_stage = idx_stage;
        a.n_meta = n_meta;
        a.n_astages = n_astages;
        a.cps = cps;
        a.lse_mode = lse_mode;
        a.pool_box_rows = (int)std::min<int64_t>(128, (int64_t)B * P);
        a.scale = scale;
        a.pool = pool;
        a.idx = idx;
        a.wl = window_lse;
        a.sink = sink;
        a.doc_start = doc_start;
        a.p = p;
        a.err = d_err;
        a.kl_scores = nullptr;
        a.kl_valid = nullptr;
        a.kl_dscores = nullptr;
        a.kl_loss = nullptr;
        a.kl_coeff = 0.f;
        a.kl_count_part = nullptr;
        a.kl_count_blocks = 0;
        a.kl_part = nullptr;
        a.kl_done = nullptr;
        a.spill = nullptr;
        a.spill_stride = 0;
        a.win = wf ? wf->W : 0;
        a.kw_lead = wf ? wf->kw_lead : 0;
        a.kw_rows = S + a.kw_lead;
        a.kw_box_rows = (int)std::min<int64_t>(128, (int64_t)B * a.kw_rows);
        a.wl_out = wf ? wf->wl_out : nullptr;
        CUtensorMap mq, mp, mk;
        if (!make_map_bf16(&mq, Q, (uint64_t)B * S * H, D, (uint32_t)H) ||
            !make_map_bf16(&mp, pool, (uint64_t)B * P, D, (uint32_t)a.pool_box_rows))
            return SAI_ERR_CUDA;
        if (wf) {
            if (!make_map_bf16(&mk, wf->Kw, (uint64_t)B * a.kw_rows, D, (uint32_t)a.kw_box_rows))
                return SAI_ERR_CUDA;
        } else {
            mk = mp;   // not read
        }
        const int grid = target_grid(a.n_tok);
        if (grid <= 0)
            return SAI_ERR_CUDA;
        const size_t spf = spill_floats_per_cta(H, K);
        if (spf && ws && ws_bytes >= (size_t)grid * spf * sizeof(float)) {
            a.spill = reinterpret_cast<float *>(ws);
            a.spill_stride = (int)spf;
        }
        if (fuse_here) {
            // N first: per-block valid-row counts (this also zeroes the counter)
            sai_status e = cuda_status(sai::launch_kl_count(kf->plan, kf->valid, kf->ws, st));
            if (e != SAI_OK)
                return e;
            uint8_t *w = reinterpret_cast<uint8_t *>(kf->ws);
            a.kl_scores = kf->scores;
            a.kl_valid = kf->valid;
            a.kl_dscores = kf->dscores;
            a.kl_loss = kf->loss;
            a.kl_coeff = kf->coeff;
            a.kl_done = reinterpret_cast<uint32_t *>(w);
            a.kl_count_part = reinterpret_cast<const int32_t *>(w + 16);
            a.kl_count_blocks = kf->plan.count_blocks;
            a.kl_part = reinterpret_cast<double *>(w + 16 + (((size_t)kf->plan.count_blocks * 4 + 15) & ~size_t(15)));
        }
        sai_status e = cuda_status(sai::launch_target_tc(mq, mp, mk, a, grid, st));
        if (e != SAI_OK || fuse_here || !kf)
            return e;
    } else if ((int)sai::target_simt_smem_bytes(H, D, K) <= smem_cap) {
        sai_status e = cuda_status(sai::launch_target_simt(Q, pool, idx, window_lse, sink, doc_start, B, S, P,
                                                           t_begin, H, D, K, cr, scale, lse_mode, p, d_err, st));
        if (e != SAI_OK || !kf)
            return e;
    } else {
        return SAI_ERR_UNSUPPORTED;
    }
    // the KL as its own pass over the target just written to p
    return cuda_status(sai::launch_distill_kl(kf->plan, p, kf->scores, kf->valid, kf->coeff, kf->loss, kf->dscores,
                                              kf->ws, st));
}

}  // namespace

sai_status sai_distill_target_ex(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start, int B, int S,
                                 int H, int D, int K, int cr, float scale, unsigned flags, float *p, int32_t *d_err,
                                 void *stream)
{
    return target_impl(Q, pool, idx, window_lse, sink, doc_start, B, S, S, 0, H, D, K, cr, scale, flags, p, d_err,
                       reinterpret_cast<cudaStream_t>(stream), nullptr);
}

sai_status sai_distill_target_range(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                    const float *window_lse, const float *sink, const int32_t *doc_start, int B,
                                    int S, int S_seq, int t_begin, int H, int D, int K, int cr, float scale,
                                    unsigned flags, float *p, int32_t *d_err, void *stream)
{
    return target_impl(Q, pool, idx, window_lse, sink, doc_start, B, S, S_seq, t_begin, H, D, K, cr, scale, flags,
                       p, d_err, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

size_t sai_distill_target_workspace_bytes(int B, int S, int H, int D, int K)
{
    if (B < 1 || S < 1 || H < 1 || D < 1 || K < 1 || (D % 64) != 0)
        return 0;
    const size_t spf = spill_floats_per_cta(H, K);
    if (!spf)
        return 0;
    const int grid = target_grid((int64_t)B * S);
    return grid > 0 ? (size_t)grid * spf * sizeof(float) : 0;
}

sai_status sai_distill_target_window_range(const uint16_t *Q, const uint16_t *Kw, const uint16_t *pool,
                                           const int32_t *idx, const float *sink, const int32_t *doc_start, int B,
                                           int S, int S_seq, int t_begin, int kw_lead, int H, int D, int K, int cr,
                                           int W, float scale, float *p, float *window_lse, int32_t *d_err,
                                           void *workspace, size_t ws_bytes, void *stream)
{
    if (workspace && !al16(workspace))
        return SAI_ERR_ALIGN;
    const WinFuse wf = {Kw, W, kw_lead, window_lse};
    return target_impl(Q, pool, idx, nullptr, sink, doc_start, B, S, S_seq, t_begin, H, D, K, cr, scale, 0u, p,
                       d_err, reinterpret_cast<cudaStream_t>(stream), nullptr, workspace, ws_bytes, &wf);
}

sai_status sai_distill_target_window(const uint16_t *Q, const uint16_t *Kw, const uint16_t *pool,
                                     const int32_t *idx, const float *sink, const int32_t *doc_start, int B, int S,
                                     int H, int D, int K, int cr, int W, float scale, float *p, float *window_lse,
                                     int32_t *d_err, void *workspace, size_t ws_bytes, void *stream)
{
    return sai_distill_target_window_range(Q, Kw, pool, idx, sink, doc_start, B, S, S, 0, 0, H, D, K, cr, W, scale,
                                           p, window_lse, d_err, workspace, ws_bytes, stream);
}

sai_status sai_distill_target_ws(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start, int B, int S,
                                 int S_seq, int t_begin, int H, int D, int K, int cr, float scale, unsigned flags,
                                 float *p, int32_t *d_err, void *workspace, size_t ws_bytes, void *stream)
{
    if (workspace && !al16(workspace))
        return SAI_ERR_ALIGN;
    return target_impl(Q, pool, idx, window_lse, sink, doc_start, B, S, S_seq, t_begin, H, D, K, cr, scale, flags,
                       p, d_err, reinterpret_cast<cudaStream_t>(stream), nullptr, workspace, ws_bytes);
}

size_t sai_distill_target_kl_workspace_bytes(int B, int S, int K)
{
    if (B < 1 || S < 1 || K < 1)
        return 0;
    return fused_ws_bytes(sai::kl_plan(B, S, K));
}

sai_status sai_distill_target_kl(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                                 const float *window_lse, const float *sink, const int32_t *doc_start, int B, int S,
                                 int H, int D, int K, int cr, float scale, unsigned flags, const float *scores,
                                 const uint8_t *valid, float coeff, float *p, float *loss, float *dscores,
                                 void *workspace, size_t ws_bytes, int32_t *d_err, void *stream)
{
    if (!scores || !valid || !loss || !dscores)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || K < 1 || !isfinite(coeff))
        return SAI_ERR_SHAPE;
    if (!al16(scores) || !al16(valid) || !al4(loss) || !al16(dscores))
        return SAI_ERR_ALIGN;
    KlFuse kf;
    kf.scores = scores;
    kf.valid = valid;
    kf.coeff = coeff;
    kf.loss = loss;
    kf.dscores = dscores;
    kf.ws = workspace;
    kf.plan = sai::kl_plan(B, S, K);
    if (!workspace || !al16(workspace) || ws_bytes < fused_ws_bytes(kf.plan))
        return SAI_ERR_WORKSPACE;
    return target_impl(Q, pool, idx, window_lse, sink, doc_start, B, S, S, 0, H, D, K, cr, scale, flags, p, d_err,
                       reinterpret_cast<cudaStream_t>(stream), &kf);
}
size_t sai_distill_kl_workspace_bytes(int B, int S, int K)
{
    if (B < 1 || S < 1 || K < 1)
        return 0;
    return sai::kl_plan(B, S, K).ws_bytes;
}

sai_status sai_distill_kl(const float *p, const float *scores, const uint8_t *valid, int B, int S, int K,
                          float coeff, float *loss, float *dscores, void *workspace, size_t ws_bytes,
                          void *stream)
{
    return sai_distill_kl_ex(p, scores, valid, B, S, K, coeff, nullptr, loss, dscores, workspace, ws_bytes, stream);
}

sai_status sai_count_valid_rows(const uint8_t *valid, int B, int S, int K, int32_t *n_rows, void *stream)
{
    if (!valid || !n_rows)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || K < 1 || (int64_t)B * S * K > INT32_MAX)
        return SAI_ERR_SHAPE;
    if (!al16(valid) || !al4(n_rows))
        return SAI_ERR_ALIGN;
    return cuda_status(sai::launch_count_rows(valid, B * S, K, n_rows, reinterpret_cast<cudaStream_t>(stream)));
}

sai_status sai_distill_kl_ex(const float *p, const float *scores, const uint8_t *valid, int B, int S, int K,
                             float coeff, const int32_t *n_rows, float *loss, float *dscores, void *workspace,
                             size_t ws_bytes, void *stream)
{
    if (n_rows && !al4(n_rows))
        return SAI_ERR_ALIGN;
    if (!p || !scores || !valid || !loss)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || K < 1 || !isfinite(coeff) || (int64_t)B * S * K > INT32_MAX)
        return SAI_ERR_SHAPE;
    if (!al16(p) || !al16(scores) || !al16(valid) || !al4(loss) || (dscores && !al16(dscores)))
        return SAI_ERR_ALIGN;
    const KlPlan pl = sai::kl_plan(B, S, K);
    if (!workspace || !al16(workspace) || ws_bytes < pl.ws_bytes)
        return SAI_ERR_WORKSPACE;
    return cuda_status(sai::launch_distill_kl(pl, p, scores, valid, coeff, loss, dscores, workspace,
                                              reinterpret_cast<cudaStream_t>(stream), n_rows));
}

sai_status sai_indexer_topk(const float *index_scores, const int32_t *doc_start, int B, int S, int cr, int K,
                            int32_t *idx, float *sel_scores, uint8_t *valid, void *stream)
{
    if (!index_scores || !idx)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || cr < 1 || K < 1 || (S % cr) != 0)
        return SAI_ERR_SHAPE;
    const int P = S / cr;
    if (K > P || (int64_t)B * S * P > INT32_MAX || (int64_t)B * S * K > INT32_MAX)
        return SAI_ERR_SHAPE;
    if (P > sai::kTopkMaxP || (int)sai::indexer_topk_smem_bytes(P) > max_smem_optin())
        return SAI_ERR_UNSUPPORTED;
    if (!al4(index_scores) || !al4(idx) || (sel_scores && !al4(sel_scores)) || (doc_start && !al4(doc_start)))
        return SAI_ERR_ALIGN;
    return cuda_status(sai::launch_indexer_topk(index_scores, doc_start, B, S, cr, K, idx, sel_scores, valid,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
