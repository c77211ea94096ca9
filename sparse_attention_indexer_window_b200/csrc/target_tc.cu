// Distillation target on tcgen05 tensor cores with an in-kernel gather of the
// selected pool rows (sm_100a).
//
// For every token (b,t) (Primus page "perf(deepseek-v4): fuse and enable the
// indexer distillation loss": first commit message -- the pool is indexed
// inside the kernel so the [B,S,K,D] gather never exists; second commit
// message / "Why the target was wrong" -- each head normalises jointly over
// its window keys, its chosen pool rows and its sink logit):
//
//   z[k,h]      = scale <pool[idx[k]], Q[t,h]>       selected slots k
//   clse[h]     = log sum_k exp z[k,h]
//   lse_full[h] = logsumexp(window_lse[t,h], clse[h], sink[h])
//   u[k]        = sum_h exp(z[k,h] - lse_full[h]),  p[k] = u[k] / max(sum u, FLT_MIN)
//
// Layout of the contraction. The problem is transposed so the MMA keeps M=128
// although a token has only H heads: A = 128 gathered pool rows (one TMEM lane
// per selected slot), B = Q[t] (N = H columns, one per head), K-dim = D in
// 64-element (128-byte, swizzled) chunks.
//
// Gather. A dedicated warp compacts each token's idx row (selected slots
// first, masked slots last), up to three tokens ahead (one at large K, where
// shared memory holds a ring of two); the idx rows arrive by its own cp.async
// copies two tokens ahead, or at large K are read from global memory, and the
// compaction turns pool rows into byte offsets. A pipeline stage is 128 selected rows x CPS 128-byte chunks of D
// (CPS = 2 where D allows: 32 KB); the A ring holds NA stages (4 at the
// V4-Flash shape) and 8 / NA gather warps fill each stage, each its share of
// the rows, copied into the swizzled K-major operand layout with 16-byte
// cp.async (eight lanes per row, four rows per instruction, every 128-byte
// row segment one coalesced request). Each warp waits for its own copies and
// arrives once on the stage's barrier. A separate warp loads the Q[t] chunks
// (contiguous) by TMA, CPS chunks per ring entry, several entries ahead. A
// tile whose selected rows are consecutive pool rows (every tile of an early
// token under a sorted top-k, whose selection is all causal blocks) is one
// TMA box per chunk instead. Masked slots are never loaded.
//
// The epilogue needs the per-head log-sum-exp over ALL selected slots before
// it can form u, so a token's scores stay in TMEM until it is done: up to
// 256/H tiles (512 slots at H=64) per accumulator. Tokens alternate between
// two 256-column accumulators, group by group (a token of one group per
// accumulator, a longer token spread over both), so the epilogue of one group
// overlaps the MMAs of the next; both epilogue warpgroups work on each group
// (half the heads each at H >= 32). Tokens with more selected slots run in groups: a first
// pass over the groups merges per-head (max, sum-exp) statistics, a second
// forms u. With a spill buffer (H >= 64, its own instantiation) the first
// pass also stores each group's raw scores there and the second reads them
// back, so every row is gathered and multiplied once; the last group's
// scores are not spilled but stay in TMEM, with their exponentials, for its
// u pass, the first of the second pass. Without a spill buffer the second
// pass gathers and multiplies each group again. When the KL stage is fused
// (sai_distill_target_kl), the epilogue then computes each row's KL and
// dscores from the target in shared memory.
//
// Window-fused instantiation (WIN, sai_distill_target_window): each token
// first runs one more tile, A = the 128 Kw rows ending at the token (one TMA
// box per chunk, rows outside the window masked), against the same Q[t]
// chunks; its per-head log-sum-exp is the window log-mass the joint merge
// needs, so window_lse is not an input and Q is read once. TMEM is then a
// ring of 512/H tile slots released one by one (TileRing), so the window
// tile's slot is free again as soon as its statistics are taken.
//
// Epilogue arithmetic (one exponential per score):
//   M[h] = max_k z[k,h]  (per 8 columns: each warp's maximum by one redux,
//          then the four lane quarters merged per head through smem)
//   e[k,h] = exp(z[k,h] - M[h]) written back to TMEM, S[h] = sum_k e[k,h]
//   a[h] = M[h] - lse_full[h],  A = max_h a[h],  w[h] = exp(a[h] - A) in (0,1]
//   u'[k] = sum_h e[k,h] w[h]   (per thread: one TMEM lane = one slot)
//   m' = sum_k u'[k] >= 1; with u = u' e^A and m = m' e^A:
//   p[k] = u'[k]/m'                     if log m' + A >= log FLT_MIN
//        = u'[k] exp(A - log FLT_MIN)   otherwise (the float32-tiny floor),
// so no intermediate is subnormal however small each head's compressed share.
// The per-branch target (SAI_TARGET_PER_BRANCH) takes a[h] = M[h] - clse[h]
// and the floor 1e-10.
//
// Warp roles (640 threads): warp 0 idx staging and compaction, warps 1..7
// and 9 row gathers, warp 11 Q loads, warps 8 (also the TMEM owner) and 10
// the two MMA issuers, warps 12..19 the epilogue (two warpgroups that split
// each token's tiles). Persistent CTAs walk tokens from the last
// (heaviest) to the first. All mbarrier waits are bounded; a timeout is
// reported through err and the CTA unwinds. Named barriers are only used
// where every participating thread is guaranteed to arrive.
#include <climits>

#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

// Warpgroups 0..2 (warps 0..11): warp 0 compaction, warps 8 and 10 MMA,
// warp 11 Q loads, the other eight warps row gathers; warpgroups 3 and 4
// (warps 12..19): epilogue.
constexpr int kMetaWarp = 0;
constexpr int kMmaWarp = 8;                         // MMA thread 0, TMEM owner
constexpr int kMmaWarp2 = 10;                       // MMA thread 1
constexpr int kQWarp = 11;
constexpr int kGatherWarps = 8;
constexpr int kEpiWarp0 = 12;
constexpr int kTgtThreads = 20 * 32;                // 640
// Register split (setmaxnreg): launched at kLaunchRegs a thread; warpgroups
// 0..2 give theirs down to kLowRegs, the two epilogue warpgroups take
// kHighRegs. 384*56 + 256*152 = 60416 <= 640*96 = 61440 (the launch total).
constexpr int kLaunchRegs = 96;
constexpr int kLowRegs = 56;
constexpr int kHighRegs = 152;
static_assert(384 * kLowRegs + 256 * kHighRegs <= kTgtThreads * kLaunchRegs, "register split");
constexpr int kMaxAStages = kGatherWarps;          // at most one A ring slot per gather warp
constexpr int kQStagesMax = 6;
// Q[t] ring: the Q warp runs this many 64-column chunks ahead, in entries of
// CPS chunks (the chunks one stage's MMAs read); at least two entries.
template <int HH, int CPS>
constexpr int q_entries() { return (HH <= 64 ? 6 : 3) / CPS >= 2 ? (HH <= 64 ? 6 : 3) / CPS : 2; }
constexpr int kMeta = 4;   // compaction ring: at most four tokens (a.n_meta: 4, or 2 for large K)
constexpr uint32_t kATile = 128 * 128;              // 128 rows x 128 bytes
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLnFltMin = -87.33654475055310898657f;  // log(2^-126)
constexpr float kLnOldFloor = -23.025850929940457f;      // log(1e-10), the per-branch target's floor

template <int HH>
struct EpiState {                 // one per epilogue warpgroup
    float red_max[8][HH];
    float red_sum[8][HH];
    float colM[HH];
    float colS[HH];
    float head_a[HH];
    float wprime[HH];
    float red_m[8];
    float klred[8][3];   // fused KL: per-warp partials of the row reductions
};

template <int HH>
struct TgtSmem {
    uint64_t a_full[kMaxAStages], a_empty[kMaxAStages];
    uint64_t q_full[kQStagesMax], q_empty[kQStagesMax];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t meta_full[kMeta], meta_empty[kMeta];
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort_flag;
    int nsel[kMeta];
    int ident[kMeta];     // 1: the selected slots are slots 0..nsel-1 (slot list not written)
    uint32_t contig[kMeta];  // bit i: tile i's rows are consecutive pool rows (one TMA box per chunk)
    EpiState<HH> epi[1];
};

// The window-fused kernel's TMEM: a ring of 512 / H tile slots of H columns
// each (at most 32). Tile n of the sequence of tiles the MMAs write lands in
// slot n % (512 / H); the epilogue releases each slot when it is done with
// it (the window tile right after its statistics, a group's tiles after its
// u pass), and the MMA threads commit each group of tiles to one barrier of
// a ring as deep as the slot count.
struct TileRing {
    uint64_t slot_empty[32];
    uint64_t grp_full[32];
    float wred_max[4][128];   // the window tile's per-quarter (max, sum) per head
    float wred_sum[4][128];
};

__device__ __forceinline__ int n_groups(int nsel, int TB)
{
    const int nt = (nsel + 127) / 128;
    return (nt + TB - 1) / TB;
}

// Selection rule for one idx entry j of token t (document start d0).
__device__ __forceinline__ bool selected(int j, int t, int d0, int P, int cr)
{
    return j >= 0 && j < P && (j + 1) * cr - 1 <= t && j * cr >= d0;
}

// FUSE_KL: the epilogue also computes the KL stage (sai_distill_target_kl);
// a separate instantiation, so the plain target kernel carries none of it.
// CPS: 64-column chunks of D per pipeline stage. One stage is CPS x 4 MMAs
// behind one barrier wait, one fence and one commit; on this part a commit
// every 4 MMAs leaves the tensor pipe idle about half the time, so CPS = 2
// whenever D allows it.
// WIN: the window-fused instantiation (window tile first, TMEM as TileRing).
template <int HH, bool FUSE_KL, int CPS, bool SPILL, bool WIN>
__global__ void __launch_bounds__(kTgtThreads, 1)
    target_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapP,
                     const __grid_constant__ CUtensorMap mapK, const TgtTcArgs a)
{
    constexpr int TB = 256 / HH;                 // tiles per accumulator
    // the raw-score spill exists only in its own instantiation (H >= 64)
    constexpr bool kSpill = SPILL && TB <= 4;
    constexpr int kSlots = 512 / HH;             // TMEM tile slots (WIN)
    constexpr uint32_t kQTile = HH * 128;        // one chunk of Q[t]: H rows x 128 bytes
    constexpr uint32_t kQEntry = CPS * kQTile;   // one Q ring entry
    constexpr uint32_t kAStage = CPS * kATile;   // one A ring stage: 128 rows x CPS chunks
    constexpr int NC16 = HH / 16;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = a.K;
    const int Kp = (K + 3) & ~3;
    const int NA = a.n_astages;              // A-stage ring depth (sized on the host; divides 8)
    uint8_t *a_buf = base;                                                   // NA x kAStage
    constexpr int QS = q_entries<HH, CPS>();
    uint8_t *q_buf = a_buf + NA * kAStage;                                   // QS x kQEntry
    // byte offset in pool of every selected slot's row, compacted per token
    const int NM = a.n_meta;                 // compaction ring depth (4, or 2 for large K)
    const bool idx_stage = a.idx_stage != 0; // idx rows staged in smem (else read from global)
    uint32_t *rowoff = reinterpret_cast<uint32_t *>(q_buf + QS * kQEntry);   // [NM][Kp]
    int32_t *slot = reinterpret_cast<int32_t *>(rowoff + NM * Kp);           // [NM][Kp]
    int32_t *idxs = slot + NM * Kp;                                          // [3][Kp] staged idx rows
    float *ubuf = reinterpret_cast<float *>(idxs + (idx_stage ? 3 * Kp : 0)); // [Kp] u' of a token
    // then [2][TB*128] partial u of the two epilogue warpgroups (H >= 32)
    TgtSmem<HH> *sm = reinterpret_cast<TgtSmem<HH> *>(ubuf + Kp + (HH >= 32 ? 2 * TB * 128 : 0));
    TileRing *ring = reinterpret_cast<TileRing *>(sm + 1);   // WIN only (no room reserved otherwise)

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_chunks = a.D / 64;
    const int n_cp = n_chunks / CPS;             // stages per tile (D / 64 is a multiple of CPS)
    const int WPS = kGatherWarps / NA;           // gather warps filling each A slot
    const bool idx_bulk = a.idx_bulk != 0;       // idx rows 16-byte aligned, K % 4 == 0

    if (threadIdx.x == 0) {
        for (int s = 0; s < NA; ++s) {
            mbar_init(&sm->a_full[s], WPS);      // lane 0 of each warp filling the slot
            mbar_init(&sm->a_empty[s], 2);       // the consumer's commit + the other MMA thread's arrival
        }
        for (int s = 0; s < QS; ++s) {
            mbar_init(&sm->q_full[s], 1);
            mbar_init(&sm->q_empty[s], 2);      // both MMA threads release a Q entry
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 2);     // both MMA threads commit a group
            mbar_init(&sm->acc_empty[b], 8);    // lane 0 of each epilogue warp
        }
        for (int b = 0; b < NM; ++b) {
            mbar_init(&sm->meta_full[b], 1);
            mbar_init(&sm->meta_empty[b], 1);
        }
        if constexpr (WIN) {
            for (int k = 0; k < kSlots; ++k) {
                mbar_init(&ring->slot_empty[k], 8);   // lane 0 of each epilogue warp
                mbar_init(&ring->grp_full[k], 2);     // both MMA threads commit a group
            }
        }
        mbar_init(&sm->drain[0], 1);
        mbar_init(&sm->drain[1], 1);
        sm->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    volatile int *abort_flag = &sm->abort_flag;

    if (warp < kEpiWarp0) {
    // warpgroups 0..2 execute this one setmaxnreg together
    regs_dec<kLowRegs>();
    if (warp == kMetaWarp) {
        // ====================================================== idx compaction
        // idx rows are staged into shared memory with this warp's own
        // 16-byte cp.async copies, two tokens ahead (three buffers), when the
        // layout has room for them (else they are read from global memory in
        // 16-byte loads). (A TMA bulk copy here queued behind the Q and pool
        // TMA traffic of the same SM and arrived late.)
        const int n_vec = K / 4;                 // 16-byte pieces of an idx row (idx_bulk: K % 4 == 0)
        auto stage_idx = [&](int gts, int buf) {
            if (idx_stage && gts < a.n_tok) {
                const int gs = a.n_tok - 1 - gts;
                const char *src = reinterpret_cast<const char *>(a.idx + (size_t)gs * K);
                const uint32_t dst = smem_u32(idxs + buf * Kp);
                for (int v = lane; v < n_vec; v += 32)
                    cp_async16(dst + v * 16, src + v * 16);
            }
            cp_async_commit();
        };
        stage_idx(blockIdx.x, 0);
        stage_idx(blockIdx.x + gridDim.x, 1);
        bool ok = true;
        int it = 0;
        for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
            const int g = a.n_tok - 1 - gt;
            const int b = g / a.S;
            const int t = g - b * a.S + a.t_begin;   // sequence position
            const int m3 = it % NM;
            int32_t *ib = idxs + (it % 3) * Kp;
            stage_idx(gt + 2 * (int)gridDim.x, (it + 2) % 3);
            cp_async_wait<2>();                  // this token's row has landed
            __syncwarp();
            ok = warp_mbar_wait(&sm->meta_empty[m3], ((it / NM) & 1) ^ 1u, abort_flag, a.err);
            if (!ok)
                break;
            int d0 = 0;
            if (a.doc_start) {
                d0 = a.doc_start[g];
                d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
            }
            uint32_t *rw = rowoff + m3 * Kp;
            int32_t *sl = slot + m3 * Kp;
            const int32_t *grow = a.idx ? a.idx + (size_t)g * K : nullptr;   // NULL: slot k is block k
            int nsel = 0, nmask = 0;
            bool bad = false;
            // Fast path. When the selected slots are exactly slots 0..n-1 (the
            // usual layout: valid entries first, -1 or masked entries after),
            // the compaction is the identity and only the row offsets are
            // written. Lane L takes 4 consecutive slots per 128-slot tile; a
            // slot j is selected when lo <= j < hi (the causal and document
            // bounds of the selection rule, turned into a block interval once
            // per token). The layout is the identity when the highest
            // selected slot is nsel - 1. A tile's rows are consecutive pool
            // rows when idx[k] - k is the same for all its selected slots.
            const uint32_t rbyte = (uint32_t)a.D * 2u;
            const uint32_t rbase = (uint32_t)(b * a.P);
            const int lo = (d0 + a.cr - 1) / a.cr;
            const int hi = min(a.P, (t + 1) / a.cr);
            const uint32_t span = hi > lo ? (uint32_t)(hi - lo) : 0u;
            int cnt = 0, kmax = -1;
            uint32_t contig = 0;                 // bit i: tile i holds consecutive blocks
            for (int k0 = 0; k0 < K; k0 += 128) {
                const int k = k0 + 4 * lane;
                int j[4];
                if (idx_bulk) {
                    int4 v = make_int4(-1, -1, -1, -1);
                    if (k < K)
                        v = idx_stage ? *reinterpret_cast<const int4 *>(ib + k)
                                      : __ldg(reinterpret_cast<const int4 *>(grow + k));
                    j[0] = v.x;
                    j[1] = v.y;
                    j[2] = v.z;
                    j[3] = v.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        j[e] = (k + e < K) ? (grow ? __ldg(grow + k + e) : k + e) : -1;
                }
                int dmin = INT_MAX, dmax = INT_MIN;
                uint4 ro;
                uint32_t *rop = &ro.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool in = k + e < K;
                    const bool sv = (uint32_t)j[e] - (uint32_t)lo < span;
                    bad |= in && j[e] != -1 && (uint32_t)j[e] >= (uint32_t)a.P;
                    cnt += sv ? 1 : 0;
                    kmax = sv ? k + e : kmax;
                    const int dd = j[e] - (k + e);
                    dmin = sv ? min(dmin, dd) : dmin;
                    dmax = sv ? max(dmax, dd) : dmax;
                    rop[e] = (rbase + (uint32_t)j[e]) * rbyte;
                }
                if (k < K)
                    *reinterpret_cast<uint4 *>(rw + k) = ro;
                const int tmin = __reduce_min_sync(0xffffffffu, dmin);
                const int tmax = __reduce_max_sync(0xffffffffu, dmax);
                if (tmin == tmax || tmax == INT_MIN)    // one offset, or no selected slot
                    contig |= 1u << (k0 >> 7);
            }
            nsel = __reduce_add_sync(0xffffffffu, cnt);
            const bool prefix = __reduce_max_sync(0xffffffffu, kmax) + 1 == nsel;
            if (prefix) {
                if (lane == 0) {
                    sm->ident[m3] = 1;
                    sm->contig[m3] = contig;
                }
            } else {
            nsel = 0;
            if (lane == 0) {
                sm->ident[m3] = 0;
                sm->contig[m3] = 0u;             // general layout: every tile by cp.async
            }
            // general case: selected slots in order at the front, masked slots
            // from the back; lane L takes 4 consecutive slots
            for (int k0 = 0; k0 < K; k0 += 128) {
                const int k = k0 + 4 * lane;
                int j[4];
                if (idx_bulk) {
                    int4 v = make_int4(-1, -1, -1, -1);
                    if (k < K)
                        v = idx_stage ? *reinterpret_cast<const int4 *>(ib + k)
                                      : __ldg(reinterpret_cast<const int4 *>(grow + k));
                    j[0] = v.x;
                    j[1] = v.y;
                    j[2] = v.z;
                    j[3] = v.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        j[e] = (k + e < K) ? (grow ? __ldg(grow + k + e) : k + e) : -1;
                }
                int cs = 0, cm = 0;
                bool sel[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool in = k + e < K;
                    sel[e] = in && selected(j[e], t, d0, a.P, a.cr);
                    bad |= in && !(j[e] == -1 || (j[e] >= 0 && j[e] < a.P));
                    cs += sel[e] ? 1 : 0;
                    cm += (in && !sel[e]) ? 1 : 0;
                }
                int sc = cs | (cm << 16);  // packed inclusive scan of both counts
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o)
                        sc += y;
                }
                const int tot = __shfl_sync(0xffffffffu, sc, 31);
                int ps = nsel + (sc & 0xffff) - cs;
                int pm = nmask + (sc >> 16) - cm;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (sel[e]) {
                        rw[ps] = (uint32_t)(b * a.P + j[e]) * (uint32_t)(a.D * 2);
                        sl[ps] = k + e;
                        ++ps;
                    } else if (k + e < K) {
                        sl[K - 1 - pm] = k + e;
                        ++pm;
                    }
                }
                nsel += tot & 0xffff;
                nmask += tot >> 16;
            }
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0 && a.err)
                atomicExch(a.err, kErrIndex);
            if (lane == 0)
                sm->nsel[m3] = nsel;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm->meta_full[m3]);
            __syncwarp();
        }
        cp_async_wait<0>();
        __syncwarp();
    } else if (warp == kQWarp) {
        // ============================================================ Q[t] chunks
        // Every (pass, group, chunk pair) of a token uses CPS H x 64 slices
        // of Q[t]; this warp loads them by TMA, QS entries ahead of the MMA.
        int qs = 0;
        uint32_t qph = 0;
        uint32_t q_issued = 0, q_last = 0;
        bool ok = true;
        int it = 0;
        if (lane == 0)
            tma_prefetch_desc(&mapQ);
        for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
            const int g = a.n_tok - 1 - gt;
            const int m3 = it % NM;
            ok = warp_mbar_wait(&sm->meta_full[m3], (it / NM) & 1, abort_flag, a.err);
            if (!ok)
                break;
            const int nsel = sm->nsel[m3];
            const int G = n_groups(nsel, TB);
            // (WIN: the window tile's group first, one more set of chunks)
            const int nq = (G > 1 && !kSpill ? 2 : 1) * G * n_cp + (WIN ? n_cp : 0);
            for (int qi = 0; qi < nq && ok; ++qi) {
                const int c0 = (qi % n_cp) * CPS;
                ok = warp_mbar_wait(&sm->q_empty[qs], qph ^ 1u, abort_flag, a.err);
                if (ok) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sm->q_full[qs], kQEntry);
#pragma unroll
                        for (int cc = 0; cc < CPS; ++cc)
                            tma_load_2d(q_buf + qs * kQEntry + cc * kQTile, &mapQ, &sm->q_full[qs], (c0 + cc) * 64,
                                        g * HH);
                    }
                    __syncwarp();
                    q_issued |= 1u << qs;
                    q_last = (q_last & ~(1u << qs)) | (qph << qs);
                }
                if (++qs == QS) {
                    qs = 0;
                    qph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < QS; ++s)
                if (q_issued & (1u << s))
                    mbar_drain(&sm->q_full[s], (q_last >> s) & 1u);
        }
        __syncwarp();
    } else if (warp != kMmaWarp && warp != kMmaWarp2 && warp < kEpiWarp0) {
        // ============================================================ gathers
        // Stage k of the MMA sequence lands in slot k % NA of the A ring. The
        // eight gather warps share the NA slots: warp gw fills part gw / NA
        // (128 / WPS consecutive rows, all CPS chunks) of every stage that
        // lands in slot gw % NA, waits for its own copies and arrives once;
        // the slot's barrier completes when all WPS parts have arrived. Every
        // producer of a slot waits for the slot's release before refilling it.
        const int gw = warp < kMmaWarp ? warp - 1 : warp - 2;   // 0..7
        const int aslot = gw % NA;
        const int part = gw / NA;
        const int rows_per = 128 / WPS;
        const int r_lo = part * rows_per;
        {
            const char *pool_bytes = reinterpret_cast<const char *>(a.pool);
            const int seg = lane & 7;            // 16-byte segment of a 128-byte row chunk
            const int r_in = lane >> 3;          // row within a 4-row group
            const uint32_t dst0 = smem_u32(a_buf + aslot * kAStage);
            const uint32_t row_bytes = (uint32_t)a.D * 2u;
            if (lane == 0) {
                tma_prefetch_desc(&mapP);
                if (WIN)
                    tma_prefetch_desc(&mapK);
            }
            uint32_t ph = 0;
            int s = 0;                           // stage index modulo NA
            bool ok = true;
            int it = 0;
            for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
                const int m3 = it % NM;
                ok = warp_mbar_wait(&sm->meta_full[m3], (it / NM) & 1, abort_flag, a.err);
                if (!ok)
                    break;
                const int nsel = sm->nsel[m3];
                const uint32_t tcontig = sm->contig[m3];
                const uint32_t *rw = rowoff + m3 * Kp;
                const int nt = (nsel + 127) / 128;
                const int G = n_groups(nsel, TB);
                const int passes = G > 1 && !kSpill ? 2 : 1;
                // WIN: Kw row of the window tile's first row (the box's last
                // row is the token's own key; negative rows read as zeros)
                int wrow0 = 0;
                if constexpr (WIN) {
                    const int g = a.n_tok - 1 - gt;
                    const int b = g / a.S;
                    wrow0 = b * a.kw_rows + a.kw_lead + (g - b * a.S) - (a.kw_box_rows - 1);
                }
                for (int pass = WIN ? -1 : 0; pass < passes && ok; ++pass) {
                    const bool wpass = WIN && pass < 0;   // the window tile
                    const int GP = wpass ? 1 : G;
                    for (int grp = 0; grp < GP && ok; ++grp) {
                        const int i0 = grp * TB;
                        const int ntg = wpass ? 1 : min(nt, i0 + TB) - i0;
                        for (int cp = 0; cp < n_cp && ok; ++cp) {
                            for (int i = 0; i < ntg; ++i) {
                                const bool mine = (s == aslot);
                                if (++s == NA)
                                    s = 0;
                                if (!mine)
                                    continue;
                                ok = warp_mbar_wait(&sm->a_empty[aslot], ph ^ 1u, abort_flag, a.err);
                                if (!ok)
                                    break;
                                const int tile_row0 = (i0 + i) * 128;
                                const int rows = min(128, nsel - tile_row0);
                                const uint32_t *ro = rw + tile_row0;
                                if (wpass) {
                                    if (lane == 0) {
                                        if (part == 0) {
                                            mbar_arrive_expect_tx(&sm->a_full[aslot],
                                                                  (uint32_t)(CPS * a.kw_box_rows) * 128u);
#pragma unroll
                                            for (int cc = 0; cc < CPS; ++cc)
                                                tma_load_2d(a_buf + aslot * kAStage + cc * kATile, &mapK,
                                                            &sm->a_full[aslot], (cp * CPS + cc) * 64, wrow0);
                                        } else {
                                            mbar_arrive(&sm->a_full[aslot]);
                                        }
                                    }
                                    __syncwarp();
                                } else if ((tcontig >> (i0 + i)) & 1u) {
                                    // a tile whose rows are consecutive pool rows (the compaction
                                    // warp marks it) is one TMA box per chunk
                                    const uint32_t ro0 = ro[0];
                                    if (lane == 0) {
                                        if (part == 0) {
                                            mbar_arrive_expect_tx(&sm->a_full[aslot],
                                                                  (uint32_t)(CPS * a.pool_box_rows) * 128u);
#pragma unroll
                                            for (int cc = 0; cc < CPS; ++cc)
                                                tma_load_2d(a_buf + aslot * kAStage + cc * kATile, &mapP,
                                                            &sm->a_full[aslot], (cp * CPS + cc) * 64,
                                                            (int32_t)(ro0 / row_bytes));
                                        } else {
                                            mbar_arrive(&sm->a_full[aslot]);
                                        }
                                    }
                                    __syncwarp();
                                } else {
                                    // one row-offset load and address computation per row, reused
                                    // for each of the stage's CPS chunks
                                    const char *src0 = pool_bytes + cp * CPS * 128 + seg * 16;
#pragma unroll 4
                                    for (int j = 0; j < rows_per / 4; ++j) {
                                        const int r = r_lo + 4 * j + r_in;
                                        if (r < rows) {
                                            const char *src = src0 + ro[r];
                                            const uint32_t d = dst0 + r * 128 + ((seg ^ (r & 7)) << 4);
#pragma unroll
                                            for (int cc = 0; cc < CPS; ++cc)
                                                cp_async16(d + cc * kATile, src + cc * 128);
                                        }
                                    }
                                    cp_async_commit();
                                    cp_async_wait<0>();
                                    fence_proxy_async_smem();
                                    __syncwarp();
                                    if (lane == 0)
                                        mbar_arrive(&sm->a_full[aslot]);
                                    __syncwarp();
                                }
                                ph ^= 1u;
                            }
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp || warp == kMmaWarp2) {
        // ============================================================ MMA
        // Two threads issue the MMAs (one cannot keep the pipe busy: an MMA
        // instruction holds its issuing thread for longer than the pipe takes
        // to run it, and every barrier wait and commit adds to that). Thread
        // mt takes the tiles i with i % 2 == mt, so each accumulator's chain of
        // chunks stays with one thread, and the other thread's MMAs keep the
        // pipe busy through this one's waits and commits. Both walk the whole
        // stage sequence of the shared A ring: each waits for every stage to be
        // filled, the owner issues its MMAs and commits the slot's release,
        // the other thread adds a plain arrival (the release barrier counts
        // two). So no slot is refilled before both threads have passed its
        // current use, and neither thread can meet a slot two phases ahead of
        // the use it waits for. Both release every Q entry and every TMEM
        // group.
        const int mt = (warp == kMmaWarp) ? 0 : 1;
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, HH);
            int as = 0, qs = 0;
            uint32_t aph = 0, qph = 0;
            bool ok = true, issued = false;
            int it = 0;
            int jobs0 = 0, jobs1 = 0;
            int gseq = 0;                        // accumulator groups so far: they alternate buffers
            int tn = 0, gq = 0;                  // WIN: tiles and groups so far (the TMEM ring)
            for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
                const int m3 = it % NM;
                if (!mbar_wait(&sm->meta_full[m3], (it / NM) & 1, abort_flag, a.err)) {
                    ok = false;
                    break;
                }
                const int nsel = sm->nsel[m3];
                const int nt = (nsel + 127) / 128;
                const int G = n_groups(nsel, TB);
                const int passes = G > 1 && !kSpill ? 2 : 1;
                for (int pass = WIN ? -1 : 0; pass < passes && ok; ++pass) {
                    const bool wpass = WIN && pass < 0;   // the window tile
                    const int GP = wpass ? 1 : G;
                    // the window tile's owner alternates token by token, so both
                    // threads issue window MMAs
                    const int wown = wpass ? (it & 1) : 0;
                    for (int grp = 0; grp < GP && ok; ++grp) {
                        const int i0 = grp * TB;
                        const int ntg = wpass ? 1 : min(nt, i0 + TB) - i0;
                        const int mb = gseq & 1;
                        ++gseq;
                        const uint32_t dbase = tmem + mb * 256;
                        int n0 = 0;
                        if constexpr (WIN) {
                            // both threads wait for every slot of the group, so neither
                            // commits a group before the epilogue has taken the group
                            // that used its commit barrier kSlots groups earlier
                            n0 = tn;
                            tn += ntg;
                            for (int i = 0; i < ntg && ok; ++i) {
                                const int n = n0 + i;
                                ok = mbar_wait(&ring->slot_empty[n & (kSlots - 1)], ((n / kSlots) & 1) ^ 1u,
                                               abort_flag, a.err);
                            }
                            if (!ok)
                                break;
                        } else {
                            const int jb = mb ? jobs1 : jobs0;
                            if (!mbar_wait(&sm->acc_empty[mb], (jb & 1) ^ 1u, abort_flag, a.err)) {
                                ok = false;
                                break;
                            }
                            if (mb)
                                ++jobs1;
                            else
                                ++jobs0;
                        }
                        for (int cp = 0; cp < n_cp && ok; ++cp) {
                            if (!mbar_wait(&sm->q_full[qs], qph, abort_flag, a.err)) {
                                ok = false;
                                break;
                            }
                            const uint64_t dq = sdesc_k_sw128(smem_u32(q_buf + qs * kQEntry));
                            for (int i = 0; i < ntg; ++i) {
                                if (!mbar_wait(&sm->a_full[as], aph, abort_flag, a.err)) {
                                    ok = false;
                                    break;
                                }
                                if (((i + wown) & 1) != mt) {
                                    mbar_arrive(&sm->a_empty[as]);
                                    if (++as == NA) {
                                        as = 0;
                                        aph ^= 1u;
                                    }
                                    continue;
                                }
                                tc_fence_after();
                                const uint64_t da = sdesc_k_sw128(smem_u32(a_buf + as * kAStage));
                                const uint32_t d_tmem =
                                    WIN ? tmem + (uint32_t)(((n0 + i) & (kSlots - 1)) * HH) : dbase + i * HH;
                                // CPS chunks x 4 K-steps; chunks are kATile bytes apart in A and
                                // kQTile in Q (descriptor start addresses are in 16-byte units)
#pragma unroll
                                for (int cc = 0; cc < CPS; ++cc)
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        umma_bf16(d_tmem, da + (uint64_t)(cc * (kATile >> 4)) + 2 * kk,
                                                  dq + (uint64_t)(cc * (kQTile >> 4)) + 2 * kk, idesc,
                                                  ((cp * CPS + cc) | kk) != 0);
                                umma_commit(&sm->a_empty[as]);
                                issued = true;
                                if (++as == NA) {
                                    as = 0;
                                    aph ^= 1u;
                                }
                            }
                            if (!ok)
                                break;
                            umma_commit(&sm->q_empty[qs]);
                            if (++qs == QS) {
                                qs = 0;
                                qph ^= 1u;
                            }
                        }
                        if (!ok)
                            break;
                        if constexpr (WIN) {
                            umma_commit(&ring->grp_full[gq & (kSlots - 1)]);
                            ++gq;
                        } else {
                            umma_commit(&sm->acc_full[mb]);
                        }
                    }
                }
            }
            if (!ok && issued) {
                umma_commit(&sm->drain[mt]);
                mbar_drain(&sm->drain[mt], 0);
            }
        }
        __syncwarp();
    }
    } else {
        // ============================================================ epilogue
        // Both epilogue warpgroups work on every token. For H >= 32 warpgroup
        // hf takes the heads [hf*H/2, (hf+1)*H/2) of every tile of a TMEM
        // group: a thread (one TMEM lane = one slot row per tile) reduces its
        // own rows first, so a column needs one cross-lane reduction per
        // warp whatever the tile count; the column max is one redux per
        // column. The two halves of each row's u are added through shared
        // memory. (For H = 16 warpgroup hf takes half the tiles instead.)
        // Per-head statistics are combined across warps through shared memory.
        // warpgroups 3 and 4 execute this one setmaxnreg together
        regs_inc<kHighRegs>();
        constexpr int TBH = TB / 2;           // tiles per warpgroup and group (H = 16)
        constexpr int IBH = TBH < 2 ? TBH : 2; // tiles per TMEM load batch (H = 16)
        // H >= 32: warpgroup hf takes heads [hf*HC, (hf+1)*HC) of every tile
        constexpr int HC = HH / 2;
        constexpr int NCB = HC >= 16 ? HC / 16 : 1;
        constexpr int IB = TB < 2 ? TB : 2;   // tiles per TMEM load batch
        const int ew = warp - kEpiWarp0;      // 0..7
        const int hf = ew >> 2;               // which half of the heads (H >= 32) or tiles (H = 16)
        const int c_lo = hf * HC;
        const int q = warp & 3;               // TMEM lane quarter
        const int r = q * 32 + lane;          // row within a 128-slot tile
        const int et = ew * 32 + lane;        // 0..255
        constexpr uint32_t bar_id = 1;
        constexpr int kEpiThreads = 256;
        EpiState<HH> &st = sm->epi[0];
        float *ub = ubuf;
        float *uh = ubuf + Kp;                // [2][TB*128] the warpgroups' partial u (H >= 32)
        const float s2 = a.scale * kLog2e;    // scale > 0 (checked on the host)
        const float sink_h = (a.sink && et < HH) ? a.sink[et] : -INFINITY;
        int jobs0 = 0, jobs1 = 0;
        int gseq = 0;                         // accumulator groups so far (as the MMA threads count)
        int tn = 0, gq = 0;                   // WIN: tiles and groups so far (the TMEM ring)
        // fused KL: the global count N of rows with a valid slot, and this
        // CTA's running KL sum (thread et == 0, fixed token order)
        const bool kl = FUSE_KL;
        float kl_c = 0.f;
        int kl_n = 0;
        double kl_acc = 0.0;
        if (kl) {
            int n = 0;
            for (int i = et; i < a.kl_count_blocks; i += kEpiThreads)
                n += a.kl_count_part[i];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
                n += __shfl_xor_sync(0xffffffffu, n, o);
            if (lane == 0)
                st.red_m[ew] = __int_as_float(n);
            named_bar_sync(bar_id, kEpiThreads);
#pragma unroll
            for (int w = 0; w < 8; ++w)
                kl_n += __float_as_int(st.red_m[w]);
            kl_c = a.kl_coeff / (float)(kl_n > 1 ? kl_n : 1);
            named_bar_sync(bar_id, kEpiThreads);
        }
        for (int it = 0; blockIdx.x + it * (int)gridDim.x < a.n_tok; ++it) {
            const int gt = blockIdx.x + it * gridDim.x;
            const int g = a.n_tok - 1 - gt;
            const int m3 = it % NM;
            // window log-mass of this token's heads, fetched early (WIN: taken
            // from the window tile)
            float wl_h = (!WIN && et < HH && a.wl) ? a.wl[(size_t)g * HH + et] : 0.f;
            // the first warp waits; the barrier hands the outcome to everyone
            bool fm = true;
            if (ew == 0)
                fm = warp_mbar_wait(&sm->meta_full[m3], (it / NM) & 1, abort_flag, a.err);
            if (!named_bar_and(bar_id, kEpiThreads, fm))
                break;
            const int nsel = sm->nsel[m3];
            const int nt = (nsel + 127) / 128;
            const int G = n_groups(nsel, TB);
            const int passes = G > 1 ? 2 : 1;
            // more than one group and a spill buffer: the second pass reads the
            // groups' raw scores back instead of waiting for them again
            const bool spill = kSpill && G > 1;
            // with the spill: the last group's scores stay in TMEM (their
            // exponentials stored there, as for a single group) until its u
            // pass, the first of the second pass; only the earlier groups
            // are spilled and read back
            const bool keep = spill;
            int mb_keep = 0, n0_keep = 0;
            float *scr = kSpill ? a.spill + (size_t)blockIdx.x * a.spill_stride : nullptr;
            float *prow = a.p + (size_t)g * K;
            const int32_t *sl = slot + m3 * Kp;
            const bool ident = sm->ident[m3] != 0;    // slot jj of the compacted order is slot jj
            const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
            // fused KL: this thread's scores and valid flags (slots et, et+256),
            // loaded now so the latency is hidden behind the token's MMAs
            constexpr int kKlReg = 2;
            float kl_s[kKlReg];
            uint8_t kl_v[kKlReg];
            if (kl) {
#pragma unroll
                for (int i = 0; i < kKlReg; ++i) {
                    const int jj = et + i * kEpiThreads;
                    const bool in = jj < K;
                    const size_t gi = (size_t)g * K + (in ? (ident ? jj : sl[jj]) : 0);
                    kl_s[i] = in ? a.kl_scores[gi] : 0.f;
                    kl_v[i] = in ? a.kl_valid[gi] : 0;
                }
            }
            // WIN: the token's window tile, its first TMEM group: wait for it,
            // take each head's log-sum-exp over the window keys into wl_h and
            // release its slot at once. Tile row r holds the key kw_box_rows - 1 - r positions
            // before the token; rows [wr_lo, kw_box_rows) are the window
            // [max(d0, t - W + 1), t]. Per 8-column block the stabiliser of a
            // column is the warp's maximum (one redux), then the warp's column
            // sums; the four lane quarters' (max, sum) pairs are merged per
            // head. False: a wait gave up.
            auto window_tile = [&](int gw, float *wl_dst) -> bool {
                if constexpr (WIN) {
                const int bw = gw / a.S;
                const int tw_pos = gw - bw * a.S + a.t_begin;
                int d0 = 0;
                if (a.doc_start) {
                    d0 = a.doc_start[gw];
                    d0 = d0 < 0 ? 0 : (d0 > tw_pos ? tw_pos : d0);
                }
                const int wr_lo = a.kw_box_rows - 1 - (tw_pos - max(d0, tw_pos - a.win + 1));
                const int nw = tn++;
                bool fw = true;
                if (ew == 0)
                    fw = warp_mbar_wait(&ring->grp_full[gq & (kSlots - 1)], (gq / kSlots) & 1, abort_flag, a.err);
                fw = named_bar_and(bar_id, kEpiThreads, fw);
                ++gq;
                if (!fw)
                    return false;
                tc_fence_after();
                const uint32_t tw = tlane + (uint32_t)((nw & (kSlots - 1)) * HH);
                const bool rv = r >= wr_lo && r < a.kw_box_rows;
#pragma unroll 1
                for (int cb = 0; cb < HC / 8; ++cb) {
                    const int col0 = c_lo + cb * 8;
                    uint32_t v[8];
                    tmem_ld8(tw + col0, v);
                    tmem_ld_wait();
                    float m8[8];
                    float mine = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        m8[e] = warp_max_f32(rv ? __uint_as_float(v[e]) : -INFINITY) * s2;
                        mine = lane == e ? m8[e] : mine;
                    }
                    float s8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        s8[e] = rv ? ex2_approx(fmaf(__uint_as_float(v[e]), s2, -m8[e])) : 0.f;
                    const float red = warp_colreduce8(s8, OpAdd());
                    if (lane < 8) {
                        ring->wred_max[q][col0 + lane] = mine;
                        ring->wred_sum[q][col0 + lane] = red;
                    }
                }
                tc_fence_before();
                named_bar_sync(bar_id, kEpiThreads);
                if (lane == 0)
                    mbar_arrive(&ring->slot_empty[nw & (kSlots - 1)]);
                __syncwarp();
                if (et < HH) {
                    float gm = ring->wred_max[0][et];
#pragma unroll
                    for (int w = 1; w < 4; ++w)
                        gm = fmaxf(gm, ring->wred_max[w][et]);
                    float gs = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        gs += ring->wred_sum[w][et] * exp2f(ring->wred_max[w][et] - gm);
                    // the token's own key is always in its window: gm is finite
                    const float wl = (gm + log2f(gs)) * 0.69314718055994531f;
                    *wl_dst = wl;
                    if (a.wl_out)
                        a.wl_out[(size_t)gw * HH + et] = wl;
                }
                // wred_* are written again only after the next window tile's
                // wait, a barrier every thread passes first
                }
                return true;
            };
            float m_part = 0.f;
            float At = 0.f;
            bool ok = true;
            for (int pass = WIN ? -1 : 0; pass < passes && ok; ++pass) {
                if constexpr (WIN) {
                    if (pass < 0) {
                        if (!window_tile(g, &wl_h))
                            ok = false;
                        continue;
                    }
                }
                for (int gi = 0; gi < G; ++gi) {
                    const int grp = (keep && pass == 1) ? (gi == 0 ? G - 1 : gi - 1) : gi;
                    const int i0 = grp * TB;
                    const int ntg = min(nt, i0 + TB) - i0;
                    // this warpgroup's tiles of the group: [t0, t1) (possibly empty)
                    const int t0 = hf * TBH;
                    const int t1 = min(ntg, t0 + TBH);
                    const bool kept = keep && grp == G - 1;       // scores stay in TMEM across the passes
                    const bool held = kept && pass == 1;          // waited for in the first pass
                    const bool from_spill = spill && pass == 1 && !kept;   // this group's scores are in scr
                    // groups alternate between the two accumulators (a spilled
                    // group's second pass reads no accumulator)
                    const int mb = held ? mb_keep : (gseq & 1);
                    if (!from_spill && !held)
                        ++gseq;
                    const uint32_t tbase = tlane + mb * 256;
                    int n0 = 0;
                    if constexpr (WIN) {
                        if (held) {
                            n0 = n0_keep;
                        } else if (!from_spill) {
                            n0 = tn;
                            tn += ntg;
                        }
                    }
                    if (kept && pass == 0) {
                        mb_keep = mb;
                        n0_keep = n0;
                    }
                    // TMEM address of tile i of the group (this thread's lane quarter)
                    auto tcol = [&](int i) -> uint32_t {
                        if constexpr (WIN)
                            return tlane + (uint32_t)(((n0 + i) & (kSlots - 1)) * HH);
                        else
                            return tbase + (uint32_t)(i * HH);
                    };
                    if (!from_spill && !held) {
                        bool fa = true;
                        if (ew == 0) {
                            if constexpr (WIN) {
                                fa = warp_mbar_wait(&ring->grp_full[gq & (kSlots - 1)], (gq / kSlots) & 1,
                                                    abort_flag, a.err);
                            } else {
                                const int jb = mb ? jobs1 : jobs0;
                                fa = warp_mbar_wait(&sm->acc_full[mb], jb & 1, abort_flag, a.err);
                            }
                        }
                        fa = named_bar_and(bar_id, kEpiThreads, fa);
                        if constexpr (WIN) {
                            ++gq;
                        } else {
                            if (mb)
                                ++jobs1;
                            else
                                ++jobs0;
                        }
                        if (!fa) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const bool single = (G == 1);
                    const bool e_tmem = single || kept;   // exponentials kept in TMEM (H >= 64)
                    if constexpr (HH >= 32) {
                    if (pass == 0) {
                    if constexpr (TB <= 4) {
                        // ---- one pass over the group's scores. Per 8-column block,
                        // every tile's values of this thread's rows come in at once;
                        // the stabiliser of a column is the warp's maximum over its
                        // 32 lanes x TB rows (one redux per column), e = 2^(v s2 -
                        // that) over valid rows (kept in TMEM for a single group),
                        // and the column sums are taken over the warp. The four TMEM
                        // lane quarters' (max, sum) pairs are merged per head below;
                        // the quarter maxima stay in red_max for the u pass.
#pragma unroll 1
                        for (int cb = 0; cb < HC / 8; ++cb) {
                            const int col0 = c_lo + cb * 8;
                            uint32_t v[TB][8];
#pragma unroll
                            for (int i = 0; i < TB; ++i)
                                if (i < ntg)
                                    tmem_ld8(tcol(i) + col0, v[i]);
                            tmem_ld_wait();
                            if (spill && !kept) {
                                // raw scores, lane-contiguous per (tile, head)
#pragma unroll
                                for (int i = 0; i < TB; ++i)
                                    if (i < ntg) {
                                        float *dst = scr + ((size_t)(grp * TB + i) * HH + col0) * 128 + r;
#pragma unroll
                                        for (int e = 0; e < 8; ++e)
                                            __stcg(dst + e * 128, __uint_as_float(v[i][e]));
                                    }
                            }
                            float m8[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                m8[e] = -INFINITY;
#pragma unroll
                            for (int i = 0; i < TB; ++i) {
                                if (i < ntg && (i0 + i) * 128 + r < nsel) {
#pragma unroll
                                    for (int e = 0; e < 8; ++e)
                                        m8[e] = fmaxf(m8[e], __uint_as_float(v[i][e]));
                                }
                            }
                            float mine = -INFINITY;
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                m8[e] = warp_max_f32(m8[e]) * s2;
                                mine = lane == e ? m8[e] : mine;
                            }
                            float s8[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                s8[e] = 0.f;
#pragma unroll
                            for (int i = 0; i < TB; ++i) {
                                if (i < ntg) {
                                    if ((i0 + i) * 128 + r < nsel) {
#pragma unroll
                                        for (int e = 0; e < 8; ++e) {
                                            const float x = ex2_approx(fmaf(__uint_as_float(v[i][e]), s2, -m8[e]));
                                            s8[e] += x;
                                            v[i][e] = __float_as_uint(x);
                                        }
                                    } else {
#pragma unroll
                                        for (int e = 0; e < 8; ++e)
                                            v[i][e] = 0u;
                                    }
                                }
                            }
                            if (e_tmem) {
#pragma unroll
                                for (int i = 0; i < TB; ++i)
                                    if (i < ntg)
                                        tmem_st8(tcol(i) + col0, v[i]);
                            }
                            const float red = warp_colreduce8(s8, OpAdd());
                            if (lane < 8) {
                                st.red_max[q][col0 + lane] = mine;
                                st.red_sum[q][col0 + lane] = red;
                            }
                        }
                        if (e_tmem)
                            tmem_st_wait();
                        named_bar_sync(bar_id, kEpiThreads);
                        if (et < HH) {
                            // group statistics in the log2 domain: max M2, sum S
                            float gm = st.red_max[0][et];
#pragma unroll
                            for (int w = 1; w < 4; ++w)
                                gm = fmaxf(gm, st.red_max[w][et]);
                            float gs = 0.f;
                            if (gm != -INFINITY) {
#pragma unroll
                                for (int w = 0; w < 4; ++w)
                                    gs += st.red_sum[w][et] * exp2f(st.red_max[w][et] - gm);
                            }
                            if (grp == 0) {
                                st.colM[et] = gm;
                                st.colS[et] = gs;
                            } else {
                                const float M0 = st.colM[et], S0 = st.colS[et];
                                const float M1 = fmaxf(M0, gm);
                                st.colS[et] = S0 * exp2f(M0 - M1) + gs * exp2f(gm - M1);
                                st.colM[et] = M1;
                            }
                        }
                    } else {
                            // ---- column max of the raw dot products over valid rows:
                            // over this thread's rows first, then across the warp's
                            // lanes in one instruction per column
#pragma unroll
                            for (int cb = 0; cb < NCB; ++cb) {
                                const int col0 = c_lo + cb * 16;
                                float m16[16];
#pragma unroll
                                for (int e = 0; e < 16; ++e)
                                    m16[e] = -INFINITY;
#pragma unroll
                                for (int ib = 0; ib < TB; ib += IB) {
                                    if (ib >= ntg)
                                        break;
                                    uint32_t v[IB][16];
#pragma unroll
                                    for (int i = 0; i < IB; ++i)
                                        if (ib + i < ntg)
                                            tmem_ld16(tcol(ib + i) + col0, v[i]);
                                    tmem_ld_wait();
#pragma unroll
                                    for (int i = 0; i < IB; ++i) {
                                        if (ib + i < ntg && (i0 + ib + i) * 128 + r < nsel) {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                m16[e] = fmaxf(m16[e], __uint_as_float(v[i][e]));
                                        }
                                    }
                                }
                                float mine = -INFINITY;
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    const float wmax = warp_max_f32(m16[e]);
                                    mine = lane == e ? wmax : mine;
                                }
                                if (lane < 16)
                                    st.red_max[q][col0 + lane] = mine;
                            }
                            named_bar_sync(bar_id, kEpiThreads);
                            if (et < HH) {
                                float mx = st.red_max[0][et];
#pragma unroll
                                for (int w = 1; w < 4; ++w)
                                    mx = fmaxf(mx, st.red_max[w][et]);
                                st.head_a[et] = mx * s2;
                            }
                            named_bar_sync(bar_id, kEpiThreads);
                            // ---- e = 2^(v s2 - max s2), column sums; one group: keep e in TMEM
#pragma unroll
                            for (int cb = 0; cb < NCB; ++cb) {
                                const int col0 = c_lo + cb * 16;
                                float s16[16], m16[16];
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    s16[e] = 0.f;
                                    m16[e] = st.head_a[col0 + e];
                                }
#pragma unroll
                                for (int ib = 0; ib < TB; ib += IB) {
                                    if (ib >= ntg)
                                        break;
                                    uint32_t v[IB][16];
#pragma unroll
                                    for (int i = 0; i < IB; ++i)
                                        if (ib + i < ntg)
                                            tmem_ld16(tcol(ib + i) + col0, v[i]);
                                    tmem_ld_wait();
#pragma unroll
                                    for (int i = 0; i < IB; ++i) {
                                        if (ib + i < ntg) {
                                            if ((i0 + ib + i) * 128 + r < nsel) {
#pragma unroll
                                                for (int e = 0; e < 16; ++e) {
                                                    const float x =
                                                        ex2_approx(fmaf(__uint_as_float(v[i][e]), s2, -m16[e]));
                                                    s16[e] += x;
                                                    v[i][e] = __float_as_uint(x);
                                                }
                                            } else {
#pragma unroll
                                                for (int e = 0; e < 16; ++e)
                                                    v[i][e] = 0u;
                                            }
                                        }
                                    }
                                    if (single) {
#pragma unroll
                                        for (int i = 0; i < IB; ++i)
                                            if (ib + i < ntg)
                                                tmem_st16(tcol(ib + i) + col0, v[i]);
                                    }
                                }
                                const float red = warp_colreduce16(s16, OpAdd());
                                if (lane < 16)
                                    st.red_sum[q][col0 + lane] = red;
                            }
                            if (single)
                                tmem_st_wait();
                            named_bar_sync(bar_id, kEpiThreads);
                            if (et < HH) {
                                // group statistics in the log2 domain: max M2, sum S
                                const float gm = st.head_a[et];
                                float gs = 0.f;
#pragma unroll
                                for (int w = 0; w < 4; ++w)
                                    gs += st.red_sum[w][et];
                                if (grp == 0) {
                                    st.colM[et] = gm;
                                    st.colS[et] = gs;
                                } else {
                                    const float M0 = st.colM[et], S0 = st.colS[et];
                                    const float M1 = fmaxf(M0, gm);
                                    st.colS[et] = S0 * exp2f(M0 - M1) + gs * exp2f(gm - M1);
                                    st.colM[et] = M1;
                                }
                            }
                    }
                        named_bar_sync(bar_id, kEpiThreads);
                    }
                    } else {
                    if (pass == 0) {
                        // ---- column max of the raw dot products over valid rows
                        for (int cc = 0; cc < NC16; ++cc) {
                            float v16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                v16[e] = -INFINITY;
                            for (int ib = t0; ib < t1; ib += IBH) {
                                uint32_t v[IBH][16];
#pragma unroll
                                for (int i = 0; i < IBH; ++i)
                                    if (ib + i < t1)
                                        tmem_ld16(tcol(ib + i) + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IBH; ++i) {
                                    if (ib + i < t1 && (i0 + ib + i) * 128 + r < nsel) {
#pragma unroll
                                        for (int e = 0; e < 16; ++e)
                                            v16[e] = fmaxf(v16[e], __uint_as_float(v[i][e]));
                                    }
                                }
                            }
                            const float red = warp_colreduce16(v16, OpMax());
                            if (lane < 16)
                                st.red_max[ew][cc * 16 + lane] = red;
                        }
                        named_bar_sync(bar_id, kEpiThreads);
                        if (et < HH) {
                            float mx = st.red_max[0][et];
#pragma unroll
                            for (int w = 1; w < 8; ++w)
                                mx = fmaxf(mx, st.red_max[w][et]);
                            st.head_a[et] = mx * s2;
                        }
                        named_bar_sync(bar_id, kEpiThreads);
                        // ---- e = 2^(v s2 - max s2), column sums; one group: keep e in TMEM
                        for (int cc = 0; cc < NC16; ++cc) {
                            float s16[16], m16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                s16[e] = 0.f;
                                m16[e] = st.head_a[cc * 16 + e];
                            }
                            for (int ib = t0; ib < t1; ib += IBH) {
                                uint32_t v[IBH][16];
#pragma unroll
                                for (int i = 0; i < IBH; ++i)
                                    if (ib + i < t1)
                                        tmem_ld16(tcol(ib + i) + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IBH; ++i) {
                                    if (ib + i < t1) {
                                        if ((i0 + ib + i) * 128 + r < nsel) {
#pragma unroll
                                            for (int e = 0; e < 16; ++e) {
                                                const float x =
                                                    ex2_approx(fmaf(__uint_as_float(v[i][e]), s2, -m16[e]));
                                                s16[e] += x;
                                                v[i][e] = __float_as_uint(x);
                                            }
                                        } else {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                v[i][e] = 0u;
                                        }
                                    }
                                }
                                if (single) {
#pragma unroll
                                    for (int i = 0; i < IBH; ++i)
                                        if (ib + i < t1)
                                            tmem_st16(tcol(ib + i) + cc * 16, v[i]);
                                }
                            }
                            const float red = warp_colreduce16(s16, OpAdd());
                            if (lane < 16)
                                st.red_sum[ew][cc * 16 + lane] = red;
                        }
                        if (single)
                            tmem_st_wait();
                        named_bar_sync(bar_id, kEpiThreads);
                        if (et < HH) {
                            // group statistics in the log2 domain: max M2, sum S
                            const float gm = st.head_a[et];
                            float gs = 0.f;
#pragma unroll
                            for (int w = 0; w < 8; ++w)
                                gs += st.red_sum[w][et];
                            if (grp == 0) {
                                st.colM[et] = gm;
                                st.colS[et] = gs;
                            } else {
                                const float M0 = st.colM[et], S0 = st.colS[et];
                                const float M1 = fmaxf(M0, gm);
                                st.colS[et] = S0 * exp2f(M0 - M1) + gs * exp2f(gm - M1);
                                st.colM[et] = M1;
                            }
                        }
                        named_bar_sync(bar_id, kEpiThreads);
                    }
                    }
                    if (pass == passes - 1) {
                        if (gi == 0) {
                            // ---- per-head merge with the window and the sink
                            if (et < HH) {
                                const float M = st.colM[et] * 0.69314718055994531f;  // natural log units
                                const float clse = M + logf(st.colS[et]);
                                if (a.lse_mode == kLsePerBranch) {
                                    // each head normalised over its selected entries alone
                                    st.head_a[et] = M - clse;
                                } else if (a.lse_mode == kLseGiven) {
                                    // the whole row's normaliser, as the attention forward gave it
                                    st.head_a[et] = M - wl_h;
                                } else {
                                    float mm = fmaxf(fmaxf(wl_h, clse), sink_h);
                                    float acc = expf(wl_h - mm) + expf(clse - mm);
                                    if (a.sink)
                                        acc += expf(sink_h - mm);
                                    st.head_a[et] = M - (mm + logf(acc));
                                }
                            }
                            named_bar_sync(bar_id, kEpiThreads);
                            float x = -INFINITY;
                            for (int h = lane; h < HH; h += 32)
                                x = fmaxf(x, st.head_a[h]);
#pragma unroll
                            for (int o = 16; o >= 1; o >>= 1)
                                x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                            At = x;
                            if (et < HH) {
                                const float wp = expf(st.head_a[et] - At);
                                st.wprime[et] = wp;
                                if constexpr (HH >= 32 && TB <= 4) {
                                    // a single (or the kept last) group's e are relative
                                    // to their lane quarter's maximum: fold the rescale
                                    // to the head's maximum into the weight, per quarter
                                    if (single || keep) {
#pragma unroll
                                        for (int w = 0; w < 4; ++w)
                                            st.red_max[w][et] = wp * exp2f(st.red_max[w][et] - st.colM[et]);
                                    }
                                }
                            }
                            named_bar_sync(bar_id, kEpiThreads);
                        }
                        if constexpr (HH >= 32) {
                        // ---- u'[k] = sum_h e[k,h] w[h]: each warpgroup sums its own
                        // heads for every tile of the group; the two partial sums of
                        // a row are added through shared memory
                        float u[TB];
#pragma unroll
                        for (int i = 0; i < TB; ++i)
                            u[i] = 0.f;
#pragma unroll
                        for (int cb = 0; cb < NCB; ++cb) {
                            const int col0 = c_lo + cb * 16;
                            float w16[16], cm16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                w16[e] = (TB <= 4 && e_tmem) ? st.red_max[q][col0 + e] : st.wprime[col0 + e];
                                cm16[e] = e_tmem ? 0.f : st.colM[col0 + e];
                            }
#pragma unroll
                            for (int ib = 0; ib < TB; ib += IB) {
                                if (ib >= ntg)
                                    break;
                                uint32_t v[IB][16];
                                if (from_spill) {
#pragma unroll
                                    for (int i = 0; i < IB; ++i)
                                        if (ib + i < ntg) {
                                            const float *src = scr + ((size_t)(grp * TB + ib + i) * HH + col0) * 128 + r;
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                v[i][e] = __float_as_uint(__ldcg(src + e * 128));
                                        }
                                } else {
#pragma unroll
                                    for (int i = 0; i < IB; ++i)
                                        if (ib + i < ntg)
                                            tmem_ld16(tcol(ib + i) + col0, v[i]);
                                    tmem_ld_wait();
                                }
#pragma unroll
                                for (int i = 0; i < IB; ++i) {
                                    if (ib + i < ntg) {
                                        float acc = u[ib + i];
                                        if (e_tmem) {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                acc = fmaf(__uint_as_float(v[i][e]), w16[e], acc);
                                        } else {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                acc = fmaf(ex2_approx(fmaf(__uint_as_float(v[i][e]), s2, -cm16[e])),
                                                           w16[e], acc);
                                        }
                                        u[ib + i] = acc;
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int i = 0; i < TB; ++i)
                            if (i < ntg)
                                uh[hf * (TB * 128) + i * 128 + r] = u[i];
                        named_bar_sync(bar_id, kEpiThreads);
                        for (int i = hf; i < ntg; i += 2) {
                            const int j = (i0 + i) * 128 + r;
                            if (j < nsel) {
                                const float uu = uh[i * 128 + r] + uh[TB * 128 + i * 128 + r];
                                ub[j] = uu;
                                m_part += uu;
                            }
                        }
                        } else {
                        // ---- u'[k] = sum_h e[k,h] w[h]
                        float u[TBH];
#pragma unroll
                        for (int i = 0; i < TBH; ++i)
                            u[i] = 0.f;
                        for (int cc = 0; cc < NC16; ++cc) {
                            float w16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                w16[e] = st.wprime[cc * 16 + e];
#pragma unroll
                            for (int ib = 0; ib < TBH; ib += IBH) {
                                if (t0 + ib >= t1)
                                    break;
                                uint32_t v[IBH][16];
#pragma unroll
                                for (int i = 0; i < IBH; ++i)
                                    if (t0 + ib + i < t1)
                                        tmem_ld16(tcol(t0 + ib + i) + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IBH; ++i) {
                                    if (t0 + ib + i < t1) {
                                        float acc = u[ib + i];
                                        if (single) {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                acc = fmaf(__uint_as_float(v[i][e]), w16[e], acc);
                                        } else {
#pragma unroll
                                            for (int e = 0; e < 16; ++e)
                                                acc = fmaf(ex2_approx(fmaf(__uint_as_float(v[i][e]), s2,
                                                                           -st.colM[cc * 16 + e])),
                                                           w16[e], acc);
                                        }
                                        u[ib + i] = acc;
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int i = 0; i < TBH; ++i) {
                            const int j = (i0 + t0 + i) * 128 + r;
                            if (t0 + i < t1 && j < nsel) {
                                ub[j] = u[i];
                                m_part += u[i];
                            }
                        }
                        }
                    }
                    if (!from_spill && !(kept && pass == 0)) {   // the kept group is released after its u pass
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (WIN) {
                                for (int i = 0; i < ntg; ++i)
                                    mbar_arrive(&ring->slot_empty[(n0 + i) & (kSlots - 1)]);
                            } else {
                                mbar_arrive(&sm->acc_empty[mb]);
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            if (!ok)
                break;
            // ---- token total and the normalised, slot-ordered output row
            float mt = m_part;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
                mt += __shfl_xor_sync(0xffffffffu, mt, o);
            if (lane == 0)
                st.red_m[ew] = mt;
            named_bar_sync(bar_id, kEpiThreads);
            float mtot = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w)
                mtot += st.red_m[w];
            float f = 0.f;
            if (nsel > 0) {
                const float ln_floor = a.lse_mode == kLsePerBranch ? kLnOldFloor : kLnFltMin;
                const bool plain = logf(mtot) + At >= ln_floor;
                f = plain ? 1.0f / mtot : expf(At - ln_floor);
            }
            if (a.p) {
                for (int jj = et; jj < K; jj += kEpiThreads)
                    prow[ident ? jj : sl[jj]] = (jj < nsel) ? ub[jj] * f : 0.f;
            }
            if (kl) {
                // ---- KL(p || softmax(scores)) over the row's valid slots and
                // its gradient, straight from the target in shared memory
                // (K <= 2 * 256 here: two slots per thread, in registers)
                const size_t rowo = (size_t)g * K;
                float pv[kKlReg];
                int kk[kKlReg];
                float mx = -INFINITY;
                bool anyv = false;
#pragma unroll
                for (int i = 0; i < kKlReg; ++i) {
                    const int jj = et + i * kEpiThreads;
                    kk[i] = jj < K ? (ident ? jj : sl[jj]) : 0;
                    pv[i] = (jj < nsel) ? ub[jj] * f : 0.f;
                    if (kl_v[i]) {
                        mx = fmaxf(mx, kl_s[i]);
                        anyv = true;
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const bool wany = __any_sync(0xffffffffu, anyv);
                if (lane == 0) {
                    st.klred[ew][0] = mx;
                    st.klred[ew][1] = wany ? 1.f : 0.f;
                }
                named_bar_sync(bar_id, kEpiThreads);
                float rmx = -INFINITY;
                bool rany = false;
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    rmx = fmaxf(rmx, st.klred[w][0]);
                    rany = rany || st.klred[w][1] != 0.f;
                }
                named_bar_sync(bar_id, kEpiThreads);
                float se = 0.f, ps = 0.f;
#pragma unroll
                for (int i = 0; i < kKlReg; ++i) {
                    if (kl_v[i]) {
                        se += __expf(kl_s[i] - rmx);
                        ps += pv[i];
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    se += __shfl_xor_sync(0xffffffffu, se, o);
                    ps += __shfl_xor_sync(0xffffffffu, ps, o);
                }
                if (lane == 0) {
                    st.klred[ew][0] = se;
                    st.klred[ew][1] = ps;
                }
                named_bar_sync(bar_id, kEpiThreads);
                float rse = 0.f, rps = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    rse += st.klred[w][0];
                    rps += st.klred[w][1];
                }
                const float lse = rany ? rmx + __logf(rse) : 0.f;
                float klv = 0.f;
#pragma unroll
                for (int i = 0; i < kKlReg; ++i) {
                    const int jj = et + i * kEpiThreads;
                    if (jj < K) {
                        const bool v = rany && kl_v[i];
                        const float logq = kl_s[i] - lse;
                        if (v && pv[i] > 0.f)
                            klv += pv[i] * (__logf(pv[i]) - logq);
                        a.kl_dscores[rowo + kk[i]] = v ? kl_c * fmaf(__expf(logq), rps, -pv[i]) : 0.f;
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
                    klv += __shfl_xor_sync(0xffffffffu, klv, o);
                named_bar_sync(bar_id, kEpiThreads);   // klred[.][0..1] read by all before reuse
                if (lane == 0)
                    st.klred[ew][2] = klv;
                named_bar_sync(bar_id, kEpiThreads);
                if (et == 0) {
                    float tk = 0.f;
#pragma unroll
                    for (int w = 0; w < 8; ++w)
                        tk += st.klred[w][2];
                    kl_acc += (double)tk;
                }
            }
            named_bar_sync(bar_id, kEpiThreads);
            if (et == 0)
                mbar_arrive(&sm->meta_empty[m3]);
            __syncwarp();
        }
        if (kl && et == 0) {
            // this CTA's KL sum; the last CTA to finish adds them in CTA order
            a.kl_part[blockIdx.x] = kl_acc;
            __threadfence();
            if (atomicAdd(a.kl_done, 1u) == gridDim.x - 1) {
                __threadfence();
                const volatile double *kp = a.kl_part;
                double tot = 0.0;
                for (int i = 0; i < (int)gridDim.x; ++i)
                    tot += kp[i];
                *a.kl_loss = (float)((double)a.kl_coeff * tot / (double)(kl_n > 1 ? kl_n : 1));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int HH, int CPS>
__host__ __device__ inline size_t fixed_smem_bytes(int K, int n_meta, int idx_stage, int win)
{
    const size_t Kp = (size_t)((K + 3) & ~3);
    const size_t uh = HH >= 32 ? (size_t)2 * (256 / HH) * 128 * 4 : 0;   // partial u of the two warpgroups
    const size_t rows = 2 * (size_t)n_meta + (idx_stage ? 3 : 0) + 1;    // row offsets, slots, idx, u'
    return 1024 + q_entries<HH, CPS>() * (size_t)(CPS * HH * 128) + Kp * 4 * rows + uh + sizeof(TgtSmem<HH>) +
           (win ? sizeof(TileRing) : 0) + 64;
}

// Deepest A-stage ring that fits the per-block smem limit, as a divisor of
// the eight gather warps (so every slot has the same number of producers),
// with two slots at least for each of the two MMA threads; 0 if none fits.
template <int HH, int CPS>
int stages_for(int K, int n_meta, int idx_stage, int win, int smem_limit)
{
    const long room = (long)smem_limit - (long)fixed_smem_bytes<HH, CPS>(K, n_meta, idx_stage, win);
    long n = room / (long)(CPS * kATile);
    if (n > kMaxAStages)
        n = kMaxAStages;
    int na = 8;
    while (na > n)
        na >>= 1;
    return na >= 4 ? na : 0;   // two slots at least for each MMA thread
}

template <int HH, int CPS>
size_t smem_bytes_for(int K, int n_meta, int idx_stage, int win, int stages)
{
    return fixed_smem_bytes<HH, CPS>(K, n_meta, idx_stage, win) + (size_t)stages * CPS * kATile;
}

template <int HH, bool FUSE_KL, int CPS, bool SPILL, bool WIN>
cudaError_t launch_hkcsw(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                         const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    auto kern = target_tc_kernel<HH, FUSE_KL, CPS, SPILL, WIN>;
    // The register split above is only safe if every thread was launched with
    // exactly kLaunchRegs registers; refuse to launch otherwise.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess)
        return e;
    if (fa.numRegs != kLaunchRegs)
        return cudaErrorInvalidConfiguration;
    if (a.n_astages < 1 || kGatherWarps % a.n_astages != 0 || (a.D / 64) % CPS != 0 ||
        (a.n_meta != 2 && a.n_meta != 4) || (a.idx_stage && !a.idx_bulk))
        return cudaErrorInvalidValue;
    // the window tile: one box of at most 128 rows, a window that fits in it
    if (WIN && (a.kw_box_rows < 1 || a.kw_box_rows > 128 || a.win < 1 || a.win > 128 || a.kw_rows < 1 ||
                a.lse_mode != kLseJoint))
        return cudaErrorInvalidValue;
    const size_t smem = smem_bytes_for<HH, CPS>(a.K, a.n_meta, a.idx_stage, WIN ? 1 : 0, a.n_astages);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<grid, kTgtThreads, smem, stream>>>(mapQ, mapP, mapK, a);
    return cudaGetLastError();
}

// The window-fused instantiation only for the plain target (no fused KL).
template <int HH, bool FUSE_KL, int CPS, bool SPILL>
cudaError_t launch_hkcs(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                        const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    if constexpr (!FUSE_KL) {
        if (a.win)
            return launch_hkcsw<HH, FUSE_KL, CPS, SPILL, true>(mapQ, mapP, mapK, a, grid, stream);
    }
    if (a.win)
        return cudaErrorInvalidValue;
    return launch_hkcsw<HH, FUSE_KL, CPS, SPILL, false>(mapQ, mapP, mapK, a, grid, stream);
}

// The spill instantiation only where it can be used (H >= 64, no fused KL).
template <int HH, bool FUSE_KL, int CPS>
cudaError_t launch_hkc(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                       const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    if constexpr (HH >= 64 && !FUSE_KL) {
        if (a.spill)
            return launch_hkcs<HH, FUSE_KL, CPS, true>(mapQ, mapP, mapK, a, grid, stream);
    }
    if (a.spill)
        return cudaErrorInvalidValue;
    return launch_hkcs<HH, FUSE_KL, CPS, false>(mapQ, mapP, mapK, a, grid, stream);
}

template <int HH, bool FUSE_KL>
cudaError_t launch_hk(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                      const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    return a.cps == 2 ? launch_hkc<HH, FUSE_KL, 2>(mapQ, mapP, mapK, a, grid, stream)
                      : launch_hkc<HH, FUSE_KL, 1>(mapQ, mapP, mapK, a, grid, stream);
}

template <int HH>
cudaError_t launch_h(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                     const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    return a.kl_scores ? launch_hk<HH, true>(mapQ, mapP, mapK, a, grid, stream)
                       : launch_hk<HH, false>(mapQ, mapP, mapK, a, grid, stream);
}

template <int HH>
int stages_h(int K, int cps, int n_meta, int idx_stage, int win, int smem_limit)
{
    return cps == 2 ? stages_for<HH, 2>(K, n_meta, idx_stage, win, smem_limit)
                    : stages_for<HH, 1>(K, n_meta, idx_stage, win, smem_limit);
}

}  // namespace

int target_tc_stages(int H, int K, int cps, int n_meta, int idx_stage, int win, int smem_limit)
{
    switch (H) {
    case 16: return stages_h<16>(K, cps, n_meta, idx_stage, win, smem_limit);
    case 32: return stages_h<32>(K, cps, n_meta, idx_stage, win, smem_limit);
    case 64: return stages_h<64>(K, cps, n_meta, idx_stage, win, smem_limit);
    case 128: return stages_h<128>(K, cps, n_meta, idx_stage, win, smem_limit);
    default: return 0;
    }
}

cudaError_t launch_target_tc(const CUtensorMap &mapQ, const CUtensorMap &mapP, const CUtensorMap &mapK,
                             const TgtTcArgs &a, int grid, cudaStream_t stream)
{
    switch (a.H) {
    case 16: return launch_h<16>(mapQ, mapP, mapK, a, grid, stream);
    case 32: return launch_h<32>(mapQ, mapP, mapK, a, grid, stream);
    case 64: return launch_h<64>(mapQ, mapP, mapK, a, grid, stream);
    case 128: return launch_h<128>(mapQ, mapP, mapK, a, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace sai
