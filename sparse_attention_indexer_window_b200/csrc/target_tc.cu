// Distillation target on tcgen05 tensor cores with an in-kernel TMA gather of
// the selected pool rows (sm_100a).
//
// For every token (b,t) (Primus page "perf(deepseek-v4): fuse and enable the
// indexer distillation loss": first commit message -- the pool is indexed
// inside the kernel so the [B,S,K,D] gather never exists; second commit
// message / "Why the target was wrong" -- one softmax over window keys,
// selected compressed entries and the per-head sink):
//
//   z[k,h]      = scale <pool[idx[k]], Q[t,h]>       selected slots k
//   clse[h]     = log sum_k exp z[k,h]
//   lse_full[h] = logsumexp(window_lse[t,h], clse[h], sink[h])
//   u[k]        = sum_h exp(z[k,h] - lse_full[h]),  p[k] = u[k] / max(sum u, FLT_MIN)
//
// Layout of the contraction. The problem is transposed so the MMA keeps M=128
// although a token has only H heads: A = 128 gathered pool rows (one TMEM lane
// per selected slot), B = Q[t] (N = H columns, one per head), K-dim = D in
// 64-element (128-byte, swizzled) chunks. The producer compacts the token's
// idx row (selected slots first, masked slots last) and gathers the selected
// rows four at a time with TMA tile::gather4 straight into the swizzled smem
// operand layout; masked slots are never loaded.
//
// The epilogue needs the per-head log-sum-exp over ALL selected slots before
// it can form u, so a token's scores stay in TMEM until it is done: up to
// 256/H tiles (512 slots at H=64) per accumulator, two accumulators so the
// epilogue of one token overlaps the MMA of the next. Tokens with more
// selected slots run in groups: a first pass over the groups merges per-head
// (max, sum-exp) statistics, a second pass recomputes each group's scores and
// forms u.
//
// Epilogue arithmetic (one exponential per score):
//   M[h] = max_k z[k,h]  (column max: transposing warp butterfly + smem)
//   e[k,h] = exp(z[k,h] - M[h]) written back to TMEM, S[h] = sum_k e[k,h]
//   a[h] = M[h] - lse_full[h],  A = max_h a[h],  w[h] = exp(a[h] - A) in (0,1]
//   u'[k] = sum_h e[k,h] w[h]   (per thread, one TMEM lane = one slot)
//   m' = sum_k u'[k] >= 1, and u = u' e^A, m = m' e^A, so
//   p[k] = u'[k]/m'              if log m' + A >= log FLT_MIN
//        = u'[k] exp(A - log FLT_MIN)   otherwise (the float32-tiny floor),
// which never forms a subnormal intermediate however small the compressed
// share of every head is.
//
// Warp roles (192 threads): warp 0 producer (idx compaction by the whole
// warp, TMA by lane 0; TMEM owner), warp 1 MMA issuer, warps 2..5 epilogue.
// Persistent CTAs walk tokens from the last (heaviest) to the first. All
// waits are bounded; a timeout is reported through err and the CTA unwinds.
#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

constexpr int kTgtThreads = 192;
constexpr int kAStages = 6;
constexpr int kQStages = 3;
constexpr uint32_t kATile = 128 * 128;  // 128 rows x 128 bytes
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLnFltMin = -87.33654475055310898657f;  // log(2^-126)

template <int HH>
struct TgtSmem {
    uint64_t a_full[kAStages], a_empty[kAStages];
    uint64_t q_full[kQStages], q_empty[kQStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t meta_full[2], meta_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int nsel[2];
    float red_max[4][HH];
    float red_sum[4][HH];
    float colM[HH];
    float colS[HH];
    float head_a[HH];
    float wprime[HH];
    float red_m[4];
};

struct Job {
    int pass;    // 0 = statistics only, 1 = final (u)
    int grp;
};

__device__ __forceinline__ int n_groups(int nsel, int TB)
{
    const int nt = (nsel + 127) / 128;
    return (nt + TB - 1) / TB;
}

template <int HH>
__global__ void __launch_bounds__(kTgtThreads, 1)
    target_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapPool,
                     const TgtTcArgs a)
{
    constexpr int TB = 256 / HH;                 // tiles per accumulator
    constexpr int IB = TB < 4 ? TB : 4;          // tiles per TMEM load batch
    constexpr uint32_t kQTile = HH * 128;        // H rows x 128 bytes
    constexpr int NC16 = HH / 16;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *a_buf = base;                               // kAStages x 16 KB
    uint8_t *q_buf = a_buf + kAStages * kATile;          // kQStages x H*128
    int32_t *rowid = reinterpret_cast<int32_t *>(q_buf + kQStages * kQTile);  // [2][K]
    int32_t *slot = rowid + 2 * a.K;                     // [2][K]
    float *ubuf = reinterpret_cast<float *>(slot + 2 * a.K);  // [K]
    TgtSmem<HH> *sm = reinterpret_cast<TgtSmem<HH> *>(
        (reinterpret_cast<uintptr_t>(ubuf + a.K) + 15) & ~uintptr_t(15));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = a.K;
    const int n_chunks = a.D / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&sm->a_full[s], 1);
            mbar_init(&sm->a_empty[s], 1);
        }
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&sm->q_full[s], 1);
            mbar_init(&sm->q_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 4);
            mbar_init(&sm->meta_full[b], 1);
            mbar_init(&sm->meta_empty[b], 1);
        }
        mbar_init(&sm->drain, 1);
        sm->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    volatile int *abort_flag = &sm->abort_flag;

    if (warp == 0) {
        // ============================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapPool);
        }
        int as = 0, qs = 0;
        uint32_t aph = 0, qph = 0;
        uint32_t a_issued = 0, a_last = 0, q_issued = 0, q_last = 0;
        bool ok = true;
        int it = 0;
        for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
            const int g = a.n_tok - 1 - gt;
            const int b = g / a.S;
            const int t = g - b * a.S;
            const int mb = it & 1;
            const uint32_t mph = (it >> 1) & 1;
            if (!mbar_wait(&sm->meta_empty[mb], mph ^ 1u, abort_flag, a.err)) {
                ok = false;
                break;
            }
            int d0 = 0;
            if (a.doc_start) {
                d0 = a.doc_start[g];
                d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
            }
            // Compact the idx row: selected slots in order at the front,
            // masked slots from the back.
            int32_t *rw = rowid + mb * K;
            int32_t *sl = slot + mb * K;
            const int32_t *irow = a.idx + (size_t)g * K;
            int nsel = 0, nmask = 0;
            const uint32_t lt = (1u << lane) - 1u;
            for (int k0 = 0; k0 < K; k0 += 32) {
                const int k = k0 + lane;
                const bool in = k < K;
                const int j = in ? __ldg(irow + k) : -1;
                const bool inr = j >= 0 && j < a.P;
                const bool sel = in && inr && (j + 1) * a.cr - 1 <= t && j * a.cr >= d0;
                if (in && !(j == -1 || inr) && a.err)
                    atomicExch(a.err, kErrIndex);
                const uint32_t sm_sel = __ballot_sync(0xffffffffu, sel);
                const uint32_t sm_msk = __ballot_sync(0xffffffffu, in && !sel);
                if (sel) {
                    const int pos = nsel + __popc(sm_sel & lt);
                    rw[pos] = b * a.P + j;
                    sl[pos] = k;
                }
                if (in && !sel)
                    sl[K - 1 - (nmask + __popc(sm_msk & lt))] = k;
                nsel += __popc(sm_sel);
                nmask += __popc(sm_msk);
            }
            if (lane == 0)
                sm->nsel[mb] = nsel;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm->meta_full[mb]);

            const int nt = (nsel + 127) / 128;
            const int G = n_groups(nsel, TB);
            const int passes = G > 1 ? 2 : 1;
            if (lane == 0) {
                for (int pass = 0; pass < passes && ok; ++pass) {
                    for (int grp = 0; grp < G && ok; ++grp) {
                        const int i0 = grp * TB;
                        const int i1 = min(nt, i0 + TB);
                        for (int c = 0; c < n_chunks && ok; ++c) {
                            if (!mbar_wait(&sm->q_empty[qs], qph ^ 1u, abort_flag, a.err)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&sm->q_full[qs], kQTile);
                            tma_load_2d(q_buf + qs * kQTile, &mapQ, &sm->q_full[qs], c * 64, g * HH);
                            q_issued |= 1u << qs;
                            q_last = (q_last & ~(1u << qs)) | (qph << qs);
                            if (++qs == kQStages) {
                                qs = 0;
                                qph ^= 1u;
                            }
                            for (int i = i0; i < i1; ++i) {
                                if (!mbar_wait(&sm->a_empty[as], aph ^ 1u, abort_flag, a.err)) {
                                    ok = false;
                                    break;
                                }
                                const int rows = min(128, nsel - i * 128);
                                const int r4 = (rows + 3) & ~3;
                                mbar_arrive_expect_tx(&sm->a_full[as], (uint32_t)r4 * 128u);
                                uint8_t *dst = a_buf + as * kATile;
                                const int base_row = i * 128;
                                const int dummy = b * a.P;
                                for (int rr = 0; rr < r4; rr += 4) {
                                    const int k = base_row + rr;
                                    const int r0 = rw[k];
                                    const int r1 = (k + 1 < nsel) ? rw[k + 1] : dummy;
                                    const int r2 = (k + 2 < nsel) ? rw[k + 2] : dummy;
                                    const int r3 = (k + 3 < nsel) ? rw[k + 3] : dummy;
                                    tma_gather4(dst + rr * 128, &mapPool, &sm->a_full[as], c * 64, r0, r1, r2, r3);
                                }
                                a_issued |= 1u << as;
                                a_last = (a_last & ~(1u << as)) | (aph << as);
                                if (++as == kAStages) {
                                    as = 0;
                                    aph ^= 1u;
                                }
                            }
                        }
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < kAStages; ++s)
                if (a_issued & (1u << s))
                    mbar_drain(&sm->a_full[s], (a_last >> s) & 1u);
            for (int s = 0; s < kQStages; ++s)
                if (q_issued & (1u << s))
                    mbar_drain(&sm->q_full[s], (q_last >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ============================================================ MMA
        const uint32_t idesc = idesc_bf16_f32(128, HH);
        int as = 0, qs = 0;
        uint32_t aph = 0, qph = 0;
        bool ok = true, issued = false;
        int it = 0, acc_it = 0;
        for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
            const int mb = it & 1;
            const uint32_t mph = (it >> 1) & 1;
            if (!mbar_wait(&sm->meta_full[mb], mph, abort_flag, a.err)) {
                ok = false;
                break;
            }
            const int nsel = sm->nsel[mb];
            const int nt = (nsel + 127) / 128;
            const int G = n_groups(nsel, TB);
            const int passes = G > 1 ? 2 : 1;
            for (int pass = 0; pass < passes && ok; ++pass) {
                for (int grp = 0; grp < G && ok; ++grp, ++acc_it) {
                    const int i0 = grp * TB;
                    const int i1 = min(nt, i0 + TB);
                    const int buf = acc_it & 1;
                    const uint32_t bph = (acc_it >> 1) & 1;
                    if (!mbar_wait(&sm->acc_empty[buf], bph ^ 1u, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int c = 0; c < n_chunks && ok; ++c) {
                        if (!mbar_wait(&sm->q_full[qs], qph, abort_flag, a.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t dq = sdesc_k_sw128(smem_u32(q_buf + qs * kQTile));
                        for (int i = i0; i < i1; ++i) {
                            if (!mbar_wait(&sm->a_full[as], aph, abort_flag, a.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            if (lane == 0) {
                                const uint64_t da = sdesc_k_sw128(smem_u32(a_buf + as * kATile));
                                const uint32_t d_tmem = tmem + buf * 256 + (i - i0) * HH;
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16(d_tmem, da + 2 * kk, dq + 2 * kk, idesc, (c | kk) != 0);
                                umma_commit(&sm->a_empty[as]);
                                issued = true;
                            }
                            __syncwarp();
                            if (++as == kAStages) {
                                as = 0;
                                aph ^= 1u;
                            }
                        }
                        if (!ok)
                            break;
                        if (lane == 0)
                            umma_commit(&sm->q_empty[qs]);
                        __syncwarp();
                        if (++qs == kQStages) {
                            qs = 0;
                            qph ^= 1u;
                        }
                    }
                    if (!ok)
                        break;
                    if (lane == 0)
                        umma_commit(&sm->acc_full[buf]);
                    __syncwarp();
                }
            }
        }
        if (!ok && lane == 0 && issued) {
            umma_commit(&sm->drain);
            mbar_drain(&sm->drain, 0);
        }
        __syncwarp();
    } else {
        // ============================================================ epilogue
        const int q = warp & 3;              // TMEM lane quarter
        const int r = q * 32 + lane;         // row within a 128-slot tile
        const int et = threadIdx.x - 64;     // 0..127
        const float scale = a.scale;
        int it = 0, acc_it = 0;
        bool ok = true;
        for (int gt = blockIdx.x; gt < a.n_tok && ok; gt += gridDim.x, ++it) {
            const int g = a.n_tok - 1 - gt;
            const int mb = it & 1;
            const uint32_t mph = (it >> 1) & 1;
            if (!mbar_wait(&sm->meta_full[mb], mph, abort_flag, a.err)) {
                ok = false;
                break;
            }
            const int nsel = sm->nsel[mb];
            const int nt = (nsel + 127) / 128;
            const int G = n_groups(nsel, TB);
            const int passes = G > 1 ? 2 : 1;
            float *prow = a.p + (size_t)g * K;
            const int32_t *sl = slot + mb * K;
            float m_part = 0.f;
            float At = 0.f;  // max_h (M[h] - lse_full[h])
            for (int pass = 0; pass < passes && ok; ++pass) {
                for (int grp = 0; grp < G; ++grp, ++acc_it) {
                    const int i0 = grp * TB;
                    const int ntg = min(nt, i0 + TB) - i0;   // tiles in this group (>= 1)
                    const int buf = acc_it & 1;
                    const uint32_t bph = (acc_it >> 1) & 1;
                    if (!mbar_wait(&sm->acc_full[buf], bph, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tbase = tmem + buf * 256 + ((uint32_t)(q * 32) << 16);
                    const bool stats = (pass == 0);
                    const bool single = (G == 1);
                    if (stats) {
                        // ---- column max over this group's rows
                        for (int cc = 0; cc < NC16; ++cc) {
                            float v16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                v16[e] = -INFINITY;
                            for (int ib = 0; ib < ntg; ib += IB) {
                                uint32_t v[IB][16];
#pragma unroll
                                for (int i = 0; i < IB; ++i)
                                    if (ib + i < ntg)
                                        tmem_ld16(tbase + (ib + i) * HH + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IB; ++i) {
                                    const bool row_ok = (ib + i < ntg) && ((i0 + ib + i) * 128 + r < nsel);
#pragma unroll
                                    for (int e = 0; e < 16; ++e)
                                        v16[e] = row_ok ? fmaxf(v16[e], __uint_as_float(v[i][e]) * scale) : v16[e];
                                }
                            }
                            const float red = warp_colreduce16(v16, OpMax());
                            if (lane < 16)
                                sm->red_max[q][cc * 16 + lane] = red;
                        }
                        named_bar_sync(1, 128);
                        if (et < HH) {
                            const float gm = fmaxf(fmaxf(sm->red_max[0][et], sm->red_max[1][et]),
                                                   fmaxf(sm->red_max[2][et], sm->red_max[3][et]));
                            sm->head_a[et] = gm;   // group max, staged
                        }
                        named_bar_sync(1, 128);
                        // ---- sum of exp(z - group max); single group: keep e in TMEM
                        for (int cc = 0; cc < NC16; ++cc) {
                            float s16[16], gm16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                s16[e] = 0.f;
                                gm16[e] = sm->head_a[cc * 16 + e] * kLog2e;
                            }
                            for (int ib = 0; ib < ntg; ib += IB) {
                                uint32_t v[IB][16];
#pragma unroll
                                for (int i = 0; i < IB; ++i)
                                    if (ib + i < ntg)
                                        tmem_ld16(tbase + (ib + i) * HH + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IB; ++i) {
                                    const bool row_ok = (ib + i < ntg) && ((i0 + ib + i) * 128 + r < nsel);
#pragma unroll
                                    for (int e = 0; e < 16; ++e) {
                                        const float x = ex2_approx(fmaf(__uint_as_float(v[i][e]) * scale, kLog2e, -gm16[e]));
                                        const float ex = row_ok ? x : 0.f;
                                        s16[e] += ex;
                                        v[i][e] = __float_as_uint(ex);
                                    }
                                }
                                if (single) {
#pragma unroll
                                    for (int i = 0; i < IB; ++i)
                                        if (ib + i < ntg)
                                            tmem_st16(tbase + (ib + i) * HH + cc * 16, v[i]);
                                }
                            }
                            const float red = warp_colreduce16(s16, OpAdd());
                            if (lane < 16)
                                sm->red_sum[q][cc * 16 + lane] = red;
                        }
                        if (single)
                            tmem_st_wait();
                        named_bar_sync(1, 128);
                        if (et < HH) {
                            const float gm = sm->head_a[et];
                            const float gs = sm->red_sum[0][et] + sm->red_sum[1][et] + sm->red_sum[2][et] +
                                             sm->red_sum[3][et];
                            if (grp == 0) {
                                sm->colM[et] = gm;
                                sm->colS[et] = gs;
                            } else {
                                const float M0 = sm->colM[et], S0 = sm->colS[et];
                                const float M1 = fmaxf(M0, gm);
                                sm->colS[et] = S0 * expf(M0 - M1) + gs * expf(gm - M1);
                                sm->colM[et] = M1;
                            }
                        }
                        named_bar_sync(1, 128);
                    }
                    if (pass == passes - 1) {
                        if (grp == 0) {
                            // ---- per-head merge with the window and the sink
                            if (et < HH) {
                                const float M = sm->colM[et];
                                const float clse = M + logf(sm->colS[et]);
                                const float wl = a.wl[(size_t)g * HH + et];
                                float mm = fmaxf(wl, clse);
                                float sk = -INFINITY;
                                if (a.sink) {
                                    sk = a.sink[et];
                                    mm = fmaxf(mm, sk);
                                }
                                float acc = expf(wl - mm) + expf(clse - mm);
                                if (a.sink)
                                    acc += expf(sk - mm);
                                const float lse_full = mm + logf(acc);
                                sm->head_a[et] = M - lse_full;
                            }
                            named_bar_sync(1, 128);
                            At = -INFINITY;
                            for (int h = 0; h < HH; ++h)
                                At = fmaxf(At, sm->head_a[h]);
                            named_bar_sync(1, 128);
                            if (et < HH)
                                sm->wprime[et] = expf(sm->head_a[et] - At);
                            named_bar_sync(1, 128);
                        }
                        // ---- u'[k] = sum_h e[k,h] w[h]
                        float u[TB];
#pragma unroll
                        for (int i = 0; i < TB; ++i)
                            u[i] = 0.f;
                        for (int cc = 0; cc < NC16; ++cc) {
                            float w16[16], m16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                w16[e] = sm->wprime[cc * 16 + e];
                                m16[e] = sm->colM[cc * 16 + e] * kLog2e;
                            }
#pragma unroll
                            for (int ib = 0; ib < TB; ib += IB) {
                                if (ib >= ntg)
                                    break;
                                uint32_t v[IB][16];
#pragma unroll
                                for (int i = 0; i < IB; ++i)
                                    if (ib + i < ntg)
                                        tmem_ld16(tbase + (ib + i) * HH + cc * 16, v[i]);
                                tmem_ld_wait();
#pragma unroll
                                for (int i = 0; i < IB; ++i) {
                                    if (ib + i < ntg) {
                                        float acc = u[ib + i];
#pragma unroll
                                        for (int e = 0; e < 16; ++e) {
                                            float ex = __uint_as_float(v[i][e]);
                                            if (!single)
                                                ex = ex2_approx(fmaf(ex * scale, kLog2e, -m16[e]));
                                            acc = fmaf(ex, w16[e], acc);
                                        }
                                        u[ib + i] = acc;
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int i = 0; i < TB; ++i) {
                            const int j = (i0 + i) * 128 + r;
                            if (i < ntg && j < nsel) {
                                ubuf[j] = u[i];
                                m_part += u[i];
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&sm->acc_empty[buf]);
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
                sm->red_m[q] = mt;
            named_bar_sync(1, 128);
            const float mtot = sm->red_m[0] + sm->red_m[1] + sm->red_m[2] + sm->red_m[3];
            if (nsel > 0) {
                const bool plain = logf(mtot) + At >= kLnFltMin;
                const float f = plain ? 0.f : expf(At - kLnFltMin);
                for (int jj = et; jj < K; jj += 128) {
                    float v = 0.f;
                    if (jj < nsel)
                        v = plain ? ubuf[jj] / mtot : ubuf[jj] * f;
                    prow[sl[jj]] = v;
                }
            } else {
                for (int jj = et; jj < K; jj += 128)
                    prow[jj] = 0.f;
            }
            named_bar_sync(1, 128);
            if (et == 0)
                mbar_arrive(&sm->meta_empty[mb]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int HH>
size_t smem_bytes_for(int K)
{
    return 1024 + kAStages * kATile + kQStages * (HH * 128) + (size_t)K * (4 + 4) * 2 + (size_t)K * 4 + 16 +
           sizeof(TgtSmem<HH>) + 64;
}

template <int HH>
cudaError_t launch_h(const CUtensorMap &mapQ, const CUtensorMap &mapPool, const TgtTcArgs &a, int grid,
                     cudaStream_t stream)
{
    const size_t smem = smem_bytes_for<HH>(a.K);
    cudaError_t e =
        cudaFuncSetAttribute(target_tc_kernel<HH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    target_tc_kernel<HH><<<grid, kTgtThreads, smem, stream>>>(mapQ, mapPool, a);
    return cudaGetLastError();
}

}  // namespace

size_t target_tc_smem_bytes(int H, int K)
{
    switch (H) {
    case 16: return smem_bytes_for<16>(K);
    case 32: return smem_bytes_for<32>(K);
    case 64: return smem_bytes_for<64>(K);
    case 128: return smem_bytes_for<128>(K);
    default: return 0;
    }
}

cudaError_t launch_target_tc(const CUtensorMap &mapQ, const CUtensorMap &mapPool, const TgtTcArgs &a, int grid,
                             cudaStream_t stream)
{
    switch (a.H) {
    case 16: return launch_h<16>(mapQ, mapPool, a, grid, stream);
    case 32: return launch_h<32>(mapQ, mapPool, a, grid, stream);
    case 64: return launch_h<64>(mapQ, mapPool, a, grid, stream);
    case 128: return launch_h<128>(mapQ, mapPool, a, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace sai
