// Banded sliding-window log-mass on tcgen05 tensor cores (sm_100a).
//
// Computes window_lse[b,t,h] = log sum_{s=lo}^{t} exp(scale <Q[b,t,h],Kw[b,s]>),
// lo = max(d0, t-W+1) (t, s and d0 are sequence positions; a token-range call
// covers positions t_begin .. t_begin+S-1 with Kw holding kw_lead keys before
// them): the log mass of the sliding-window keys that the joint
// softmax of a CSA layer carries in its denominator (Primus page "perf(
// deepseek-v4): fuse and enable the indexer distillation loss", second commit
// message: computing the window mass eagerly materialises per-head window
// logits that are mostly masked; the fused kernel never writes them and reads
// only the keys each tile of queries can see).
//
// Tile: M = 128 rows = TQ = 128/H consecutive tokens x H heads, contiguous in
// Q viewed as [B*S*H, D]. The key band of the tile is the NB = roundup16(W +
// TQ - 1) consecutive Kw rows starting at t0 - W + 1 (one TMA box; rows before
// the sequence are zero-filled or belong to the previous sequence and are
// masked). One MMA chain of D/64 x 4 steps (M=128, N=NB, K=16) puts the
// 128 x NB logits in TMEM; the epilogue reads one row per thread and reduces
// it with a masked two-pass max / sum-exp over the columns of its window.
//
// Warp roles (320 threads): warp 0 TMA producer (and TMEM owner), warp 1 MMA
// issuer, warps 2..5 and 6..9 two epilogue groups that take alternate tiles,
// each with its own 256-column TMEM accumulator. The kernel is bound by
// reading Q from HBM once; the stage ring keeps about 200 KB in flight.
// Every wait is bounded; on timeout the kernel writes NaN rows and unwinds.
#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

constexpr int kWinStages = 6;
constexpr int kWinThreads = 320;
constexpr uint32_t kATileBytes = 128 * 128;  // 128 rows x 64 bf16

struct WinSmem {
    uint64_t full[kWinStages];
    uint64_t empty[kWinStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kWinThreads, 1)
    window_lse_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                         const WinTcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t b_bytes = a.b_stage_bytes;  // NB x 128, rounded to 1024
    const uint32_t chunk_bytes = kATileBytes + b_bytes;   // one 64-column chunk of D: Q tile + key band
    // A stage carries two chunks when D allows it (three stages), else one
    // (six stages): the same bytes in flight, half the barrier waits, fences
    // and commits per MMA, which cost the issuing thread ~150 cycles each.
    const int cps = ((a.D / 64) % 2 == 0) ? 2 : 1;
    const int n_stages = kWinStages / cps;
    const uint32_t stage_bytes = cps * chunk_bytes;
    WinSmem *sm = reinterpret_cast<WinSmem *>(base + kWinStages * chunk_bytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWinStages; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 4);
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

    const int n_tiles = a.n_tiles;
    const int n_chunks = a.D / 64;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapK);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, last_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                const int g0 = tile * a.TQ;
                const int b = g0 / a.S;
                const int t0 = g0 - b * a.S;
                const int rowQ = g0 * a.H;
                // Kw is [B, S + kw_lead, D]: local token t sits at Kw row t + kw_lead
                const int rowK = b * (a.S + a.kw_lead) + t0 + a.kw_lead - a.W + 1;
                for (int c = 0; c < n_chunks; c += cps) {
                    if (!mbar_wait(&sm->empty[stage], phase ^ 1u, abort_flag, nullptr)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = base + stage * stage_bytes;
                    mbar_arrive_expect_tx(&sm->full[stage], (uint32_t)cps * (kATileBytes + a.NB * 128u));
                    for (int cc = 0; cc < cps; ++cc) {
                        tma_load_2d(sa + cc * chunk_bytes, &mapQ, &sm->full[stage], (c + cc) * 64, rowQ);
                        tma_load_2d(sa + cc * chunk_bytes + kATileBytes, &mapK, &sm->full[stage], (c + cc) * 64,
                                    rowK);
                    }
                    issued_mask |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == n_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < n_stages; ++s)
                    if (issued_mask & (1u << s))
                        mbar_drain(&sm->full[s], (last_parity >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, a.NB);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, issued = false;
        int j = 0;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++j) {
            const int buf = j & 1;
            const uint32_t aphase = (j >> 1) & 1;
            if (!mbar_wait(&sm->acc_empty[buf], aphase ^ 1u, abort_flag, nullptr)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + buf * 256;
            for (int c = 0; c < n_chunks; c += cps) {
                if (!mbar_wait(&sm->full[stage], phase, abort_flag, nullptr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    for (int cc = 0; cc < cps; ++cc) {
                        const uint32_t sa = smem_u32(base + stage * stage_bytes + cc * chunk_bytes);
                        const uint64_t da = sdesc_k_sw128(sa);
                        const uint64_t db = sdesc_k_sw128(sa + kATileBytes);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d_tmem, da + 2 * kk, db + 2 * kk, idesc, ((c + cc) | kk) != 0);
                    }
                    umma_commit(&sm->empty[stage]);
                    issued = true;
                }
                __syncwarp();
                if (++stage == n_stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok)
                break;
            if (lane == 0)
                umma_commit(&sm->acc_full[buf]);
            __syncwarp();
        }
        if (!ok && lane == 0 && issued) {
            umma_commit(&sm->drain);
            mbar_drain(&sm->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int wg = (warp - 2) >> 2;    // takes tiles j with j & 1 == wg
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int r = q * 32 + lane;       // tile row
        const float s2 = a.scale * 1.4426950408889634f;  // scale > 0 (checked on the host)
        const int ncol16 = a.NB / 16;
        const int rt = r / a.H;            // token of this row within the tile
        const int h = r - rt * a.H;
        int j = wg;
        int uses = 0;
        for (int tile = blockIdx.x + wg * gridDim.x; tile < n_tiles; tile += 2 * gridDim.x, j += 2, ++uses) {
            const int g0 = tile * a.TQ;
            const int g = g0 + rt;
            const int b = g0 / a.S;
            const int t = g - b * a.S + a.t_begin;       // sequence positions
            const int t0 = g0 - b * a.S + a.t_begin;
            int d0 = 0;
            if (a.doc_start) {
                d0 = a.doc_start[g];
                d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
            }
            d0 = max(d0, a.t_begin - a.kw_lead);         // the first key the caller passed
            if (!mbar_wait(&sm->acc_full[wg], uses & 1, abort_flag, nullptr)) {
                a.out[(size_t)g * a.H + h] = __int_as_float(0x7fc00000);
                break;
            }
            tc_fence_after();
            const int lo = max(d0, t - a.W + 1);
            const int band0 = t0 - a.W + 1;      // key of band column 0
            const int clo = lo - band0, chi = t - band0;
            // chunks any row of this warp needs
            int wlo = clo, whi = chi;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                wlo = min(wlo, __shfl_xor_sync(0xffffffffu, wlo, o));
                whi = max(whi, __shfl_xor_sync(0xffffffffu, whi, o));
            }
            const int c_begin = wlo >> 4, c_end = min(ncol16 - 1, whi >> 4);
            const uint32_t taddr = tmem + wg * 256 + ((uint32_t)(q * 32) << 16);
            // two passes (max, then sum of exponentials) over the row's window
            // columns, three 16-column TMEM loads per wait
            float mx = -INFINITY;
            for (int cb = c_begin; cb <= c_end; cb += 3) {
                uint32_t v[3][16];
#pragma unroll
                for (int u = 0; u < 3; ++u)
                    if (cb + u <= c_end)
                        tmem_ld16(taddr + (cb + u) * 16, v[u]);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 3; ++u) {
                    const int c0 = (cb + u) * 16;
                    if (cb + u > c_end)
                        break;
                    if (c0 >= clo && c0 + 15 <= chi) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            mx = fmaxf(mx, __uint_as_float(v[u][e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c0 + e >= clo && c0 + e <= chi)
                                mx = fmaxf(mx, __uint_as_float(v[u][e]));
                    }
                }
            }
            const float m2 = mx * s2;
            float sum = 0.f;
            for (int cb = c_begin; cb <= c_end; cb += 3) {
                uint32_t v[3][16];
#pragma unroll
                for (int u = 0; u < 3; ++u)
                    if (cb + u <= c_end)
                        tmem_ld16(taddr + (cb + u) * 16, v[u]);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 3; ++u) {
                    const int c0 = (cb + u) * 16;
                    if (cb + u > c_end)
                        break;
                    if (c0 >= clo && c0 + 15 <= chi) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            sum += ex2_approx(fmaf(__uint_as_float(v[u][e]), s2, -m2));
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c0 + e >= clo && c0 + e <= chi)
                                sum += ex2_approx(fmaf(__uint_as_float(v[u][e]), s2, -m2));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm->acc_empty[wg]);
            a.out[(size_t)g * a.H + h] = mx * a.scale + logf(sum);
        }
        (void)j;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

size_t window_tc_smem_bytes(int NB)
{
    const size_t b_bytes = ((size_t)NB * 128 + 1023) & ~size_t(1023);
    return 1024 + kWinStages * (kATileBytes + b_bytes) + sizeof(WinSmem) + 64;
}

cudaError_t launch_window_lse_tc(const CUtensorMap &mapQ, const CUtensorMap &mapK, const WinTcArgs &a,
                                 int grid, cudaStream_t stream)
{
    const size_t smem = window_tc_smem_bytes(a.NB);
    cudaError_t e = cudaFuncSetAttribute(window_lse_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    window_lse_tc_kernel<<<grid, kWinThreads, smem, stream>>>(mapQ, mapK, a);
    return cudaGetLastError();
}

}  // namespace sai
