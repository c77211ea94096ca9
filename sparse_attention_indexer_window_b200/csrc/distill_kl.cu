// KL(attention || indexer) and its analytic gradient in one pass over each
// row (Primus page "perf(deepseek-v4): fuse and enable the indexer
// distillation loss", first commit message: the KL tail is fused with an
// analytic backward and saves nothing beyond its inputs; MaxText page "Add
// Indexer Loss [Deepseek v4]", review: log-softmax gives the exact gradient
// Q - P, and the valid mask includes the indexer mask).
//
// Per row over valid slots: lse = log sum exp s; q = exp(s - lse);
//   KL_row = sum_{p>0} p (log p - s + lse);  dscores = c (q sum(p) - p),
//   c = coeff / max(N, 1), N = rows with a valid slot.
//
// One cooperative launch on the caller's stream (all blocks resident at
// once), after a 16-byte reset of the workspace's counters:
//   A. every warp takes its rows and counts those with a valid slot (one
//      atomic per block into N). When the grid has a warp per row, the warp
//      also loads its row into registers and forms everything that does not
//      need N: lse, sum(p), KL_row and q = exp(s - lse);
//   B. a grid barrier (bounded: on a timeout the loss is NaN and dscores is
//      not written), after which N is read once;
//   C. dscores from the registers, or (rows streamed) KL and dscores per
//      row; each block stores its partial KL sum (fp64); the last block to
//      finish adds the partials in block order and writes the loss. The
//      result is deterministic run to run.
// With N given by the caller, A and B are skipped.
// HBM-bound: per row it reads p, scores (4K bytes each) and valid (K bytes)
// once (valid twice when rows outnumber warps) and writes dscores (4K bytes).
#include <math.h>

#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

constexpr int kKlThreads = 256;
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlMaxBlocks = 148 * 4;

struct KlWs {
    uint32_t *done;       // blocks finished (the last one writes the loss)
    uint32_t *bar_count;  // grid barrier: arrivals
    uint32_t *bar_gen;    // grid barrier: generation
    int32_t *n_rows;      // rows with a valid slot (the single-launch form's N)
    int32_t *count_part;
    double *kl_part;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline KlWs ws_layout(void *ws, int count_blocks)
{
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    KlWs w;
    w.done = reinterpret_cast<uint32_t *>(b);
    w.bar_count = reinterpret_cast<uint32_t *>(b + 4);
    w.bar_gen = reinterpret_cast<uint32_t *>(b + 8);
    w.n_rows = reinterpret_cast<int32_t *>(b + 12);
    w.count_part = reinterpret_cast<int32_t *>(b + 16);
    w.kl_part = reinterpret_cast<double *>(b + 16 + align16((size_t)count_blocks * 4));
    return w;
}

__global__ void __launch_bounds__(kKlThreads)
    kl_count_kernel(const uint8_t *__restrict__ valid, int rows, int K, void *ws, int count_blocks)
{
    KlWs w = ws_layout(ws, count_blocks);
    __shared__ int wcount[kKlWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int c = 0;
    const bool vec = (K & 15) == 0;
    for (int r = blockIdx.x * kKlWarps + warp; r < rows; r += gridDim.x * kKlWarps) {
        const uint8_t *vr = valid + (size_t)r * K;
        bool any = false;
        if (vec) {
            for (int k = lane * 16; k < K; k += 32 * 16) {
                const uint4 x = __ldg(reinterpret_cast<const uint4 *>(vr + k));
                any |= (x.x | x.y | x.z | x.w) != 0;
            }
        } else {
            for (int k = lane; k < K; k += 32)
                any |= vr[k] != 0;
        }
        c += __any_sync(0xffffffffu, any) ? 1 : 0;
    }
    if (lane == 0)
        wcount[warp] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int i = 0; i < kKlWarps; ++i)
            s += wcount[i];
        w.count_part[blockIdx.x] = s;
        if (blockIdx.x == 0)
            *w.done = 0u;
    }
}

// Rows with a valid slot, added into *n (zeroed by the caller's stream first).
__global__ void __launch_bounds__(kKlThreads)
    count_rows_kernel(const uint8_t *__restrict__ valid, int rows, int K, int32_t *n)
{
    __shared__ int wcount[kKlWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int c = 0;
    const bool vec = (K & 15) == 0;
    for (int r = blockIdx.x * kKlWarps + warp; r < rows; r += gridDim.x * kKlWarps) {
        const uint8_t *vr = valid + (size_t)r * K;
        bool any = false;
        if (vec) {
            for (int k = lane * 16; k < K; k += 32 * 16) {
                const uint4 x = __ldg(reinterpret_cast<const uint4 *>(vr + k));
                any |= (x.x | x.y | x.z | x.w) != 0;
            }
        } else {
            for (int k = lane; k < K; k += 32)
                any |= vr[k] != 0;
        }
        c += __any_sync(0xffffffffu, any) ? 1 : 0;
    }
    if (lane == 0)
        wcount[warp] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int i = 0; i < kKlWarps; ++i)
            s += wcount[i];
        if (s)
            atomicAdd(n, s);
    }
}

__device__ __forceinline__ float warp_max(float v)
{
    for (int o = 16; o >= 1; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v)
{
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One row in registers: NV float4 groups per lane, element 4*lane + 128*j + e
// (K % 4 == 0, K <= 128*NV).
template <int NV>
struct RowRegs {
    float4 p[NV], s[NV];
    uint32_t v[NV];
};

// Loads a row; true (in every lane) if it has a valid slot.
template <int NV>
__device__ __forceinline__ bool row_load(RowRegs<NV> &R, const float *__restrict__ pr,
                                         const float *__restrict__ sr, const uint8_t *__restrict__ vr, int K)
{
    const int lane = threadIdx.x & 31;
    bool any = false;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int k = 4 * lane + 128 * j;
        if (k < K) {
            R.p[j] = __ldcs(reinterpret_cast<const float4 *>(pr + k));
            R.s[j] = __ldcs(reinterpret_cast<const float4 *>(sr + k));
            R.v[j] = __ldcs(reinterpret_cast<const unsigned int *>(vr + k));
        } else {
            R.p[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            R.s[j] = R.p[j];
            R.v[j] = 0u;
        }
        any |= R.v[j] != 0u;
    }
    return __any_sync(0xffffffffu, any);
}

// KL of a loaded row; writes its dscores (zeros for a row with no valid slot).
template <int NV>
__device__ __forceinline__ float row_kl(const RowRegs<NV> &R, bool any, float *dr, int K, float c)
{
    const int lane = threadIdx.x & 31;
    if (!any) {
        if (dr) {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int k = 4 * lane + 128 * j;
                if (k < K)
                    __stcs(reinterpret_cast<float4 *>(dr + k), make_float4(0.f, 0.f, 0.f, 0.f));
            }
        }
        return 0.f;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            mx = v ? fmaxf(mx, s4[e]) : mx;
        }
    }
    mx = warp_max(mx);
    float se = 0.f, ps = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
        const float p4[4] = {R.p[j].x, R.p[j].y, R.p[j].z, R.p[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            se += v ? __expf(s4[e] - mx) : 0.f;
            ps += v ? p4[e] : 0.f;
        }
    }
    se = warp_sum(se);
    ps = warp_sum(ps);
    const float lse = mx + __logf(se);
    float kl = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
        const float p4[4] = {R.p[j].x, R.p[j].y, R.p[j].z, R.p[j].w};
        float d4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            const float logq = s4[e] - lse;
            kl += (v && p4[e] > 0.f) ? p4[e] * (__logf(p4[e]) - logq) : 0.f;
            d4[e] = v ? c * fmaf(__expf(logq), ps, -p4[e]) : 0.f;
        }
        const int k = 4 * lane + 128 * j;
        if (dr && k < K)
            __stcs(reinterpret_cast<float4 *>(dr + k), make_float4(d4[0], d4[1], d4[2], d4[3]));
    }
    return warp_sum(kl);
}

// The part of a loaded row's KL that needs no N: returns KL_row (in every
// lane), sets lse and sum(p) over valid slots, and turns the scores in R into
// q = exp(s - lse). Call only for a row with a valid slot.
template <int NV>
__device__ __forceinline__ float row_stats(RowRegs<NV> &R, int K, float &ps_out)
{
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            mx = v ? fmaxf(mx, s4[e]) : mx;
        }
    }
    mx = warp_max(mx);
    float se = 0.f, ps = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
        const float p4[4] = {R.p[j].x, R.p[j].y, R.p[j].z, R.p[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            se += v ? __expf(s4[e] - mx) : 0.f;
            ps += v ? p4[e] : 0.f;
        }
    }
    se = warp_sum(se);
    ps_out = warp_sum(ps);
    const float lse = mx + __logf(se);
    float kl = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        float *s4 = &R.s[j].x;
        const float p4[4] = {R.p[j].x, R.p[j].y, R.p[j].z, R.p[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (R.v[j] >> (8 * e)) & 0xffu;
            const float logq = s4[e] - lse;
            kl += (v && p4[e] > 0.f) ? p4[e] * (__logf(p4[e]) - logq) : 0.f;
            s4[e] = __expf(logq);
        }
    }
    return warp_sum(kl);
}

// dscores of a row after row_stats: c (q sum(p) - p) on valid slots, else 0
// (the whole row 0 when it has no valid slot).
template <int NV>
__device__ __forceinline__ void row_dscores(const RowRegs<NV> &R, bool any, float ps, float c, float *dr, int K)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int k = 4 * lane + 128 * j;
        if (k >= K)
            continue;
        const float q4[4] = {R.s[j].x, R.s[j].y, R.s[j].z, R.s[j].w};
        const float p4[4] = {R.p[j].x, R.p[j].y, R.p[j].z, R.p[j].w};
        float d4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = any && ((R.v[j] >> (8 * e)) & 0xffu);
            d4[e] = v ? c * fmaf(q4[e], ps, -p4[e]) : 0.f;
        }
        __stcs(reinterpret_cast<float4 *>(dr + k), make_float4(d4[0], d4[1], d4[2], d4[3]));
    }
}

// Whether a row has a valid slot (in every lane of the warp).
__device__ __forceinline__ bool row_any_valid(const uint8_t *__restrict__ vr, int K)
{
    const int lane = threadIdx.x & 31;
    bool any = false;
    if ((K & 15) == 0) {
        for (int k = lane * 16; k < K; k += 32 * 16) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(vr + k));
            any |= (x.x | x.y | x.z | x.w) != 0;
        }
    } else {
        for (int k = lane; k < K; k += 32)
            any |= vr[k] != 0;
    }
    return __any_sync(0xffffffffu, any);
}

// Barrier over all blocks of a cooperative launch (every block resident).
// The generation is read before arriving, so it can only move once this
// block has arrived; the last arrival resets the count and moves it. Bounded:
// false (in every thread of the block) after the wait limit.
__device__ bool grid_barrier(uint32_t *count, uint32_t *gen)
{
    __shared__ int ok_s;
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile uint32_t *g = gen;
        const uint32_t g0 = *g;
        __threadfence();
        bool ok = true;
        if (atomicAdd(count, 1u) == gridDim.x - 1) {
            atomicExch(count, 0u);
            __threadfence();
            atomicAdd(gen, 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while (*g == g0) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
        ok_s = ok ? 1 : 0;
    }
    __syncthreads();
    return ok_s != 0;
}

// Any K: two passes over the row (the second pass hits L1/L2).
__device__ __forceinline__ float kl_row_any(const float *__restrict__ pr, const float *__restrict__ sr,
                                            const uint8_t *__restrict__ vr, float *dr, int K, float c)
{
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY, se = 0.f, ps = 0.f;
    bool any = false;
    for (int k = lane; k < K; k += 32) {
        if (vr[k]) {
            const float s = sr[k];
            any = true;
            if (s > mx) {
                se = se * __expf(mx - s) + 1.f;
                mx = s;
            } else {
                se += __expf(s - mx);
            }
            ps += pr[k];
        }
    }
    if (!__any_sync(0xffffffffu, any)) {
        if (dr)
            for (int k = lane; k < K; k += 32)
                dr[k] = 0.f;
        return 0.f;
    }
    const float gmx = warp_max(mx);
    se = (mx == -INFINITY) ? 0.f : se * __expf(mx - gmx);
    se = warp_sum(se);
    ps = warp_sum(ps);
    const float lse = gmx + __logf(se);
    float kl = 0.f;
    for (int k = lane; k < K; k += 32) {
        const bool v = vr[k] != 0;
        const float p = pr[k];
        const float logq = sr[k] - lse;
        kl += (v && p > 0.f) ? p * (__logf(p) - logq) : 0.f;
        if (dr)
            dr[k] = v ? c * fmaf(__expf(logq), ps, -p) : 0.f;
    }
    return warp_sum(kl);
}

// RES: one warp per row (rows <= warps of the grid), the row held in
// registers from the count to the KL; else rows are streamed after the
// count. NV: float4 groups per lane of the register row form (0: any K).
template <int NV, bool RES>
__global__ void __launch_bounds__(kKlThreads, 4)
    kl_fused_kernel(const float *__restrict__ p, const float *__restrict__ scores, const uint8_t *__restrict__ valid,
                    int rows, int K, float coeff, float *loss, float *dscores, void *ws, int count_blocks,
                    const int32_t *n_given)
{
    constexpr int NV1 = NV > 0 ? NV : 1;     // the register form's width
    constexpr int NR = RES ? NV1 : 1;         // registers kept across the barrier
    KlWs w = ws_layout(ws, count_blocks);
    __shared__ double wkl[kKlWarps];
    __shared__ int wcnt[kKlWarps];
    __shared__ bool last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kKlWarps + warp;
    const int nw = gridDim.x * kKlWarps;
    const size_t off = (size_t)gw * K;

    // RES: the row's loads, and all of its KL that does not need N, come
    // before the barrier; only the dscores stores wait for N
    RowRegs<NR> R;
    bool rany = false;
    float rps = 0.f;
    double acc = 0.0;
    if (RES && gw < rows) {
        rany = row_load<NR>(R, p + off, scores + off, valid + off, K);
        if (rany)
            acc = (double)row_stats<NR>(R, K, rps);
    }

    int N;
    if (!n_given) {
        // A. rows with a valid slot: one atomic per block
        int c = 0;
        if (RES)
            c = rany ? 1 : 0;
        else
            for (int r = gw; r < rows; r += nw)
                c += row_any_valid(valid + (size_t)r * K, K) ? 1 : 0;
        if (lane == 0)
            wcnt[warp] = c;
        __syncthreads();
        if (threadIdx.x == 0) {
            int sb = 0;
            for (int i = 0; i < kKlWarps; ++i)
                sb += wcnt[i];
            if (sb)
                atomicAdd(w.n_rows, sb);
        }
        // B. every block's count is in before any block reads N
        if (!grid_barrier(w.bar_count, w.bar_gen)) {
            if (threadIdx.x == 0)
                *loss = __int_as_float(0x7fc00000);
            return;
        }
        N = __ldcg(w.n_rows);
    } else {
        N = *n_given;
    }
    const float c = coeff / (float)(N > 1 ? N : 1);

    // C. dscores (RES), or the whole row (streamed)
    if (RES) {
        if (gw < rows && dscores)
            row_dscores<NR>(R, rany, rps, c, dscores + off, K);
    } else {
        for (int r = gw; r < rows; r += nw) {
            const size_t ro = (size_t)r * K;
            float kl;
            if (NV > 0) {
                RowRegs<NV1> T;
                const bool any = row_load<NV1>(T, p + ro, scores + ro, valid + ro, K);
                kl = row_kl<NV1>(T, any, dscores ? dscores + ro : nullptr, K, c);
            } else {
                kl = kl_row_any(p + ro, scores + ro, valid + ro, dscores ? dscores + ro : nullptr, K, c);
            }
            acc += (double)kl;
        }
    }
    if (lane == 0)
        wkl[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double sb = 0.0;
        for (int i = 0; i < kKlWarps; ++i)
            sb += wkl[i];
        w.kl_part[blockIdx.x] = sb;
        __threadfence();
        const uint32_t prev = atomicAdd(w.done, 1u);
        last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (last) {
        // fixed-order parallel sum of the per-block partials
        __threadfence();
        const volatile double *kp = w.kl_part;
        double sb = 0.0;
        for (int i = threadIdx.x; i < (int)gridDim.x; i += blockDim.x)
            sb += kp[i];
        for (int o = 16; o >= 1; o >>= 1)
            sb += __shfl_xor_sync(0xffffffffu, sb, o);
        if (lane == 0)
            wkl[warp] = sb;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int i = 0; i < kKlWarps; ++i)
                t += wkl[i];
            *loss = (float)((double)coeff * t / (double)(N > 1 ? N : 1));
        }
    }
}

// Blocks of `kern` that fit on the device at once (cooperative launch bound),
// looked up once per device.
template <int NV, bool RES>
int coop_capacity()
{
    static int cap[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    if (cap[dev] == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kl_fused_kernel<NV, RES>, kKlThreads, 0) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        cap[dev] = per_sm * sms;
    }
    return cap[dev];
}

template <int NV, bool RES>
cudaError_t launch_fused(const KlPlan &pl, const float *p, const float *scores, const uint8_t *valid, float coeff,
                         float *loss, float *dscores, void *ws, cudaStream_t stream, const int32_t *n_given, int grid)
{
    int rows = pl.rows, K = pl.K, cb = pl.count_blocks;
    void *args[] = {(void *)&p, (void *)&scores, (void *)&valid, (void *)&rows, (void *)&K, (void *)&coeff,
                    (void *)&loss, (void *)&dscores, (void *)&ws, (void *)&cb, (void *)&n_given};
    return cudaLaunchCooperativeKernel((const void *)kl_fused_kernel<NV, RES>, dim3(grid), dim3(kKlThreads), args, 0,
                                       stream);
}

template <int NV>
cudaError_t launch_nv(const KlPlan &pl, const float *p, const float *scores, const uint8_t *valid, float coeff,
                      float *loss, float *dscores, void *ws, cudaStream_t stream, const int32_t *n_given)
{
    // one warp per row when the whole grid fits at once, else streamed rows
    const int cap_res = coop_capacity<NV, true>();
    const int need = (pl.rows + kKlWarps - 1) / kKlWarps;
    if (NV > 0 && need <= pl.row_blocks && need <= cap_res)
        return launch_fused<NV, true>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given,
                                      need > 0 ? need : 1);
    const int cap = coop_capacity<NV, false>();
    if (cap <= 0)
        return cudaErrorLaunchOutOfResources;
    const int grid = pl.row_blocks < cap ? pl.row_blocks : cap;
    return launch_fused<NV, false>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given, grid);
}

}  // namespace

KlPlan kl_plan(int B, int S, int K)
{
    KlPlan pl;
    pl.rows = B * S;
    pl.K = K;
    const int need = (pl.rows + kKlWarps - 1) / kKlWarps;
    pl.count_blocks = need < kKlMaxBlocks ? need : kKlMaxBlocks;
    pl.row_blocks = pl.count_blocks;
    if (pl.count_blocks < 1)
        pl.count_blocks = pl.row_blocks = 1;
    pl.ws_bytes = 16 + align16((size_t)pl.count_blocks * 4) + align16((size_t)pl.row_blocks * 8);
    return pl;
}

cudaError_t launch_kl_count(const KlPlan &pl, const uint8_t *valid, void *ws, cudaStream_t stream)
{
    kl_count_kernel<<<pl.count_blocks, kKlThreads, 0, stream>>>(valid, pl.rows, pl.K, ws, pl.count_blocks);
    return cudaGetLastError();
}

cudaError_t launch_count_rows(const uint8_t *valid, int rows, int K, int32_t *n, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(n, 0, sizeof(int32_t), stream);
    if (e != cudaSuccess)
        return e;
    const int need = (rows + kKlWarps - 1) / kKlWarps;
    const int blocks = need < kKlMaxBlocks ? (need > 0 ? need : 1) : kKlMaxBlocks;
    count_rows_kernel<<<blocks, kKlThreads, 0, stream>>>(valid, rows, K, n);
    return cudaGetLastError();
}

cudaError_t launch_distill_kl(const KlPlan &pl, const float *p, const float *scores, const uint8_t *valid,
                              float coeff, float *loss, float *dscores, void *ws, cudaStream_t stream,
                              const int32_t *n_given)
{
    // completion counter and grid-barrier words start at zero
    cudaError_t e = cudaMemsetAsync(ws, 0, 16, stream);
    if (e != cudaSuccess)
        return e;
    const int K = pl.K;
    if ((K & 3) == 0 && K <= 128)
        return launch_nv<1>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given);
    if ((K & 3) == 0 && K <= 256)
        return launch_nv<2>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given);
    if ((K & 3) == 0 && K <= 512)
        return launch_nv<4>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given);
    return launch_nv<0>(pl, p, scores, valid, coeff, loss, dscores, ws, stream, n_given);
}

}  // namespace sai
