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
// Two launches on the caller's stream:
//   1. count: per-block counts of valid rows into the workspace; block 0 also
//      resets the completion counter used below (so the workspace needs no
//      initialisation by the caller);
//   2. rows: every block sums the counts (N), one warp per row computes KL and
//      writes dscores, each block stores its partial KL sum (fp64, fixed
//      order); the last block to finish adds the partials in block order and
//      writes the loss. The result is deterministic run to run.
// HBM-bound: per row it reads p, scores (4K bytes each) and valid (K bytes)
// once and writes dscores (4K bytes).
#include <math.h>

#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

constexpr int kKlThreads = 256;
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlMaxBlocks = 148 * 4;

struct KlWs {
    uint32_t *done;
    int32_t *count_part;
    double *kl_part;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline KlWs ws_layout(void *ws, int count_blocks)
{
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    KlWs w;
    w.done = reinterpret_cast<uint32_t *>(b);
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

// One row, elements held in registers: NV float4 groups per lane, element
// 4*lane + 128*j + e (K % 4 == 0, K <= 128*NV).
template <int NV>
__device__ __forceinline__ float kl_row_vec(const float *__restrict__ pr, const float *__restrict__ sr,
                                            const uint8_t *__restrict__ vr, float *dr, int K, float c)
{
    const int lane = threadIdx.x & 31;
    float4 pv[NV], sv[NV];
    uint32_t vv[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int k = 4 * lane + 128 * j;
        if (k < K) {
            pv[j] = __ldcs(reinterpret_cast<const float4 *>(pr + k));
            sv[j] = __ldcs(reinterpret_cast<const float4 *>(sr + k));
            vv[j] = __ldcs(reinterpret_cast<const unsigned int *>(vr + k));
        } else {
            pv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            sv[j] = pv[j];
            vv[j] = 0u;
        }
    }
    float mx = -INFINITY;
    bool any = false;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {sv[j].x, sv[j].y, sv[j].z, sv[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (vv[j] >> (8 * e)) & 0xffu;
            mx = v ? fmaxf(mx, s4[e]) : mx;
            any |= v;
        }
    }
    mx = warp_max(mx);
    if (!__any_sync(0xffffffffu, any)) {
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
    float se = 0.f, ps = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const float s4[4] = {sv[j].x, sv[j].y, sv[j].z, sv[j].w};
        const float p4[4] = {pv[j].x, pv[j].y, pv[j].z, pv[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (vv[j] >> (8 * e)) & 0xffu;
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
        const float s4[4] = {sv[j].x, sv[j].y, sv[j].z, sv[j].w};
        const float p4[4] = {pv[j].x, pv[j].y, pv[j].z, pv[j].w};
        float d4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool v = (vv[j] >> (8 * e)) & 0xffu;
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

template <int NV>
__global__ void __launch_bounds__(kKlThreads, 4)
    kl_rows_kernel(const float *__restrict__ p, const float *__restrict__ scores, const uint8_t *__restrict__ valid,
                   int rows, int K, float coeff, float *loss, float *dscores, void *ws, int count_blocks,
                   const int32_t *n_given)
{
    KlWs w = ws_layout(ws, count_blocks);
    __shared__ double wkl[kKlWarps];
    __shared__ int nshare;
    __shared__ bool last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // N = number of valid rows: the caller's (e.g. summed over ranks), else
    // from the count kernel's partials.
    int n = 0;
    if (!n_given)
        for (int i = threadIdx.x; i < count_blocks; i += blockDim.x)
            n += w.count_part[i];
    for (int o = 16; o >= 1; o >>= 1)
        n += __shfl_xor_sync(0xffffffffu, n, o);
    if (threadIdx.x == 0)
        nshare = n_given ? *n_given : 0;
    __syncthreads();
    if (lane == 0 && !n_given)
        atomicAdd(&nshare, n);
    __syncthreads();
    const int N = nshare;
    const float c = coeff / (float)(N > 1 ? N : 1);

    double acc = 0.0;
    for (int r = blockIdx.x * kKlWarps + warp; r < rows; r += gridDim.x * kKlWarps) {
        const size_t off = (size_t)r * K;
        float kl;
        if (NV > 0)
            kl = kl_row_vec<(NV > 0 ? NV : 1)>(p + off, scores + off, valid + off, dscores ? dscores + off : nullptr,
                                               K, c);
        else
            kl = kl_row_any(p + off, scores + off, valid + off, dscores ? dscores + off : nullptr, K, c);
        acc += (double)kl;
    }
    if (lane == 0)
        wkl[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int i = 0; i < kKlWarps; ++i)
            s += wkl[i];
        w.kl_part[blockIdx.x] = s;
        __threadfence();
        const uint32_t prev = atomicAdd(w.done, 1u);
        last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (last) {
        // fixed-order parallel sum of the per-block partials
        __threadfence();
        const volatile double *kp = w.kl_part;
        double s = 0.0;
        for (int i = threadIdx.x; i < (int)gridDim.x; i += blockDim.x)
            s += kp[i];
        for (int o = 16; o >= 1; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0)
            wkl[warp] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int i = 0; i < kKlWarps; ++i)
                t += wkl[i];
            *loss = (float)((double)coeff * t / (double)(N > 1 ? N : 1));
        }
    }
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
    cudaError_t e;
    if (n_given) {
        // N is the caller's: only the completion counter needs resetting
        e = cudaMemsetAsync(ws, 0, 16, stream);
    } else {
        kl_count_kernel<<<pl.count_blocks, kKlThreads, 0, stream>>>(valid, pl.rows, pl.K, ws, pl.count_blocks);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess)
        return e;
    const int K = pl.K;
    if ((K & 3) == 0 && K <= 128)
        kl_rows_kernel<1><<<pl.row_blocks, kKlThreads, 0, stream>>>(p, scores, valid, pl.rows, K, coeff, loss,
                                                                     dscores, ws, pl.count_blocks, n_given);
    else if ((K & 3) == 0 && K <= 256)
        kl_rows_kernel<2><<<pl.row_blocks, kKlThreads, 0, stream>>>(p, scores, valid, pl.rows, K, coeff, loss,
                                                                     dscores, ws, pl.count_blocks, n_given);
    else if ((K & 3) == 0 && K <= 512)
        kl_rows_kernel<4><<<pl.row_blocks, kKlThreads, 0, stream>>>(p, scores, valid, pl.rows, K, coeff, loss,
                                                                     dscores, ws, pl.count_blocks, n_given);
    else
        kl_rows_kernel<0><<<pl.row_blocks, kKlThreads, 0, stream>>>(p, scores, valid, pl.rows, K, coeff, loss,
                                                                     dscores, ws, pl.count_blocks, n_given);
    return cudaGetLastError();
}

}  // namespace sai
