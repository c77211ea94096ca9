// CUDA-core kernels for shapes the tensor-core kernels do not take (few
// heads, D not a multiple of 64). One CTA per token, fp32 arithmetic, the
// same formulas as the tensor-core path:
//   window_lse[t,h] = log sum_{window} exp(scale <q_h, k_s>)
//   p[k] = u[k] / max(m, FLT_MIN), u[k] = sum_h exp(z[k,h] - lse_full[h])
// (Primus page "perf(deepseek-v4): fuse and enable the indexer distillation
// loss", first and second commit messages.)
#include <math.h>

#include "sai_device.cuh"
#include "sai_kernels.h"

namespace sai {
namespace {

constexpr int kGenThreads = 128;
constexpr float kLnFltMinG = -87.33654475055310898657f;
constexpr float kLnOldFloorG = -23.025850929940457f;  // log(1e-10), the per-branch target's floor

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

__device__ __forceinline__ float block_sum(float v, float *scratch)
{
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0)
        scratch[w] = v;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i)
        s += scratch[i];
    return s;
}

__global__ void __launch_bounds__(kGenThreads)
    window_lse_generic_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ Kw,
                              const int32_t *__restrict__ doc_start, int S, int H, int D, int W, int t_begin,
                              int kw_lead, float scale, float *__restrict__ out)
{
    extern __shared__ float gsm[];
    float *qs = gsm;               // [H][D]
    float *zs = qs + H * D;        // [H][W]
    const int g = blockIdx.x;
    const int b = g / S;
    const int t = g - b * S + t_begin;   // sequence position
    int d0 = 0;
    if (doc_start) {
        d0 = doc_start[g];
        d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
    }
    const int lo = max(max(d0, t - W + 1), t_begin - kw_lead);
    const int nw = t - lo + 1;
    for (int i = threadIdx.x; i < H * D; i += blockDim.x)
        qs[i] = bf16f(Q[(size_t)g * H * D + i]);
    __syncthreads();
    for (int pr = threadIdx.x; pr < H * nw; pr += blockDim.x) {
        const int h = pr / nw, s = lo + pr % nw;
        // Kw is [B, S + kw_lead, D]; position s is row s - t_begin + kw_lead
        const uint16_t *k = Kw + ((size_t)b * (S + kw_lead) + (s - t_begin + kw_lead)) * D;
        float acc = 0.f;
        for (int d = 0; d < D; ++d)
            acc = fmaf(qs[h * D + d], bf16f(k[d]), acc);
        zs[h * W + (s - lo)] = acc * scale;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < H; h += blockDim.x >> 5) {
        float mx = -INFINITY;
        for (int i = lane; i < nw; i += 32)
            mx = fmaxf(mx, zs[h * W + i]);
        for (int o = 16; o >= 1; o >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float se = 0.f;
        for (int i = lane; i < nw; i += 32)
            se += expf(zs[h * W + i] - mx);
        for (int o = 16; o >= 1; o >>= 1)
            se += __shfl_xor_sync(0xffffffffu, se, o);
        if (lane == 0)
            out[(size_t)g * H + h] = mx + logf(se);
    }
}

__global__ void __launch_bounds__(kGenThreads)
    target_generic_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ pool,
                          const int32_t *__restrict__ idx, const float *__restrict__ wl,
                          const float *__restrict__ sink, const int32_t *__restrict__ doc_start, int S, int P,
                          int t_begin, int H, int D, int K, int cr, float scale, int lse_mode,
                          float *__restrict__ p, int32_t *err)
{
    extern __shared__ float gsm[];
    float *qs = gsm;                              // [H][D]
    float *zs = qs + H * D;                       // [K][H] (compacted rows)
    float *hM = zs + K * H;                       // [H]
    float *hA = hM + H;                           // [H]
    float *us = hA + H;                           // [K]
    float *scratch = us + K;                      // [32]
    int *rows = reinterpret_cast<int *>(scratch + 32);  // [K]
    int *slots = rows + K;                        // [K]
    int *cnt = slots + K;                         // [1]
    const int g = blockIdx.x;
    const int b = g / S;
    const int t = g - b * S + t_begin;   // sequence position
    int d0 = 0;
    if (doc_start) {
        d0 = doc_start[g];
        d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
    }
    if (threadIdx.x == 0)
        *cnt = 0;
    for (int i = threadIdx.x; i < H * D; i += blockDim.x)
        qs[i] = bf16f(Q[(size_t)g * H * D + i]);
    __syncthreads();
    float *prow = p + (size_t)g * K;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const int j = idx ? idx[(size_t)g * K + k] : k;   // NULL: dense, slot k is block k
        const bool inr = j >= 0 && j < P;
        if (!(j == -1 || inr) && err)
            atomicExch(err, kErrIndex);
        if (inr && (j + 1) * cr - 1 <= t && j * cr >= d0) {
            const int pos = atomicAdd(cnt, 1);
            rows[pos] = b * P + j;
            slots[pos] = k;
        } else {
            prow[k] = 0.f;
        }
    }
    __syncthreads();
    const int nsel = *cnt;
    if (nsel == 0)
        return;
    for (int pr = threadIdx.x; pr < nsel * H; pr += blockDim.x) {
        const int j = pr / H, h = pr - j * H;
        const uint16_t *pv = pool + (size_t)rows[j] * D;
        float acc = 0.f;
        for (int d = 0; d < D; ++d)
            acc = fmaf(qs[h * D + d], bf16f(pv[d]), acc);
        zs[j * H + h] = acc * scale;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        float M = -INFINITY;
        for (int j = 0; j < nsel; ++j)
            M = fmaxf(M, zs[j * H + h]);
        float se = 0.f;
        for (int j = 0; j < nsel; ++j)
            se += expf(zs[j * H + h] - M);
        const float clse = M + logf(se);
        hM[h] = M;
        if (lse_mode == kLsePerBranch) {
            hA[h] = M - clse;                     // each head normalised over its selected entries
            continue;
        }
        const float w = wl[(size_t)g * H + h];
        if (lse_mode == kLseGiven) {
            hA[h] = M - w;                        // the whole row's normaliser, as given
            continue;
        }
        float mm = fmaxf(w, clse);
        if (sink)
            mm = fmaxf(mm, sink[h]);
        float acc = expf(w - mm) + expf(clse - mm);
        if (sink)
            acc += expf(sink[h] - mm);
        hA[h] = M - (mm + logf(acc));
    }
    __syncthreads();
    float At = -INFINITY;
    for (int h = 0; h < H; ++h)
        At = fmaxf(At, hA[h]);
    float mpart = 0.f;
    for (int j = threadIdx.x; j < nsel; j += blockDim.x) {
        float u = 0.f;
        for (int h = 0; h < H; ++h)
            u = fmaf(expf(zs[j * H + h] - hM[h]), expf(hA[h] - At), u);
        us[j] = u;
        mpart += u;
    }
    const float mt = block_sum(mpart, scratch);
    const float ln_floor = lse_mode == kLsePerBranch ? kLnOldFloorG : kLnFltMinG;
    const bool plain = logf(mt) + At >= ln_floor;
    const float f = plain ? 0.f : expf(At - ln_floor);
    for (int j = threadIdx.x; j < nsel; j += blockDim.x)
        prow[slots[j]] = plain ? us[j] / mt : us[j] * f;
}

}  // namespace

size_t window_simt_smem_bytes(int H, int D, int W) { return (size_t)(H * D + H * W) * 4; }

cudaError_t launch_window_lse_simt(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start, int B, int S,
                                   int H, int D, int W, int t_begin, int kw_lead, float scale, float *out,
                                   cudaStream_t stream)
{
    const size_t smem = window_simt_smem_bytes(H, D, W);
    cudaError_t e = cudaFuncSetAttribute(window_lse_generic_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    window_lse_generic_kernel<<<B * S, kGenThreads, smem, stream>>>(Q, Kw, doc_start, S, H, D, W, t_begin, kw_lead,
                                                                    scale, out);
    return cudaGetLastError();
}

size_t target_simt_smem_bytes(int H, int D, int K)
{
    return (size_t)(H * D + K * H + 2 * H + K + 32) * 4 + (size_t)(2 * K + 1) * 4;
}

cudaError_t launch_target_simt(const uint16_t *Q, const uint16_t *pool, const int32_t *idx, const float *wl,
                               const float *sink, const int32_t *doc_start, int B, int S, int P, int t_begin,
                               int H, int D, int K, int cr, float scale, int lse_mode, float *p, int32_t *err,
                               cudaStream_t stream)
{
    const size_t smem = target_simt_smem_bytes(H, D, K);
    cudaError_t e =
        cudaFuncSetAttribute(target_generic_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    target_generic_kernel<<<B * S, kGenThreads, smem, stream>>>(Q, pool, idx, wl, sink, doc_start, S, P, t_begin, H,
                                                                D, K, cr, scale, lse_mode, p, err);
    return cudaGetLastError();
}

}  // namespace sai
