// Top-K compressed-block selection per token from given indexer scores
// (MaxText page "Add Indexer Loss [Deepseek v4]": the indexer keeps its
// top-k block indices, writes -1 wherever the choice is invalid and returns
// the scores alongside; its commit messages give the causal block mask and
// the packing mask). The indexer's own score formula is not on the pages;
// its output is this kernel's input.
//
// Rule: block j of token (b,t) is a candidate iff (j+1)*cr - 1 <= t,
// j*cr >= d0 (the token's document start) and its score is neither NaN nor
// -inf. The K candidates with the largest scores are selected, an equal
// score going to the lower block (+0 and -0 are equal). Slot k holds the
// k-th selected block in ascending block order; the slots past the number
// selected hold -1.
//
// One CTA per token row. HBM-bound: a row's candidate scores are read once
// (about half the row on average, since later blocks are in the future; only
// the candidate range is read and walked), kept in shared memory as
// order-preserving 32-bit keys, and selected with an 8-bit radix select
// (up to four histogram passes; it stops early once the crossing bin holds
// exactly the keys still needed) for the K-th largest key.
// A block-wide scan then compacts the selected blocks in block order, which
// gives the ascending slot order without a sort.
#include <cuda_runtime.h>
#include <stdint.h>

#include "indexer_topk.h"

namespace sai {
namespace {

constexpr int kTkThreads = 256;
constexpr int kTkWarps = kTkThreads / 32;

// Order-preserving key of a score: a larger score gives a larger key, +0 and
// -0 give the same key, and 0 marks an entry that cannot be selected (NaN or
// -inf). Every selectable key is at least the key of -FLT_MAX, 0x00800000.
__device__ __forceinline__ uint32_t order_key(float x)
{
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7fffffffu) > 0x7f800000u || u == 0xff800000u)   // NaN, -inf
        return 0u;
    if ((u << 1) == 0u)                                         // -0 -> +0
        u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of v over the block (thread order), and the total
// (unsigned: callers pack two counts of at most 16 bits each into one word).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_buf, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        warp_buf[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w) {
        const uint32_t x = warp_buf[w];
        before += (w < warp) ? x : 0u;
        tot += x;
    }
    total = tot;
    return before + incl - v;
}

// Sum of v over the block, in every thread, with one barrier. The caller
// must pass another barrier before warp_buf is written again.
__device__ __forceinline__ int block_total(int v, uint32_t *warp_buf)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0)
        warp_buf[warp] = (uint32_t)v;
    __syncthreads();
    int tot = 0;
#pragma unroll
    for (int w = 0; w < kTkWarps; ++w)
        tot += (int)warp_buf[w];
    return tot;
}

__global__ void __launch_bounds__(kTkThreads)
    indexer_topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ doc_start, int S, int cr,
                        int P, int K, int32_t *__restrict__ idx, float *__restrict__ sel,
                        uint8_t *__restrict__ valid)
{
    extern __shared__ uint32_t keys[];   // [jhi - jlo] (at most P)
    __shared__ int hist[2][256];         // one per radix pass, in turn
    __shared__ uint32_t warp_buf[kTkWarps];
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem;
    __shared__ int s_done;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x;
    const int t = g % S;
    int d0 = 0;
    if (doc_start) {
        d0 = doc_start[g];
        d0 = d0 < 0 ? 0 : (d0 > t ? t : d0);
    }
    // candidates are the blocks j in [jlo, jhi): (j+1)*cr - 1 <= t and j*cr >= d0
    const int jhi = min(P, (t + 1) / cr);
    const int jlo = min(jhi, (d0 + cr - 1) / cr);
    const int L = jhi - jlo;                          // keys[i] is block jlo + i
    const float *row = scores + (size_t)g * P + jlo;

    int cnt = 0;
    for (int i = tid; i < L; i += kTkThreads) {
        const uint32_t k = order_key(__ldg(row + i));
        keys[i] = k;
        cnt += k != 0u;
    }
    hist[0][tid] = 0;                                // the first pass's bins (256 threads, 256 bins)
    // one barrier: the candidate count, and the key writes ordered before the
    // reads below (warp_buf is next written after the radix passes' barriers)
    const int n_cand = block_total(cnt, warp_buf);

    // Threshold key T and the number `rem` of entries equal to T to take.
    // With no more candidates than K, every candidate is taken (T = 0).
    uint32_t T = 0u;
    int rem = 0;
    if (n_cand > K) {
        uint32_t prefix = 0u, mask = 0u;
        rem = K;
        int pass = 0;
        for (int shift = 24; shift >= 0; shift -= 8, ++pass) {
            int *h = hist[pass & 1];
            // the next pass's bins, cleared now: nothing reads them until the
            // barrier after this pass's scan
            hist[(pass + 1) & 1][tid] = 0;
            for (int i = tid; i < L; i += kTkThreads) {
                const uint32_t k = keys[i];
                if (k != 0u && (k & mask) == prefix)
                    atomicAdd(&h[(k >> shift) & 255u], 1);
            }
            __syncthreads();
            if (warp == 0) {
                // lane l holds bins 255-8l, 254-8l, ..., 248-8l (high to low)
                int c[8], sum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    c[e] = h[255 - 8 * lane - e];
                    sum += c[e];
                }
                int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o)
                        incl += y;
                }
                const int excl = incl - sum;
                // the keys matching the prefix number at least rem, so exactly
                // one lane holds the bin where the count from the top reaches rem
                const unsigned here = __ballot_sync(0xffffffffu, excl < rem && rem <= incl);
                if (lane == __ffs(here) - 1) {
                    int acc = excl, e = 0;
                    while (e < 7 && acc + c[e] < rem)
                        acc += c[e++];
                    s_prefix = prefix | ((uint32_t)(255 - 8 * lane - e) << shift);
                    s_rem = rem - acc;
                    // every key of the crossing bin is needed: the keys above the
                    // bin's lowest value are exactly the selection
                    s_done = (rem - acc == c[e]) ? 1 : 0;
                }
            }
            __syncthreads();
            prefix = s_prefix;
            rem = s_rem;
            mask |= 255u << shift;
            if (s_done && shift > 0 && prefix != 0u) {
                // take every key with this prefix: k > prefix - 1 (the keys
                // below the bin are smaller)
                prefix -= 1u;
                rem = 0;
                break;
            }
        }
        T = prefix;
    }

    // warp_buf is written again below: with no radix pass since block_total's
    // reads, a barrier first (n_cand is the same in every thread)
    if (n_cand <= K)
        __syncthreads();

    // Compaction in block order: thread n owns candidates [n*E, (n+1)*E).
    const int E = (L + kTkThreads - 1) / kTkThreads;
    const int i0 = min(L, tid * E), i1 = min(L, i0 + E);
    int cgt = 0, ceq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t k = keys[i];
        cgt += k > T;
        ceq += (k != 0u && k == T);
    }
    // one scan of both counts, packed (each below 2^16: L <= P, and P keys
    // fit the shared memory only below that)
    uint32_t packed_total = 0;
    const uint32_t packed_before =
        block_excl_scan(((uint32_t)cgt << 16) | (uint32_t)ceq, warp_buf, packed_total);
    const int eq_before = (int)(packed_before & 0xffffu);
    // keys before this thread's: every key above T, and the first `rem` equal to T
    int slot = (int)(packed_before >> 16) + min(eq_before, rem);
    const int n_out = (int)(packed_total >> 16) + min((int)(packed_total & 0xffffu), rem);
    int32_t *irow = idx + (size_t)g * K;
    float *srow = sel ? sel + (size_t)g * K : nullptr;
    uint8_t *vrow = valid ? valid + (size_t)g * K : nullptr;
    int eq_seen = eq_before;
    for (int i = i0; i < i1; ++i) {
        const uint32_t k = keys[i];
        bool take = k > T;
        if (!take && k != 0u && k == T)
            take = eq_seen++ < rem;
        if (take) {
            irow[slot] = jlo + i;
            if (srow)
                srow[slot] = __ldg(row + i);
            if (vrow)
                vrow[slot] = 1;
            ++slot;
        }
    }
    for (int k = n_out + tid; k < K; k += kTkThreads) {
        irow[k] = -1;
        if (srow)
            srow[k] = 0.f;
        if (vrow)
            vrow[k] = 0;
    }
}

}  // namespace

size_t indexer_topk_smem_bytes(int P) { return (size_t)P * 4; }

cudaError_t launch_indexer_topk(const float *scores, const int32_t *doc_start, int B, int S, int cr, int K,
                                int32_t *idx, float *sel, uint8_t *valid, cudaStream_t stream)
{
    const int P = S / cr;
    const size_t smem = indexer_topk_smem_bytes(P);
    cudaError_t e = cudaFuncSetAttribute(indexer_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    indexer_topk_kernel<<<B * S, kTkThreads, smem, stream>>>(scores, doc_start, S, cr, P, K, idx, sel, valid);
    return cudaGetLastError();
}

}  // namespace sai
