// sai_distill_kl_noalloc: sai_distill_kl without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they need the
// loss: a framework plugin whose host owns every device allocation (and would
// see a stray cudaMalloc as a leak or an out-of-budget failure), code that must
// not take cudaMalloc's implicit device-wide synchronisation on a latency
// path, or a caller that simply has no allocator handy. This entry point runs
// the same two kernels as sai_distill_kl with their scratch words in a fixed,
// file-scope device array instead of a workspace argument.
//
// The array (kNoallocScratchBytes) is part of the library's device image, so
// every GPU that loads the library holds it until the process exits. All calls
// on a device share it: two calls that run at the same time on that device
// (different streams, or different host threads) race on it and may corrupt
// each other's loss. The kernels overwrite every scratch word they read, so
// nothing needs clearing between calls.
//
// The device address of the array is looked up once per device, on the first
// call made with that device current (cudaGetSymbolAddress). Make that first
// call before any stream capture begins.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <mutex>

#include "sai.h"
#include "sai_kernels.h"

namespace {

// Largest scratch the KL kernels use: their block counts are capped, so this
// bound holds for every (B, S, K) that sai_distill_kl accepts.
constexpr size_t kNoallocScratchBytes = 8192;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_kl_scratch[kNoallocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_kl_scratch for the current device (looked up once).
sai_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return SAI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kl_scratch) != cudaSuccess || !p)
            return SAI_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SAI_OK;
}

}  // namespace

extern "C" size_t sai_distill_kl_noalloc_max_scratch_bytes(void) { return kNoallocScratchBytes; }

extern "C" sai_status sai_distill_kl_noalloc(const float *p, const float *scores, const uint8_t *valid, int B, int S,
                                             int K, float coeff, float *loss, float *dscores, void *stream)
{
    if (!p || !scores || !valid || !loss)
        return SAI_ERR_NULL;
    if (B < 1 || S < 1 || K < 1 || !isfinite(coeff) || (int64_t)B * S * K > INT32_MAX)
        return SAI_ERR_SHAPE;
    const uintptr_t m16 = 15u;
    if ((reinterpret_cast<uintptr_t>(p) & m16) || (reinterpret_cast<uintptr_t>(scores) & m16) ||
        (reinterpret_cast<uintptr_t>(valid) & m16) || (reinterpret_cast<uintptr_t>(loss) & 3u) ||
        (dscores && (reinterpret_cast<uintptr_t>(dscores) & m16)))
        return SAI_ERR_ALIGN;
    const sai::KlPlan pl = sai::kl_plan(B, S, K);
    if (pl.ws_bytes > kNoallocScratchBytes)
        return SAI_ERR_WORKSPACE;  // sizes whose scratch would not fit the static array
    void *ws = nullptr;
    const sai_status st = scratch_for_current_device(&ws);
    if (st != SAI_OK)
        return st;
    return sai::launch_distill_kl(pl, p, scores, valid, coeff, loss, dscores, ws,
                                  reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAI_OK
               : SAI_ERR_CUDA;
}
