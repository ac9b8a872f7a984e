// route_noalloc.cu -- the router entry point for callers that cannot allocate
// device memory.
//
// Some callers may not call cudaMalloc at the point where they run the layer:
// a runtime whose allocator owns all device memory (a caching or pooled
// allocator sized at start-up), a decode loop that must not allocate between
// steps to keep its latency predictable, or code running where the CUDA
// allocation calls are not allowed.  moe_route uses a library-owned workspace
// that is grown with cudaMalloc on first use; moe_route_noalloc runs the same
// two router kernels but keeps their scratch -- the router's partial-logit slices
// and the call's status word -- in a fixed device array compiled into the library.
#include <mutex>

#include "moe.h"
#include "moe_internal.h"

namespace moe {

// Scratch of moe_route_noalloc: 256 bytes of status, then the partial logits
// [splits][M][E] fp32 (splits from route_plan).  Every GPU that loads the library holds
// these 4 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr size_t kNoAllocStatusBytes = 256;
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

// Device address of g_route_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
static int route_scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED_SHAPE;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        addr[dev] = p;
    }
    *out = addr[dev];
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" int moe_route_noalloc(const void *x_bf16, const float *router_w, const float *router_bias,
                                 int32_t *topk_ids, float *topk_w, int M, int H, int E, int k, cudaStream_t stream)
{
    int rc = check_dims(M, H, 32, E, k, false);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    if (!x_bf16 || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    const uintptr_t ax = reinterpret_cast<uintptr_t>(x_bf16), aw = reinterpret_cast<uintptr_t>(router_w);
    if ((ax % 16) || (aw % 16) || (reinterpret_cast<uintptr_t>(topk_ids) % 4) ||
        (reinterpret_cast<uintptr_t>(topk_w) % 4) || (router_bias && reinterpret_cast<uintptr_t>(router_bias) % 4))
        return MOE_ERR_INVALID_ARG;
    const int splits = route_plan(M, H, E).splits;
    const size_t need = kNoAllocStatusBytes + static_cast<size_t>(splits) * M * E * sizeof(float);
    if (need > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
    void *base = nullptr;
    rc = route_scratch_address(&base);
    if (rc != MOE_OK) return rc;
    int *status = static_cast<int *>(base);
    float *partial = reinterpret_cast<float *>(static_cast<unsigned char *>(base) + kNoAllocStatusBytes);
    // every partial logit the top-k kernel reads is written first by the logits kernel, so
    // nothing in the array has to start at zero
    cudaError_t e = launch_route_logits(x_bf16, router_w, partial, nullptr, nullptr, status, nullptr, M, H, E, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_route_topk(partial, splits, router_bias, topk_ids, topk_w, nullptr, nullptr, M, E, k, stream, false);
    if (e != cudaSuccess) return cuda_fail(e);
    return MOE_OK;
}
