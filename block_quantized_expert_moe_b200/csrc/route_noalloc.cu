// moe_route_topk_noalloc: the router + top-k of moe_route_topk with its
// scratch (the logits matrix and the last-CTA ticket) in a fixed device array
// instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory: code that runs while a stream
// capture in global mode is open (cudaMalloc is an illegal call there), or a
// host framework that forbids allocation once it is serving, because
// cudaMalloc and cudaFree can synchronise the device and stall every stream.
// Such callers pass only their inputs and outputs; the scratch below is part
// of the loaded library.
//
// Limits and sharing:
//   * the array holds kNoallocLogits floats: n_tokens * n_experts must not
//     exceed 65,536 (for example 64 tokens x 1,024 experts); larger calls
//     return MOE_ERR_INVALID_ARG before anything is enqueued;
//   * every GPU that loads the library holds the array (256 KiB + 256 B)
//     until the process exits;
//   * all calls on a device share the array and it keeps the last call's
//     contents: each call clears the ticket (with cudaMemsetAsync on the
//     caller's stream) and overwrites every logit it reads, but two calls that
//     overlap on the GPU (different streams with no ordering between them)
//     race on the array and give wrong results;
//   * the first call on a device looks up the array's device address and sets
//     the router kernel's shared-memory limit (once per device, with that
//     device current; a failed set-up is retried by the next call); make that
//     first call before any stream capture begins;
//   * every call runs the CUDA-core router kernel (route_kernel), also for more
//     than 64 bf16 tokens, where moe_route_topk uses the tensor-core GEMM;
//   * a time-out of the kernel's bounded wait is recorded in word 1 of the
//     array (each call clears it first); moe_route_noalloc_status reads it.
#include <cuda_runtime.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kNoallocLogits = 65536;
constexpr int kNoallocHeader = 256;  // bytes in front of the logits: the ticket

// The scratch itself.  In host code `g_route_scratch` only names the symbol;
// kernels get the device address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kNoallocHeader + kNoallocLogits * sizeof(float)];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[64];
bool g_noalloc_attr[64];  // the router kernel's shared-memory limit is set on this device

}  // namespace

cudaError_t route_set_attributes();
cudaError_t launch_wait_probe(int32_t *err, cudaStream_t s);

namespace {

// Device address of the scratch on `dev` (the current device), looked up once
// per device, and the router kernel's attributes, set once per device; only
// successes are remembered, so a failed set-up is retried by the next call.
cudaError_t noalloc_scratch(int dev, unsigned char **out)
{
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    if (!g_noalloc_attr[dev]) {
        cudaError_t e = route_set_attributes();
        if (e != cudaSuccess) return e;
        g_noalloc_attr[dev] = true;
    }
    *out = static_cast<unsigned char *>(g_noalloc_ptr[dev]);
    return cudaSuccess;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_topk_noalloc(const void *x, moe_dtype x_dtype, const uint16_t *router_w,
                                              int n_tokens, int hidden, int n_experts, int top_k,
                                              int32_t *idx_out, float *gate_out, void *stream)
{
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n_tokens < 0 || hidden < 8 || hidden % 8 || hidden > 16384) return MOE_ERR_INVALID_ARG;
    if (n_experts < 1 || n_experts > 1024 || top_k < 1 || top_k > n_experts) return MOE_ERR_INVALID_ARG;
    if (n_tokens == 0) return MOE_OK;  // an empty batch: nothing to enqueue
    if (!x || !router_w || !idx_out || !gate_out) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(router_w)) & 15u) return MOE_ERR_INVALID_ARG;
    if ((long long)n_tokens * n_experts > kNoallocLogits) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    unsigned char *scratch = nullptr;
    if (noalloc_scratch(dev, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    RouteArgs a{};
    a.x = x;
    a.x_dtype = x_dtype;
    a.wr = router_w;
    a.T = n_tokens;
    a.H = hidden;
    a.E = n_experts;
    a.k = top_k;
    a.rt = route_tokens_per_pass(hidden);
    a.ticket = reinterpret_cast<int32_t *>(scratch);
    a.logits = reinterpret_cast<float *>(scratch + kNoallocHeader);
    a.idx = idx_out;
    a.gate = gate_out;
    a.do_plan = 0;
    a.err = a.ticket + 1;  // word 1: a timed-out wait
    if (cudaMemsetAsync(a.ticket, 0, 64, s) != cudaSuccess) return MOE_ERR_CUDA;  // the tickets (words 0, 2..)
    return launch_route(a, route_grid(n_experts, n_tokens, a.rt, sms), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_route_noalloc_status(void)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    unsigned char *scratch = nullptr;
    if (noalloc_scratch(dev, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int32_t e = 0;
    if (cudaMemcpy(&e, scratch + 4, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (e && cudaMemset(scratch + 4, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status>(e);
}

extern "C" moe_status moe_debug_noalloc_wait_timeout(void *stream)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    unsigned char *scratch = nullptr;
    if (noalloc_scratch(dev, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
    return launch_wait_probe(reinterpret_cast<int32_t *>(scratch + 4), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}
