// Routing (router logits + softmax top-k) that allocates nothing.
//
// Some callers cannot call cudaMalloc at all: code that runs inside another
// runtime's memory pool or a fixed-budget service, callers that forbid device
// allocation after start-up so that memory use stays predictable, and plain C
// hosts that only hold device pointers handed to them.  moe_route_static
// serves them: it takes the router weights and the tokens as device pointers
// and keeps its one intermediate (the logits) in a fixed array in device
// memory that the library reserves when it is loaded.
#include <mutex>
#include <stdio.h>

#include "moe_internal.cuh"

// The logits scratch (plus a zero bias row for callers without a bias):
// MOE_ROUTE_STATIC_MAX_LOGITS floats, i.e. tokens x experts of one call.
// Every device that loads the library holds this array until the process
// exits.
static __device__ __align__(256) float g_route_scratch[MOE_ROUTE_STATIC_MAX_LOGITS + 1024];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scratch_ptr[kMaxDevices] = {};   // device address of g_route_scratch, per device

// Host code cannot take the device address of a __device__ array directly;
// ask the runtime for it once per device, with that device current.  The
// address belongs to the device's primary context: after cudaDeviceReset on a
// device this library must not be used on that device again in the process.
int scratch_for_current_device(float **out) {
    int dev = 0;
    QE_CHECK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return qeffn::set_cuda_error(e, "cudaGetSymbolAddress(g_route_scratch)");
        g_scratch_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" int moe_route_static(const uint16_t *x_bf16, int T, int d_model, const float *router_w,
                                const float *router_bias, int n_experts, int top_k, int32_t *ids,
                                float *w, void *stream) {
    if (!x_bf16 || !router_w || !ids || !w || T < 0 || d_model <= 0 || n_experts <= 0 || top_k <= 0 ||
        top_k > n_experts || top_k > 32 || n_experts > 1024 || d_model % 4 != 0 || d_model > 16384)
        return MOE_ERR_INVALID_ARG;
    // the router reads its weight rows with 16-byte loads
    if (reinterpret_cast<uintptr_t>(router_w) % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if ((long long)T * n_experts > MOE_ROUTE_STATIC_MAX_LOGITS) {
        return qeffn::set_too_many(
            "moe_route_static: T * n_experts exceeds the fixed scratch of MOE_ROUTE_STATIC_MAX_LOGITS");
    }
    float *scratch = nullptr;
    int s = scratch_for_current_device(&scratch);
    if (s != MOE_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    float *logits = scratch + 1024;
    const float *bias = router_bias;
    if (!bias) {   // the zero row at the front of the scratch; cleared on every call
        QE_CHECK(cudaMemsetAsync(scratch, 0, sizeof(float) * n_experts, st));
        bias = scratch;
    }
    return qeffn::launch_route_raw(x_bf16, T, d_model, n_experts, top_k, router_w, bias, logits, ids, w, st);
}
