// decode_noalloc.cu -- rat_decode_step_noalloc: the decode step with its
// scratch memory in a static device array instead of a caller workspace.
//
// Some callers cannot allocate device memory at the moment they run a decode
// step: a plugin inside an inference engine that owns every byte of device
// memory and hands its plugins no scratch buffer, or a serving loop whose
// memory budget is fixed at start-up and forbids cudaMalloc afterwards.  For
// them this entry point takes only the step's inputs and outputs; the split
// partials that rat_decode_step keeps in its workspace live here in
// g_decode_scratch, a file-scope __device__ array of kScratchBytes that every
// GPU loading this library holds until the process exits.
//
// Host code must not hand the array's name to a kernel: on the host it names a
// stand-in, not device memory.  The device address is fetched with
// cudaGetSymbolAddress on the first call made while a device is current, and
// cached together with that device's current context: a call that finds a
// different context there (the old one was destroyed, e.g. by
// cudaDeviceReset, and the module loaded again) fetches the address anew.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "rat_internal.cuh"

using namespace rat;

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices];   // device address of g_decode_scratch, per device
CUcontext g_scratch_ctx[kMaxDevices];  // the context that address belongs to

// The driver's cuCtxGetCurrent, looked up once through the runtime.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

// Device address of the scratch on the current device: looked up on the first
// call in each context of the device, then reused.
rat_status scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices)
        return set_last_error(RAT_ERR_UNSUPPORTED, "rat_decode_step_noalloc: device ordinal above 63");
    CtxGetCurrentFn get_ctx = ctx_get_current();
    if (!get_ctx) return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cuCtxGetCurrent unavailable");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    CUcontext ctx = nullptr;
    if (g_scratch_addr[dev]) {
        // a context is current once the device has been used; compare it
        if (get_ctx(&ctx) != CUDA_SUCCESS)
            return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cuCtxGetCurrent failed");
        if (ctx == g_scratch_ctx[dev]) {
            *out = g_scratch_addr[dev];
            return RAT_OK;
        }
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);  // also makes the device's primary context current
    if (e != cudaSuccess || !p)
        return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cudaGetSymbolAddress of the scratch failed");
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
        return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cuCtxGetCurrent failed");
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
    *out = p;
    return RAT_OK;
}

}  // namespace

extern "C" rat_status rat_decode_step_noalloc(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                                              const void *g, float *state_k, float *state_v, void *cache_k,
                                              void *cache_v, int cache_cap, const int32_t *pos, void *o,
                                              float *lse, rat_stream_t stream) {
    // the argument rules of rat_decode_step, from the same checker
    rat_status st = check_decode_args(cfg, q, k, v, g, state_k, state_v, cache_k, cache_v, cache_cap, pos, o, lse);
    if (st != RAT_OK) return st;
    if (cfg->B == 0) return RAT_OK;

    DecodeParams p;
    memset(&p, 0, sizeof(p));
    const size_t need = sizeof(WsHeader) + decode_plan(cfg, cache_cap, &p);
    if (need > kScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "rat_decode_step_noalloc: needs %zu bytes of scratch, the static scratch holds %zu (16 MiB); "
                 "use rat_decode_step with a workspace", need, kScratchBytes);
        return set_last_error(RAT_ERR_UNSUPPORTED, msg);
    }
    void *scratch = nullptr;
    st = scratch_on_current_device(&scratch);
    if (st != RAT_OK) return st;

    p.q = q; p.k = k; p.v = v; p.g = g;
    p.state[0] = state_k; p.state[1] = state_v;
    p.cache[0] = cache_k; p.cache[1] = cache_v;
    p.pos = pos; p.o = o; p.lse = lse;
    char *w = static_cast<char *>(scratch);
    p.hdr = reinterpret_cast<WsHeader *>(w);
    p.part = reinterpret_cast<float *>(w + sizeof(WsHeader));
    const size_t part_bytes = ((size_t)cfg->B * p.items_per_b * (cfg->d + 2) * sizeof(float) + 255) & ~(size_t)255;
    p.counter = reinterpret_cast<int *>(w + sizeof(WsHeader) + part_bytes);
    p.cap = cache_cap; p.B = cfg->B; p.H = cfg->H; p.d = cfg->d;
    const float scale = cfg->scale > 0.f ? cfg->scale : 1.0f / sqrtf((float)cfg->d);
    p.scale_log2 = scale * 1.4426950408889634f;
    // the per-(b,h) completion counters must start from zero
    cudaError_t ez = cudaMemsetAsync(p.counter, 0, (size_t)cfg->B * cfg->H * sizeof(int), (cudaStream_t)stream);
    if (ez != cudaSuccess) return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: counter reset failed");
    cudaError_t e = launch_decode(p, cfg->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: launch failed");
    return RAT_OK;
}
