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
// stand-in, not device memory.  The device address is fetched once per device
// with cudaGetSymbolAddress, on the first call made while that device is
// current, and cached.
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
void *g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// Device address of the scratch on the current device (set up on first use).
rat_status scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices)
        return set_last_error(RAT_ERR_UNSUPPORTED, "rat_decode_step_noalloc: device ordinal above 63");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p)
            return set_last_error(RAT_ERR_CUDA, "rat_decode_step_noalloc: cudaGetSymbolAddress of the scratch failed");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return RAT_OK;
}

bool a16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" rat_status rat_decode_step_noalloc(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                                              const void *g, float *state_k, float *state_v, void *cache_k,
                                              void *cache_v, int cache_cap, const int32_t *pos, void *o,
                                              float *lse, rat_stream_t stream) {
    // the same argument rules as rat_decode_step
    const char *bad = nullptr;
    if (!cfg) bad = "cfg is NULL";
    else if (cfg->B < 0 || cfg->H < 1 || cfg->H > kMaxHeads || (cfg->d != 64 && cfg->d != 128))
        bad = "need B >= 0, 1 <= H <= 256, d in {64, 128}";
    else if (cfg->dtype != RAT_F32 && cfg->dtype != RAT_BF16) bad = "invalid dtype";
    else if (!cfg->dil || !cfg->win) bad = "cfg->dil / cfg->win is NULL";
    else if (!(cfg->scale == cfg->scale)) bad = "scale is NaN";
    else if (cache_cap < 1) bad = "cache_cap < 1";
    if (!bad && cfg->B > 0) {
        for (int h = 0; h < cfg->H && !bad; ++h)
            if (cfg->dil[h] < 1 || cfg->win[h] < 0) bad = "dil[h] must be >= 1 and win[h] >= 0";
        const void *req[] = {q, k, v, g, state_k, state_v, cache_k, cache_v, pos, o};
        for (const void *ptr : req)
            if (!bad && (!ptr || !a16(ptr))) bad = "a required pointer is NULL or not 16-byte aligned";
        if (!bad && lse && !a16(lse)) bad = "lse is not 16-byte aligned";
    }
    if (bad) return set_last_error(RAT_ERR_INVALID, bad);
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
    rat_status st = scratch_on_current_device(&scratch);
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
