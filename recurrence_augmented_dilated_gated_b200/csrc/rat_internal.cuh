// rat_internal.cuh -- parameter blocks and device helpers shared by the kernels
// of librat.so.  Nothing here is part of the public ABI (include/rat.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "rat.h"

namespace rat {

// Raise a kernel's dynamic shared-memory limit once per device.  The setting
// persists, so repeating it on every launch would only add a host call to
// every step (and one more call that stream capture has to tolerate).
// `done` holds one bit per device and must be distinct per kernel.
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, size_t bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

constexpr int kMaxHeads = 256;
constexpr long long kDefaultSpinNs = 1000000000LL;  // 1 s bound on every device-side wait

// First 256 bytes of every workspace.
struct WsHeader {
    int status;                    // first device-side error (a rat_status), 0 = none
    int detail;                    // which unit reported it (e.g. a scan ticket)
    long long stall_ticket_plus1;  // failure injection for the scan look-back, 0 = off
    long long spin_limit_ns;       // 0 = kDefaultSpinNs
    long long pad[29];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

__device__ __forceinline__ void report_error(WsHeader *hdr, int code, int detail) {
    if (atomicCAS(&hdr->status, 0, code) == 0) hdr->detail = detail;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- 4-wide I/O
// Four consecutive channels of a token row: 8 bytes of bf16 or 16 bytes of f32.
template <typename T> struct IO4;

template <> struct IO4<float> {
    static __device__ __forceinline__ float4 load(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ void store(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
};

template <> struct IO4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p) {
        uint2 raw = *reinterpret_cast<const uint2 *>(p);
        float2 lo = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
        float2 hi = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 raw;
        raw.x = *reinterpret_cast<uint32_t *>(&lo);
        raw.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(p) = raw;
    }
};

__device__ __forceinline__ float f4get(const float4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Decode-cache rows of position j for a head with dilation D, window W and
// S = ceil(cap / D) (layout in include/rat.h).  Residue-major: one row.  Fixed
// grid: the grid row when j is on the grid (j mod D == D - 1), and the window
// ring row when the head keeps a ring (D > 1, W > 0); -1 where there is none.
__host__ __device__ __forceinline__ void cache_rows_of(long long j, int D, int W, long long S, int grid,
                                                       long long &grid_row, long long &ring_row) {
    if (!grid) {
        grid_row = (j % D) * S + j / D;
        ring_row = -1;
        return;
    }
    grid_row = (j % D == D - 1) ? j / D : -1;
    ring_row = (D > 1 && W > 0) ? S + j % W : -1;
}

// Element offset of (logical row `row`, channel 0) of (b, h) in a cache: the
// dense [B,H,R,d] block, or the page the table names ([num_pages,H,P,d]); -1
// when the table names no valid page.
__host__ __device__ __forceinline__ long long cache_offset(const int *table, int pps, int page_rows, int num_pages,
                                                           long long cache_R, int H, int d, int b, int h,
                                                           long long row) {
    if (!table) return (((long long)b * H + h) * cache_R + row) * d;
    // one 32-bit division (a row of one sequence's cache fits in 32 bits; a
    // 64-bit division and remainder cost several times as many instructions)
    long long pi, pr;
    if (row >= 0 && row <= 0x7fffffffLL) {
        const unsigned r32 = (unsigned)row, q = r32 / (unsigned)page_rows;
        pi = q;
        pr = r32 - q * (unsigned)page_rows;
    } else {
        pi = row / page_rows;
        pr = row % page_rows;
    }
    const int pg = table[(long long)b * pps + pi];
    if (pg < 0 || pg >= num_pages) return -1;
    return (((long long)pg * H + h) * page_rows + pr) * d;
}

// --------------------------------------------------------------- scan (K1)
struct ScanParams {
    // 4-D TMA maps (d, H, T, B) of k, v, g (loads) and kt, vt (stores), box
    // (d, 1, chunk_len, 1); the T extent clips every box at its batch's end
    CUtensorMap tmap[5];
    int use_tma_out;        // kt / vt maps are valid
    const void *x[2];       // k, v            [B,T,H,d]
    const void *g;          // gate logits     [B,T,H,d]
    const float *init[2];   // [B,H,d] or null
    void *out[2];           // kt, vt or null
    float *fin[2];          // final state [B,H,d] or null
    void *cache[2];         // decode cache [B,H,R,d] or null
    long long cache_R;      // rows per (b,h) cache block
    int cap;
    int grid;               // cache layout of the fixed-grid reading (grid rows + window ring)
    int one;                // one-tensor form: x[0], g -> out[0] (separate gates, run per tensor)
    int t0;                 // position of the call's first token: out rows and cache positions are t0 + t
    const int *page_table;  // paged cache (null: dense), as DecodeParams
    int page_rows, pps, num_pages;
    int B, T, H, d;
    int nslices;            // B * nheads
    int nchunks;            // chunks along T per slice
    int chunk_len;          // timesteps per chunk
    int nheads;             // heads taken by this launch
    unsigned char head_list[kMaxHeads];
    unsigned char head_recur[kMaxHeads];
    int head_dil[kMaxHeads];
    int head_win[kMaxHeads];
    unsigned int *ticket;   // dynamic chunk ticket counter (zeroed per launch)
    int *flags;             // [nslices * nchunks] 0 none, 1 aggregate, 2 inclusive
    float *agg;             // [nslices * nchunks][3][d]  (A, b_k, b_v)
    float *incl;            // [nslices * nchunks][2][d]  state after the chunk
    WsHeader *hdr;
};

// ---------------------------------------------------------- attention (K2/K3)
struct AttnParams {
    const void *q;          // [B,T,H,d]
    const void *kt, *vt;    // augmented keys / values [B,T,H,d]
    const void *kraw, *vraw;// raw keys / values for heads with use_raw (or null)
    void *o;                // [B,T,H,d]
    float *lse;             // [B,H,T] or null
    int B, T, H, d;
    float scale_log2;       // scale * log2(e)
    int t0;                 // chunked prefill: rows are positions t0 + t; kt/vt hold t0 + T rows
    int Th;                 // rows per batch entry of kt/vt
    int grid;               // fixed-grid reading of dilation
    int dedupe;             // the window part skips the dilated set's keys
    int dil[kMaxHeads];
    int win[kMaxHeads];
    unsigned char use_raw[kMaxHeads];
    unsigned char skip[kMaxHeads];   // heads another kernel computes
    WsHeader *hdr;
};

// -------------------------------------------------------------- decode (K4/K5)
struct DecodeParams {
    const void *q, *k, *v, *g;   // [B,H,d]
    float *state[2];             // [B,H,d] fp32, in place
    void *cache[2];              // [B,H,R,d]
    const int *pos;              // device [B]
    void *o;                     // [B,H,d]
    float *lse;                  // [B,H] or null
    float *part;                 // [B][items][d + 2]  (acc[d], m, l) per work item
    int *counter;                // [B][H] items finished (the last one combines and resets it)
    long long cache_R;
    int cap, B, H, d;
    int items_per_b;             // sum over heads of nsplit
    int grid;                    // fixed-grid reading and its cache layout
    int dedupe;                  // the window part skips the dilated set's keys
    int sep;                     // separate key and value gates: g is [2,B,H,d]
    // paged cache (null table: one dense [B,H,R,d] block): logical row r of
    // (b, h) at page table[b * pps + r / page_rows], [num_pages, H, page_rows, d]
    const int *page_table;
    int page_rows, pps, num_pages;
    float scale_log2;
    int dil[kMaxHeads];
    int win[kMaxHeads];
    int slab[kMaxHeads];         // ceil(cap / dil)
    int nsplit[kMaxHeads];       // work items of head h (the last also does the step update)
    int rows_per_item[kMaxHeads];// slab rows per work item
    int item0[kMaxHeads + 1];    // first item of head h within a batch entry
    unsigned char recur[kMaxHeads];
    WsHeader *hdr;
};

// -------------------------------------------------- top-k block decode (K6)
constexpr int kTopkMaxK = 64;          // selected blocks per query, at most
constexpr int kTopkMaxBlocks = 16384;  // blocks of one (b, h) cache, at most (scores in shared memory)

struct TopkParams {
    const void *q, *k, *v, *g;   // [B,H,d]
    float *state[2];             // [B,H,d] fp32, in place
    void *cache[2];              // [B,H,R,d], dense layout: position j at row j
    float *stats;                // [B,H,nblk,2,d] fp32 block statistics
    const int *pos;              // device [B]
    void *o;                     // [B,H,d]
    float *lse;                  // [B,H] or null
    int *sel;                    // [B,H,K] selected blocks or null
    long long cache_R;
    int cap, B, H, d;
    int bs, K, mode, nblk;       // block size, blocks to select, RAT_TOPK_*, ceil(cap / bs)
    int sep;                     // separate key and value gates: g is [2,B,H,d]
    float scale_log2;
    unsigned char recur[kMaxHeads];
    WsHeader *hdr;
};

// Fills the per-head split plan, items_per_b and cache_R of `p` for a decode
// step with capacity `cap` (host).  Returns the scratch bytes the step needs
// after the workspace header: partials plus per-(b,h) counters.
size_t decode_plan(const rat_cfg *c, int cap, DecodeParams *p);

// Process-wide count of kernels this library has launched (rat_launch_count).
void count_launches(int n);

// Record the calling thread's rat_last_error() message; returns s.
rat_status set_last_error(rat_status s, const char *msg);
// Argument checks of a decode step (cfg, pointers, cache_cap), the same for
// every decode entry point; sets the last-error string on failure.
rat_status check_decode_args(const rat_cfg *cfg, const void *q, const void *k, const void *v, const void *g,
                             const float *state_k, const float *state_v, const void *cache_k, const void *cache_v,
                             int cache_cap, const int32_t *pos, const void *o, const float *lse);

// launchers (defined in the kernel files); return cudaGetLastError()
cudaError_t launch_scan(const ScanParams &p, int dtype, cudaStream_t s);
// tokens per scan chunk for head dimension d
int scan_chunk_tokens(int d);
// 4-D TMA map (d, H, T, B) of the first T rows of a [B,Ts,H,d] tensor (Ts rows
// per batch entry), box (d, 1, box_rows, 1), no swizzle
bool encode_map_tokens(CUtensorMap *map, const void *base, int dtype, int B, int T, int Ts, int H, int d,
                       int box_rows);
// final state of the heads in p.head_list, which have no recurrence
cudaError_t launch_final_of_plain_heads(const ScanParams &p, int dtype, cudaStream_t s);
cudaError_t launch_attn_simt(const AttnParams &p, int dtype, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t s);
// block statistics of positions [0, n_tok) of the cache
cudaError_t launch_topk_stats(const TopkParams &p, int n_tok, int dtype, cudaStream_t s);
cudaError_t launch_topk_decode(const TopkParams &p, int dtype, cudaStream_t s);

}  // namespace rat
