// attn_simt.cu -- K2f: the attention step on CUDA cores in fp32.
//
// "RAT+: Train Dense, Infer Sparse", Abstract and Figure 1(c): query t attends
// to the dilated set { j <= t : (t-j) mod D == 0 } and, when the head has a
// window W > 0, in a second softmax to { max(0, t-W+1) <= j <= t }; the two
// softmaxes are merged by log-sum-exp.  Under the fixed-grid reading the
// dilated set is { j <= t : j mod D == D-1 } plus t itself (once).  With
// dedupe the window part skips the keys of the dilated set.
//
// One warp owns one query row: each lane holds d/32 channels of q and of the
// running output, the score of every key is a warp-wide dot product, and the
// softmax is accumulated online in the log2 domain.  This is the path for fp32
// operands (tensor cores would round them) and it needs no particular d.
#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kWarps = 8;

template <typename T> __device__ __forceinline__ float ld1(const T *p);
template <> __device__ __forceinline__ float ld1<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
template <typename T> __device__ __forceinline__ void st1(T *p, float v);
template <> __device__ __forceinline__ void st1<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

template <int CPL>
struct RowState {
    float m, l, acc[CPL];
    __device__ __forceinline__ void init() {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
    }
};

// Online softmax over keys j = jhi, jhi - step, ..., >= jlo (log2-domain scores);
// with skip_d > 0, keys in the dilated set of row t (dilation skip_d; fixed
// grid when grid) are left out.
template <typename T, int CPL>
__device__ __forceinline__ void attend(RowState<CPL> &st, const float *q, const T *kb, const T *vb,
                                       size_t rs, long long jlo, long long jhi, long long step, int lane,
                                       int skip_d = 0, long long t = 0, int grid = 0) {
    for (long long j = jhi; j >= jlo; j -= step) {
        if (skip_d > 0 && (grid ? (j % skip_d == skip_d - 1 || j == t) : ((t - j) % skip_d == 0))) continue;
        const T *kr = kb + (size_t)j * rs;
        const T *vr = vb + (size_t)j * rs;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) s += q[i] * ld1<T>(kr + lane + 32 * i);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float mn = fmaxf(st.m, s);
        const float corr = exp2f(st.m - mn);
        const float pj = exp2f(s - mn);
        st.l = st.l * corr + pj;
#pragma unroll
        for (int i = 0; i < CPL; ++i) st.acc[i] = st.acc[i] * corr + pj * ld1<T>(vr + lane + 32 * i);
        st.m = mn;
    }
}

template <typename T, int CPL>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(const AttnParams p) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long nrows = (long long)p.B * p.H * p.T;
    if (row >= nrows) return;
    // rows ordered (b, h, t); t is the position, tl the row of this call
    const long long tl = row % p.T;
    const long long t = p.t0 + tl;
    const int h = (int)((row / p.T) % p.H);
    const int b = (int)(row / ((long long)p.T * p.H));
    if (p.skip[h]) return;  // uniform across the warp (one row per warp)
    const int d = p.d;
    const size_t rs = (size_t)p.H * d;
    const size_t hb = ((size_t)b * p.T * p.H + h) * d;                        // (b, row 0, h, 0) of q and o
    // (b, position 0, h, 0) of kt, vt: Th rows per batch entry (raw k, v: the call's T)
    const size_t hk = ((size_t)b * (size_t)(p.use_raw[h] ? p.T : p.Th) * p.H + h) * d;
    const T *qb = static_cast<const T *>(p.q) + hb;
    const T *kb = static_cast<const T *>(p.use_raw[h] ? p.kraw : p.kt) + hk;
    const T *vb = static_cast<const T *>(p.use_raw[h] ? p.vraw : p.vt) + hk;

    float q[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) q[i] = ld1<T>(qb + (size_t)tl * rs + lane + 32 * i) * p.scale_log2;

    const int D = p.dil[h], W = p.win[h];
    RowState<CPL> dil, wnd;
    dil.init();
    if (p.grid && D > 1) {
        // the grid keys up to t, then t itself unless it is on the grid
        const long long g_hi = (t + 1) / D * D - 1;
        attend<T, CPL>(dil, q, kb, vb, rs, D - 1, g_hi, D, lane);
        if (t % D != D - 1) attend<T, CPL>(dil, q, kb, vb, rs, t, t, 1, lane);
    } else {
        attend<T, CPL>(dil, q, kb, vb, rs, t % D, t, D, lane);
    }
    float m = dil.m, l = dil.l;
    float acc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = dil.acc[i];
    if (W > 0) {
        wnd.init();
        attend<T, CPL>(wnd, q, kb, vb, rs, max(0LL, t - W + 1), t, 1, lane, p.dedupe ? D : 0, t, p.grid);
        // log-sum-exp merge of two (unnormalised) softmax accumulators
        const float mn = fmaxf(dil.m, wnd.m);
        const float c1 = exp2f(dil.m - mn), c2 = exp2f(wnd.m - mn);
        l = dil.l * c1 + wnd.l * c2;
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[i] = dil.acc[i] * c1 + wnd.acc[i] * c2;
        m = mn;
    }
    const float inv = 1.f / l;
    T *ob = static_cast<T *>(p.o) + hb + (size_t)tl * rs;
#pragma unroll
    for (int i = 0; i < CPL; ++i) st1<T>(ob + lane + 32 * i, acc[i] * inv);
    if (p.lse && lane == 0)
        p.lse[((size_t)b * p.H + h) * p.T + tl] = (m + log2f(l)) * 0.69314718055994531f;
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams &p, int dtype, cudaStream_t s) {
    const long long nrows = (long long)p.B * p.H * p.T;
    const unsigned grid = (unsigned)((nrows + kWarps - 1) / kWarps);
    if (grid == 0) return cudaSuccess;
    if (dtype == RAT_BF16) {
        if (p.d == 128) attn_simt_kernel<__nv_bfloat16, 4><<<grid, kWarps * 32, 0, s>>>(p);
        else attn_simt_kernel<__nv_bfloat16, 2><<<grid, kWarps * 32, 0, s>>>(p);
    } else {
        if (p.d == 128) attn_simt_kernel<float, 4><<<grid, kWarps * 32, 0, s>>>(p);
        else attn_simt_kernel<float, 2><<<grid, kWarps * 32, 0, s>>>(p);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
