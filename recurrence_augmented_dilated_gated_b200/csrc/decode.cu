// decode.cu -- K4/K5: one decode step of the temporal-mixing operator
// ("RAT+: Train Dense, Infer Sparse", Figure 2: decode updates the recurrence
// with a simple step and attends over the dilated KV cache; Abstract: the
// dilated pattern cuts the KV cache a step reads by D).
//
// For batch entry b, head h, new token at t = pos[b], dilation D, window W:
//   s <- a*s + (1-a)*x (x = k, v; a = sigmoid(g), a = 0 without recurrence),
//   the new augmented row is stored at cache row (t mod D)*S + t/D,
//   o = softmax over the multiset  { j <= t, j == t mod D }  (+)  { t-W+1..t }.
// Softmaxes over disjoint pieces of a key multiset combine exactly by
// log-sum-exp, so the step is split into independent work items whose partial
// (unnormalised accumulator, running max, running sum) are merged by K5:
//   * items 0..nsplit_h-1 : consecutive runs of `rows_per_split` old rows of the
//     residue slab (t mod D) -- one contiguous, coalesced stream per item;
//   * the tail item       : the step update of the recurrent state, the append
//     of the new row, the new row's dilated score, and the window rows.
// Only the tail item touches the state and the new cache row, and no other
// item reads that row, so the items need no ordering among themselves.
// The work is HBM-bound: each cache row is read once, 2*d bytes of bf16 per
// row and tensor (K~ and V~).
#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kThreads = 128;
constexpr int kUnroll = 4;

// 8 consecutive channels (16 bytes of bf16, 32 bytes of f32) as floats
template <typename T> struct IO8;
template <> struct IO8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *f) {
        uint4 raw = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <> struct IO8<float> {
    static __device__ __forceinline__ void load(const float *p, float *f) {
        float4 a = reinterpret_cast<const float4 *>(p)[0];
        float4 b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <typename T> __device__ __forceinline__ float round_to(float x);
template <> __device__ __forceinline__ float round_to<float>(float x) { return x; }
template <> __device__ __forceinline__ float round_to<__nv_bfloat16>(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}
template <typename T> __device__ __forceinline__ T to_t(float x);
template <> __device__ __forceinline__ float to_t<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 to_t<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ int find_head(const DecodeParams &p, int it) {
    int lo = 0, hi = p.H - 1;  // largest h with item0[h] <= it
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (p.item0[mid] <= it) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Per row-group online softmax state (log2-domain scores).
struct Acc8 {
    float m, l, o[8];
};

// Sum over the LPR lanes of one row group.  The row groups of a warp can take
// different branches (their rows differ), so the shuffle names only the lanes
// of the calling group; every xor partner (offset < LPR) lies inside it.
template <int LPR>
__device__ __forceinline__ unsigned group_mask() {
    const unsigned lane = threadIdx.x & 31u;
    const unsigned ones = LPR == 32 ? 0xffffffffu : ((1u << LPR) - 1u);
    return ones << (lane / LPR * LPR);
}

template <int LPR>
__device__ __forceinline__ float group_sum(float s) {
    const unsigned mask = group_mask<LPR>();
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(mask, s, off);
    return s;
}

__device__ __forceinline__ void acc_add(Acc8 &a, float s, const float *v) {
    const float mn = fmaxf(a.m, s);
    const float corr = exp2f(a.m - mn);
    const float pj = exp2f(s - mn);
    a.l = a.l * corr + pj;
#pragma unroll
    for (int i = 0; i < 8; ++i) a.o[i] = a.o[i] * corr + pj * v[i];
    a.m = mn;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    constexpr int LPR = D / 8;                 // lanes per cache row (8 channels each)
    constexpr int NG = kThreads / LPR;         // row groups per CTA
    __shared__ float s_new[2][D];              // new augmented key / value (rounded)
    __shared__ float s_m[NG], s_l[NG];
    __shared__ float s_o[NG][D];

    const int tid = threadIdx.x;
    const int b = blockIdx.x / p.items_per_b;
    const int it = blockIdx.x % p.items_per_b;
    const int h = find_head(p, it);
    const int li = it - p.item0[h];
    const bool tail = li == p.nsplit[h];
    float *part = p.part + ((size_t)b * p.items_per_b + it) * (D + 2);
    const int t = p.pos[b];
    if (t < 0 || t >= p.cap) {
        if (tid == 0) report_error(p.hdr, RAT_ERR_INVALID, b);
        for (int c = tid; c < D; c += kThreads) part[c] = 0.f;
        if (tid == 0) { part[D] = -INFINITY; part[D + 1] = 0.f; }
        return;
    }
    const int Dh = p.dil[h], W = p.win[h];
    const long long S = p.slab[h];
    const int r = t % Dh;
    const int n_old = t / Dh;                  // old rows of the residue slab
    const size_t bh = (size_t)b * p.H + h;
    const T *ck = static_cast<const T *>(p.cache[0]) + bh * (size_t)p.cache_R * D;
    const T *cv = static_cast<const T *>(p.cache[1]) + bh * (size_t)p.cache_R * D;

    const int grp = tid / LPR, gl = tid % LPR, c0 = gl * 8;
    float q[8];
    {
        const T *qp = static_cast<const T *>(p.q) + bh * D + c0;
        IO8<T>::load(qp, q);
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] *= p.scale_log2;
    }
    Acc8 acc;
    acc.m = -INFINITY;
    acc.l = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc.o[i] = 0.f;

    if (!tail) {
        // a run of old rows of the residue slab: rows [i0, i1) at cache rows r*S + i
        const int i0 = li * p.rows_per_split;
        const int i1 = min(i0 + p.rows_per_split, n_old);
        const T *kb = ck + ((size_t)r * S) * D + c0;
        const T *vb = cv + ((size_t)r * S) * D + c0;
        for (int i = i0 + grp; i < i1; i += NG * kUnroll) {
            float kf[kUnroll][8], vf[kUnroll][8];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int ii = i + u * NG;
                if (ii < i1) {
                    IO8<T>::load(kb + (size_t)ii * D, kf[u]);
                    IO8<T>::load(vb + (size_t)ii * D, vf[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int ii = i + u * NG;
                if (ii < i1) {  // uniform across the row group
                    float s = 0.f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) s += q[c] * kf[u][c];
                    s = group_sum<LPR>(s);
                    acc_add(acc, s, vf[u]);
                }
            }
        }
    } else {
        // step update of the recurrent state and append of the new row
        for (int c = tid; c < D; c += kThreads) {
            const size_t e = bh * D + c;
            const float xk = (float)static_cast<const T *>(p.k)[e];
            const float xv = (float)static_cast<const T *>(p.v)[e];
            float a = 0.f, oma = 1.f;
            if (p.recur[h]) {
                float gl_ = fminf(fmaxf((float)static_cast<const T *>(p.g)[e], -80.f), 80.f);
                float ex = expf(-gl_);
                a = 1.f / (1.f + ex);
                oma = ex * a;
            }
            const float sk = a * p.state[0][e] + oma * xk;
            const float sv = a * p.state[1][e] + oma * xv;
            p.state[0][e] = sk;
            p.state[1][e] = sv;
            const size_t row = (size_t)r * S + n_old;
            static_cast<T *>(p.cache[0])[bh * (size_t)p.cache_R * D + row * D + c] = to_t<T>(sk);
            static_cast<T *>(p.cache[1])[bh * (size_t)p.cache_R * D + row * D + c] = to_t<T>(sv);
            s_new[0][c] = round_to<T>(sk);
            s_new[1][c] = round_to<T>(sv);
        }
        __syncthreads();
        // old rows of the window: j in [max(0, t-W+1), t-1]
        if (W > 0) {
            const int j0 = max(0, t - W + 1);
            for (int j = j0 + grp; j < t; j += NG) {
                const size_t row = (size_t)(j % Dh) * S + (size_t)(j / Dh);
                float kf[8], vf[8];
                IO8<T>::load(ck + row * D + c0, kf);
                IO8<T>::load(cv + row * D + c0, vf);
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) s += q[c] * kf[c];
                s = group_sum<LPR>(s);
                acc_add(acc, s, vf);
            }
        }
        // the new row: once in the dilated set, once more in the window
        if (grp == 0) {
            float kf[8], vf[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                kf[c] = s_new[0][c0 + c];
                vf[c] = s_new[1][c0 + c];
            }
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) s += q[c] * kf[c];
            s = group_sum<LPR>(s);
            acc_add(acc, s, vf);
            if (W > 0) acc_add(acc, s, vf);
        }
    }

    // fold the row groups of this CTA into one partial
    if (gl == 0) {
        s_m[grp] = acc.m;
        s_l[grp] = acc.l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_o[grp][c0 + i] = acc.o[i];
    __syncthreads();
    float M = -INFINITY;
    for (int g2 = 0; g2 < NG; ++g2) M = fmaxf(M, s_m[g2]);
    for (int c = tid; c < D; c += kThreads) {
        float o = 0.f;
        for (int g2 = 0; g2 < NG; ++g2)
            if (s_m[g2] != -INFINITY) o += s_o[g2][c] * exp2f(s_m[g2] - M);
        part[c] = o;
    }
    if (tid == 0) {
        float L = 0.f;
        for (int g2 = 0; g2 < NG; ++g2)
            if (s_m[g2] != -INFINITY) L += s_l[g2] * exp2f(s_m[g2] - M);
        part[D] = M;
        part[D + 1] = L;
    }
}

// K5: log-sum-exp combine of the items of one (b, h).
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int c = threadIdx.x;
    const int i0 = p.item0[h], i1 = p.item0[h + 1];
    const float *base = p.part + (size_t)b * p.items_per_b * (D + 2);
    float M = -INFINITY;
    for (int i = i0; i < i1; ++i) M = fmaxf(M, base[(size_t)i * (D + 2) + D]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
        for (int i = i0; i < i1; ++i) {
            const float *pi = base + (size_t)i * (D + 2);
            if (pi[D] == -INFINITY) continue;
            const float w = exp2f(pi[D] - M);
            L += pi[D + 1] * w;
            o += pi[c] * w;
        }
    }
    const size_t e = ((size_t)b * p.H + h) * D + c;
    static_cast<T *>(p.o)[e] = to_t<T>(L > 0.f ? o / L : 0.f);
    if (p.lse && c == 0) p.lse[(size_t)b * p.H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace

cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t s) {
    const unsigned grid = (unsigned)p.B * (unsigned)p.items_per_b;
    const unsigned grid2 = (unsigned)p.B * (unsigned)p.H;
    if (grid == 0) return cudaSuccess;
    if (dtype == RAT_BF16) {
        if (p.d == 128) {
            decode_kernel<__nv_bfloat16, 128><<<grid, kThreads, 0, s>>>(p);
            decode_combine_kernel<__nv_bfloat16, 128><<<grid2, 128, 0, s>>>(p);
        } else {
            decode_kernel<__nv_bfloat16, 64><<<grid, kThreads, 0, s>>>(p);
            decode_combine_kernel<__nv_bfloat16, 64><<<grid2, 64, 0, s>>>(p);
        }
    } else {
        if (p.d == 128) {
            decode_kernel<float, 128><<<grid, kThreads, 0, s>>>(p);
            decode_combine_kernel<float, 128><<<grid2, 128, 0, s>>>(p);
        } else {
            decode_kernel<float, 64><<<grid, kThreads, 0, s>>>(p);
            decode_combine_kernel<float, 64><<<grid2, 64, 0, s>>>(p);
        }
    }
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace rat
