// topk.cu -- K6: top-k block attention for decoding over the augmented
// keys/values ("RAT+: Train Dense, Infer Sparse", Figure 3 and Tables 17-18:
// top-k block attention on RAT+ with block size and number of blocks;
// "Augmenting Attention with Exponentially Decaying Memory", section 2.2:
// Quest ranks blocks by per-dimension min/max key statistics, MoBA by
// mean-pooled keys, and both keep the first and the local block).
//
// Keys of a dense head are grouped in blocks of `bs` consecutive positions.
// The new query at t (block c = t / bs) attends to block 0, block c (rows up
// to t) and the K best-scoring of blocks 1 .. c-1:
//   Quest  score = sum_ch max(q_ch * kmin_ch, q_ch * kmax_ch)
//   MoBA   score = q . (sum of the block's keys) / bs
// equal scores going to the lower block.  Per-block statistics live in a
// caller buffer [B, H, nblk, 2, d] fp32 (min and max, or sum and unused): the
// prefill builds them from the cache, each decode step folds its new key into
// its block's entry.
//
// One CTA per (b, h) runs the step: (A) recurrence update, cache append and
// statistics update of block c; (B) candidate scores into shared memory, one
// warp per block; (C) K rounds of a block-wide argmax; (D) an online softmax
// over the kept blocks' rows, row groups of d/8 lanes, folded by LSE.  (B)
// and (D) read contiguous runs (the candidates' statistics; each kept block's
// rows), which stream through a shared-memory double buffer by cp.async.
#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// The candidates' statistics and the kept blocks' K~/V~ rows are contiguous
// runs in global memory: they stream through a double buffer in shared memory
// (cp.async, 16 bytes per thread and copy), the next chunk in flight while the
// CTA works on the current one.
constexpr int kStageBytes = 16384;

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// this thread's copies of all but the most recent `n` groups have landed
template <int n>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

template <typename T> struct Row8;
template <> struct Row8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *f) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <> struct Row8<float> {
    static __device__ __forceinline__ void load(const float *p, float *f) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ------------------------------------------------------------ statistics
// One warp per (b, h, block): lane l covers channels l, l + 32, ...
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) topk_stats_kernel(const TopkParams p, int n_tok) {
    const long long w = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long nblk_tok = (n_tok + p.bs - 1) / p.bs;
    if (w >= (long long)p.B * p.H * nblk_tok) return;
    const int g = (int)(w % nblk_tok);
    const long long bh = w / nblk_tok;
    const T *ck = static_cast<const T *>(p.cache[0]) + (size_t)bh * p.cache_R * D;
    float *st = p.stats + ((size_t)bh * p.nblk + g) * 2 * D;
    const int j0 = g * p.bs, j1 = min(j0 + p.bs, n_tok);
    constexpr int CPL = D / 32;
    float a[CPL], b[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        a[i] = p.mode == RAT_TOPK_QUEST ? INFINITY : 0.f;
        b[i] = -INFINITY;
    }
    for (int j = j0; j < j1; ++j) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const float x = to_f<T>(ck[(size_t)j * D + lane + 32 * i]);
            if (p.mode == RAT_TOPK_QUEST) {
                a[i] = fminf(a[i], x);
                b[i] = fmaxf(b[i], x);
            } else {
                a[i] += x;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        st[lane + 32 * i] = a[i];
        st[D + lane + 32 * i] = p.mode == RAT_TOPK_QUEST ? b[i] : 0.f;
    }
}

// ------------------------------------------------------------ decode step
// Online softmax state of one row group (log2-domain scores).
struct Acc {
    float m, l, o[8];
};

__device__ __forceinline__ void acc_add(Acc &a, float s, const float *v) {
    const float mn = fmaxf(a.m, s);
    const float corr = a.m == -INFINITY ? 0.f : exp2f(a.m - mn);
    const float pj = exp2f(s - mn);
    a.l = a.l * corr + pj;
#pragma unroll
    for (int i = 0; i < 8; ++i) a.o[i] = a.o[i] * corr + pj * v[i];
    a.m = mn;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) topk_decode_kernel(const TopkParams p) {
    constexpr int LPR = D / 8;             // lanes per row (8 channels each)
    constexpr int NG = kThreads / LPR;     // row groups
    extern __shared__ __align__(16) unsigned char s_dyn[];   // double buffer, then the candidate scores
    unsigned char *ring = s_dyn;                            // 2 x kStageBytes
    float *s_score = reinterpret_cast<float *>(s_dyn + 2 * kStageBytes);   // [nblk]
    __shared__ float s_q[D];
    __shared__ float s_rv[kWarps];
    __shared__ int s_ri[kWarps];
    __shared__ int s_pick[kTopkMaxK];
    __shared__ int s_blk[kTopkMaxK + 2], s_off[kTopkMaxK + 3], s_nb;
    __shared__ float s_m[NG], s_l[NG], s_o[NG][D];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const size_t bh = (size_t)blockIdx.x;
    const int t = p.pos[b];
    T *o_out = static_cast<T *>(p.o) + bh * D;
    if (t < 0 || t >= p.cap) {   // uniform over the CTA: skip the entry, report it
        for (int c = tid; c < D; c += kThreads) o_out[c] = from_f<T>(0.f);
        if (tid == 0) {
            if (p.lse) p.lse[bh] = -INFINITY;
            report_error(p.hdr, RAT_ERR_INVALID, b);
        }
        if (p.sel)
            for (int i = tid; i < p.K; i += kThreads) p.sel[bh * p.K + i] = -1;
        return;
    }
    const int bs = p.bs, c = t / bs;
    T *ck = static_cast<T *>(p.cache[0]) + bh * p.cache_R * D;
    T *cv = static_cast<T *>(p.cache[1]) + bh * p.cache_R * D;
    float *st = p.stats + bh * (size_t)p.nblk * 2 * D;

    // (A) step update of channel tid, append of row t, statistics of block c
    if (tid < D) {
        const size_t e = bh * D + tid;
        float a[2] = {0.f, 0.f}, oma[2] = {1.f, 1.f};   // keys, values
        if (p.recur[h]) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                // separate gates: the value gate is the second [B,H,d] tensor
                const size_t ge = (p.sep && i == 1) ? (size_t)p.B * p.H * D + e : e;
                const float g = fminf(fmaxf(to_f<T>(static_cast<const T *>(p.g)[ge]), -80.f), 80.f);
                const float ex = expf(-g);
                a[i] = 1.f / (1.f + ex);
                oma[i] = ex * a[i];
            }
        }
        const float sk = a[0] * p.state[0][e] + oma[0] * to_f<T>(static_cast<const T *>(p.k)[e]);
        const float sv = a[1] * p.state[1][e] + oma[1] * to_f<T>(static_cast<const T *>(p.v)[e]);
        p.state[0][e] = sk;
        p.state[1][e] = sv;
        const T rk = from_f<T>(sk);
        ck[(size_t)t * D + tid] = rk;
        cv[(size_t)t * D + tid] = from_f<T>(sv);
        const float x = to_f<T>(rk);
        float *sc = st + (size_t)c * 2 * D;
        const bool first = t % bs == 0;
        if (p.mode == RAT_TOPK_QUEST) {
            sc[tid] = first ? x : fminf(sc[tid], x);
            sc[D + tid] = first ? x : fmaxf(sc[D + tid], x);
        } else {
            sc[tid] = first ? x : sc[tid] + x;
            sc[D + tid] = 0.f;
        }
        s_q[tid] = to_f<T>(static_cast<const T *>(p.q)[e]);
    }
    __syncthreads();

    // (B) scores of the candidate blocks 1 .. c-1, block g by warp (g - 1) mod
    // kWarps; their statistics stream through the double buffer, CB blocks
    // per chunk
    const int ncand = c > 1 ? c - 1 : 0;
    {
        constexpr int CB = kStageBytes / (2 * D * (int)sizeof(float));
        const int nch = (ncand + CB - 1) / CB;
        auto load = [&](int sidx, int buf) {
            const int g0 = 1 + sidx * CB, n = min(CB, c - g0);
            const unsigned char *src = reinterpret_cast<const unsigned char *>(st + (size_t)g0 * 2 * D);
            unsigned char *dst = ring + buf * kStageBytes;
            const int pieces = n * 2 * D * (int)sizeof(float) / 16;
            for (int i = tid; i < pieces; i += kThreads) cp_async16(dst + 16 * i, src + 16 * i);
            cp_async_commit();
        };
        if (nch > 0) load(0, 0);
        for (int sidx = 0; sidx < nch; ++sidx) {
            if (sidx + 1 < nch) {
                load(sidx + 1, (sidx + 1) & 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();   // every thread's copies of this chunk have landed
            const float *base = reinterpret_cast<const float *>(ring + (sidx & 1) * kStageBytes);
            const int g0 = 1 + sidx * CB, g1 = min(c, g0 + CB);
            for (int g = g0 + (((1 + warp - g0) % kWarps) + kWarps) % kWarps; g < g1; g += kWarps) {
                const float *sg = base + (size_t)(g - g0) * 2 * D;
                float s = 0.f;
                for (int ch = lane; ch < D; ch += 32) {
                    const float qc = s_q[ch];
                    if (p.mode == RAT_TOPK_QUEST) s += fmaxf(qc * sg[ch], qc * sg[D + ch]);
                    else s += qc * sg[ch];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                if (lane == 0) s_score[g] = p.mode == RAT_TOPK_QUEST ? s : s / (float)bs;
            }
            __syncthreads();   // the buffer is free for the chunk after next
        }
    }
    __syncthreads();

    // (C) K rounds: the best remaining candidate, equal scores to the lower block
    const int npick = min(p.K, ncand);
    for (int k = 0; k < npick; ++k) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int g = 1 + tid; g < c; g += kThreads) {
            const float v = s_score[g];
            if (v > bv || (v == bv && g < bi)) {   // taken blocks hold NaN and never win
                bv = v;
                bi = g;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == 0) {
            s_rv[warp] = bv;
            s_ri[warp] = bi;
        }
        __syncthreads();
        if (tid == 0) {
            float v = s_rv[0];
            int i = s_ri[0];
            for (int w = 1; w < kWarps; ++w)
                if (s_rv[w] > v || (s_rv[w] == v && s_ri[w] < i)) {
                    v = s_rv[w];
                    i = s_ri[w];
                }
            // every remaining score NaN (NaN inputs): take a block in range
            // rather than index past the score array
            if (i < 1 || i >= c) i = 1 + k;
            s_pick[k] = i;
            s_score[i] = __int_as_float(0x7fffffff);   // NaN: out of the later rounds
        }
        __syncthreads();
    }
    if (p.sel)
        for (int i = tid; i < p.K; i += kThreads) p.sel[bh * p.K + i] = i < npick ? s_pick[i] : -1;

    // (D) the kept blocks: 0, the picks, and c (rows up to t)
    if (tid == 0) {
        int nb = 0;
        s_blk[nb++] = 0;
        for (int k = 0; k < npick; ++k) s_blk[nb++] = s_pick[k];
        if (c > 0) s_blk[nb++] = c;
        s_off[0] = 0;
        for (int i = 0; i < nb; ++i) {
            const int j0 = s_blk[i] * bs;
            const int j1 = min(j0 + bs, t + 1);
            s_off[i + 1] = s_off[i] + (j1 - j0);
        }
        s_nb = nb;
    }
    __syncthreads();
    const int nb = s_nb;
    const int grp = tid / LPR, c0 = (tid % LPR) * 8;
    float q8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q8[i] = s_q[c0 + i] * p.scale_log2;
    const unsigned gmask = (LPR == 32 ? 0xffffffffu : ((1u << LPR) - 1u)) << ((lane / LPR) * LPR);
    Acc acc;
    acc.m = -INFINITY;
    acc.l = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc.o[i] = 0.f;
    // The kept rows in order (block by block), cut into chunks of at most SR
    // rows that stream through the double buffer (K~ rows, then V~ rows).  Row
    // r of the concatenation still goes to group r mod NG, in order.
    {
        constexpr int SR = kStageBytes / (2 * D * (int)sizeof(T));
        auto rows_of = [&](int bi, int ro) { return min(SR, (s_off[bi + 1] - s_off[bi]) - ro); };
        auto advance = [&](int &bi, int &ro) {
            ro += SR;
            if (ro >= s_off[bi + 1] - s_off[bi]) {
                ++bi;
                ro = 0;
            }
        };
        auto load = [&](int bi, int ro, int buf) {
            const int n = rows_of(bi, ro);
            const size_t j0 = (size_t)s_blk[bi] * bs + ro;   // first cache row
            const unsigned char *sk = reinterpret_cast<const unsigned char *>(ck + j0 * D);
            const unsigned char *sv = reinterpret_cast<const unsigned char *>(cv + j0 * D);
            unsigned char *dk = ring + buf * kStageBytes, *dv = dk + SR * D * sizeof(T);
            const int pieces = n * D * (int)sizeof(T) / 16;
            for (int i = tid; i < pieces; i += kThreads) {
                cp_async16(dk + 16 * i, sk + 16 * i);
                cp_async16(dv + 16 * i, sv + 16 * i);
            }
            cp_async_commit();
        };
        int lb = 0, lr = 0;   // next chunk to load
        int cb = 0, cr = 0;   // chunk to score
        if (nb > 0) {
            load(0, 0, 0);
            advance(lb, lr);
        }
        for (int k = 0; cb < nb; ++k) {
            const bool more = lb < nb;
            if (more) {
                load(lb, lr, (k + 1) & 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();   // every thread's copies of this chunk have landed
            const T *bkr = reinterpret_cast<const T *>(ring + (k & 1) * kStageBytes);
            const T *bvr = bkr + SR * D;
            const int n = rows_of(cb, cr), rg0 = s_off[cb] + cr;   // the chunk's first row in the concatenation
            for (int rr = ((grp - rg0) % NG + NG) % NG; rr < n; rr += NG) {
                float kf[8], vf[8];
                Row8<T>::load(bkr + (size_t)rr * D + c0, kf);
                Row8<T>::load(bvr + (size_t)rr * D + c0, vf);
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) s += q8[i] * kf[i];
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(gmask, s, off);
                acc_add(acc, s, vf);
            }
            __syncthreads();   // the buffer is free for the chunk after next
            if (more) advance(lb, lr);
            advance(cb, cr);
        }
    }
    if (tid % LPR == 0) {
        s_m[grp] = acc.m;
        s_l[grp] = acc.l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_o[grp][c0 + i] = acc.o[i];
    __syncthreads();
    float M = -INFINITY;
    for (int g2 = 0; g2 < NG; ++g2) M = fmaxf(M, s_m[g2]);
    for (int ch = tid; ch < D; ch += kThreads) {
        float L = 0.f, o = 0.f;
        for (int g2 = 0; g2 < NG; ++g2)
            if (s_m[g2] != -INFINITY) {
                const float w = exp2f(s_m[g2] - M);
                L += s_l[g2] * w;
                o += s_o[g2][ch] * w;
            }
        o_out[ch] = from_f<T>(L > 0.f ? o / L : 0.f);
        if (p.lse && ch == 0) p.lse[bh] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
}

template <typename T, int D>
cudaError_t launch_decode_typed(const TopkParams &p, cudaStream_t s) {
    const size_t smem = 2 * (size_t)kStageBytes + (size_t)p.nblk * sizeof(float);
    // the limit is raised once per device, so to the largest score array any call can need
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(topk_decode_kernel<T, D>,
                                      2 * (size_t)kStageBytes + (size_t)kTopkMaxBlocks * sizeof(float), smem_set);
    if (e != cudaSuccess) return e;
    topk_decode_kernel<T, D><<<(unsigned)(p.B * p.H), kThreads, smem, s>>>(p);
    return cudaSuccess;
}

template <typename T, int D>
void launch_stats_typed(const TopkParams &p, int n_tok, cudaStream_t s) {
    const long long warps = (long long)p.B * p.H * ((n_tok + p.bs - 1) / p.bs);
    const unsigned grid = (unsigned)((warps + kWarps - 1) / kWarps);
    if (grid > 0) topk_stats_kernel<T, D><<<grid, kThreads, 0, s>>>(p, n_tok);
}

}  // namespace

cudaError_t launch_topk_stats(const TopkParams &p, int n_tok, int dtype, cudaStream_t s) {
    if ((long long)p.B * p.H * n_tok == 0) return cudaSuccess;
    if (dtype == RAT_BF16) {
        if (p.d == 128) launch_stats_typed<__nv_bfloat16, 128>(p, n_tok, s);
        else launch_stats_typed<__nv_bfloat16, 64>(p, n_tok, s);
    } else {
        if (p.d == 128) launch_stats_typed<float, 128>(p, n_tok, s);
        else launch_stats_typed<float, 64>(p, n_tok, s);
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_topk_decode(const TopkParams &p, int dtype, cudaStream_t s) {
    if (p.B * p.H == 0) return cudaSuccess;
    cudaError_t e;
    if (dtype == RAT_BF16) e = p.d == 128 ? launch_decode_typed<__nv_bfloat16, 128>(p, s) : launch_decode_typed<__nv_bfloat16, 64>(p, s);
    else e = p.d == 128 ? launch_decode_typed<float, 128>(p, s) : launch_decode_typed<float, 64>(p, s);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
