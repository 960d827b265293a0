// scan.cu -- K1: the gated linear recurrence over keys and values for a whole
// prefill ("RAT+: Train Dense, Infer Sparse", Figure 1(a): full-sequence
// recurrence with L = T; Figure 2: prefill runs the recurrence as a scan;
// "Augmenting Attention with Exponentially Decaying Memory", section 2.1: key
// and value states updated with one input-dependent gate).
//
//   s_t = a_t * s_{t-1} + (1 - a_t) * x_t,  a_t = sigmoid(g_t),  per channel.
//
// The recurrence is an affine map per step, s -> a*s + (1-a)*x, and affine maps
// compose associatively: (A2,b2) o (A1,b1) = (A2*A1, A2*b1 + b2).  One launch
// runs a single-pass scan over chunks of time with decoupled look-back
// (Merrill & Garland, "Single-pass Parallel Prefix Scan with Decoupled
// Look-back", 2016):
//   * a CTA takes a dynamic ticket -> (slice = one (b,h) head, chunk of time);
//     tickets are handed out in launch order, so every predecessor chunk of a
//     running CTA has already started (forward progress);
//   * pass 1: each group of d/4 threads (4 channels per thread, one token row
//     per group) folds its sub-chunk into (A, b_k, b_v), reading g, k, v once;
//   * the CTA folds its groups, publishes its aggregate, looks back over
//     predecessor chunks (aggregates or inclusive states) to get the state
//     entering the chunk, and publishes its inclusive state;
//   * pass 2: each group replays its sub-chunk from its carried-in state and
//     writes the augmented rows (and decode-cache rows).  The pass-2 reads hit
//     L2: the chunk was read microseconds earlier by the same CTA.
// HBM traffic is the algorithmic 3 reads + 2 writes per (token, channel).
// Every wait on a predecessor is bounded by the workspace's spin limit; on
// expiry the CTA records RAT_ERR_TIMEOUT, continues from a zero state and still
// publishes, so no successor waits forever.
#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;

template <bool kAccurate>
__device__ __forceinline__ void gate(float g, float &a, float &oma) {
    // a = sigmoid(g), 1 - a = e * a with e = exp(-g): no cancellation as a -> 1.
    // Clamping to +-80 changes nothing representable in fp32 and keeps e finite.
    g = fminf(fmaxf(g, -80.f), 80.f);
    if (kAccurate) {
        float e = expf(-g);
        a = 1.f / (1.f + e);
        oma = e * a;
    } else {
        float e = __expf(-g);
        a = __fdividef(1.f, 1.f + e);
        oma = e * a;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) scan_kernel(const ScanParams p) {
    constexpr int LPR = D / 4;            // threads per token row
    constexpr int G = kThreads / LPR;     // thread groups (sub-chunks) per CTA
    constexpr bool kAccurate = sizeof(T) == 4;
    __shared__ unsigned s_ticket;
    __shared__ float s_agg[G][3][D];      // per group (A, b_k, b_v)
    __shared__ float s_carry[G][2][D];    // state entering each group's sub-chunk

    const int tid = threadIdx.x;
    if (tid == 0) s_ticket = atomicAdd(p.ticket, 1u);
    __syncthreads();
    const unsigned ticket = s_ticket;
    const int slice = (int)(ticket % (unsigned)p.nslices);
    const int chunk = (int)(ticket / (unsigned)p.nslices);
    const int b = slice / p.nheads;
    const int h = p.head_list[slice % p.nheads];
    const bool rec = p.head_recur[h] != 0;
    const int grp = tid / LPR, c0 = (tid % LPR) * 4;

    const T *xk = static_cast<const T *>(p.x[0]);
    const T *xv = static_cast<const T *>(p.x[1]);
    const T *gg = static_cast<const T *>(p.g);
    const size_t rs = (size_t)p.H * D;                         // stride between tokens
    const size_t base = ((size_t)b * p.T * p.H + h) * D + c0;  // (b, t=0, h, c0)
    const long long t0 = (long long)chunk * p.chunk_len + (long long)grp * p.sub_len;
    const long long t1 = min(t0 + (long long)p.sub_len, (long long)p.T);

    // ---- pass 1: fold the sub-chunk into one affine map per channel
    float A[4] = {1.f, 1.f, 1.f, 1.f}, bk[4] = {0.f, 0.f, 0.f, 0.f}, bv[4] = {0.f, 0.f, 0.f, 0.f};
    for (long long t = t0; t < t1; t += kUnroll) {
        float4 kk[kUnroll], vv[kUnroll], ga[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (t + u < t1) {
                size_t e = base + (size_t)(t + u) * rs;
                kk[u] = IO4<T>::load(xk + e);
                vv[u] = IO4<T>::load(xv + e);
                ga[u] = rec ? IO4<T>::load(gg + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (t + u < t1) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = 0.f, oma = 1.f;
                    if (rec) gate<kAccurate>(f4get(ga[u], c), a, oma);
                    A[c] *= a;
                    bk[c] = a * bk[c] + oma * f4get(kk[u], c);
                    bv[c] = a * bv[c] + oma * f4get(vv[u], c);
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        s_agg[grp][0][c0 + c] = A[c];
        s_agg[grp][1][c0 + c] = bk[c];
        s_agg[grp][2][c0 + c] = bv[c];
    }
    __syncthreads();

    // ---- chunk aggregate, look-back, inclusive publish (warp 0)
    if (tid < 32) {
        const int lane = tid;
        const bool owns = lane < LPR;          // lanes holding 4 channels each
        const int cc = lane * 4;
        float TA[4] = {1.f, 1.f, 1.f, 1.f}, Tk[4] = {0.f, 0.f, 0.f, 0.f}, Tv[4] = {0.f, 0.f, 0.f, 0.f};
        if (owns) {
            for (int gi = 0; gi < G; ++gi) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = s_agg[gi][0][cc + c];
                    TA[c] *= a;
                    Tk[c] = a * Tk[c] + s_agg[gi][1][cc + c];
                    Tv[c] = a * Tv[c] + s_agg[gi][2][cc + c];
                }
            }
        }
        const size_t my = (size_t)slice * p.nchunks + chunk;
        const bool stalled = p.hdr->stall_ticket_plus1 == (long long)ticket + 1;
        float sk[4] = {0.f, 0.f, 0.f, 0.f}, sv[4] = {0.f, 0.f, 0.f, 0.f};  // state entering the chunk
        if (chunk == 0) {
            if (owns) {
                const size_t ib = ((size_t)b * p.H + h) * D + cc;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    sk[c] = p.init[0] ? p.init[0][ib + c] : 0.f;
                    sv[c] = p.init[1] ? p.init[1][ib + c] : 0.f;
                }
            }
        } else if (!stalled) {
            // publish the aggregate so successors need not wait for our look-back
            if (owns) {
                float *ag = p.agg + my * 3 * D + cc;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ag[c] = TA[c];
                    ag[D + c] = Tk[c];
                    ag[2 * D + c] = Tv[c];
                }
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release(p.flags + my, 1);

            // look back: fold predecessor aggregates until an inclusive state
            float accA[4] = {1.f, 1.f, 1.f, 1.f}, acck[4] = {0.f, 0.f, 0.f, 0.f}, accv[4] = {0.f, 0.f, 0.f, 0.f};
            const long long limit = p.hdr->spin_limit_ns > 0 ? p.hdr->spin_limit_ns : kDefaultSpinNs;
            const unsigned long long start = global_ns();
            int pred = chunk - 1;
            bool timed_out = false;
            while (true) {
                const int *fp = p.flags + (size_t)slice * p.nchunks + pred;
                int f = ld_acquire(fp);
                int spins = 0;
                while (__any_sync(0xffffffffu, f == 0)) {
                    if (__any_sync(0xffffffffu, (long long)(global_ns() - start) > limit)) {
                        timed_out = true;
                        break;
                    }
                    if (++spins > 8) __nanosleep(64);
                    f = ld_acquire(fp);
                }
                if (timed_out) break;
                f = __reduce_min_sync(0xffffffffu, f);
                const size_t pi = (size_t)slice * p.nchunks + pred;
                if (f == 2) {
                    if (owns) {
                        const float *in = p.incl + pi * 2 * D + cc;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            sk[c] = accA[c] * in[c] + acck[c];
                            sv[c] = accA[c] * in[D + c] + accv[c];
                        }
                    }
                    break;
                }
                // aggregate of chunk `pred`: acc <- acc o agg(pred)
                if (owns) {
                    const float *ag = p.agg + pi * 3 * D + cc;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float a = ag[c];
                        acck[c] = accA[c] * ag[D + c] + acck[c];
                        accv[c] = accA[c] * ag[2 * D + c] + accv[c];
                        accA[c] *= a;
                    }
                }
                --pred;  // chunk 0 always publishes inclusive, so pred stays >= 0
            }
            if (timed_out) {
                if (lane == 0) report_error(p.hdr, RAT_ERR_TIMEOUT, (int)ticket);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    sk[c] = acck[c];
                    sv[c] = accv[c];
                }
            }
        }
        // inclusive state after this chunk
        float ik[4], iv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            ik[c] = TA[c] * sk[c] + Tk[c];
            iv[c] = TA[c] * sv[c] + Tv[c];
        }
        if (!stalled) {
            if (owns) {
                float *in = p.incl + my * 2 * D + cc;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    in[c] = ik[c];
                    in[D + c] = iv[c];
                }
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release(p.flags + my, 2);
        }
        if (owns && chunk == p.nchunks - 1) {
            const size_t ib = ((size_t)b * p.H + h) * D + cc;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (p.fin[0]) p.fin[0][ib + c] = ik[c];
                if (p.fin[1]) p.fin[1][ib + c] = iv[c];
            }
        }
        // state entering each group's sub-chunk
        if (owns) {
            for (int gi = 0; gi < G; ++gi) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    s_carry[gi][0][cc + c] = sk[c];
                    s_carry[gi][1][cc + c] = sv[c];
                    float a = s_agg[gi][0][cc + c];
                    sk[c] = a * sk[c] + s_agg[gi][1][cc + c];
                    sv[c] = a * sv[c] + s_agg[gi][2][cc + c];
                }
            }
        }
    }
    __syncthreads();

    // ---- pass 2: replay the sub-chunk from its carried-in state, write rows
    float sk[4], sv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        sk[c] = s_carry[grp][0][c0 + c];
        sv[c] = s_carry[grp][1][c0 + c];
    }
    T *ok = static_cast<T *>(p.out[0]);
    T *ov = static_cast<T *>(p.out[1]);
    T *ck = static_cast<T *>(p.cache[0]);
    T *cv = static_cast<T *>(p.cache[1]);
    const int Dh = p.head_dil[h];
    const long long S = ((long long)p.cap + Dh - 1) / Dh;
    const size_t cbase = ((size_t)b * p.H + h) * (size_t)p.cache_R * D + c0;
    for (long long t = t0; t < t1; t += kUnroll) {
        float4 kk[kUnroll], vv[kUnroll], ga[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (t + u < t1) {
                size_t e = base + (size_t)(t + u) * rs;
                kk[u] = IO4<T>::load(xk + e);
                vv[u] = IO4<T>::load(xv + e);
                ga[u] = rec ? IO4<T>::load(gg + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (t + u < t1) {
                float rk[4], rv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = 0.f, oma = 1.f;
                    if (rec) gate<kAccurate>(f4get(ga[u], c), a, oma);
                    sk[c] = a * sk[c] + oma * f4get(kk[u], c);
                    sv[c] = a * sv[c] + oma * f4get(vv[u], c);
                    rk[c] = sk[c];
                    rv[c] = sv[c];
                }
                const float4 wk = make_float4(rk[0], rk[1], rk[2], rk[3]);
                const float4 wv = make_float4(rv[0], rv[1], rv[2], rv[3]);
                const long long tt = t + u;
                if (ok) {
                    size_t e = base + (size_t)tt * rs;
                    IO4<T>::store(ok + e, wk);
                    IO4<T>::store(ov + e, wv);
                }
                if (ck) {
                    long long row = (tt % Dh) * S + tt / Dh;
                    size_t e = cbase + (size_t)row * D;
                    IO4<T>::store(ck + e, wk);
                    IO4<T>::store(cv + e, wv);
                }
            }
        }
    }
}

// Final state of heads without recurrence (a = 0): s_{T-1} = x_{T-1}.  Used
// when the scan itself skips those heads (their attention reads k, v directly).
template <typename T>
__global__ void final_of_plain_heads_kernel(const ScanParams p) {
    const int b = blockIdx.x;
    const T *xs[2] = {static_cast<const T *>(p.x[0]), static_cast<const T *>(p.x[1])};
    for (int i = threadIdx.x; i < p.nheads * p.d; i += blockDim.x) {
        const int h = p.head_list[i / p.d], c = i % p.d;
        const size_t src = (((size_t)b * p.T + (p.T - 1)) * p.H + h) * p.d + c;
        const size_t dst = ((size_t)b * p.H + h) * p.d + c;
        for (int j = 0; j < 2; ++j)
            if (p.fin[j]) p.fin[j][dst] = (float)xs[j][src];
    }
}

}  // namespace

cudaError_t launch_final_of_plain_heads(const ScanParams &p, int dtype, cudaStream_t s) {
    if (p.B == 0 || p.T == 0 || p.nheads == 0) return cudaSuccess;
    if (dtype == RAT_BF16) final_of_plain_heads_kernel<__nv_bfloat16><<<p.B, 256, 0, s>>>(p);
    else final_of_plain_heads_kernel<float><<<p.B, 256, 0, s>>>(p);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_scan(const ScanParams &p, int dtype, cudaStream_t s) {
    const unsigned grid = (unsigned)p.nslices * (unsigned)p.nchunks;
    if (grid == 0) return cudaSuccess;
    if (dtype == RAT_BF16) {
        if (p.d == 128) scan_kernel<__nv_bfloat16, 128><<<grid, kThreads, 0, s>>>(p);
        else scan_kernel<__nv_bfloat16, 64><<<grid, kThreads, 0, s>>>(p);
    } else {
        if (p.d == 128) scan_kernel<float, 128><<<grid, kThreads, 0, s>>>(p);
        else scan_kernel<float, 64><<<grid, kThreads, 0, s>>>(p);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
