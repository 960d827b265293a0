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
//   * TMA loads stage the chunk's k and v rows (d channels of one head) in
//     shared memory; the gate logits g either go the same way or, for bf16
//     with d = 128, straight from global memory into the registers of the
//     thread that uses them (coalesced across the warp), which leaves room
//     for three CTAs per SM instead of two;
//   * pass 1: each group of d/4 threads (4 channels per thread) folds its
//     sub-chunk of rows into (A, b_k, b_v);
//   * the CTA folds its groups, publishes its aggregate, looks back over
//     predecessor chunks (aggregates or inclusive states) to get the state
//     entering the chunk, and publishes its inclusive state;
//   * pass 2: each group replays its sub-chunk from its carried-in state,
//     overwriting k and v in shared memory with K~ and V~, which two TMA
//     stores write back (and decode-cache rows are written directly).  The
//     gate comes from an fp16 copy of 1 - a that pass 1 left over g in shared
//     memory, or, when g was not staged, from the logits read again (an L2
//     hit) and the same fp32 arithmetic as pass 1.
// HBM traffic is the algorithmic 3 reads + 2 writes per (token, channel).
// With separate gates for keys and values the scan runs twice in its
// one-tensor form (kOne: x and g in, x~ out), once per tensor: 2 reads and 1
// write each, again the algorithmic traffic.
// Every wait is bounded by the workspace's spin limit; on expiry the CTA
// records RAT_ERR_TIMEOUT, continues from a zero state and still publishes, so
// no successor waits forever.
#include <cuda_fp16.h>

#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kThreads = 256;
constexpr int kSub = 16;   // tokens per thread group

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

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

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one issue for two channels).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_split(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// a bf16 pair (one 32-bit word, low half first) as an fp32 pair
__device__ __forceinline__ uint64_t bf2_f2(uint32_t w) {
    return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_bf2(uint64_t v) {
    const float2 x = f2_split(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(x.x, x.y);
    return *reinterpret_cast<const uint32_t *>(&b);
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One gate pair of the bf16 path: a = sigmoid(g), 1 - a = e * a with
// e = 2^(-g log2 e).  Only g >= -80 needs clamping (e stays finite); large g
// gives e -> 0, a -> 1, 1 - a -> 0 without it.
__device__ __forceinline__ void gate2(uint32_t gw, uint64_t &a, uint64_t &oma) {
    const uint64_t g = bf2_f2(gw);
    const float2 gs = f2_split(g);
    const float2 t = f2_split(f2_mul(f2(fmaxf(gs.x, -80.f), fmaxf(gs.y, -80.f)),
                                     f2(-1.4426950408889634f, -1.4426950408889634f)));
    const uint64_t e = f2(ex2_approx(t.x), ex2_approx(t.y));
    const float2 den = f2_split(f2_add(e, f2(1.f, 1.f)));
    a = f2(rcp_approx(den.x), rcp_approx(den.y));
    oma = f2_mul(e, a);
}

// 4 consecutive channels of one token row in shared memory
template <typename T> struct Smem4;
template <> struct Smem4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p) { return IO4<__nv_bfloat16>::load(p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v) { IO4<__nv_bfloat16>::store(p, v); }
};
template <> struct Smem4<float> {
    static __device__ __forceinline__ float4 load(const float *p) { return IO4<float>::load(p); }
    static __device__ __forceinline__ void store(float *p, float4 v) { IO4<float>::store(p, v); }
};

// bf16 with d = 128: the gate logits bypass shared memory (each thread reads
// its own, coalesced across the warp, in both passes; the second read hits
// L2), so a chunk stages only k and v and three CTAs fit on an SM; group 0
// (warp 0, which runs the look-back) keeps its aggregate in registers, which
// keeps the static shared memory small enough for the third CTA.
template <typename T, int D>
constexpr bool gate_in_regs() { return sizeof(T) == 2 && D == 128; }

template <typename T, int D, bool kOne>
__global__ void __launch_bounds__(kThreads, gate_in_regs<T, D>() ? 3 : 1)
    scan_kernel(const __grid_constant__ ScanParams p) {
    constexpr int LPR = D / 4;             // threads per token row (4 channels each)
    constexpr int G = kThreads / LPR;      // thread groups (sub-chunks) per CTA
    constexpr int C = G * kSub;            // tokens per chunk
    constexpr uint32_t kTile = C * D * sizeof(T);
    constexpr bool kAccurate = sizeof(T) == 4;
    constexpr bool kRegG = gate_in_regs<T, D>();
    static_assert(!kRegG || LPR == 32, "group 0 is warp 0");
    constexpr int G0 = kRegG ? 1 : 0;      // groups whose aggregate stays in registers
    extern __shared__ __align__(128) uint8_t sbuf[];
    T *tile_k = reinterpret_cast<T *>(sbuf);
    T *tile_v = reinterpret_cast<T *>(sbuf + kTile);
    T *tile_g = reinterpret_cast<T *>(sbuf + 2 * kTile);   // staged only when !kRegG
    __shared__ unsigned s_ticket;
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_load_ok;
    // per group g >= G0, at index g - G0: (A, b_k, b_v); after the look-back,
    // slots 1 and 2 hold the state entering the group's sub-chunk (k and v)
    __shared__ float s_agg[G - G0][3][D];
    // three CTAs per SM: staged k and v, this table and the small words above,
    // plus the 1 KB the hardware reserves per CTA, within the SM's 228 KB
    static_assert(!kRegG || 3 * (2 * (size_t)kTile + sizeof(s_agg) + 64 + 1024) <= 228 * 1024,
                  "three CTAs must fit in an SM's shared memory");

    const int tid = threadIdx.x;
    if (tid == 0) {
        s_ticket = atomicAdd(p.ticket, 1u);
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s_bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const unsigned ticket = s_ticket;
    const int slice = (int)(ticket % (unsigned)p.nslices);
    const int chunk = (int)(ticket / (unsigned)p.nslices);
    const int b = slice / p.nheads;
    const int h = p.head_list[slice % p.nheads];
    const bool rec = p.head_recur[h] != 0;
    const int grp = tid / LPR, c0 = (tid % LPR) * 4;
    const int tc0 = chunk * C;                                   // first token of the chunk
    const int r0 = grp * kSub;                                   // first row of this group
    const int r1 = min(r0 + kSub, p.T - tc0);                    // rows of this group (may be <= r0)
    const long long limit = p.hdr->spin_limit_ns > 0 ? p.hdr->spin_limit_ns : kDefaultSpinNs;

    // gate logits of this thread's rows and channels (kRegG), read while the
    // chunk's k and v are being staged
    const __nv_bfloat16 *grow = nullptr;   // row r0 of this thread's channels
    const size_t gstride = (size_t)p.H * D;
    uint2 gr[kSub];
    if constexpr (kRegG) {
        if (rec) {
            grow = static_cast<const __nv_bfloat16 *>(p.g) + (((size_t)b * p.T + tc0 + r0) * p.H + h) * D + c0;
#pragma unroll
            for (int i = 0; i < kSub; ++i)
                gr[i] = r0 + i < r1 ? __ldg(reinterpret_cast<const uint2 *>(grow + i * gstride)) : make_uint2(0u, 0u);
        }
    }

    // ---- stage the chunk: TMA loads of k, v (and g) rows of this head
    if (tid == 0) {
        const uint32_t bar = smem_u32(&s_bar);
        const int ntile = rec && !kRegG ? 3 : 2;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                     "r"((uint32_t)ntile * kTile - (kOne ? kTile : 0u))
                     : "memory");
        for (int i = 0; i < ntile; ++i)
            if (!kOne || i != 1)   // the one-tensor form has no second tensor
            asm volatile(
                "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(sbuf + i * kTile)),
                "l"(reinterpret_cast<uint64_t>(&p.tmap[i])), "r"(0), "r"(h), "r"(tc0), "r"(b), "r"(bar)
                : "memory");
        // bounded wait for the bytes to land
        auto landed = [&]() -> int {
            const unsigned long long t0 = global_ns();
            for (uint32_t w = 0;; ++w) {
                uint32_t done;
                asm volatile(
                    "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n\t"
                    "selp.u32 %0, 1, 0, q;\n\t}\n"
                    : "=r"(done)
                    : "r"(bar)
                    : "memory");
                if (done) return 1;
                if ((w & 63u) == 63u && (long long)(global_ns() - t0) > limit) return 0;
            }
        };
        const int ok = landed();
        s_load_ok = ok;
        if (!ok) {
            report_error(p.hdr, RAT_ERR_TIMEOUT, (int)ticket);
            // the chunk is skipped, but the CTA must not exit while its copies
            // may still write its shared memory: one more bounded wait for them
            (void)landed();
        }
    }
    __syncthreads();
    const bool loaded = s_load_ok != 0;

    // ---- pass 1: fold the sub-chunk into one affine map per channel
    float A[4] = {1.f, 1.f, 1.f, 1.f}, bk[4] = {0.f, 0.f, 0.f, 0.f}, bv[4] = {0.f, 0.f, 0.f, 0.f};
    if (loaded && !kAccurate && rec) {
        // bf16: channel pairs in f32x2 arithmetic
        uint64_t A2[2] = {f2(1.f, 1.f), f2(1.f, 1.f)}, bk2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)},
                 bv2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int r = r0; r < r0 + kSub; ++r) {
            if (r < r1) {
                const uint2 kw = *reinterpret_cast<const uint2 *>(tile_k + r * D + c0);
                const uint2 vw = kOne ? make_uint2(0u, 0u) : *reinterpret_cast<const uint2 *>(tile_v + r * D + c0);
                const uint2 gw = kRegG ? gr[r - r0] : *reinterpret_cast<const uint2 *>(tile_g + r * D + c0);
                const uint32_t kq[2] = {kw.x, kw.y}, vq[2] = {vw.x, vw.y}, gq[2] = {gw.x, gw.y};
                uint32_t oh[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint64_t a, oma;
                    gate2(gq[h], a, oma);
                    A2[h] = f2_mul(A2[h], a);
                    bk2[h] = f2_fma(a, bk2[h], f2_mul(oma, bf2_f2(kq[h])));
                    bv2[h] = f2_fma(a, bv2[h], f2_mul(oma, bf2_f2(vq[h])));
                    const float2 o = f2_split(oma);
                    const __half2 hh = __floats2half2_rn(o.x, o.y);
                    oh[h] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                // keep 1 - a for pass 2 (fp16: relative precision 2^-11)
                // over the gate logits this thread has just consumed
                if constexpr (!kRegG) *reinterpret_cast<uint2 *>(tile_g + r * D + c0) = make_uint2(oh[0], oh[1]);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 x = f2_split(A2[h]), y = f2_split(bk2[h]), z = f2_split(bv2[h]);
            A[2 * h] = x.x; A[2 * h + 1] = x.y;
            bk[2 * h] = y.x; bk[2 * h + 1] = y.y;
            bv[2 * h] = z.x; bv[2 * h + 1] = z.y;
        }
    } else if (loaded) {
#pragma unroll
        for (int r = r0; r < r0 + kSub; ++r) {
            if (r < r1) {
                const float4 kk = Smem4<T>::load(tile_k + r * D + c0);
                const float4 vv = kOne ? make_float4(0.f, 0.f, 0.f, 0.f) : Smem4<T>::load(tile_v + r * D + c0);
                const float4 gg = rec ? Smem4<T>::load(tile_g + r * D + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
                float om[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = 0.f, oma = 1.f;
                    if (rec) gate<kAccurate>(f4get(gg, c), a, oma);
                    om[c] = oma;
                    A[c] *= a;
                    bk[c] = a * bk[c] + oma * f4get(kk, c);
                    bv[c] = a * bv[c] + oma * f4get(vv, c);
                }
                if (!kAccurate && rec) {
                    // keep 1 - a for pass 2 (fp16: relative precision 2^-11)
                    // over the gate logit this thread has just consumed
                    __half2 *gh = reinterpret_cast<__half2 *>(tile_g + r * D + c0);
                    gh[0] = __floats2half2_rn(om[0], om[1]);
                    gh[1] = __floats2half2_rn(om[2], om[3]);
                }
            }
        }
    }
    if (grp >= G0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            s_agg[grp - G0][0][c0 + c] = A[c];
            s_agg[grp - G0][1][c0 + c] = bk[c];
            s_agg[grp - G0][2][c0 + c] = bv[c];
        }
    }
    __syncthreads();

    // ---- chunk aggregate, look-back, inclusive publish (warp 0)
    float sk0[4], sv0[4];   // kRegG: the state entering group 0's sub-chunk (warp 0)
    if (tid < 32) {
        const int lane = tid;
        const bool owns = lane < LPR;          // lanes holding 4 channels each
        const int cc = lane * 4;
        float TA[4] = {1.f, 1.f, 1.f, 1.f}, Tk[4] = {0.f, 0.f, 0.f, 0.f}, Tv[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (kRegG) {
            // group 0 is this warp: its aggregate is in registers
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                TA[c] = A[c];
                Tk[c] = bk[c];
                Tv[c] = bv[c];
            }
        }
        if (owns) {
            for (int gi = G0; gi < G; ++gi) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = s_agg[gi - G0][0][cc + c];
                    TA[c] *= a;
                    Tk[c] = a * Tk[c] + s_agg[gi - G0][1][cc + c];
                    Tv[c] = a * Tv[c] + s_agg[gi - G0][2][cc + c];
                }
            }
        }
        const size_t sbase = (size_t)slice * p.nchunks;
        const size_t my = sbase + chunk;
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
            // the warp barrier orders every lane's stores before lane 0's
            // release store of the flag, whose release is cumulative
            __syncwarp();
            if (lane == 0) st_release(p.flags + my, 1);

            // Warp-parallel look-back: lane l inspects chunk base - l, so one
            // round trip finds the nearest inclusive state among 32
            // predecessors; every aggregate in between is folded in.
            float accA[4] = {1.f, 1.f, 1.f, 1.f}, acck[4] = {0.f, 0.f, 0.f, 0.f}, accv[4] = {0.f, 0.f, 0.f, 0.f};
            const unsigned long long start = global_ns();
            int base = chunk - 1;
            bool timed_out = false;
            int spins = 0;
            while (true) {
                const int mine = base - lane;
                const int f = mine >= 0 ? ld_acquire(p.flags + sbase + mine) : 0;
                const unsigned incl = __ballot_sync(0xffffffffu, f == 2);
                const unsigned none = __ballot_sync(0xffffffffu, f == 0);
                const int lstar = incl ? __ffs(incl) - 1 : 32;   // nearest inclusive predecessor
                const unsigned before = lstar == 32 ? 0xffffffffu : ((1u << lstar) - 1u);
                if (none & before) {  // an aggregate in between is not out yet: look again
                    if ((long long)(global_ns() - start) > limit) {
                        timed_out = true;
                        break;
                    }
                    if (++spins > 4) __nanosleep(32);
                    continue;
                }
                __syncwarp();  // the flags acquired by every lane order the reads below
                // the inclusive state found, loaded with the aggregates (one round trip)
                float inK[4] = {0.f, 0.f, 0.f, 0.f}, inV[4] = {0.f, 0.f, 0.f, 0.f};
                if (lstar < 32 && owns) {
                    const float *in = p.incl + (sbase + (base - lstar)) * 2 * D + cc;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        inK[c] = in[c];
                        inV[c] = in[D + c];
                    }
                }
                // fold aggregates of chunks base, base-1, ..., base-lstar+1
                if (owns) {
                    int j = 0;
                    for (; j + 4 <= lstar; j += 4) {
                        float ag4[4][12];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float *ag = p.agg + (sbase + (base - j - q)) * 3 * D + cc;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                ag4[q][c] = ag[c];
                                ag4[q][4 + c] = ag[D + c];
                                ag4[q][8 + c] = ag[2 * D + c];
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                acck[c] = accA[c] * ag4[q][4 + c] + acck[c];
                                accv[c] = accA[c] * ag4[q][8 + c] + accv[c];
                                accA[c] *= ag4[q][c];
                            }
                    }
                    for (; j < lstar; ++j) {
                        const float *ag = p.agg + (sbase + (base - j)) * 3 * D + cc;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            acck[c] = accA[c] * ag[D + c] + acck[c];
                            accv[c] = accA[c] * ag[2 * D + c] + accv[c];
                            accA[c] *= ag[c];
                        }
                    }
                }
                if (lstar < 32) {
                    if (owns) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            sk[c] = accA[c] * inK[c] + acck[c];
                            sv[c] = accA[c] * inV[c] + accv[c];
                        }
                    }
                    break;
                }
                base -= 32;  // 32 aggregates folded, none inclusive: next window
                spins = 0;
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
        // state entering each group's sub-chunk (over the consumed b_k, b_v slots)
        if constexpr (kRegG) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                sk0[c] = sk[c];
                sv0[c] = sv[c];
                sk[c] = A[c] * sk[c] + bk[c];
                sv[c] = A[c] * sv[c] + bv[c];
            }
        }
        if (owns) {
            for (int gi = G0; gi < G; ++gi) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float a = s_agg[gi - G0][0][cc + c];
                    const float ak = s_agg[gi - G0][1][cc + c], av = s_agg[gi - G0][2][cc + c];
                    s_agg[gi - G0][1][cc + c] = sk[c];
                    s_agg[gi - G0][2][cc + c] = sv[c];
                    sk[c] = a * sk[c] + ak;
                    sv[c] = a * sv[c] + av;
                }
            }
        }
    }
    __syncthreads();

    // ---- pass 2: replay the sub-chunk from its carried-in state; K~ and V~
    // overwrite k and v in shared memory (same thread, same slot)
    float sk[4], sv[4];
    if (kRegG && grp == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sk[c] = sk0[c];
            sv[c] = sv0[c];
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            sk[c] = s_agg[grp - G0][1][c0 + c];
            sv[c] = s_agg[grp - G0][2][c0 + c];
        }
    }
    T *ck = static_cast<T *>(p.cache[0]);
    T *cv = static_cast<T *>(p.cache[1]);
    const int Dh = p.head_dil[h], Wh = p.head_win[h];
    const long long S = ((long long)p.cap + Dh - 1) / Dh;
    // the window ring keeps the prefill's last W positions (one writer per row)
    const long long ring_from = (long long)p.t0 + p.T - Wh;
    // element offset of (cache row `row`, channel c0) of this head: the dense
    // block or a page of a paged cache; a page the table does not name validly
    // is reported and the row left unwritten
    auto crow = [&](long long row) -> long long {
        const long long o = cache_offset(p.page_table, p.pps, p.page_rows, p.num_pages, p.cache_R, p.H, D, b, h, row);
        if (o < 0) report_error(p.hdr, RAT_ERR_INVALID, (int)ticket);
        return o < 0 ? -1 : o + c0;
    };
    if (loaded && !kAccurate && rec) {
        // bf16: a = 1 - (1 - a) from the fp16 cache, channel pairs in f32x2;
        // kRegG: the gate recomputed from the logits, read again (from L2)
        uint64_t sk2[2] = {f2(sk[0], sk[1]), f2(sk[2], sk[3])}, sv2[2] = {f2(sv[0], sv[1]), f2(sv[2], sv[3])};
        if constexpr (kRegG) {
#pragma unroll
            for (int i = 0; i < kSub; ++i)
                gr[i] = r0 + i < r1 ? __ldg(reinterpret_cast<const uint2 *>(grow + i * gstride)) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int r = r0; r < r0 + kSub; ++r) {
            if (r < r1) {
                const uint2 kw = *reinterpret_cast<const uint2 *>(tile_k + r * D + c0);
                const uint2 vw = kOne ? make_uint2(0u, 0u) : *reinterpret_cast<const uint2 *>(tile_v + r * D + c0);
                const uint2 ow = kRegG ? gr[r - r0] : *reinterpret_cast<const uint2 *>(tile_g + r * D + c0);
                const uint32_t kq[2] = {kw.x, kw.y}, vq[2] = {vw.x, vw.y}, oq[2] = {ow.x, ow.y};
                uint32_t wk[2], wv[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint64_t a, oma;
                    if constexpr (kRegG) {
                        gate2(oq[h], a, oma);   // the same arithmetic as pass 1
                    } else {
                        const float2 of = __half22float2(*reinterpret_cast<const __half2 *>(&oq[h]));
                        oma = f2(of.x, of.y);
                        a = f2_fma(oma, f2(-1.f, -1.f), f2(1.f, 1.f));
                    }
                    sk2[h] = f2_fma(a, sk2[h], f2_mul(oma, bf2_f2(kq[h])));
                    sv2[h] = f2_fma(a, sv2[h], f2_mul(oma, bf2_f2(vq[h])));
                    wk[h] = f2_bf2(sk2[h]);
                    wv[h] = f2_bf2(sv2[h]);
                }
                *reinterpret_cast<uint2 *>(tile_k + r * D + c0) = make_uint2(wk[0], wk[1]);
                *reinterpret_cast<uint2 *>(tile_v + r * D + c0) = make_uint2(wv[0], wv[1]);
                if (ck) {
                    const long long tt = (long long)p.t0 + tc0 + r;
                    long long row0, row1;
                    cache_rows_of(tt, Dh, Wh, S, p.grid, row0, row1);
                    const long long e0 = row0 >= 0 ? crow(row0) : -1;
                    if (e0 >= 0) {
                        *reinterpret_cast<uint2 *>(ck + e0) = make_uint2(wk[0], wk[1]);
                        if (!kOne) *reinterpret_cast<uint2 *>(cv + e0) = make_uint2(wv[0], wv[1]);
                    }
                    const long long e1 = (row1 >= 0 && tt >= ring_from) ? crow(row1) : -1;
                    if (e1 >= 0) {
                        *reinterpret_cast<uint2 *>(ck + e1) = make_uint2(wk[0], wk[1]);
                        if (!kOne) *reinterpret_cast<uint2 *>(cv + e1) = make_uint2(wv[0], wv[1]);
                    }
                }
            }
        }
    } else if (loaded) {
#pragma unroll
        for (int r = r0; r < r0 + kSub; ++r) {
            if (r < r1) {
                const float4 kk = Smem4<T>::load(tile_k + r * D + c0);
                const float4 vv = Smem4<T>::load(tile_v + r * D + c0);
                float4 gg = make_float4(0.f, 0.f, 0.f, 0.f);
                float omc[4] = {1.f, 1.f, 1.f, 1.f};
                if (rec) {
                    if (kAccurate) {
                        gg = Smem4<T>::load(tile_g + r * D + c0);
                    } else {
                        const __half2 *gh = reinterpret_cast<const __half2 *>(tile_g + r * D + c0);
                        const float2 o01 = __half22float2(gh[0]), o23 = __half22float2(gh[1]);
                        omc[0] = o01.x; omc[1] = o01.y; omc[2] = o23.x; omc[3] = o23.y;
                    }
                }
                float rk[4], rv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a = 0.f, oma = 1.f;
                    if (rec) {
                        if (kAccurate) gate<kAccurate>(f4get(gg, c), a, oma);
                        else { oma = omc[c]; a = 1.f - oma; }
                    }
                    sk[c] = a * sk[c] + oma * f4get(kk, c);
                    sv[c] = a * sv[c] + oma * f4get(vv, c);
                    rk[c] = sk[c];
                    rv[c] = sv[c];
                }
                const float4 wk = make_float4(rk[0], rk[1], rk[2], rk[3]);
                const float4 wv = make_float4(rv[0], rv[1], rv[2], rv[3]);
                Smem4<T>::store(tile_k + r * D + c0, wk);
                Smem4<T>::store(tile_v + r * D + c0, wv);
                if (ck) {
                    const long long tt = (long long)p.t0 + tc0 + r;
                    long long row0, row1;
                    cache_rows_of(tt, Dh, Wh, S, p.grid, row0, row1);
                    const long long e0 = row0 >= 0 ? crow(row0) : -1;
                    if (e0 >= 0) {
                        IO4<T>::store(ck + e0, wk);
                        if (!kOne) IO4<T>::store(cv + e0, wv);
                    }
                    const long long e1 = (row1 >= 0 && tt >= ring_from) ? crow(row1) : -1;
                    if (e1 >= 0) {
                        IO4<T>::store(ck + e1, wk);
                        if (!kOne) IO4<T>::store(cv + e1, wv);
                    }
                }
            }
        }
    }
    if (p.use_tma_out && loaded) {
        // generic-proxy writes of K~ / V~ must be visible to the TMA engine
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            for (int i = 0; i < (kOne ? 1 : 2); ++i)
                asm volatile(
                    "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                        reinterpret_cast<uint64_t>(&p.tmap[3 + i])),
                    "r"(0), "r"(h), "r"(p.t0 + tc0), "r"(b), "r"(smem_u32(sbuf + i * kTile))
                    : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // the stores must have read shared memory before the CTA exits
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    }
}

// Final state of heads without recurrence (a = 0): s_{T-1} = x_{T-1}.  Used
// when the scan itself skips those heads (their attention reads k, v directly).
template <typename T>
__global__ void final_of_plain_heads_kernel(const __grid_constant__ ScanParams p) {
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

template <typename T, int D>
size_t scan_smem() {
    constexpr int C = (kThreads / (D / 4)) * kSub;
    // k, v (and g unless each thread reads its own gate logits) of one chunk
    return (gate_in_regs<T, D>() ? 2 : 3) * (size_t)C * D * sizeof(T);
}

template <typename T, int D, bool kOne>
cudaError_t launch_form(const ScanParams &p, unsigned tickets, cudaStream_t s) {
    const size_t smem = scan_smem<T, D>();
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(scan_kernel<T, D, kOne>, smem, smem_set);
    if (e != cudaSuccess) return e;
    if (gate_in_regs<T, D>()) {
        // three CTAs per SM need the largest shared-memory carve-out
        static std::atomic<unsigned long long> carve_set{0};
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
        if (!bit || !(carve_set.load(std::memory_order_acquire) & bit)) {
            e = cudaFuncSetAttribute(scan_kernel<T, D, kOne>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return e;
            if (bit) carve_set.fetch_or(bit, std::memory_order_acq_rel);
        }
    }
    scan_kernel<T, D, kOne><<<tickets, kThreads, smem, s>>>(p);
    return cudaSuccess;
}

template <typename T, int D>
cudaError_t launch_one(const ScanParams &p, unsigned tickets, cudaStream_t s) {
    return p.one ? launch_form<T, D, true>(p, tickets, s) : launch_form<T, D, false>(p, tickets, s);
}

}  // namespace

int scan_chunk_tokens(int d) { return (kThreads / (d / 4)) * kSub; }

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
    cudaError_t e;
    if (dtype == RAT_BF16) e = p.d == 128 ? launch_one<__nv_bfloat16, 128>(p, grid, s) : launch_one<__nv_bfloat16, 64>(p, grid, s);
    else e = p.d == 128 ? launch_one<float, 128>(p, grid, s) : launch_one<float, 64>(p, grid, s);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
