// decode.cu -- K4: one decode step of the temporal-mixing operator
// ("RAT+: Train Dense, Infer Sparse", Figure 2: decode updates the recurrence
// with a simple step and attends over the dilated KV cache; Abstract: the
// dilated pattern cuts the KV cache a step reads by D).
//
// For batch entry b, head h, new token at t = pos[b], dilation D, window W:
//   s <- a*s + (1-a)*x (x = k, v; a = sigmoid(g), a = 0 without recurrence),
//   the new augmented row is stored at cache row (t mod D)*S + t/D,
//   o = softmax over the multiset  { j <= t, j == t mod D }  (+)  { t-W+1..t }.
// Under the fixed-grid reading the dilated set is { j < t, j mod D == D-1 }
// plus t, the slab is the grid (rows 0 .. t/D - 1, the same count), the new
// row is stored at its grid row only when t is on the grid, and the window
// rows come from a ring of the last W positions (D > 1).  A paged cache
// (kPaged) keeps the same logical rows in pages named by a page table; the
// ring's bulk copies split where a run of rows crosses a page.  With dedupe the
// window part skips the keys of the dilated set, the new row among them.
// Softmaxes over disjoint pieces of a key multiset combine exactly by
// log-sum-exp, so the step is split into independent work items:
//   * item i of (b, h) streams its run of old rows of the residue slab
//     (t mod D), one contiguous coalesced region;
//   * the last item also does the step update of the recurrent state, the
//     append of the new row, the new row's dilated score and the window rows.
// Only the last item touches the state and the new cache row, and no other
// item reads that row, so the items need no ordering among themselves.  Each
// item writes a partial (unnormalised accumulator, max, sum); the last item
// of a (b, h) to finish (a per-(b,h) atomic counter, reset by that item)
// combines the partials by log-sum-exp and writes o and lse.
// The work is HBM-bound: each cache row is read once, 2*d bytes of bf16 per
// row and tensor (K~ and V~).
#include "rat_internal.cuh"

namespace rat {

namespace {

constexpr int kCompute = 128;        // threads that score rows (4 warps)
constexpr int kThreads = kCompute + 32;  // plus one producer warp
constexpr int kBatch = 4;            // rows scored together per row group
constexpr int kRowsMax = 2048;       // slab rows per work item, at most ...
constexpr int kRowsMin = 256;        // ... and at least, when the batch alone cannot fill the GPU
constexpr int kItemsWanted = 4 * 148;  // work items per step that keep every SM busy
constexpr int kStages = 4;           // shared-memory ring of K/V row blocks
constexpr long long kWaitNs = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with `parity`; false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if ((long long)(global_ns() - t0) > kWaitNs) return false;
        }
    }
}

__device__ __forceinline__ void compute_sync() {  // the kCompute scoring threads only
    asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory");
}

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
__device__ __forceinline__ float group_sum(float s, unsigned mask) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(mask, s, off);
    return s;
}

// Online softmax state of one row group (log2-domain scores); o holds this
// lane's 8 channels of the unnormalised accumulator.
struct Acc8 {
    float m, l, o[8];
};

// Adds the first n <= NB keys (scores s[], values v[][]) in one rescale,
// leaving out key u when bit u of `skip` is set; fully unrolled and predicated
// so the arrays stay in registers.
template <int NB>
__device__ __forceinline__ void acc_add_batch(Acc8 &a, const float *s, const float (*v)[8], int n,
                                              unsigned skip = 0u) {
    float mb = -INFINITY;
#pragma unroll
    for (int u = 0; u < NB; ++u) mb = (u < n && !((skip >> u) & 1u)) ? fmaxf(mb, s[u]) : mb;
    const float mn = fmaxf(a.m, mb);
    const float corr = a.m == -INFINITY ? 0.f : exp2f(a.m - mn);
    a.l *= corr;
#pragma unroll
    for (int i = 0; i < 8; ++i) a.o[i] *= corr;
#pragma unroll
    for (int u = 0; u < NB; ++u) {
        const float pj = (u < n && !((skip >> u) & 1u)) ? exp2f(s[u] - mn) : 0.f;
        a.l += pj;
#pragma unroll
        for (int i = 0; i < 8; ++i) a.o[i] += pj * v[u][i];
    }
    a.m = mn;
}

template <typename T, int D, bool kPaged>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    constexpr int LPR = D / 8;                 // lanes per cache row (8 channels each)
    constexpr int NG = kCompute / LPR;         // row groups
    constexpr int RS = NG * kBatch;            // rows per ring stage
    constexpr uint32_t kRowBytes = D * sizeof(T);
    constexpr uint32_t kStageBytes = 2 * RS * kRowBytes;   // K and V rows
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t s_full[kStages], s_empty[kStages];
    __shared__ float s_new[2][D];              // new augmented key / value (rounded)
    __shared__ float s_m[NG], s_l[NG];
    __shared__ float s_o[NG][D];
    __shared__ int s_last;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int b = blockIdx.x / p.items_per_b;
    const int it = blockIdx.x % p.items_per_b;
    const int h = find_head(p, it);
    const int li = it - p.item0[h];
    const bool last = li == p.nsplit[h] - 1;
    float *part = p.part + ((size_t)b * p.items_per_b + it) * (D + 2);
    const int t = p.pos[b];
    const bool valid_pos = t >= 0 && t < p.cap;
    const size_t bh = (size_t)b * p.H + h;
    const int Dh = p.dil[h], W = p.win[h];
    const long long S = p.slab[h];
    const int r = valid_pos ? t % Dh : 0;
    const int n_old = valid_pos ? t / Dh : 0;    // old rows of the residue slab (or grid)
    const size_t slab0 = p.grid ? 0 : (size_t)r * S;   // first cache row of the slab
    const int i0 = li * p.rows_per_item[h];      // this item's run of old rows: [i0, i1)
    const int i1 = min(i0 + p.rows_per_item[h], n_old);
    const int nrows = max(0, i1 - i0);
    const int nst = (nrows + RS - 1) / RS;       // ring stages this item streams
    const T *ck = static_cast<const T *>(p.cache[0]);   // cache bases: rows at row_off(row)
    const T *cv = static_cast<const T *>(p.cache[1]);
    // element offset of logical cache row `row` of (b, h); -1 for a page the
    // table does not name validly
    auto row_off = [&](long long row) -> long long {
        if (kPaged) return cache_offset(p.page_table, p.pps, p.page_rows, p.num_pages, p.cache_R, p.H, D, b, h, row);
        return ((long long)bh * p.cache_R + row) * D;
    };
    // a paged cache: every page the step of (b, h) touches must be valid, else
    // the pair is skipped (o = 0) and reported like an invalid position.  Every
    // item checks the pages of the whole step, so all items of (b, h) agree.
    int bad = 0;
    if (kPaged && valid_pos) {
        if (n_old > 0) {
            // first and last page of the step's slab (32-bit divisions when the
            // rows fit, as they do for any cache a sequence can hold)
            const long long r_lo = (long long)slab0, r_hi = (long long)slab0 + n_old - 1;
            const bool fits = r_hi <= 0x7fffffffLL;
            const long long pg_lo = fits ? (long long)((unsigned)r_lo / (unsigned)p.page_rows) : r_lo / p.page_rows;
            const long long pg_hi = fits ? (long long)((unsigned)r_hi / (unsigned)p.page_rows) : r_hi / p.page_rows;
            for (long long pg = pg_lo + tid; pg <= pg_hi; pg += kThreads) bad |= row_off(pg * p.page_rows) < 0;
        }
        long long ra, rb;
        cache_rows_of(t, Dh, W, S, p.grid, ra, rb);
        // the new row's two slots, each by a thread of another warp than the
        // slab's first pages, so that every page-table load is in flight at once
        if (tid == 32 && ra >= 0) bad |= row_off(ra) < 0;
        if (tid == 64 && rb >= 0) bad |= row_off(rb) < 0;
        if (W > 0) {
            // the window's old rows, four independent lookups per thread at a time
            const int jlo = max(0, t - W + 1);
#pragma unroll 4
            for (int jj = jlo + tid; jj < t; jj += kThreads) {
                cache_rows_of(jj, Dh, W, S, p.grid, ra, rb);
                bad |= row_off(rb >= 0 ? rb : ra) < 0;
            }
        }
    }

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < kStages; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&s_full[i])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&s_empty[i])), "r"(kCompute / 32)
                         : "memory");
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (!valid_pos) report_error(p.hdr, RAT_ERR_INVALID, b);
    }
    bad = __syncthreads_or(bad);
    const bool valid = valid_pos && !bad;
    if (tid == 0 && valid_pos && bad) report_error(p.hdr, RAT_ERR_INVALID, b);

    Acc8 acc;
    acc.m = -INFINITY;
    acc.l = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc.o[i] = 0.f;
    const int grp = tid / LPR, gl = tid % LPR, c0 = gl * 8;

    if (warp == kCompute / 32) {
        // ------------------------------------------------ producer: stream the
        // item's contiguous run of K~ and V~ rows through the ring
        if ((tid & 31) == 0 && valid) {
            const char *kb = reinterpret_cast<const char *>(ck + (kPaged ? 0 : row_off(slab0 + i0)));
            const char *vb = reinterpret_cast<const char *>(cv + (kPaged ? 0 : row_off(slab0 + i0)));
            int sidx = 0;
            bool ok = true;
            for (; sidx < nst; ++sidx) {
                const int st = sidx % kStages;
                if (sidx >= kStages &&
                    !mbar_wait(smem_u32(&s_empty[st]), (uint32_t)(sidx / kStages - 1) & 1u, &s_abort)) {
                    ok = false;
                    break;
                }
                const int nr = min(RS, nrows - sidx * RS);
                const uint32_t bytes = (uint32_t)nr * kRowBytes;
                const uint32_t full = smem_u32(&s_full[st]);
                const uint32_t dk = smem_u32(ring + st * kStageBytes);
                const uint32_t dv = dk + RS * kRowBytes;
                const size_t off = (size_t)sidx * RS * kRowBytes;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full), "r"(2 * bytes)
                             : "memory");
                if (!kPaged) {
                    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                                     dk),
                                 "l"(kb + off), "r"(bytes), "r"(full)
                                 : "memory");
                    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                                     dv),
                                 "l"(vb + off), "r"(bytes), "r"(full)
                                 : "memory");
                } else {
                    // one copy per page the stage's rows touch (all validated above)
                    const long long ra = (long long)(slab0 + i0) + (long long)sidx * RS;
                    for (int done = 0; done < nr;) {
                        const long long row = ra + done;
                        const long long in_page = row <= 0x7fffffffLL
                                                      ? (long long)((unsigned)row % (unsigned)p.page_rows)
                                                      : row % p.page_rows;
                        const int n = (int)min((long long)(nr - done), (long long)p.page_rows - in_page);
                        const long long ofs = row_off(row);
                        const uint32_t nb = (uint32_t)n * kRowBytes, so = (uint32_t)done * kRowBytes;
                        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                                         dk + so),
                                     "l"(ck + ofs), "r"(nb), "r"(full)
                                     : "memory");
                        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                                         dv + so),
                                     "l"(cv + ofs), "r"(nb), "r"(full)
                                     : "memory");
                        done += n;
                    }
                }
            }
            if (!ok) {
                s_abort = 1;
                report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
                volatile int never = 0;
                for (int q = max(0, sidx - kStages); q < sidx; ++q)  // copies still in flight
                    mbar_wait(smem_u32(&s_full[q % kStages]), (uint32_t)(q / kStages) & 1u, &never);
            }
        }
    } else if (valid) {
        // ------------------------------------------------ scoring warps
        const unsigned gmask = group_mask<LPR>();
        float q[8];
        IO8<T>::load(static_cast<const T *>(p.q) + bh * D + c0, q);
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] *= p.scale_log2;

        // The last item's step update of the recurrent state: its inputs are
        // loaded now and used after the old rows, so their latency overlaps
        // the stream (channel tid; kCompute >= D)
        static_assert(kCompute >= D, "one channel per scoring thread");
        float in_k = 0.f, in_v = 0.f, in_g = 0.f, in_gv = 0.f, st_k = 0.f, st_v = 0.f;
        const size_t e_new = bh * D + tid;
        if (last && tid < D) {
            in_k = (float)static_cast<const T *>(p.k)[e_new];
            in_v = (float)static_cast<const T *>(p.v)[e_new];
            if (p.recur[h]) {
                in_g = (float)static_cast<const T *>(p.g)[e_new];
                // separate gates: the value gate is the second [B,H,d] tensor
                in_gv = p.sep ? (float)static_cast<const T *>(p.g)[(size_t)p.B * p.H * D + e_new] : in_g;
            }
            st_k = p.state[0][e_new];
            st_v = p.state[1][e_new];
        }

        // the item's old rows, one ring stage at a time; group grp takes rows
        // [grp*kBatch, grp*kBatch + kBatch) of each stage
        bool ok = true;
        for (int sidx = 0; sidx < nst; ++sidx) {
            const int st = sidx % kStages;
            ok = __all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&s_full[st]), (uint32_t)(sidx / kStages) & 1u, &s_abort));
            if (!ok) break;
            const int nr = min(RS, nrows - sidx * RS);
            const int n = max(0, min(kBatch, nr - grp * kBatch));
            const T *sk_ = reinterpret_cast<const T *>(ring + st * kStageBytes);
            const T *sv_ = sk_ + RS * D;
            float kf[kBatch][8], vf[kBatch][8], sc[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                if (u < n) {
                    IO8<T>::load(sk_ + (grp * kBatch + u) * D + c0, kf[u]);
                    IO8<T>::load(sv_ + (grp * kBatch + u) * D + c0, vf[u]);
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) kf[u][c] = vf[u][c] = 0.f;
                }
            }
            __syncwarp();
            if ((tid & 31) == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&s_empty[st])) : "memory");
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                float s2 = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) s2 += q[c] * kf[u][c];
                sc[u] = group_sum<LPR>(s2, gmask);
            }
            acc_add_batch<kBatch>(acc, sc, vf, n);
        }
        if (!ok) {
            s_abort = 1;
            if (tid == 0) report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
        }

        if (last) {
            // step update and append of the new row (no item reads it this step)
            if (tid < D) {
                float a = 0.f, oma = 1.f, av = 0.f, omav = 1.f;
                if (p.recur[h]) {
                    const float gl_ = fminf(fmaxf(in_g, -80.f), 80.f);
                    const float ex = expf(-gl_);
                    a = 1.f / (1.f + ex);
                    oma = ex * a;
                    av = a;
                    omav = oma;
                    if (p.sep) {
                        const float gv_ = fminf(fmaxf(in_gv, -80.f), 80.f);
                        const float exv = expf(-gv_);
                        av = 1.f / (1.f + exv);
                        omav = exv * av;
                    }
                }
                const float sk = a * st_k + oma * in_k;
                const float sv = av * st_v + omav * in_v;
                p.state[0][e_new] = sk;
                p.state[1][e_new] = sv;
                long long row0, row1;
                cache_rows_of(t, Dh, W, S, p.grid, row0, row1);
                T *dk = static_cast<T *>(p.cache[0]) + tid;
                T *dv = static_cast<T *>(p.cache[1]) + tid;
                if (row0 >= 0) {
                    dk[row_off(row0)] = to_t<T>(sk);
                    dv[row_off(row0)] = to_t<T>(sv);
                }
                if (row1 >= 0) {  // the ring slot of t - W, which no window needs any more
                    dk[row_off(row1)] = to_t<T>(sk);
                    dv[row_off(row1)] = to_t<T>(sv);
                }
                s_new[0][tid] = round_to<T>(sk);
                s_new[1][tid] = round_to<T>(sv);
            }
            compute_sync();  // the new row is in shared memory
            // old rows of the window: j in [max(0, t-W+1), t-1]
            if (W > 0) {
                const int j0 = max(0, t - W + 1);
                for (int j = j0 + grp * kBatch; j < t; j += NG * kBatch) {
                    float kf[kBatch][8], vf[kBatch][8], sc[kBatch];
                    const int n = min(kBatch, t - j);
                    unsigned skip = 0u;
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        if (u < n) {
                            const int jj = j + u;
                            if (p.dedupe && (p.grid ? jj % Dh == Dh - 1 : (t - jj) % Dh == 0)) skip |= 1u << u;
                            long long row0, row1;
                            cache_rows_of(jj, Dh, W, S, p.grid, row0, row1);
                            const long long ofs = row_off(row1 >= 0 ? row1 : row0);
                            IO8<T>::load(ck + ofs + c0, kf[u]);
                            IO8<T>::load(cv + ofs + c0, vf[u]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) kf[u][c] = vf[u][c] = 0.f;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        float s2 = 0.f;
#pragma unroll
                        for (int c = 0; c < 8; ++c) s2 += q[c] * kf[u][c];
                        sc[u] = group_sum<LPR>(s2, gmask);
                    }
                    acc_add_batch<kBatch>(acc, sc, vf, n, skip);
                }
            }
            // the new row: once in the dilated set, once more in the window
            // (not with dedupe)
            if (grp == 0) {
                float kv[2][8], sc[2];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    kv[0][c] = s_new[1][c0 + c];
                    kv[1][c] = kv[0][c];
                }
                float s2 = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) s2 += q[c] * s_new[0][c0 + c];
                s2 = group_sum<LPR>(s2, gmask);
                sc[0] = s2;
                sc[1] = s2;
                acc_add_batch<2>(acc, sc, kv, W > 0 && !p.dedupe ? 2 : 1);
            }
        }
    }

    // fold the row groups into one partial (scoring threads)
    if (tid < kCompute) {
        if (gl == 0) {
            s_m[grp] = acc.m;
            s_l[grp] = acc.l;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) s_o[grp][c0 + i] = acc.o[i];
        compute_sync();
        float M = -INFINITY;
        for (int g2 = 0; g2 < NG; ++g2) M = fmaxf(M, s_m[g2]);
        if (p.nsplit[h] == 1) {
            // the only item of (b, h): write o and lse directly (an invalid
            // position leaves every row group empty: o = 0, lse = -inf)
            float L = 0.f;
            for (int g2 = 0; g2 < NG; ++g2)
                if (s_m[g2] != -INFINITY) L += s_l[g2] * exp2f(s_m[g2] - M);
            for (int c = tid; c < D; c += kCompute) {
                float o = 0.f;
                for (int g2 = 0; g2 < NG; ++g2)
                    if (s_m[g2] != -INFINITY) o += s_o[g2][c] * exp2f(s_m[g2] - M);
                static_cast<T *>(p.o)[bh * D + c] = to_t<T>(L > 0.f ? o / L : 0.f);
                if (p.lse && c == 0) p.lse[bh] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
            }
        } else {
            for (int c = tid; c < D; c += kCompute) {
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
    }
    if (p.nsplit[h] == 1) return;   // nothing to combine

    // the last item of (b, h) to finish combines all of them
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int done = atomicAdd(p.counter + bh, 1);
        s_last = done == p.nsplit[h] - 1;
    }
    __syncthreads();
    if (!s_last || tid >= kCompute) return;
    __threadfence();
    const float *base = p.part + ((size_t)b * p.items_per_b + p.item0[h]) * (D + 2);
    const int ni = p.nsplit[h];
    float Mx = -INFINITY;
    for (int i = 0; i < ni; ++i) Mx = fmaxf(Mx, __ldcg(base + (size_t)i * (D + 2) + D));
    for (int c = tid; c < D; c += kCompute) {
        float L = 0.f, o = 0.f;
        if (Mx != -INFINITY) {
            for (int i = 0; i < ni; ++i) {
                const float *pi = base + (size_t)i * (D + 2);
                const float mi = __ldcg(pi + D);
                if (mi == -INFINITY) continue;
                const float w = exp2f(mi - Mx);
                L += __ldcg(pi + D + 1) * w;
                o += __ldcg(pi + c) * w;
            }
        }
        static_cast<T *>(p.o)[bh * D + c] = to_t<T>(L > 0.f ? o / L : 0.f);
        if (p.lse && c == 0) p.lse[bh] = L > 0.f ? (Mx + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    if (tid == 0) p.counter[bh] = 0;  // ready for the next step
}

template <typename T, int D, bool kPaged>
cudaError_t launch_form(const DecodeParams &p, unsigned grid, cudaStream_t s) {
    constexpr int RS = (kCompute / (D / 8)) * kBatch;
    const size_t smem = (size_t)kStages * 2 * RS * D * sizeof(T);
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(decode_kernel<T, D, kPaged>, smem, smem_set);
    if (e != cudaSuccess) return e;
    decode_kernel<T, D, kPaged><<<grid, kThreads, smem, s>>>(p);
    return cudaSuccess;
}

template <typename T, int D>
cudaError_t launch_typed(const DecodeParams &p, unsigned grid, cudaStream_t s) {
    return p.page_table ? launch_form<T, D, true>(p, grid, s) : launch_form<T, D, false>(p, grid, s);
}

}  // namespace

size_t decode_plan(const rat_cfg *c, int cap, DecodeParams *p) {
    // Longer items mean fewer partial results to merge; split further only
    // while the batch's items would leave SMs idle.
    int target = kRowsMax;
    while (target > kRowsMin) {
        long long n_items = 0;
        for (int h = 0; h < c->H; ++h) {
            const long long slab = ((long long)cap + c->dil[h] - 1) / c->dil[h];
            n_items += slab > 0 ? (slab + target - 1) / target : 1;
        }
        if (n_items * c->B >= kItemsWanted) break;
        target /= 2;
    }
    int items = 0;
    long long R = 0;
    for (int h = 0; h < c->H; ++h) {
        const int D = c->dil[h];
        const int slab = (cap + D - 1) / D;
        const int ns = (slab + target - 1) / target;
        const int n = ns > 0 ? ns : 1;
        p->dil[h] = D;
        // with dedupe a D = 1 head's window keys are all in its dilated set
        p->win[h] = (c->flags & RAT_FLAG_DEDUPE) && D == 1 ? 0 : c->win[h];
        p->slab[h] = slab;
        p->nsplit[h] = n;
        p->rows_per_item[h] = (slab + n - 1) / n;   // balanced runs
        p->item0[h] = items;
        p->recur[h] = (c->recur == nullptr || c->recur[h] != 0) ? 1 : 0;
        items += n;
        const bool grid = (c->flags & RAT_FLAG_GRID_DILATION) != 0;
        const long long rows = grid ? (long long)slab + (D > 1 ? c->win[h] : 0) : (long long)D * slab;
        R = R > rows ? R : rows;
    }
    p->grid = (c->flags & RAT_FLAG_GRID_DILATION) ? 1 : 0;
    p->dedupe = (c->flags & RAT_FLAG_DEDUPE) ? 1 : 0;
    p->sep = (c->flags & RAT_FLAG_SEPARATE_GATES) ? 1 : 0;
    p->item0[c->H] = items;
    p->items_per_b = items;
    p->cache_R = R;
    const size_t part = (size_t)c->B * items * (c->d + 2) * sizeof(float);
    const size_t part_al = (part + 255) & ~(size_t)255;
    return part_al + (size_t)c->B * c->H * sizeof(int);
}

cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t s) {
    const unsigned grid = (unsigned)p.B * (unsigned)p.items_per_b;
    if (grid == 0) return cudaSuccess;
    cudaError_t e;
    if (dtype == RAT_BF16) e = p.d == 128 ? launch_typed<__nv_bfloat16, 128>(p, grid, s) : launch_typed<__nv_bfloat16, 64>(p, grid, s);
    else e = p.d == 128 ? launch_typed<float, 128>(p, grid, s) : launch_typed<float, 64>(p, grid, s);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
