// attn_tc.cu -- K2/K3: the attention step on the 5th-generation tensor cores
// (tcgen05 + TMEM, operands staged by TMA), bf16 operands, fp32 softmax.
//
// "RAT+: Train Dense, Infer Sparse", Abstract and Figure 1(c): query t attends
// to its dilated set { j <= t : (t-j) mod D == 0 } and, for heads with a local
// window W > 0, in a second softmax to { max(0,t-W+1) <= j <= t }; the two are
// merged by log-sum-exp.  The dilated set of residue r = t mod D is a dense
// causal problem on the interleaved subsequence r, r+D, r+2D, ..., so the
// dilated part is D independent causal flash attentions per head.  A 5-D TMA
// map (d, H, D, T/D, B) turns the residue into a coordinate: one box load
// fetches 128 rows of one subsequence.
//
// One CTA computes one 128-row query tile (one work unit):
//   warp 0      TMA producer: the Q tile once, then K and V tiles (2-stage rings)
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into a double-buffered
//               TMEM S, then O += P V into TMEM O (one elected thread)
//   warps 2..5  softmax: thread i owns query row i (TMEM lane i); online
//               softmax in the log2 domain, P written to shared memory in the
//               128B-swizzled K-major layout the tensor core reads; O is
//               rescaled in TMEM only when the running max grows by more than
//               2^8 (the stale max bounds every P by 256).
// Launch 1 (dilated part): work units are (b, h, residue, query tile), issued
// heaviest first.  Heads without a window write o and lse directly; heads with
// one write o (bf16) and lse into scratch.  Launch 2 (window part): 128
// consecutive query positions against the ceil((W+127)/128) key tiles ending
// at the diagonal; the epilogue merges with launch 1's (o, lse) by LSE.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA records
// RAT_ERR_TIMEOUT, raises a shared abort flag, waits (bounded) for its own
// copies and MMAs in flight, frees its TMEM and exits.
#include <cuda.h>

#include "attn_tc.cuh"

#include <mutex>

namespace rat {

namespace {

constexpr int BM = 128, BN = 128;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;   // S0 [0,128) S1 [128,256) O [256, 256+d)
constexpr long long kWaitNs = 2000000000LL;

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with `parity` to complete.  False on timeout or
// when another role has raised the abort flag.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
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

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane; the load and its
// completion wait are one asm statement, so no use can move above the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Shared-memory matrix descriptors (tcgen05 "matrix descriptor"): start
// address, leading / stride byte offsets (16-byte units), version 1, and the
// 128-byte swizzle layout (2).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B,
// A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ work units
struct Unit {
    int m;       // query tile index within the subsequence (dilated) or sequence (window)
    int cls;     // class
    int b, h, r; // batch, head, residue
};

__device__ __forceinline__ Unit decode_unit(const TcParams &p, long long u) {
    // Classes are sorted by mtiles descending; units go level by level from the
    // top query tile down, and within a level class by class.
    Unit out{0, 0, 0, 0, 0};
    long long rem = u;
    int k = 0;
    for (; k < p.ncls; ++k) {
        const int hi = p.cls[k].mtiles;
        const int lo = (k + 1 < p.ncls) ? p.cls[k + 1].mtiles : 0;
        const long long S = p.prefix[k + 1];
        const long long seg = (long long)(hi - lo) * S;
        if (rem < seg) {
            out.m = hi - 1 - (int)(rem / S);
            rem %= S;
            break;
        }
        rem -= seg;
    }
    int c = 0;
    while (c < k && p.prefix[c + 1] <= rem) ++c;
    long long idx = rem - p.prefix[c];
    const TcClass &C = p.cls[c];
    out.cls = c;
    out.r = (int)(idx % C.D);
    idx /= C.D;
    out.h = p.heads[C.head0 + (int)(idx % C.nheads)];
    out.b = (int)(idx / C.nheads);
    return out;
}

// KV tiles of a unit: first key row (subsequence row for the dilated part,
// position for the window part) of tile j, and the tile count.
struct KvPlan {
    int nkv, ks0;
};

__device__ __forceinline__ KvPlan kv_plan(const TcParams &p, const Unit &u) {
    if (!p.window_mode) return KvPlan{u.m + 1, 0};
    const int W = p.win[u.h];
    const int nwt = (W + BN - 1 + BM - 1) / BN;  // tiles covering [t0 - W + 1, t0 + 127]
    const int j0 = max(0, nwt - u.m - 1);        // skip tiles entirely before position 0
    return KvPlan{nwt - j0, BM * (u.m + 1 - nwt + j0)};
}

template <int HD>
struct Smem {
    static constexpr int kTile = BM * HD * 2;         // one Q/K/V tile (bytes)
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTile;              // 2 stages
    static constexpr int kV = kK + 2 * kTile;          // 2 stages
    static constexpr int kP = kV + 2 * kTile;          // 128 x 128 bf16
    static constexpr int kBytes = kP + BM * BN * 2;
};

// ------------------------------------------------------------------ kernel
template <int HD>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
    using L = Smem<HD>;
    constexpr int NCB = HD / 64;  // 64-column (128-byte) blocks of a head row
    extern __shared__ uint8_t dsmem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);

    __shared__ uint64_t bar_q, bar_kfull[2], bar_kempty[2], bar_vfull[2], bar_vempty[2];
    __shared__ uint64_t bar_sfull[2], bar_sfree[2], bar_pfull, bar_pvdone, bar_drain;
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a bounded wait of an earlier CTA on this workspace gave up: skip the
    // remaining work units (the error is already recorded for rat_check_status)
    if (*reinterpret_cast<volatile int *>(&p.hdr->status) == RAT_ERR_TIMEOUT) return;
    const Unit u = decode_unit(p, blockIdx.x);
    const KvPlan plan = kv_plan(p, u);
    const TcClass &C = p.cls[u.cls];

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(&bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_kfull[i], 1);
            mbar_init(&bar_kempty[i], 1);
            mbar_init(&bar_vfull[i], 1);
            mbar_init(&bar_vempty[i], 1);
            mbar_init(&bar_sfull[i], 1);
            mbar_init(&bar_sfree[i], 4);
        }
        mbar_init(&bar_pfull, 4);
        mbar_init(&bar_pvdone, 1);
        mbar_init(&bar_drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const CUtensorMap *mq = &p.tq[u.cls];
            const CUtensorMap *mk = &p.tk[u.cls];
            const CUtensorMap *mv = &p.tv[u.cls];
            const int qrow = BM * u.m;
            mbar_expect_tx(&bar_q, L::kTile);
            for (int cb = 0; cb < NCB; ++cb)
                tma_load_5d(sbase + L::kQ + cb * BM * 128, mq, &bar_q, cb * 64, u.h, u.r, qrow, u.b);
            bool ok = true;
            int j = 0;
            for (; j < plan.nkv && ok; ++j) {
                const int st = j & 1;
                const uint32_t ph = (uint32_t)(j >> 1) & 1u;
                const int krow = plan.ks0 + BN * j;
                if (j >= 2) ok = mbar_wait(&bar_kempty[st], ph ^ 1u, &s_abort);
                if (!ok) break;
                mbar_expect_tx(&bar_kfull[st], L::kTile);
                for (int cb = 0; cb < NCB; ++cb)
                    tma_load_5d(sbase + L::kK + st * L::kTile + cb * BN * 128, mk, &bar_kfull[st], cb * 64, u.h,
                                u.r, krow, u.b);
                if (j >= 2) ok = mbar_wait(&bar_vempty[st], ph ^ 1u, &s_abort);
                if (!ok) {
                    // K of this tile is in flight: let it land before leaving
                    mbar_wait(&bar_kfull[st], ph, &s_abort);
                    break;
                }
                mbar_expect_tx(&bar_vfull[st], L::kTile);
                for (int cb = 0; cb < NCB; ++cb)
                    tma_load_5d(sbase + L::kV + st * L::kTile + cb * BN * 128, mv, &bar_vfull[st], cb * 64, u.h,
                                u.r, krow, u.b);
            }
            if (!ok) {
                s_abort = 1;
                report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
                // copies already issued complete on their own: wait for the last of each ring
                for (int jj = max(0, j - 2); jj < j; ++jj) {
                    const int st = jj & 1;
                    const uint32_t ph = (uint32_t)(jj >> 1) & 1u;
                    volatile int never = 0;
                    mbar_wait(&bar_kfull[st], ph, &never);
                    mbar_wait(&bar_vfull[st], ph, &never);
                }
                volatile int never = 0;
                mbar_wait(&bar_q, 0, &never);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(BM, BN, 0);
            const uint32_t id_pv = idesc_bf16(BM, HD, 1);
            const uint32_t tq = sbase + L::kQ, tp = sbase + L::kP;
            bool ok = mbar_wait(&bar_q, 0, &s_abort);
            int issued_pv = 0;
            auto issue_pv = [&](int jj) -> bool {
                const int st = jj & 1;
                if (!mbar_wait(&bar_pfull, (uint32_t)jj & 1u, &s_abort)) return false;
                if (!mbar_wait(&bar_vfull[st], (uint32_t)(jj >> 1) & 1u, &s_abort)) return false;
                tc_fence_after();
                const uint32_t tv = sbase + L::kV + st * L::kTile;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t a = sdesc(tp + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = sdesc(tv + kk * 16 * 128, BN * 128, 1024);
                    umma_f16(tmem + 256, a, b, id_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bar_pvdone);
                umma_commit(&bar_vempty[st]);
                issued_pv = jj + 1;
                return true;
            };
            for (int j = 0; j < plan.nkv && ok; ++j) {
                const int st = j & 1, sb = j & 1;
                ok = mbar_wait(&bar_kfull[st], (uint32_t)(j >> 1) & 1u, &s_abort);
                if (ok && j >= 2) ok = mbar_wait(&bar_sfree[sb], (uint32_t)((j >> 1) - 1) & 1u, &s_abort);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tk = sbase + L::kK + st * L::kTile;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t a = sdesc(tq + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = sdesc(tk + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024);
                    umma_f16(tmem + sb * BN, a, b, id_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bar_sfull[sb]);
                umma_commit(&bar_kempty[st]);
                if (j >= 1) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(plan.nkv - 1);
            if (!ok) {
                s_abort = 1;
                report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
                // let every MMA already issued finish before TMEM is released:
                // a commit arrives once all prior tcgen05 operations are done
                (void)issued_pv;
                umma_commit(&bar_drain);
                volatile int never = 0;
                mbar_wait(&bar_drain, 0, &never);
            }
        }
    } else {
        // ------------------------------------------------ softmax warps 2..5
        const int q4 = warp & 3;                 // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;          // query row of this thread
        const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
        const int qi = BM * u.m + row;           // subsequence row (dilated) / position (window)
        const int W = p.win[u.h];
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        uint8_t *prow = smem + L::kP + row * 128;
        for (int j = 0; j < plan.nkv; ++j) {
            const int sb = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfull[sb], (uint32_t)(j >> 1) & 1u, &s_abort));
            if (!ok) break;
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem + lane_base + sb * BN + c * 32, s + c * 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sfree[sb]);

            // mask: dilated part is causal on subsequence rows; window part keeps
            // keys in (qi - W, qi]
            const int ks = plan.ks0 + BN * j;
            bool full;
            if (!p.window_mode) full = (j < u.m);
            else full = (ks + BN - 1 <= BM * u.m) && (ks > BM * u.m + BM - 1 - W);
            float mx = -INFINITY;
            if (full) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    s[c] *= p.scale_log2;
                    mx = fmaxf(mx, s[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int kp = ks + c;
                    const bool valid = p.window_mode ? (kp <= qi && kp > qi - W) : (kp <= qi);
                    s[c] = valid ? s[c] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
            }
            // running max with lazy rescale: keep the stale max unless the new
            // one exceeds it by more than 8 (P stays <= 2^8)
            float m_new = m_run;
            bool rescale = false;
            if (mx > m_run + 8.f || m_run == -INFINITY) {
                m_new = mx;
                rescale = (j > 0) && (m_run != -INFINITY);
            }
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                s[c] = ex2(s[c] - m_use);
                rs += s[c];
            }
            const float alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_use);
            l_run = l_run * alpha + rs;
            m_run = m_new;
            // O and the P buffer are free once the previous PV has completed
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_pvdone, (uint32_t)(j - 1) & 1u, &s_abort));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    const float f = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        float o[32];
                        tmem_ld32(tmem + lane_base + 256 + c * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= f;
                        tmem_st32(tmem + lane_base + 256 + c * 32, o);
                    }
                }
            }
            // P row -> shared memory, 128B-swizzled K-major (16-byte chunk q of a
            // 128-byte row lands at chunk q ^ (row & 7))
#pragma unroll
            for (int q = 0; q < BN / 8; ++q) {
                uint4 w;
                w.x = pack_bf16(s[8 * q + 0], s[8 * q + 1]);
                w.y = pack_bf16(s[8 * q + 2], s[8 * q + 3]);
                w.z = pack_bf16(s[8 * q + 4], s[8 * q + 5]);
                w.w = pack_bf16(s[8 * q + 6], s[8 * q + 7]);
                const int blk = q >> 3, ch = (q & 7) ^ (row & 7);
                *reinterpret_cast<uint4 *>(prow + blk * (BM * 128) + ch * 16) = w;
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_pfull);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar_pvdone, (uint32_t)(plan.nkv - 1) & 1u, &s_abort));
        if (!ok) {
            s_abort = 1;
            report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
        } else {
            tc_fence_after();
            // ---- epilogue: o = O / l, lse = ln(2) * (m + log2 l)
            const bool valid_row = qi < C.n;
            const long long t = p.window_mode ? (long long)qi : (long long)u.r + (long long)C.D * qi;
            const size_t orow = (((size_t)u.b * p.T + (size_t)t) * p.H + u.h) * HD;
            const size_t lrow = ((size_t)u.b * p.H + u.h) * p.T + (size_t)t;
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
            float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;   // log2 domain
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);
            const bool merge = p.window_mode != 0;
            float w_self = 1.f, w_dil = 0.f;
            if (merge && valid_row) {
                // merge with the dilated part: weights e^(lse_i - max) / sum
                const float ld2 = p.lse_dil[lrow] * 1.4426950408889634f;
                const float mm = fmaxf(ld2, lse2);
                const float e1 = ex2(ld2 - mm), e2 = ex2(lse2 - mm);
                w_dil = e1 / (e1 + e2);
                w_self = e2 / (e1 + e2);
                lse2 = mm + __log2f(e1 + e2);
            }
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                float ov[32];
                tmem_ld32(tmem + lane_base + 256 + c * 32, ov);
                if (valid_row) {
                    uint4 *dst = reinterpret_cast<uint4 *>(o + orow + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float v8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) v8[i] = ov[8 * q + i] * inv_l * w_self;
                        if (merge) {
                            const uint4 prev = dst[q];
                            const uint32_t pw[4] = {prev.x, prev.y, prev.z, prev.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pw[i]));
                                v8[2 * i] += w_dil * f.x;
                                v8[2 * i + 1] += w_dil * f.y;
                            }
                        }
                        uint4 w;
                        w.x = pack_bf16(v8[0], v8[1]);
                        w.y = pack_bf16(v8[2], v8[3]);
                        w.z = pack_bf16(v8[4], v8[5]);
                        w.w = pack_bf16(v8[6], v8[7]);
                        dst[q] = w;
                    }
                }
            }
            if (valid_row) {
                const float lse = lse2 * 0.69314718055994531f;
                if (!merge && p.win[u.h] > 0) p.lse_dil[lrow] = lse;   // the window launch merges later
                else if (p.lse_user) p.lse_user[lrow] = lse;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

// ------------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

bool encode_map_5d(CUtensorMap *map, const void *base, int B, int T, int H, int d, int D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || D < 1 || T % D != 0) return false;
    const cuuint64_t e = 2;  // bf16
    const cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)D, (cuuint64_t)(T / D), (cuuint64_t)B};
    const cuuint64_t strides[4] = {e * d, e * d * H, e * d * H * D, e * d * H * T};
    const cuuint32_t box[5] = {64, 1, 1, 128, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One CTA per SM: each CTA allocates all 512 TMEM columns, so the d = 64
// variant also asks for more than half of the shared memory.
size_t attn_tc_smem_bytes(int hd) {
    const size_t need = (hd == 128 ? (size_t)Smem<128>::kBytes : (size_t)Smem<64>::kBytes) + 1024;
    return need > 120 * 1024 ? need : 120 * 1024;
}

cudaError_t launch_attn_tc(const TcParams &p, int hd, cudaStream_t s) {
    if (p.total_units == 0) return cudaSuccess;
    const size_t smem = attn_tc_smem_bytes(hd);
    cudaError_t e;
    if (hd == 128) {
        e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attn_tc_kernel<128><<<(unsigned)p.total_units, kThreads, smem, s>>>(p);
    } else {
        e = cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attn_tc_kernel<64><<<(unsigned)p.total_units, kThreads, smem, s>>>(p);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
