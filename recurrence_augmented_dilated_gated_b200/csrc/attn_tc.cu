// attn_tc.cu -- K2/K3: the attention step on the 5th-generation tensor cores
// (tcgen05 + TMEM, operands staged by TMA), bf16 operands, fp32 softmax.
//
// "RAT+: Train Dense, Infer Sparse", Abstract and Figure 1(c): query t attends
// to its dilated set { j <= t : (t-j) mod D == 0 } and, for heads with a local
// window W > 0, in a second softmax to { max(0,t-W+1) <= j <= t }; the two are
// merged by log-sum-exp.  The dilated set of residue r = t mod D is a dense
// causal problem on the interleaved subsequence r, r+D, r+2D, ..., so the
// dilated part is D independent causal flash attentions per head.  A 5-D TMA
// map (d, H, D, T/D, B) makes the residue a coordinate: one box load fetches
// 128 rows of one subsequence.
//
// One CTA computes one work unit: 256 query rows as two 128-row sub-tiles that
// share every K/V tile load (ping-pong, as in FlashAttention-4):
//   warp 0      TMA producer: Q0/Q1 once, then K and V tiles (2-stage rings)
//   warp 1      TMEM owner and MMA issuer (the warp runs converged; one
//               elected lane issues every MMA and commit), in the order
//               PV0(j) QK0(j+1) PV1(j) QK1(j+1), so the tensor core works on
//               one sub-tile while the softmax of the other runs
//   warps 2..9  two softmax warpgroups, one per sub-tile; thread i of a group
//               owns query row i (TMEM lane i).  Online softmax in the log2
//               domain; P (bf16) is written back into TMEM over its own S and
//               read from there by the PV MMA.  A row's first tile takes two
//               passes (its max, then P), and O is rescaled in TMEM only when
//               the running max grows by more than 8; every later tile, masked
//               or not, takes one pass against the running reference, raised
//               only where a 32-key chunk's sum of P would pass 2^32.
// TMEM: S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d).
// Launch 1 (dilated part): units are (b, h, residue, 256-row block), grouped
// by (b, h, residue) with the heaviest block first, so the blocks that share a
// subsequence's K/V run together and hit L2.  Heads without a window write o
// and lse; heads with one write o (bf16) and lse into scratch.  Launch 2
// (window part): 256 consecutive positions against the key tiles covering
// [t0-W+1, t0+255]; the epilogue merges with launch 1's (o, lse) by LSE.
// Under the fixed-grid reading of dilation (query t attends to the keys
// j <= t with j mod D == D-1, plus its own key) the dilated launch is replaced
// by a grid launch: units are 256 consecutive positions against the key tiles
// of the residue-(D-1) subsequence up to the last row's grid key, masked per
// row; the epilogue adds the row's own key (when it is off the grid) by LSE,
// scoring it from q and K~ in global memory.
// With dedupe the window launch also masks, in every tile, the keys of the
// row's dilated set (a periodic bit pattern per 32-column chunk), so a key in
// both sets counts once.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA records
// RAT_ERR_TIMEOUT, raises a shared abort flag, waits (bounded) for its own
// copies and MMAs in flight, frees its TMEM and exits.
#include <cuda.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "attn_tc.cuh"
#include "tmem_io.cuh"

namespace rat {

namespace {

constexpr int BM = kTcRowsQ, BN = kTcRowsKV;   // query rows per sub-tile, keys per K/V tile (128 each)
constexpr int kSub = 2;                        // query sub-tiles per CTA
constexpr int kThreads = 64 + kSub * 128;      // TMA warp, MMA warp, two softmax warpgroups
constexpr uint32_t kTmemCols = 512;
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

// The MMA issuer's warp runs converged; one elected lane issues each MMA and
// commit (always the same lane, so its commits track its own MMAs), while the
// descriptors and TMEM addresses are warp-uniform values.
__device__ __forceinline__ void umma_commit_e(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(
            smem_u32(bar))
        : "memory");
}

// One K/V tile's worth of MMAs of one sub-tile in one statement: a single
// lane election and predicate set-up for the group instead of one per MMA.
// QK: S (+)= Q K^T over NK K steps of 16 (both operands in shared memory);
// descriptors a[i] / b[i] address step i.  The first step overwrites S.
template <int NK>
__device__ __forceinline__ void umma_ss_group(uint32_t d_tmem, const uint64_t *a, const uint64_t *b, uint32_t idesc);
template <>
__device__ __forceinline__ void umma_ss_group<8>(uint32_t d_tmem, const uint64_t *a, const uint64_t *b, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred e, z, t;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 z, %1, %1;\n\t"
        "setp.eq.b32 t, %1, %1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %3, %1, z;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %5, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %7, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %9, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %10, %11, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %12, %13, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %14, %15, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %16, %17, %1, t;\n\t}\n" ::"r"(d_tmem),
        "r"(idesc), "l"(a[0]), "l"(b[0]), "l"(a[1]), "l"(b[1]), "l"(a[2]), "l"(b[2]), "l"(a[3]), "l"(b[3]),
        "l"(a[4]), "l"(b[4]), "l"(a[5]), "l"(b[5]), "l"(a[6]), "l"(b[6]), "l"(a[7]), "l"(b[7])
        : "memory");
}
template <>
__device__ __forceinline__ void umma_ss_group<4>(uint32_t d_tmem, const uint64_t *a, const uint64_t *b, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred e, z, t;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 z, %1, %1;\n\t"
        "setp.eq.b32 t, %1, %1;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %3, %1, z;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %5, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %7, %1, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %9, %1, t;\n\t}\n" ::"r"(d_tmem),
        "r"(idesc), "l"(a[0]), "l"(b[0]), "l"(a[1]), "l"(b[1]), "l"(a[2]), "l"(b[2]), "l"(a[3]), "l"(b[3])
        : "memory");
}
// PV: O (+)= P V over the tile's 128 keys in 8 K steps of 16, P from TMEM
// columns a_tmem + 8 i (bf16 pairs), V descriptors b[i]; the first step
// accumulates only when acc != 0.
__device__ __forceinline__ void umma_ts_group8(uint32_t d_tmem, uint32_t a_tmem, const uint64_t *b, uint32_t idesc,
                                               uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, f, t;\n\t.reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 f, %3, 0;\n\t"
        "setp.eq.b32 t, %2, %2;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\tadd.u32 a4, %1, 32;\n\t"
        "add.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\tadd.u32 a7, %1, 56;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %4, %2, f;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %5, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], %6, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], %7, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], %8, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], %9, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], %10, %2, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], %11, %2, t;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(idesc), "r"(acc), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]),
        "l"(b[6]), "l"(b[7])
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

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start
// address, leading / stride byte offsets (16-byte units), version 1, and the
// 128-byte swizzle layout (2).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B, A
// K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ work units
struct Unit {
    int m;        // 256-row block index within the subsequence (dilated) or sequence (window)
    int cls;      // class
    int b, h, r;  // batch, head, residue
};

// Units of class c occupy [prefix[c], prefix[c+1]); inside a class, groups of
// units share (b, h, residue) and list their blocks heaviest (last) first.
__device__ __forceinline__ Unit decode_unit(const TcParams &p, long long u) {
    int c = 0;
    while (c + 1 < p.ncls && p.prefix[c + 1] <= u) ++c;
    const TcClass &C = p.cls[c];
    const long long rem = u - p.prefix[c];
    long long g = rem / C.mtiles;
    Unit out;
    out.cls = c;
    out.m = C.mtiles - 1 - (int)(rem % C.mtiles);
    out.r = (int)(g % C.nres);
    g /= C.nres;
    out.h = p.heads[C.head0 + (int)(g % C.nheads)];
    out.b = (int)(g / C.nheads);
    return out;
}

// Key tiles (128 key rows each, first row 128*j) of a unit: tiles [jlo, jhi];
// sub-tile i takes [lo[i], hi[i]] (none when its rows all lie past the end).
struct Plan {
    int jlo, jhi;
    int lo[kSub], hi[kSub];
    bool valid[kSub];
};

// Where a unit's query rows sit in the key rows: a chunked prefill's queries
// start at position t0, i.e. subsequence row t0 / D of the dilated part (t0 is
// a multiple of D there) and position t0 of the window and grid parts.
template <int kKind>
__device__ __forceinline__ int query_offset(const TcParams &p, const TcClass &C) {
    return kKind == kTcDilated ? p.t0 / C.D : p.t0;
}

template <int kKind>
__device__ __forceinline__ Plan make_plan(const TcParams &p, const Unit &u) {
    Plan pl;
    const TcClass &C = p.cls[u.cls];
    const int n = C.n;
    const int q0 = 2 * BM * u.m;
    const int W = p.win[u.h];
    const int qo = query_offset<kKind>(p, C);
    for (int i = 0; i < kSub; ++i) {
        const int qmin = q0 + BM * i;
        pl.valid[i] = qmin < n;
        const int qlast = qo + min(qmin + BM - 1, n - 1);   // the sub-tile's last row, in key units
        if (kKind == kTcGrid) {
            // grid keys g <= (t+1)/D - 1 for the sub-tile's last row t; a tile
            // whose rows have no grid key yet keeps tile 0, fully masked
            pl.hi[i] = max(0, ((qlast + 1) / C.D - 1) / BN);
        } else {
            pl.hi[i] = qlast / BN;
        }
        if (kKind != kTcWindow && kKind != kTcWindowDedupe) {
            pl.lo[i] = 0;
        } else {
            const int first = qo + qmin - W + 1;  // earliest key of the sub-tile's first row
            pl.lo[i] = first > 0 ? first / BN : 0;
        }
    }
    pl.jlo = pl.lo[0];
    pl.jhi = pl.valid[1] ? pl.hi[1] : pl.hi[0];
    return pl;
}

__device__ __forceinline__ bool takes(const Plan &pl, int i, int j) {
    return pl.valid[i] && j >= pl.lo[i] && j <= pl.hi[i];
}

// Softmax passes over one 128-key row of S in TMEM, in four 32-column chunks
// in a loop that is not unrolled: the small code keeps both softmax
// warpgroups' instruction streams in cache, which measured faster than 64-
// or 128-column bodies unrolled per mask mode.  MODE: 0 = every key valid,
// 2 = masked, key k valid iff lo < k <= lim (causal: lo below every key).  k
// counts keys from the tile's first column and the limits are this row's, so
// each test is at most two compares per element.
template <int MODE>
__device__ __forceinline__ bool key_ok(int k, int lo, int lim) {
    return MODE == 0 ? true : (k <= lim && k > lo);
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one issue for two elements).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max of three (sm_100 three-input max)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Max of the valid raw scores of this thread's row.
template <int MODE>
__device__ __forceinline__ float row_max_s(uint32_t t_s, int lo, int lim) {
    float mx4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mx4[k] = -INFINITY;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float a = __uint_as_float(sr[2 * k]), b = __uint_as_float(sr[2 * k + 1]);
            if (MODE != 0) {
                a = key_ok<MODE>(32 * q + 2 * k, lo, lim) ? a : -INFINITY;
                b = key_ok<MODE>(32 * q + 2 * k + 1, lo, lim) ? b : -INFINITY;
            }
            mx4[k & 3] = max3(mx4[k & 3], a, b);
        }
    }
    return max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
}

// P = 2^(s * c - m) (0 for masked keys), packed to bf16 pairs over the first
// 64 columns of the row: chunk q lands on columns [16q, 16q+16), which this
// and the earlier chunks have already consumed.  Returns the row sum of P.
template <int MODE>
__device__ __forceinline__ float row_exp_s(uint32_t t_s, int lo, int lim, float c, float m) {
    uint64_t rs2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rs2[k] = f2_pack(0.f, 0.f);
    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2), t0, t1);
            float e0 = ex2(t0), e1 = ex2(t1);
            if (MODE != 0) {
                e0 = key_ok<MODE>(32 * q + 2 * k, lo, lim) ? e0 : 0.f;
                e1 = key_ok<MODE>(32 * q + 2 * k + 1, lo, lim) ? e1 : 0.f;
            }
            rs2[k & 3] = f2_add(rs2[k & 3], f2_pack(e0, e1));
            pk[k] = pack_bf16(e0, e1);
        }
        tmem_st16_async(t_s + 16 * q, pk);
    }
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) f2_unpack(rs2[k], r[2 * k], r[2 * k + 1]);
    return ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
}

// A masked tile, 32 columns at a time.  The 32 rows of a warp are
// consecutive, so a causal or window boundary crosses at most one or two
// 32-column chunks of the warp's rows: every other chunk is either valid for
// all 32 rows (the unmasked body) or masked for all of them (skipped: no TMEM
// load, no exponentials, P = 0).  Only the chunks the boundary crosses run the
// masked body.  The decision is warp-uniform (votes), as the TMEM loads need.
// 0: every key masked for every row of the warp; 1: every key valid; 2: mixed.
__device__ __forceinline__ int chunk_kind(int q, int lo, int lim) {
    const int k0 = 32 * q, k1 = 32 * q + 31;
    if (__all_sync(0xffffffffu, k1 <= lo || k0 > lim)) return 0;
    if (__all_sync(0xffffffffu, k0 > lo && k1 <= lim)) return 1;
    return 2;
}

// row_max_s over a masked tile, chunk by chunk (same result, bit for bit).
__device__ __forceinline__ float row_max_m(uint32_t t_s, int lo, int lim) {
    float mx4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mx4[k] = -INFINITY;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        const int kind = chunk_kind(q, lo, lim);
        if (kind == 0) continue;
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        if (kind == 1) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
                mx4[k & 3] = max3(mx4[k & 3], __uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float a = __uint_as_float(sr[2 * k]), b = __uint_as_float(sr[2 * k + 1]);
                a = key_ok<2>(32 * q + 2 * k, lo, lim) ? a : -INFINITY;
                b = key_ok<2>(32 * q + 2 * k + 1, lo, lim) ? b : -INFINITY;
                mx4[k & 3] = max3(mx4[k & 3], a, b);
            }
        }
    }
    return max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
}

// row_exp_s over a masked tile, chunk by chunk (same P and row sum, bit for
// bit: a skipped chunk's zeros add nothing to the sum).
__device__ __forceinline__ float row_exp_m(uint32_t t_s, int lo, int lim, float c, float m) {
    uint64_t rs2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rs2[k] = f2_pack(0.f, 0.f);
    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        const int kind = chunk_kind(q, lo, lim);
        uint32_t pk[16];
        if (kind == 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) pk[k] = 0u;
        } else {
            uint32_t sr[32];
            tmem_ld32(t_s + 32 * q, sr);
            if (kind == 1) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    float t0, t1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2),
                              t0, t1);
                    const float e0 = ex2(t0), e1 = ex2(t1);
                    rs2[k & 3] = f2_add(rs2[k & 3], f2_pack(e0, e1));
                    pk[k] = pack_bf16(e0, e1);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    float t0, t1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2),
                              t0, t1);
                    float e0 = ex2(t0), e1 = ex2(t1);
                    e0 = key_ok<2>(32 * q + 2 * k, lo, lim) ? e0 : 0.f;
                    e1 = key_ok<2>(32 * q + 2 * k + 1, lo, lim) ? e1 : 0.f;
                    rs2[k & 3] = f2_add(rs2[k & 3], f2_pack(e0, e1));
                    pk[k] = pack_bf16(e0, e1);
                }
            }
        }
        tmem_st16_async(t_s + 16 * q, pk);
    }
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) f2_unpack(rs2[k], r[2 * k], r[2 * k + 1]);
    return ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// P of this row's first `nq` chunks of a tile (bf16 pairs in TMEM columns
// [0, 16 nq)) times f (1 leaves a row's P unchanged, bit for bit).  Rare path
// of the one-pass softmax, kept out of line; called by all lanes of a warp.
__device__ __noinline__ void rescale_p(uint32_t t_s, int nq, float f) {
    tmem_wait_st();   // the chunks' P stores have landed
    for (int q = 0; q < nq; ++q) {
        uint32_t pk[16];
        tmem_ld16(t_s + 16 * q, pk);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&pk[k]);
            const float2 x = __bfloat1622float2(v);
            pk[k] = pack_bf16(x.x * f, x.y * f);
        }
        tmem_st16(t_s + 16 * q, pk);
    }
}

// One-pass softmax of a tile against the row's running reference m (log2
// domain, finite): P = 2^(s c - m), with no separate pass for the tile's max.
// The reference need not be the maximum (softmax does not depend on it) as
// long as P stays bounded: a chunk whose sum of P exceeds 2^32 (some score far
// above m) first raises m for its rows to an upper bound of their maximum so
// far (the earlier chunks' scores lie below m + 32), rescales the P already
// written and the partial sum, and is computed again.  Returns the row sum of
// P against the final m, which the caller compares with the m it passed in.
// kMasked: a masked tile (key k valid iff lo < k <= lim), its 32-column chunks
// classified as in row_exp_m: chunks masked for every row of the warp are
// skipped (P = 0), chunks valid for all of them take the unmasked body.
template <bool kMasked>
__device__ __forceinline__ float row_exp_1p(uint32_t t_s, float c, float &m, int lo, int lim) {
    uint64_t rs2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rs2[k] = f2_pack(0.f, 0.f);
    const uint64_t c2 = f2_pack(c, c);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        const int kind = kMasked ? chunk_kind(q, lo, lim) : 1;
        uint32_t pk[16];
        uint64_t cs2[4];
        if (kMasked && kind == 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) pk[k] = 0u;
            tmem_st16_async(t_s + 16 * q, pk);
            continue;
        }
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        if (kMasked && kind == 2) {
            // masked scores out of the way once: -inf gives P = 0 and no max
#pragma unroll
            for (int k = 0; k < 32; ++k)
                if (!key_ok<2>(32 * q + k, lo, lim)) sr[k] = __float_as_uint(-INFINITY);
        }
#pragma unroll 1
        for (int pass = 0;; ++pass) {
            const uint64_t nm2 = f2_pack(-m, -m);
#pragma unroll
            for (int k = 0; k < 4; ++k) cs2[k] = f2_pack(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float t0, t1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2), t0,
                          t1);
                const float e0 = ex2(t0), e1 = ex2(t1);
                cs2[k & 3] = f2_add(cs2[k & 3], f2_pack(e0, e1));
                pk[k] = pack_bf16(e0, e1);
            }
            float a[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) f2_unpack(cs2[k], a[2 * k], a[2 * k + 1]);
            const float csum = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
            const bool hit = csum > 4294967296.f;   // 2^32 (an infinite sum too)
            if (pass > 0 || !__any_sync(0xffffffffu, hit)) break;
            float mn = m;
            if (hit) {
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < 16; ++k) mx = max3(mx, __uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
                mn = fmaxf(m + 32.f, mx * c);
            }
            const float f = hit ? ex2(m - mn) : 1.f;
            if (q > 0) rescale_p(t_s, q, f);
            const uint64_t f2v = f2_pack(f, f);
#pragma unroll
            for (int k = 0; k < 4; ++k) rs2[k] = f2_mul(rs2[k], f2v);
            m = mn;
        }
        tmem_st16_async(t_s + 16 * q, pk);
#pragma unroll
        for (int k = 0; k < 4; ++k) rs2[k] = f2_add(rs2[k], cs2[k]);
    }
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) f2_unpack(rs2[k], r[2 * k], r[2 * k + 1]);
    return ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
}

// Keys the dilated set already holds, for the window part with dedupe: in a
// tile, key k is excluded when k == e0 (mod xd).  base has a bit at every
// multiple of xd below 32 (one bit when xd > 32); e is the offset of the first
// excluded key of the current 32-column chunk, d32 = 32 mod xd steps it on.
struct Excl {
    uint32_t base;
    int d32, xd;
};

__device__ __forceinline__ Excl make_excl(int xd) {
    Excl x;
    x.xd = xd;
    x.d32 = 32 % xd;
    x.base = 0u;
    for (int k = 0; k < 32; k += xd) x.base |= 1u << k;
    return x;
}

__device__ __forceinline__ uint32_t excl_word(const Excl &x, int e) { return e < 32 ? x.base << e : 0u; }

__device__ __forceinline__ int excl_next(const Excl &x, int e) {
    e -= x.d32;
    return e < 0 ? e + x.xd : e;
}

// row_max_s / row_exp_s with the masked test and the exclusion pattern
// starting at offset e0 of the tile.
__device__ __forceinline__ float row_max_x(uint32_t t_s, int lo, int lim, const Excl &x, int e0) {
    float mx4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mx4[k] = -INFINITY;
    int e = e0;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        const uint32_t xw = excl_word(x, e);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float a = __uint_as_float(sr[2 * k]), b = __uint_as_float(sr[2 * k + 1]);
            a = key_ok<2>(32 * q + 2 * k, lo, lim) && !((xw >> (2 * k)) & 1u) ? a : -INFINITY;
            b = key_ok<2>(32 * q + 2 * k + 1, lo, lim) && !((xw >> (2 * k + 1)) & 1u) ? b : -INFINITY;
            mx4[k & 3] = max3(mx4[k & 3], a, b);
        }
        e = excl_next(x, e);
    }
    return max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
}

__device__ __forceinline__ float row_exp_x(uint32_t t_s, int lo, int lim, const Excl &x, int e0, float c,
                                           float m) {
    uint64_t rs2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rs2[k] = f2_pack(0.f, 0.f);
    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
    int e = e0;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        const uint32_t xw = excl_word(x, e);
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2), t0, t1);
            float e0_ = ex2(t0), e1_ = ex2(t1);
            e0_ = key_ok<2>(32 * q + 2 * k, lo, lim) && !((xw >> (2 * k)) & 1u) ? e0_ : 0.f;
            e1_ = key_ok<2>(32 * q + 2 * k + 1, lo, lim) && !((xw >> (2 * k + 1)) & 1u) ? e1_ : 0.f;
            rs2[k & 3] = f2_add(rs2[k & 3], f2_pack(e0_, e1_));
            pk[k] = pack_bf16(e0_, e1_);
        }
        tmem_st16_async(t_s + 16 * q, pk);
        e = excl_next(x, e);
    }
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) f2_unpack(rs2[k], r[2 * k], r[2 * k + 1]);
    return ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
}

// row_exp_1p for the dedupe window: keys outside (lo, lim] and the dilated
// set's keys (the exclusion pattern from offset e0) get score -inf, then one
// pass against the running reference m, as in row_exp_1p.
__device__ __forceinline__ float row_exp_1px(uint32_t t_s, float c, float &m, int lo, int lim, const Excl &x, int e0) {
    uint64_t rs2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rs2[k] = f2_pack(0.f, 0.f);
    const uint64_t c2 = f2_pack(c, c);
    int e = e0;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t sr[32];
        tmem_ld32(t_s + 32 * q, sr);
        const uint32_t xw = excl_word(x, e);
#pragma unroll
        for (int k = 0; k < 32; ++k)
            if (!(key_ok<2>(32 * q + k, lo, lim) && !((xw >> k) & 1u))) sr[k] = __float_as_uint(-INFINITY);
        uint32_t pk[16];
        uint64_t cs2[4];
#pragma unroll 1
        for (int pass = 0;; ++pass) {
            const uint64_t nm2 = f2_pack(-m, -m);
#pragma unroll
            for (int k = 0; k < 4; ++k) cs2[k] = f2_pack(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float t0, t1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nm2), t0,
                          t1);
                const float e0_ = ex2(t0), e1_ = ex2(t1);
                cs2[k & 3] = f2_add(cs2[k & 3], f2_pack(e0_, e1_));
                pk[k] = pack_bf16(e0_, e1_);
            }
            float a[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) f2_unpack(cs2[k], a[2 * k], a[2 * k + 1]);
            const float csum = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
            const bool hit = csum > 4294967296.f;   // 2^32 (an infinite sum too)
            if (pass > 0 || !__any_sync(0xffffffffu, hit)) break;
            float mn = m;
            if (hit) {
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < 16; ++k) mx = max3(mx, __uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
                mn = fmaxf(m + 32.f, mx * c);
            }
            const float f = hit ? ex2(m - mn) : 1.f;
            if (q > 0) rescale_p(t_s, q, f);
            const uint64_t f2v = f2_pack(f, f);
#pragma unroll
            for (int k = 0; k < 4; ++k) rs2[k] = f2_mul(rs2[k], f2v);
            m = mn;
        }
        tmem_st16_async(t_s + 16 * q, pk);
#pragma unroll
        for (int k = 0; k < 4; ++k) rs2[k] = f2_add(rs2[k], cs2[k]);
        e = excl_next(x, e);
    }
    float r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) f2_unpack(rs2[k], r[2 * k], r[2 * k + 1]);
    return ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
}

template <int HD>
struct Smem {
    static constexpr int kTile = BM * HD * 2;   // one 128-row tile of Q, K or V (bytes)
    static constexpr int kQ = 0;                 // kSub tiles
    static constexpr int kK = kQ + kSub * kTile; // 2 stages
    static constexpr int kV = kK + 2 * kTile;    // 2 stages
    static constexpr int kBytes = kV + 2 * kTile;
};

// ------------------------------------------------------------------ kernel
// Persistent: one CTA per SM takes work units from a ticket counter in the
// order of the unit list (so the blocks of one subsequence still run close
// together and share its K/V in L2).  The roles run ahead across units: the
// producer loads the next unit's Q as soon as the last QK of the current one
// has read its Q, and K/V tiles flow through the same rings; the MMA issuer
// starts the next unit's first QK while the softmax warps write the current
// unit's output.  O_i needs no barrier of its own: the next PV into O_i waits
// for that warpgroup's next P, which it writes only after its epilogue has
// read O_i (ordered by the tcgen05 fences around bar_pfull).  Unit tickets
// reach the other roles through a 2-slot ring in shared memory.
template <int HD, int kKind>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
    using L = Smem<HD>;
    constexpr bool kWin = kKind == kTcWindow || kKind == kTcWindowDedupe;
    constexpr bool kGrid = kKind == kTcGrid;
    constexpr bool kDedupe = kKind == kTcWindowDedupe;
    constexpr int NCB = HD / 64;  // 64-column (128-byte) blocks of a head row
    extern __shared__ uint8_t dsmem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);

    __shared__ uint64_t bar_q, bar_qempty, bar_kfull[2], bar_kempty[2], bar_vfull[2], bar_vempty[2];
    __shared__ uint64_t bar_sfull[kSub], bar_pfull[kSub], bar_pvdone[kSub], bar_drain;
    __shared__ uint64_t bar_ufull[2], bar_uempty[2];
    __shared__ long long s_unit[2];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a bounded wait of an earlier launch on this workspace gave up: skip the
    // work (the error is already recorded for rat_check_status)
    if (*reinterpret_cast<volatile int *>(&p.hdr->status) == RAT_ERR_TIMEOUT) return;

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(&bar_q, 1);
        mbar_init(&bar_qempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_kfull[i], 1);
            mbar_init(&bar_kempty[i], 1);
            mbar_init(&bar_vfull[i], 1);
            mbar_init(&bar_vempty[i], 1);
            mbar_init(&bar_ufull[i], 1);
            mbar_init(&bar_uempty[i], 1 + 4 * kSub);  // MMA issuer + every softmax warp
        }
        for (int i = 0; i < kSub; ++i) {
            mbar_init(&bar_sfull[i], 1);
            mbar_init(&bar_pfull[i], 4);
            mbar_init(&bar_pvdone[i], 1);
        }
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
            int nk = 0, nv = 0, nqu = 0;  // K tiles, V tiles, Q units issued so far
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int slot = it & 1;
                if (it >= 2 && !(ok = mbar_wait(&bar_uempty[slot], (uint32_t)((it >> 1) - 1) & 1u, &s_abort)))
                    break;
                const long long un = (long long)atomicAdd(p.ticket, 1u);
                s_unit[slot] = un;
                mbar_arrive(&bar_ufull[slot]);
                if (un >= p.total_units) break;
                const Unit u = decode_unit(p, un);
                const Plan pl = make_plan<kKind>(p, u);
                const int ntiles = pl.jhi - pl.jlo + 1;
                const CUtensorMap *mq = &p.tq[u.cls];
                const CUtensorMap *mk = &p.tk[u.cls];
                const CUtensorMap *mv = &p.tv[u.cls];
                const int rk = u.r + p.cls[u.cls].kres;   // K/V residue coordinate
                // Q of the previous unit has been read by its last QK
                if (it >= 1 && !(ok = mbar_wait(&bar_qempty, (uint32_t)(it - 1) & 1u, &s_abort))) break;
                const int nq = pl.valid[1] ? 2 : 1;
                mbar_expect_tx(&bar_q, nq * L::kTile);
                for (int i = 0; i < nq; ++i)
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_5d(sbase + L::kQ + i * L::kTile + cb * BM * 128, mq, &bar_q, cb * 64, u.h, u.r,
                                    2 * BM * u.m + BM * i, u.b);
                ++nqu;
                for (int t = 0; t < ntiles; ++t) {
                    const int krow = BN * (pl.jlo + t);
                    const int st = nk & 1;
                    const uint32_t ph = (uint32_t)(nk >> 1) & 1u;
                    if (nk >= 2 && !(ok = mbar_wait(&bar_kempty[st], ph ^ 1u, &s_abort))) break;
                    mbar_expect_tx(&bar_kfull[st], L::kTile);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_5d(sbase + L::kK + st * L::kTile + cb * BN * 128, mk, &bar_kfull[st], cb * 64,
                                    u.h, rk, krow, u.b);
                    ++nk;
                    if (nv >= 2 && !(ok = mbar_wait(&bar_vempty[st], ph ^ 1u, &s_abort))) break;
                    mbar_expect_tx(&bar_vfull[st], L::kTile);
                    for (int cb = 0; cb < NCB; ++cb)
                        tma_load_5d(sbase + L::kV + st * L::kTile + cb * BN * 128, mv, &bar_vfull[st], cb * 64,
                                    u.h, rk, krow, u.b);
                    ++nv;
                }
            }
            if (!ok) {
                s_abort = 1;
                report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
            }
            // Before the CTA exits, every copy it issued must have landed (the
            // consumers have waited for all of them unless a role gave up): the
            // last one issued into each ring slot and the last Q; bounded.
            volatile int never = 0;
            for (int n = max(0, nk - 2); n < nk; ++n) mbar_wait(&bar_kfull[n & 1], (uint32_t)(n >> 1) & 1u, &never);
            for (int n = max(0, nv - 2); n < nv; ++n) mbar_wait(&bar_vfull[n & 1], (uint32_t)(n >> 1) & 1u, &never);
            if (nqu > 0) mbar_wait(&bar_q, (uint32_t)(nqu - 1) & 1u, &never);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        {
            const uint32_t id_qk = idesc_bf16(BM, BN, 0);
            const uint32_t id_pv = idesc_bf16(BM, HD, 1);
            int n_pv[kSub] = {0, 0};   // PV MMAs issued per sub-tile (pfull phases)
            // Descriptors of the tiles at their first K step; later steps add
            // their byte offset / 16 to the start-address field (shared memory
            // lies below 256 KB, so the field never carries into the next).
            const uint64_t dq0 = sdesc(sbase + L::kQ, 16, 1024);
            const uint64_t dk0 = sdesc(sbase + L::kK, 16, 1024);
            const uint64_t dv0 = sdesc(sbase + L::kV, BN * 128, 1024);
            constexpr uint64_t kTileD = L::kTile >> 4;   // one tile, in 16-byte units
            auto qk = [&](int i, int n) {  // S_i = Q_i K(ring tile n)
                const uint64_t aq = dq0 + i * kTileD, bk = dk0 + (n & 1) * kTileD;
                uint64_t a[HD / 16], b[HD / 16];
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    a[kk] = aq + (uint64_t)(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
                    b[kk] = bk + (uint64_t)(((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4);
                }
                umma_ss_group<HD / 16>(tmem + BM * i, a, b, id_qk);
                umma_commit_e(&bar_sfull[i]);
            };
            // O_i (+)= P_i V(ring tile n), P_i read from TMEM over S_i.  Only the
            // unit's last PV of a sub-tile signals bar_pvdone (for the epilogue):
            // the commit after QK_i(j+1), issued after PV_i(j), already tells the
            // softmax that O_i holds tile j when S_i(j+1) is ready.
            auto pv = [&](int i, int n, bool acc, bool last) -> bool {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_pfull[i], (uint32_t)n_pv[i] & 1u, &s_abort))) return false;
                tc_fence_after();
                const uint64_t bv = dv0 + (n & 1) * kTileD;
                uint64_t b[BN / 16];
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) b[kk] = bv + (uint64_t)((kk * 16 * 128) >> 4);
                static_assert(BN / 16 == 8, "eight K steps of P V per tile");
                umma_ts_group8(tmem + 256 + HD * i, tmem + BM * i, b, id_pv, acc ? 1u : 0u);
                if (last) umma_commit_e(&bar_pvdone[i]);
                ++n_pv[i];
                return true;
            };
            int kv = 0;  // K/V ring tiles consumed before this unit
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int slot = it & 1;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bar_ufull[slot], (uint32_t)(it >> 1) & 1u, &s_abort)))) break;
                const long long un = s_unit[slot];
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_uempty[slot]);
                if (un >= p.total_units) break;
                const Unit u = decode_unit(p, un);
                const Plan pl = make_plan<kKind>(p, u);
                const int ntiles = pl.jhi - pl.jlo + 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_q, (uint32_t)it & 1u, &s_abort));
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar_kfull[kv & 1], (uint32_t)(kv >> 1) & 1u, &s_abort));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int i = 0; i < kSub; ++i)
                    if (takes(pl, i, pl.jlo)) qk(i, kv);
                umma_commit_e(&bar_kempty[kv & 1]);
                if (ntiles == 1) umma_commit_e(&bar_qempty);
                bool started[kSub] = {false, false};  // a PV of this unit has written O_i (accumulate)
                for (int t = 0; t < ntiles && ok; ++t) {
                    const int j = pl.jlo + t;
                    const int cur = kv + t, nxt = cur + 1;
                    bool v_ready = false, k_ready = false;
#pragma unroll
                    for (int i = 0; i < kSub; ++i) {
                        if (!ok) break;
                        if (takes(pl, i, j)) {
                            if (!v_ready) {
                                ok = __all_sync(0xffffffffu, mbar_wait(&bar_vfull[cur & 1], (uint32_t)(cur >> 1) & 1u, &s_abort));
                                if (!ok) break;
                                v_ready = true;
                            }
                            ok = pv(i, cur, started[i], !takes(pl, i, j + 1));
                            if (!ok) break;
                            started[i] = true;
                        }
                        if (t + 1 < ntiles && takes(pl, i, j + 1)) {
                            if (!k_ready) {
                                ok = __all_sync(0xffffffffu, mbar_wait(&bar_kfull[nxt & 1], (uint32_t)(nxt >> 1) & 1u, &s_abort));
                                if (!ok) break;
                                tc_fence_after();
                                k_ready = true;
                            }
                            qk(i, nxt);
                        }
                    }
                    if (!ok) break;
                    umma_commit_e(&bar_vempty[cur & 1]);
                    if (t + 1 < ntiles) {
                        if (!k_ready) ok = __all_sync(0xffffffffu, mbar_wait(&bar_kfull[nxt & 1], (uint32_t)(nxt >> 1) & 1u, &s_abort));
                        umma_commit_e(&bar_kempty[nxt & 1]);
                        if (t + 2 == ntiles) umma_commit_e(&bar_qempty);  // the unit's last QK is issued
                    }
                }
                kv += ntiles;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok && lane == 0) {
                s_abort = 1;
                report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
            }
            // every MMA already issued must finish before TMEM is released
            // (a commit arrives once all prior tcgen05 operations are done)
            umma_commit_e(&bar_drain);
            volatile int never = 0;
            __all_sync(0xffffffffu, mbar_wait(&bar_drain, 0, &never));
        }
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int sub = (warp - 2) >> 2;         // sub-tile of this warpgroup
        const int q4 = warp & 3;                 // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;          // query row within the sub-tile
        const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
        const uint32_t t_s = tmem + lane_base + BM * sub;         // S (and P) of this row
        const uint32_t t_o = tmem + lane_base + 256 + HD * sub;   // O of this row
        int n_s = 0, n_pv = 0;   // S tiles, and units whose last PV was awaited, of this sub-tile
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int slot = it & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_ufull[slot], (uint32_t)(it >> 1) & 1u, &s_abort));
            if (!ok) break;
            const long long un = s_unit[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_uempty[slot]);
            if (un >= p.total_units) break;
            const Unit u = decode_unit(p, un);
            const TcClass &C = p.cls[u.cls];
            const Plan pl = make_plan<kKind>(p, u);
            const int qmin = 2 * BM * u.m + BM * sub;                 // first row of the sub-tile
            const int qi = qmin + row;                                // subsequence row / position
            const int W = p.win[u.h];
            const int qo = query_offset<kKind>(p, C);
            const int lo_s = sub ? pl.lo[1] : pl.lo[0];
            const int nt = (sub ? pl.valid[1] : pl.valid[0]) ? (sub ? pl.hi[1] : pl.hi[0]) - lo_s + 1 : 0;
            Excl xcl;
            if constexpr (kDedupe) xcl = make_excl(C.xd);
            float m_run = -INFINITY, l_run = 0.f;
            for (int c = 0; c < nt; ++c) {
                const int j = lo_s + c;
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfull[sub], (uint32_t)n_s & 1u, &s_abort));
                if (!ok) break;
                ++n_s;
                tc_fence_after();
                // mask: causal on subsequence rows (dilated part); keys in (qi - W, qi] (window
                // part); grid keys g <= (qi+1)/D - 1 (grid part)
                const int ks = BN * j;
                const int qa = qo + qi, qamin = qo + qmin;   // the row and the sub-tile's first, in key units
                const bool full = kGrid ? (ks + BN - 1 <= (qamin + 1) / C.D - 1)
                                  : !kWin ? (ks + BN - 1 <= qamin)
                                          : (ks + BN - 1 <= qamin && ks > qamin + BM - 1 - W);
                // row limits in keys from the tile's first column: key k valid iff k <= lim
                const int lim = kGrid ? (qa + 1) / C.D - 1 - ks : qa - ks;
                // window part: and k > lo (no lower limit in the dilated part)
                const int lo = kWin ? qa - W - ks : INT_MIN / 2;
                const int mode = full ? 0 : 2;
                // dedupe: the dilated set's keys in this tile are k == e0 (mod xd):
                // k == lim for the residue reading (the row's own key among them);
                // the grid positions ks + k == xd - 1 (mod xd) for the fixed grid,
                // whose own key leaves through the limit instead
                int e0 = 0, limx = lim;
                if constexpr (kDedupe) {
                    const int r0 = p.grid ? (C.xd - 1 - ks) % C.xd : lim % C.xd;
                    e0 = r0 < 0 ? r0 + C.xd : r0;
                    if (p.grid) limx = lim - 1;
                }
                {
                    // a tile after the row's first: one pass against the
                    // running reference (warp-uniform choice: TMEM accesses are
                    // warp-collective)
                    if (__all_sync(0xffffffffu, m_run != -INFINITY)) {
                        float m = m_run;
                        float rs;
                        if constexpr (kDedupe) rs = row_exp_1px(t_s, p.scale_log2, m, lo, limx, xcl, e0);
                        else rs = mode == 0 ? row_exp_1p<false>(t_s, p.scale_log2, m, lo, lim)
                                            : row_exp_1p<true>(t_s, p.scale_log2, m, lo, lim);
                        const bool raised = m != m_run;
                        const float alpha = raised ? ex2(m_run - m) : 1.f;
                        // O holds tiles 0..c-1 (S(c) completes after every earlier
                        // MMA): bring it to the raised reference before PV(c)
                        if (__any_sync(0xffffffffu, raised)) {
#pragma unroll 1
                            for (int cc = 0; cc < HD / 32; ++cc) {
                                uint32_t o[32];
                                tmem_ld32(t_o + cc * 32, o);
#pragma unroll
                                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                                tmem_st32(t_o + cc * 32, o);
                            }
                        }
                        l_run = l_run * alpha + rs;
                        m_run = m;
                        tmem_wait_st();   // P is in TMEM before the MMA warp reads it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar_pfull[sub]);
                        continue;
                    }
                }
                float mraw;
                if constexpr (kDedupe) mraw = row_max_x(t_s, lo, limx, xcl, e0);
                else mraw = mode == 0 ? row_max_s<0>(t_s, lo, lim) : row_max_m(t_s, lo, lim);
                const float mx = mraw * p.scale_log2;   // scale > 0 commutes with max
                // running max with lazy rescale: keep the stale max unless the new
                // one exceeds it by more than 8 (P stays <= 2^8)
                float m_new = m_run;
                bool rescale = false;
                if (mx > m_run + 8.f || m_run == -INFINITY) {
                    m_new = mx;
                    rescale = (c > 0) && (m_run != -INFINITY);
                }
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_use);
                // S(c) is complete only after every earlier MMA of this CTA, so O
                // already holds tiles 0..c-1: rescale it before PV(c) adds to it
                if (c > 0) {
                    if (__any_sync(0xffffffffu, rescale)) {
                        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                        for (int cc = 0; cc < HD / 32; ++cc) {
                            uint32_t o[32];
                            tmem_ld32(t_o + cc * 32, o);
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                            tmem_st32(t_o + cc * 32, o);
                        }
                    }
                }
                float rs;
                if constexpr (kDedupe) rs = row_exp_x(t_s, lo, limx, xcl, e0, p.scale_log2, m_use);
                else rs = mode == 0 ? row_exp_s<0>(t_s, lo, lim, p.scale_log2, m_use)
                                    : row_exp_m(t_s, lo, lim, p.scale_log2, m_use);
                l_run = l_run * alpha + rs;
                m_run = m_new;
                tmem_wait_st();   // P is in TMEM before the MMA warp reads it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_pfull[sub]);
            }
            if (!ok) break;
            if (nt > 0) {
                const bool valid_row = qi < C.n;
                const long long t = kKind != kTcDilated ? (long long)qi : (long long)(u.r + C.r0) + (long long)C.D * qi;
                const size_t orow = (((size_t)u.b * p.T + (size_t)t) * p.H + u.h) * HD;
                const size_t lrow = ((size_t)u.b * p.H + u.h) * p.T + (size_t)t;
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);
                constexpr bool merge = kWin || kGrid;
                // The row's other part, merged by LSE: for the window launch the
                // dilated part's row (o, lse) written by the previous launch; for
                // the grid launch the row's own key (V~_t, score s q_t.K~_t) when
                // t is off the grid.  Fetched while the last PV runs.
                const bool mrow = merge && valid_row && (!kGrid || (p.t0 + t) % C.D != C.D - 1);
                uint4 prev[HD / 8];
                float ld2 = 0.f;
                if (mrow) {
                    if constexpr (kGrid) {
                        const uint4 *qs = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) + orow);
                        // the row's own key and value: row t0 + t of the [B, t0+T, H, d] history
                        const size_t hrow = (((size_t)u.b * p.Th + (size_t)(p.t0 + t)) * p.H + u.h) * HD;
                        const uint4 *ks4 =
                            reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.kself[u.cls]) + hrow);
                        const uint4 *vs4 =
                            reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.vself[u.cls]) + hrow);
                        float z = 0.f;
#pragma unroll
                        for (int q = 0; q < HD / 8; ++q) {
                            const uint4 a = qs[q], k4 = ks4[q];
                            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, kw[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&aw[i]));
                                const float2 fk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kw[i]));
                                z = fmaf(fa.x, fk.x, z);
                                z = fmaf(fa.y, fk.y, z);
                            }
                            prev[q] = vs4[q];
                        }
                        ld2 = z * p.scale_log2;
                    } else {
                        const uint4 *src = reinterpret_cast<const uint4 *>(o + orow);
#pragma unroll
                        for (int q = 0; q < HD / 8; ++q) prev[q] = src[q];
                        ld2 = p.lse_dil[lrow] * 1.4426950408889634f;
                    }
                } else if constexpr (merge) {
#pragma unroll
                    for (int q = 0; q < HD / 8; ++q) prev[q] = make_uint4(0u, 0u, 0u, 0u);
                }
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_pvdone[sub], (uint32_t)n_pv & 1u, &s_abort));
                if (!ok) break;
                ++n_pv;
                tc_fence_after();
                // ---- epilogue: o = O / l, lse = ln(2) * (m + log2 l)
                const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;  // log2 domain
                // weights of this launch's part (w_self) and of the other part (w_dil)
                float w_self = 1.f, w_dil = 0.f;
                if (mrow) {
                    // merge with the other part: weights e^(lse_i - max) / sum
                    const float mm = fmaxf(ld2, lse2);
                    const float e1 = ex2(ld2 - mm), e2 = ex2(lse2 - mm);
                    w_dil = e1 / (e1 + e2);
                    w_self = e2 / (e1 + e2);
                    lse2 = mm + __log2f(e1 + e2);
                }
                if constexpr (merge) {
#pragma unroll
                    for (int cc = 0; cc < HD / 32; ++cc) {
                        float ov[32];
                        {
                            uint32_t raw[32];
                            tmem_ld32(t_o + cc * 32, raw);
#pragma unroll
                            for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(raw[i]);
                        }
                        if (valid_row) {
                            uint4 *dst = reinterpret_cast<uint4 *>(o + orow + cc * 32);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                float v8[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) v8[i] = ov[8 * q + i] * inv_l * w_self;
                                if constexpr (merge) {
                                    const uint4 pq = prev[cc * 4 + q];
                                    const uint32_t pw[4] = {pq.x, pq.y, pq.z, pq.w};
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        const float2 f =
                                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pw[i]));
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
                } else {
#pragma unroll 1
                    for (int cc = 0; cc < HD / 32; ++cc) {
                        float ov[32];
                        {
                            uint32_t raw[32];
                            tmem_ld32(t_o + cc * 32, raw);
#pragma unroll
                            for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(raw[i]);
                        }
                        if (valid_row) {
                            uint4 *dst = reinterpret_cast<uint4 *>(o + orow + cc * 32);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                float v8[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) v8[i] = ov[8 * q + i] * inv_l * w_self;
                                if constexpr (merge) {
                                    const uint4 pq = prev[cc * 4 + q];
                                    const uint32_t pw[4] = {pq.x, pq.y, pq.z, pq.w};
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        const float2 f =
                                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pw[i]));
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
                }
                if (valid_row) {
                    const float lse = lse2 * 0.69314718055994531f;
                    if (!kWin && p.win[u.h] > 0) p.lse_dil[lrow] = lse;  // the window launch merges later
                    else if (p.lse_user) p.lse_user[lrow] = lse;
                }
            }
        }
        if (!ok) {
            s_abort = 1;
            report_error(p.hdr, RAT_ERR_TIMEOUT, (int)blockIdx.x);
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

bool encode_map_res(CUtensorMap *map, const void *base, int B, int Ts, int H, int d, int D, int r0, int nres, int n,
                    int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || D < 1 || r0 < 0 || nres < 1 || n < 1 || (long long)r0 + nres - 1 + (long long)(n - 1) * D >= Ts)
        return false;
    const cuuint64_t e = 2;  // bf16
    const cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)nres, (cuuint64_t)n, (cuuint64_t)B};
    const cuuint64_t strides[4] = {e * d, e * d * H, e * d * H * D, e * d * H * Ts};
    const cuuint32_t box[5] = {64, 1, 1, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const char *origin = static_cast<const char *>(base) + (size_t)r0 * H * d * e;
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<char *>(origin), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_map_5d(CUtensorMap *map, const void *base, int B, int T, int Ts, int H, int d, int D, int box_rows) {
    if (D < 1 || T % D != 0 || T < D) return false;
    return encode_map_res(map, base, B, Ts, H, d, D, 0, D, T / D, box_rows);
}

// One CTA per SM: each CTA allocates all 512 TMEM columns, so the d = 64
// variant also asks for more than half of the shared memory.
bool encode_map_tokens(CUtensorMap *map, const void *base, int dtype, int B, int T, int Ts, int H, int d,
                       int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t e = dtype == RAT_BF16 ? 2 : 4;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {e * d, e * d * H, e * d * H * Ts};
    const cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, dtype == RAT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_tc_smem_bytes(int hd) {
    const size_t need = (hd == 128 ? (size_t)Smem<128>::kBytes : (size_t)Smem<64>::kBytes) + 1024;
    return need > 120 * 1024 ? need : 120 * 1024;
}

template <int HD, int kKind>
cudaError_t launch_inst(const TcParams &p, unsigned grid, size_t smem, cudaStream_t s) {
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t e = ensure_smem_limit(attn_tc_kernel<HD, kKind>, smem, smem_set);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<HD, kKind><<<grid, kThreads, smem, s>>>(p);
    return cudaSuccess;
}

template <int HD>
cudaError_t launch_kind(const TcParams &p, unsigned grid, size_t smem, cudaStream_t s) {
    switch (p.kind) {
    case kTcWindow: return launch_inst<HD, kTcWindow>(p, grid, smem, s);
    case kTcGrid: return launch_inst<HD, kTcGrid>(p, grid, smem, s);
    case kTcWindowDedupe: return launch_inst<HD, kTcWindowDedupe>(p, grid, smem, s);
    default: return launch_inst<HD, kTcDilated>(p, grid, smem, s);
    }
}

cudaError_t launch_attn_tc(const TcParams &p, int hd, cudaStream_t s) {
    if (p.total_units == 0) return cudaSuccess;
    const size_t smem = attn_tc_smem_bytes(hd);
    int dev = 0, nsm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (the shared memory and TMEM of one CTA fill an SM)
    const unsigned grid = (unsigned)std::min<long long>(p.total_units, (long long)nsm);
    // each launch kind is its own instantiation, carrying only its own
    // epilogue and masks (instruction-cache footprint)
    e = hd == 128 ? launch_kind<128>(p, grid, smem, s) : launch_kind<64>(p, grid, smem, s);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace rat
