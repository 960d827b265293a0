// api.cu -- the C ABI of librat.so (declared in include/rat.h): argument
// checks, workspace layout and kernel dispatch.  Every step of the operator
// runs in this library's kernels; there is no host or library fallback.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "attn_tc.cuh"
#include "rat_internal.cuh"

using namespace rat;

namespace rat {
static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace rat

namespace {

thread_local char g_last_error[256] = "";

rat_status fail(rat_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

}  // namespace

rat_status rat::set_last_error(rat_status s, const char *msg) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
    return s;
}

namespace {

rat_status cuda_fail(cudaError_t e, const char *what) {
    return fail(RAT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

size_t elt_size(int dtype) { return dtype == RAT_F32 ? 4 : 2; }

int scan_chunk_len(int d) { return scan_chunk_tokens(d); }

// Work-unit counters for the tensor-core attention launches of one call
// (each launch takes up to 8 classes of heads, so 256 heads need at most 64).
constexpr int kAttnTickets = 128;


rat_status check_cfg(const rat_cfg *c, bool need_T = true) {
    if (!c) return fail(RAT_ERR_INVALID, "cfg is NULL");
    if (c->B < 0 || c->H < 1 || c->d < 1 || (need_T && c->T < 0))
        return fail(RAT_ERR_INVALID, "need B >= 0, T >= 0, H >= 1, d >= 1 (B=%d T=%d H=%d d=%d)", c->B, c->T,
                    c->H, c->d);
    if (c->H > kMaxHeads) return fail(RAT_ERR_UNSUPPORTED, "H=%d exceeds %d heads", c->H, kMaxHeads);
    if (c->d != 64 && c->d != 128) return fail(RAT_ERR_UNSUPPORTED, "head_dim d=%d (supported: 64, 128)", c->d);
    if (c->dtype != RAT_F32 && c->dtype != RAT_BF16) return fail(RAT_ERR_INVALID, "dtype %d", c->dtype);
    if (!c->dil || !c->win) return fail(RAT_ERR_INVALID, "cfg->dil / cfg->win is NULL");
    for (int h = 0; h < c->H; ++h) {
        if (c->dil[h] < 1) return fail(RAT_ERR_INVALID, "dil[%d]=%d < 1", h, c->dil[h]);
        if (c->win[h] < 0) return fail(RAT_ERR_INVALID, "win[%d]=%d < 0", h, c->win[h]);
    }
    const double elems = (double)c->B * (need_T ? (double)c->T : 1.0) * c->H * c->d;
    if (elems >= 1099511627776.0) return fail(RAT_ERR_INVALID, "B*T*H*d too large");
    if (!(c->scale == c->scale)) return fail(RAT_ERR_INVALID, "scale is NaN");
    if (c->t0 < 0 || (long long)c->t0 + c->T > 0x7fffffffLL) return fail(RAT_ERR_INVALID, "t0 %d out of range", c->t0);
    if (c->t_cap != 0 && (long long)c->t_cap < (long long)c->t0 + c->T)
        return fail(RAT_ERR_INVALID, "t_cap %d < t0 + T", c->t_cap);
    if (need_T && (double)c->B * ((double)c->t0 + c->T + c->t_cap) * c->H * c->d >= 1099511627776.0)
        return fail(RAT_ERR_INVALID, "B*(t0+T)*H*d too large");
    if (c->flags & ~(RAT_FLAG_GRID_DILATION | RAT_FLAG_DEDUPE | RAT_FLAG_SEPARATE_GATES))
        return fail(RAT_ERR_INVALID, "unknown flags 0x%x", c->flags);
    return RAT_OK;
}

bool head_recur(const rat_cfg *c, int h) { return c->recur == nullptr || c->recur[h] != 0; }

bool grid_mode(const rat_cfg *c) { return (c->flags & RAT_FLAG_GRID_DILATION) != 0; }

// rows per batch entry of the kt/vt history (t0 + T unless the caller's buffer is longer)
int hist_rows(const rat_cfg *c) { return c->t_cap ? c->t_cap : c->t0 + c->T; }

bool dedupe_mode(const rat_cfg *c) { return (c->flags & RAT_FLAG_DEDUPE) != 0; }

// The window a head's attention runs: with dedupe a D = 1 head's window keys
// all lie in its dilated set, so it has no window part.
int attn_window(const rat_cfg *c, int h) { return dedupe_mode(c) && c->dil[h] == 1 ? 0 : c->win[h]; }

float scale_of(const rat_cfg *c) { return c->scale > 0.f ? c->scale : 1.0f / sqrtf((float)c->d); }

// Rows of one (b, h) block of the decode cache: residue-major, all positions;
// or, under the fixed grid, the grid rows plus the window ring (D > 1, W > 0).
int64_t cache_rows(const rat_cfg *c, int cap) {
    int64_t R = 0;
    for (int h = 0; h < c->H; ++h) {
        const int64_t D = c->dil[h], S = (cap + D - 1) / D;
        const int64_t rows = grid_mode(c) ? S + (D > 1 ? (int64_t)c->win[h] : 0) : D * S;
        R = std::max<int64_t>(R, rows);
    }
    return R;
}

struct Layout {
    size_t ticket = 0, flags = 0, agg = 0, incl = 0;  // scan
    size_t lse_dil = 0, att_ticket = 0;               // attention
    size_t kt = 0, vt = 0;                            // mix scratch
    size_t part = 0;                                  // decode
    int nchunks = 0, items_per_b = 0;
    size_t total = 0;
};

Layout layout(const rat_cfg *c, int op, int cap) {
    Layout L;
    size_t off = sizeof(WsHeader);
    const size_t elt = elt_size(c->dtype);
    if (op == RAT_OP_SCAN || op == RAT_OP_MIX || op == RAT_OP_MIX_CALLER_KV) {
        const int clen = scan_chunk_len(c->d);
        L.nchunks = (c->T + clen - 1) / clen;
        const size_t units = (size_t)c->B * c->H * L.nchunks;
        L.ticket = off; off += 256;
        L.flags = off; off = align256(off + units * sizeof(int));
        L.agg = off; off = align256(off + units * 3 * c->d * sizeof(float));
        L.incl = off; off = align256(off + units * 2 * c->d * sizeof(float));
    }
    if (op == RAT_OP_ATTN || op == RAT_OP_MIX || op == RAT_OP_MIX_CALLER_KV) {
        L.lse_dil = off; off = align256(off + (size_t)c->B * c->H * c->T * sizeof(float));
        L.att_ticket = off; off += kAttnTickets * sizeof(unsigned);   // one work counter per launch
    }
    if (op == RAT_OP_MIX) {
        const size_t bytes = (size_t)c->B * c->T * c->H * c->d * elt;
        L.kt = off; off = align256(off + bytes);
        L.vt = off; off = align256(off + bytes);
    }
    if (op == RAT_OP_DECODE) {
        DecodeParams tmp;
        memset(&tmp, 0, sizeof(tmp));
        L.part = off;
        off = align256(off + decode_plan(c, cap, &tmp));
        L.items_per_b = tmp.items_per_b;
    }
    L.total = off;
    return L;
}

rat_status check_ws(const rat_cfg *c, int op, int cap, void *ws, size_t ws_bytes, Layout *L) {
    if (!ws) return fail(RAT_ERR_INVALID, "workspace is NULL");
    if (((uintptr_t)ws & 255u) != 0) return fail(RAT_ERR_INVALID, "workspace must be 256-byte aligned");
    *L = layout(c, op, cap);
    if (ws_bytes < L->total)
        return fail(RAT_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L->total);
    return RAT_OK;
}

#define CHECK_PTR(p, name)                                                                   \
    do {                                                                                     \
        if (!(p)) return fail(RAT_ERR_INVALID, "%s is NULL", name);                         \
        if (!aligned16(p)) return fail(RAT_ERR_INVALID, "%s is not 16-byte aligned", name); \
    } while (0)
#define CHECK_OPT(p, name)                                                                   \
    do {                                                                                     \
        if ((p) && !aligned16(p)) return fail(RAT_ERR_INVALID, "%s is not 16-byte aligned", name); \
    } while (0)

bool empty(const rat_cfg *c) { return (size_t)c->B * (size_t)c->T == 0; }

// An empty prefill leaves the state where it was: final = init (or zero).
rat_status empty_prefill_state(const rat_cfg *c, const float *ik, const float *iv, float *fk, float *fv,
                               cudaStream_t s) {
    const size_t bytes = (size_t)c->B * c->H * c->d * sizeof(float);
    if (bytes == 0) return RAT_OK;
    const float *src[2] = {ik, iv};
    float *dst[2] = {fk, fv};
    for (int i = 0; i < 2; ++i) {
        if (!dst[i]) continue;
        cudaError_t e = src[i] ? cudaMemcpyAsync(dst[i], src[i], bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(dst[i], 0, bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "empty prefill state copy");
    }
    return RAT_OK;
}

bool separate_gates(const rat_cfg *c) { return (c->flags & RAT_FLAG_SEPARATE_GATES) != 0; }

// One scan launch: tensor maps of its operands, zeroed ticket and chunk flags.
rat_status scan_pass(const rat_cfg *c, const Layout &L, ScanParams &p, char *ws, cudaStream_t s) {
    // the one-tensor form reads slot 1 of neither list: repeat slot 0 there
    const void *srcs[5] = {p.x[0], p.x[1] ? p.x[1] : p.x[0], p.g, p.out[0], p.out[1] ? p.out[1] : p.out[0]};
    p.use_tma_out = p.out[0] != nullptr ? 1 : 0;
    // inputs hold the call's T positions; kt / vt are the [B, t0+T, H, d] history
    for (int i = 0; i < (p.use_tma_out ? 5 : 3); ++i)
        if (!encode_map_tokens(&p.tmap[i], srcs[i], c->dtype, c->B, i < 3 ? c->T : c->t0 + c->T,
                               i < 3 ? c->T : hist_rows(c), c->H, c->d, p.chunk_len))
            return fail(RAT_ERR_CUDA, "cuTensorMapEncodeTiled failed (scan operand %d)", i);
    // zero the ticket and the chunk flags (one contiguous range)
    cudaError_t e = cudaMemsetAsync(ws + L.ticket, 0, L.agg - L.ticket, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(scan flags)");
    e = launch_scan(p, c->dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return RAT_OK;
}

// Scan of the selected heads into kt/vt and/or the cache.
rat_status run_scan(const rat_cfg *c, const Layout &L, const void *k, const void *v, const void *g,
                    const float *ik, const float *iv, void *kt, void *vt, float *fk, float *fv,
                    void *ck, void *cv, int cap, char *ws, bool only_recurrent, cudaStream_t s,
                    const rat_paged_cache *pc = nullptr) {
    ScanParams p;
    memset(&p, 0, sizeof(p));
    if (pc) {
        p.page_table = pc->page_table;
        p.page_rows = pc->page_rows;
        p.pps = pc->pages_per_seq;
        p.num_pages = pc->num_pages;
    }
    p.x[0] = k; p.x[1] = v; p.g = g;
    p.init[0] = ik; p.init[1] = iv;
    p.out[0] = kt; p.out[1] = vt;
    p.fin[0] = fk; p.fin[1] = fv;
    p.cache[0] = ck; p.cache[1] = cv;
    p.cap = cap;
    p.cache_R = ck ? cache_rows(c, cap) : 0;
    p.grid = grid_mode(c) ? 1 : 0;
    p.B = c->B; p.T = c->T; p.H = c->H; p.d = c->d;
    p.t0 = c->t0;
    int n = 0, n_plain = 0;
    unsigned char plain[kMaxHeads];
    for (int h = 0; h < c->H; ++h) {
        p.head_recur[h] = head_recur(c, h) ? 1 : 0;
        p.head_dil[h] = c->dil[h];
        p.head_win[h] = c->win[h];
        if (!only_recurrent || p.head_recur[h]) p.head_list[n++] = (unsigned char)h;
        else plain[n_plain++] = (unsigned char)h;
    }
    if (n_plain > 0 && (fk || fv)) {
        // skipped heads still report their final state (a = 0: the last token)
        ScanParams pp = p;
        memcpy(pp.head_list, plain, n_plain);
        pp.nheads = n_plain;
        cudaError_t e = launch_final_of_plain_heads(pp, c->dtype, s);
        if (e != cudaSuccess) return cuda_fail(e, "final-state launch");
    }
    if (n == 0) return RAT_OK;
    p.nheads = n;
    p.nslices = c->B * n;
    p.nchunks = L.nchunks;
    p.chunk_len = scan_chunk_len(c->d);
    p.ticket = reinterpret_cast<unsigned *>(ws + L.ticket);
    p.flags = reinterpret_cast<int *>(ws + L.flags);
    p.agg = reinterpret_cast<float *>(ws + L.agg);
    p.incl = reinterpret_cast<float *>(ws + L.incl);
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    if (!separate_gates(c)) return scan_pass(c, L, p, ws, s);
    // separate gates: the keys with g[0], then the values with g[1], each in
    // the one-tensor form of the scan (ordered on the stream, one workspace)
    ScanParams pk = p, pv = p;
    pk.one = pv.one = 1;
    pk.x[1] = nullptr; pk.init[1] = nullptr; pk.out[1] = nullptr; pk.fin[1] = nullptr; pk.cache[1] = nullptr;
    pv.x[0] = v; pv.init[0] = iv; pv.out[0] = vt; pv.fin[0] = fv; pv.cache[0] = cv;
    pv.x[1] = nullptr; pv.init[1] = nullptr; pv.out[1] = nullptr; pv.fin[1] = nullptr; pv.cache[1] = nullptr;
    pv.g = static_cast<const char *>(g) + (size_t)c->B * c->T * c->H * c->d * elt_size(c->dtype);
    rat_status st = scan_pass(c, L, pk, ws, s);
    if (st != RAT_OK) return st;
    return scan_pass(c, L, pv, ws, s);
}

// Kind of a head's dilated part on the tensor cores: the residue subsequences,
// or (fixed grid, D > 1) every position against the grid subsequence.
bool grid_head(const rat_cfg *c, int h) { return grid_mode(c) && c->dil[h] > 1; }

// A head runs on the tensor-core kernel when its operands are bf16; otherwise
// the fp32 CUDA-core kernel computes it.  Any T works: the residues of a
// dilation D that does not divide T fall into two classes of equal length
// (ceil(T/D) and floor(T/D) rows), each read through its own strided view.
// A chunked prefill also needs t0 % D == 0, so that the chunk's residues line
// up with the history's.
bool tc_head(const rat_cfg *c, int h) { return c->dtype == RAT_BF16 && c->t0 % c->dil[h] == 0; }

// One tensor-core launch over `heads` (kind kTcDilated, kTcWindow or kTcGrid),
// grouped into classes of equal (dilation, K/V source).
rat_status launch_tc_part(const rat_cfg *c, const int *heads, int nheads, int kind, const void *q,
                          const void *kt, const void *vt, const void *kraw, const void *vraw,
                          const bool *raw_head, void *o, float *lse, float *lse_dil, char *ws, unsigned *tickets,
                          int *n_launch, cudaStream_t s) {
    // part: 0 every residue of the dilation (or natural order); with D not
    // dividing T, 1 the residues r < T mod D (ceil(T/D) rows) and 2 the rest
    struct Key { int D; int raw; int xd; int part; };
    int done = 0;
    bool taken[kMaxHeads] = {false};
    while (done < nheads) {
        TcParams P;
        memset(&P, 0, sizeof(P));
        P.B = c->B; P.T = c->T; P.H = c->H;
        P.kind = kind;
        P.q = q;
        P.t0 = c->t0;
        P.Tk = c->t0 + c->T;
        P.Th = hist_rows(c);
        P.scale_log2 = scale_of(c) * 1.4426950408889634f;
        P.o = o; P.lse_user = lse; P.lse_dil = lse_dil;
        P.hdr = reinterpret_cast<WsHeader *>(ws);
        if (*n_launch >= kAttnTickets) return fail(RAT_ERR_UNSUPPORTED, "more than %d attention launches", kAttnTickets);
        P.ticket = tickets + (*n_launch)++;
        P.grid = grid_mode(c) ? 1 : 0;
        for (int h = 0; h < c->H; ++h) P.win[h] = attn_window(c, h);
        // collect up to kTcMaxClasses classes
        Key keys[kTcMaxClasses];
        int ncls = 0, nh = 0;
        int cls_heads[kTcMaxClasses][kMaxHeads];
        int cls_n[kTcMaxClasses] = {0};
        for (int i = 0; i < nheads; ++i) {
            const int h = heads[i];
            if (taken[i]) continue;
            const bool win_kind = kind == kTcWindow || kind == kTcWindowDedupe;
            // the dedupe window launch also tells the heads' dilations apart
            const int D = win_kind ? 1 : c->dil[h];
            const int xd = kind == kTcWindowDedupe ? c->dil[h] : 1;
            const int rem = c->T % D, qd = c->T / D;
            Key want[2];
            int nk = 0;
            if (kind != kTcDilated || rem == 0) {
                want[nk++] = Key{D, raw_head[h] ? 1 : 0, xd, 0};
            } else {
                want[nk++] = Key{D, raw_head[h] ? 1 : 0, xd, 1};
                if (qd > 0) want[nk++] = Key{D, raw_head[h] ? 1 : 0, xd, 2};
            }
            // the head joins a launch only with all of its classes
            int ci[2] = {-1, -1}, fresh = 0;
            for (int w = 0; w < nk; ++w)
                for (int j = 0; j < ncls; ++j)
                    if (keys[j].D == want[w].D && keys[j].raw == want[w].raw && keys[j].xd == want[w].xd &&
                        keys[j].part == want[w].part)
                        ci[w] = j;
            for (int w = 0; w < nk; ++w) fresh += ci[w] < 0;
            if (ncls + fresh > kTcMaxClasses) continue;  // next launch
            for (int w = 0; w < nk; ++w) {
                if (ci[w] < 0) {
                    ci[w] = ncls++;
                    keys[ci[w]] = want[w];
                }
                cls_heads[ci[w]][cls_n[ci[w]]++] = h;
            }
            taken[i] = true;
            ++done;
        }
        // order classes by query tiles per subsequence, descending (heaviest first)
        int order[kTcMaxClasses];
        for (int i = 0; i < ncls; ++i) order[i] = i;
        std::sort(order, order + ncls, [&](int a, int b) {
            return keys[a].D != keys[b].D ? keys[a].D < keys[b].D : keys[a].part < keys[b].part;
        });
        P.ncls = ncls;
        long long pref = 0;
        for (int oi = 0; oi < ncls; ++oi) {
            const int ci = order[oi];
            TcClass &C = P.cls[oi];
            C.D = keys[ci].D;
            const int part = keys[ci].part, rem = c->T % C.D, qd = c->T / C.D;
            // query rows per group: a residue subsequence, or every position;
            // residues r0 .. r0+nres-1 (with D not dividing T: those before
            // T mod D have one row more than the rest)
            C.r0 = part == 2 ? rem : 0;
            C.nres = kind != kTcDilated ? 1 : part == 0 ? C.D : part == 1 ? rem : C.D - rem;
            C.n = kind != kTcDilated ? c->T : part == 1 ? qd + 1 : qd;
            C.kres = 0;   // every K/V map starts at its class's first residue
            C.xd = keys[ci].xd;
            C.mtiles = (C.n + 255) / 256;   // 256-row units per (b, h, residue) group
            C.nheads = cls_n[ci];
            C.head0 = nh;
            for (int j = 0; j < cls_n[ci]; ++j) P.heads[nh++] = (unsigned char)cls_heads[ci][j];
            P.prefix[oi] = pref;
            pref += (long long)c->B * C.nheads * C.nres * C.mtiles;
            const void *kb = keys[ci].raw ? kraw : kt;
            const void *vb = keys[ci].raw ? vraw : vt;
            P.kself[oi] = kb;
            P.vself[oi] = vb;
            // raw k / v (heads without recurrence, mix prefill) hold the call's rows only
            const int kv_rows = keys[ci].raw ? c->T : P.Th;
            // K/V views over the history's Tk = t0 + T positions: the class's
            // residues (dilated part; t0 is a multiple of D, so they are the
            // queries' residues), the grid (residue D - 1), or natural order
            const int krem = P.Tk % C.D, kq = P.Tk / C.D;
            int kr0 = 0, knres = 1, kn = P.Tk;
            if (kind == kTcDilated) {
                kr0 = C.r0;
                knres = C.nres;
                kn = part == 0 ? kq : part == 1 ? kq + 1 : kq;
            } else if (kind == kTcGrid) {
                kr0 = C.D - 1;
                kn = kq;
            }
            (void)krem;
            // Q: the class's residues of the call's T rows, or natural order
            const bool ok_q = kind == kTcDilated
                                  ? encode_map_res(&P.tq[oi], q, c->B, c->T, c->H, c->d, C.D, C.r0, C.nres, C.n, kTcRowsQ)
                                  : encode_map_res(&P.tq[oi], q, c->B, c->T, c->H, c->d, 1, 0, 1, c->T, kTcRowsQ);
            if (kn < 1) {
                // a grid with no key yet (Tk < D): every row attends to itself
                // only; point the maps at the first row (never read: the plan
                // of every row masks its one tile completely)
                kr0 = 0;
                kn = 1;
            }
            if (!ok_q || !encode_map_res(&P.tk[oi], kb, c->B, kv_rows, c->H, c->d, C.D, kr0, knres, kn, kTcRowsKV) ||
                !encode_map_res(&P.tv[oi], vb, c->B, kv_rows, c->H, c->d, C.D, kr0, knres, kn, kTcRowsKV))
                return fail(RAT_ERR_CUDA, "cuTensorMapEncodeTiled failed (dilation %d)", C.D);
        }
        P.prefix[ncls] = pref;
        P.total_units = pref;
        cudaError_t e = launch_attn_tc(P, c->d, s);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core attention launch");
    }
    return RAT_OK;
}

rat_status run_attn(const rat_cfg *c, const Layout &L, const void *q, const void *kt, const void *vt,
                    const void *kraw, const void *vraw, bool raw_for_plain_heads, void *o, float *lse,
                    char *ws, cudaStream_t s) {
    bool raw_head[kMaxHeads];
    int tc_all[kMaxHeads], tc_grid[kMaxHeads], tc_win[kMaxHeads];
    int n_tc = 0, n_grid = 0, n_win = 0, n_simt = 0;
    for (int h = 0; h < c->H; ++h) {
        raw_head[h] = raw_for_plain_heads && !head_recur(c, h);
        if (tc_head(c, h)) {
            if (grid_head(c, h)) tc_grid[n_grid++] = h;
            else tc_all[n_tc++] = h;
            if (attn_window(c, h) > 0) tc_win[n_win++] = h;
        } else {
            ++n_simt;
        }
    }
    float *lse_dil = reinterpret_cast<float *>(ws + L.lse_dil);
    if (n_tc + n_grid > 0) {
        unsigned *tickets = reinterpret_cast<unsigned *>(ws + L.att_ticket);
        int n_launch = 0;
        cudaError_t e = cudaMemsetAsync(tickets, 0, kAttnTickets * sizeof(unsigned), s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(attention tickets)");
        // The sort in launch_tc_part orders classes by dilation; with T fixed,
        // a smaller dilation means longer subsequences, i.e. more query tiles.
        rat_status st = RAT_OK;
        if (n_tc > 0)
            st = launch_tc_part(c, tc_all, n_tc, kTcDilated, q, kt, vt, kraw, vraw, raw_head, o, lse, lse_dil, ws,
                                tickets, &n_launch, s);
        if (st != RAT_OK) return st;
        if (n_grid > 0)
            st = launch_tc_part(c, tc_grid, n_grid, kTcGrid, q, kt, vt, kraw, vraw, raw_head, o, lse, lse_dil, ws,
                                tickets, &n_launch, s);
        if (st != RAT_OK) return st;
        if (n_win > 0) {
            st = launch_tc_part(c, tc_win, n_win, dedupe_mode(c) ? kTcWindowDedupe : kTcWindow, q, kt, vt, kraw, vraw, raw_head, o, lse, lse_dil, ws,
                                tickets, &n_launch, s);
            if (st != RAT_OK) return st;
        }
    }
    if (n_simt > 0) {
        AttnParams p;
        memset(&p, 0, sizeof(p));
        p.q = q; p.kt = kt; p.vt = vt; p.kraw = kraw; p.vraw = vraw;
        p.o = o; p.lse = lse;
        p.B = c->B; p.T = c->T; p.H = c->H; p.d = c->d;
        p.t0 = c->t0;
        p.Th = hist_rows(c);
        p.scale_log2 = scale_of(c) * 1.4426950408889634f;
        p.grid = grid_mode(c) ? 1 : 0;
        p.dedupe = dedupe_mode(c) ? 1 : 0;
        for (int h = 0; h < c->H; ++h) {
            p.dil[h] = c->dil[h];
            p.win[h] = attn_window(c, h);
            p.use_raw[h] = raw_head[h] ? 1 : 0;
            p.skip[h] = tc_head(c, h) ? 1 : 0;
        }
        p.hdr = reinterpret_cast<WsHeader *>(ws);
        cudaError_t e = launch_attn_simt(p, c->dtype, s);
        if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    }
    return RAT_OK;
}

// A paged cache descriptor: pools and table given, pages cover the logical rows.
rat_status check_paged(const rat_cfg *c, const rat_paged_cache *pc, int cap) {
    if (!pc) return fail(RAT_ERR_INVALID, "paged cache descriptor is NULL");
    CHECK_PTR(pc->pool_k, "pool_k"); CHECK_PTR(pc->pool_v, "pool_v"); CHECK_PTR(pc->page_table, "page_table");
    if (pc->page_rows < 1 || pc->num_pages < 1 || pc->pages_per_seq < 1)
        return fail(RAT_ERR_INVALID, "page_rows %d, num_pages %d, pages_per_seq %d must be >= 1", pc->page_rows,
                    pc->num_pages, pc->pages_per_seq);
    if (cap < 1) return fail(RAT_ERR_INVALID, "cache_cap %d < 1", cap);
    const long long R = cache_rows(c, cap);
    if ((long long)pc->pages_per_seq * pc->page_rows < R)
        return fail(RAT_ERR_INVALID, "pages_per_seq x page_rows < %lld cache rows", R);
    return RAT_OK;
}

// rat_decode_step with a dense cache (pc = NULL) or a paged one.
rat_status decode_step(const rat_cfg *cfg, const void *q, const void *k, const void *v, const void *g,
                       float *state_k, float *state_v, void *cache_k, void *cache_v, const rat_paged_cache *pc,
                       int cache_cap, const int32_t *pos, void *o, float *lse, void *ws, size_t ws_bytes,
                       rat_stream_t stream) {
    rat_status st = check_decode_args(cfg, q, k, v, g, state_k, state_v, cache_k, cache_v, cache_cap, pos, o, lse);
    if (st != RAT_OK) return st;
    if (cfg->B == 0) return RAT_OK;
    Layout L;
    st = check_ws(cfg, RAT_OP_DECODE, cache_cap, ws, ws_bytes, &L);
    if (st != RAT_OK) return st;
    DecodeParams p;
    memset(&p, 0, sizeof(p));
    decode_plan(cfg, cache_cap, &p);
    p.q = q; p.k = k; p.v = v; p.g = g;
    p.state[0] = state_k; p.state[1] = state_v;
    p.cache[0] = cache_k; p.cache[1] = cache_v;
    if (pc) {
        p.page_table = pc->page_table;
        p.page_rows = pc->page_rows;
        p.pps = pc->pages_per_seq;
        p.num_pages = pc->num_pages;
    }
    p.pos = pos; p.o = o; p.lse = lse;
    char *w = static_cast<char *>(ws);
    p.part = reinterpret_cast<float *>(w + L.part);
    const size_t part_bytes = align256((size_t)cfg->B * p.items_per_b * (cfg->d + 2) * sizeof(float));
    p.counter = reinterpret_cast<int *>(w + L.part + part_bytes);
    p.cap = cache_cap; p.B = cfg->B; p.H = cfg->H; p.d = cfg->d;
    p.scale_log2 = scale_of(cfg) * 1.4426950408889634f;
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    // per-(b,h) completion counters start from zero on every call
    cudaError_t ez = cudaMemsetAsync(p.counter, 0, (size_t)cfg->B * cfg->H * sizeof(int), (cudaStream_t)stream);
    if (ez != cudaSuccess) return cuda_fail(ez, "cudaMemsetAsync(decode counters)");
    cudaError_t e = launch_decode(p, cfg->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return RAT_OK;
}

// rat_scan_prefill with a dense cache (pc = NULL) or a paged one.
rat_status scan_prefill(const rat_cfg *cfg, const void *k, const void *v, const void *g, const float *init_k,
                        const float *init_v, void *kt, void *vt, float *final_k, float *final_v, void *cache_k,
                        void *cache_v, const rat_paged_cache *pc, int cache_cap, void *ws, size_t ws_bytes,
                        rat_stream_t stream) {
    rat_status st = check_cfg(cfg);
    if (st != RAT_OK) return st;
    CHECK_OPT(init_k, "init_k"); CHECK_OPT(init_v, "init_v");
    CHECK_OPT(final_k, "final_k"); CHECK_OPT(final_v, "final_v");
    if (empty(cfg)) return empty_prefill_state(cfg, init_k, init_v, final_k, final_v, (cudaStream_t)stream);
    CHECK_PTR(k, "k"); CHECK_PTR(v, "v"); CHECK_PTR(g, "g");
    CHECK_OPT(init_k, "init_k"); CHECK_OPT(init_v, "init_v");
    CHECK_OPT(kt, "kt"); CHECK_OPT(vt, "vt");
    CHECK_OPT(final_k, "final_k"); CHECK_OPT(final_v, "final_v");
    CHECK_OPT(cache_k, "cache_k"); CHECK_OPT(cache_v, "cache_v");
    if ((kt == nullptr) != (vt == nullptr)) return fail(RAT_ERR_INVALID, "kt and vt must be given together");
    if ((cache_k == nullptr) != (cache_v == nullptr))
        return fail(RAT_ERR_INVALID, "cache_k and cache_v must be given together");
    if (!kt && !cache_k) return fail(RAT_ERR_INVALID, "no output: give kt/vt and/or cache_k/cache_v");
    if (cache_k && cache_cap < (long long)cfg->t0 + cfg->T)
        return fail(RAT_ERR_INVALID, "cache_cap %d < t0 + T = %lld", cache_cap, (long long)cfg->t0 + cfg->T);
    Layout L;
    st = check_ws(cfg, RAT_OP_SCAN, 0, ws, ws_bytes, &L);
    if (st != RAT_OK) return st;
    return run_scan(cfg, L, k, v, g, init_k, init_v, kt, vt, final_k, final_v, cache_k, cache_v,
                    cache_cap, static_cast<char *>(ws), false, (cudaStream_t)stream, pc);
}

}  // namespace

// The argument rules of a decode step, shared by every decode entry point
// (with and without a workspace) so that they accept and refuse alike.
rat_status rat::check_decode_args(const rat_cfg *cfg, const void *q, const void *k, const void *v, const void *g,
                                  const float *state_k, const float *state_v, const void *cache_k,
                                  const void *cache_v, int cache_cap, const int32_t *pos, const void *o,
                                  const float *lse) {
    rat_status st = check_cfg(cfg, false);
    if (st != RAT_OK) return st;
    if (cfg->B == 0) return RAT_OK;
    CHECK_PTR(q, "q"); CHECK_PTR(k, "k"); CHECK_PTR(v, "v"); CHECK_PTR(g, "g");
    CHECK_PTR(state_k, "state_k"); CHECK_PTR(state_v, "state_v");
    CHECK_PTR(cache_k, "cache_k"); CHECK_PTR(cache_v, "cache_v");
    CHECK_PTR(pos, "pos"); CHECK_PTR(o, "o"); CHECK_OPT(lse, "lse");
    if (cache_cap < 1) return fail(RAT_ERR_INVALID, "cache_cap %d < 1", cache_cap);
    return RAT_OK;
}

extern "C" {

int rat_version(void) { return 101; }

long long rat_launch_count(void) { return rat::g_launches.load(std::memory_order_relaxed); }

const char *rat_last_error(void) { return g_last_error; }

const char *rat_status_string(rat_status s) {
    switch (s) {
    case RAT_OK: return "RAT_OK";
    case RAT_ERR_INVALID: return "RAT_ERR_INVALID: invalid argument";
    case RAT_ERR_UNSUPPORTED: return "RAT_ERR_UNSUPPORTED: no kernel for this configuration";
    case RAT_ERR_CUDA: return "RAT_ERR_CUDA: CUDA runtime or launch failure";
    case RAT_ERR_TIMEOUT: return "RAT_ERR_TIMEOUT: a bounded device-side wait gave up";
    case RAT_ERR_WORKSPACE: return "RAT_ERR_WORKSPACE: workspace too small";
    }
    return "unknown rat_status";
}

size_t rat_workspace_size(const rat_cfg *cfg, int op, int cache_cap) {
    if (op < RAT_OP_SCAN || op > RAT_OP_TOPK_DECODE) return 0;
    const bool dec = op == RAT_OP_DECODE || op == RAT_OP_TOPK_DECODE;
    if (check_cfg(cfg, !dec) != RAT_OK) return 0;
    if (dec && cache_cap < 1) return 0;
    if (op == RAT_OP_TOPK_DECODE) return sizeof(WsHeader);   // the status word only
    return layout(cfg, op, cache_cap).total;
}

rat_status rat_workspace_init(void *ws, size_t ws_bytes, rat_stream_t stream) {
    if (!ws || ws_bytes < sizeof(WsHeader)) return fail(RAT_ERR_INVALID, "workspace NULL or < 256 bytes");
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace header)");
    return RAT_OK;
}

int64_t rat_cache_rows(const rat_cfg *cfg, int cap) {
    if (check_cfg(cfg, false) != RAT_OK || cap < 1) return 0;
    return cache_rows(cfg, cap);
}

rat_status rat_scan_prefill(const rat_cfg *cfg, const void *k, const void *v, const void *g,
                            const float *init_k, const float *init_v, void *kt, void *vt,
                            float *final_k, float *final_v, void *cache_k, void *cache_v,
                            int cache_cap, void *ws, size_t ws_bytes, rat_stream_t stream) {
    return scan_prefill(cfg, k, v, g, init_k, init_v, kt, vt, final_k, final_v, cache_k, cache_v, nullptr,
                        cache_cap, ws, ws_bytes, stream);
}

rat_status rat_scan_prefill_paged(const rat_cfg *cfg, const void *k, const void *v, const void *g,
                                  const float *init_k, const float *init_v, void *kt, void *vt, float *final_k,
                                  float *final_v, const rat_paged_cache *cache, int cache_cap, void *ws,
                                  size_t ws_bytes, rat_stream_t stream) {
    rat_status st = check_cfg(cfg);
    if (st != RAT_OK) return st;
    st = check_paged(cfg, cache, cache_cap);
    if (st != RAT_OK) return st;
    return scan_prefill(cfg, k, v, g, init_k, init_v, kt, vt, final_k, final_v, cache->pool_k, cache->pool_v,
                        cache, cache_cap, ws, ws_bytes, stream);
}

rat_status rat_dilated_attn_prefill(const rat_cfg *cfg, const void *q, const void *kt, const void *vt,
                                    void *o, float *lse, void *ws, size_t ws_bytes, rat_stream_t stream) {
    rat_status st = check_cfg(cfg);
    if (st != RAT_OK) return st;
    if (empty(cfg)) return RAT_OK;
    CHECK_PTR(q, "q"); CHECK_PTR(kt, "kt"); CHECK_PTR(vt, "vt"); CHECK_PTR(o, "o");
    CHECK_OPT(lse, "lse");
    Layout L;
    st = check_ws(cfg, RAT_OP_ATTN, 0, ws, ws_bytes, &L);
    if (st != RAT_OK) return st;
    return run_attn(cfg, L, q, kt, vt, nullptr, nullptr, false, o, lse, static_cast<char *>(ws),
                    (cudaStream_t)stream);
}

rat_status rat_mix_prefill(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                           const void *g, const float *init_k, const float *init_v, void *o,
                           float *lse, void *kt, void *vt, float *final_k, float *final_v,
                           void *ws, size_t ws_bytes, rat_stream_t stream) {
    rat_status st = check_cfg(cfg);
    if (st != RAT_OK) return st;
    CHECK_OPT(init_k, "init_k"); CHECK_OPT(init_v, "init_v");
    CHECK_OPT(final_k, "final_k"); CHECK_OPT(final_v, "final_v");
    if (empty(cfg)) return empty_prefill_state(cfg, init_k, init_v, final_k, final_v, (cudaStream_t)stream);
    CHECK_PTR(q, "q"); CHECK_PTR(k, "k"); CHECK_PTR(v, "v"); CHECK_PTR(g, "g"); CHECK_PTR(o, "o");
    CHECK_OPT(lse, "lse");
    CHECK_OPT(kt, "kt"); CHECK_OPT(vt, "vt");
    CHECK_OPT(final_k, "final_k"); CHECK_OPT(final_v, "final_v");
    if ((kt == nullptr) != (vt == nullptr)) return fail(RAT_ERR_INVALID, "kt and vt must be given together");
    const bool caller_kv = kt != nullptr;
    if (cfg->t0 > 0 && !caller_kv)
        return fail(RAT_ERR_INVALID, "a chunked prefill (t0 > 0) needs the caller's kt/vt history");
    if (!caller_kv && cfg->t_cap != 0 && cfg->t_cap != cfg->T)
        return fail(RAT_ERR_INVALID, "t_cap describes the caller's kt/vt; the workspace keeps T rows");
    Layout L;
    st = check_ws(cfg, caller_kv ? RAT_OP_MIX_CALLER_KV : RAT_OP_MIX, 0, ws, ws_bytes, &L);
    if (st != RAT_OK) return st;
    char *w = static_cast<char *>(ws);
    if (!caller_kv) {
        kt = w + L.kt;
        vt = w + L.vt;
    }
    const cudaStream_t s = (cudaStream_t)stream;
    // Heads without recurrence attend to k/v directly, unless the caller asked
    // for the complete augmented tensors.
    st = run_scan(cfg, L, k, v, g, init_k, init_v, kt, vt, final_k, final_v, nullptr, nullptr, 0, w,
                  !caller_kv, s);
    if (st != RAT_OK) return st;
    return run_attn(cfg, L, q, kt, vt, k, v, !caller_kv, o, lse, w, s);
}

rat_status rat_decode_step(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                           const void *g, float *state_k, float *state_v, void *cache_k,
                           void *cache_v, int cache_cap, const int32_t *pos, void *o, float *lse,
                           void *ws, size_t ws_bytes, rat_stream_t stream) {
    return decode_step(cfg, q, k, v, g, state_k, state_v, cache_k, cache_v, nullptr, cache_cap, pos, o, lse, ws,
                       ws_bytes, stream);
}

rat_status rat_decode_step_paged(const rat_cfg *cfg, const void *q, const void *k, const void *v, const void *g,
                                 float *state_k, float *state_v, const rat_paged_cache *cache, int cache_cap,
                                 const int32_t *pos, void *o, float *lse, void *ws, size_t ws_bytes,
                                 rat_stream_t stream) {
    rat_status st = check_cfg(cfg, false);
    if (st != RAT_OK) return st;
    st = check_paged(cfg, cache, cache_cap);
    if (st != RAT_OK) return st;
    return decode_step(cfg, q, k, v, g, state_k, state_v, cache->pool_k, cache->pool_v, cache, cache_cap, pos, o,
                       lse, ws, ws_bytes, stream);
}

// ---------------------------------------------------------- top-k block decode

namespace {

rat_status check_topk(const rat_cfg *c, int block, int topk, int mode, int cap) {
    rat_status st = check_cfg(c, false);
    if (st != RAT_OK) return st;
    if (block < 1) return fail(RAT_ERR_INVALID, "block %d < 1", block);
    if (topk < 0 || topk > kTopkMaxK) return fail(RAT_ERR_INVALID, "topk %d outside [0, %d]", topk, kTopkMaxK);
    if (mode != RAT_TOPK_QUEST && mode != RAT_TOPK_MOBA) return fail(RAT_ERR_INVALID, "top-k mode %d", mode);
    if (cap < 1) return fail(RAT_ERR_INVALID, "cache_cap %d < 1", cap);
    if ((cap + (long long)block - 1) / block > kTopkMaxBlocks)
        return fail(RAT_ERR_UNSUPPORTED, "ceil(cache_cap / block) exceeds %d blocks", kTopkMaxBlocks);
    for (int h = 0; h < c->H; ++h)
        if (c->dil[h] != 1 || c->win[h] != 0)
            return fail(RAT_ERR_INVALID, "top-k decoding needs dil = 1 and win = 0 (head %d)", h);
    return RAT_OK;
}

TopkParams topk_params(const rat_cfg *c, int block, int topk, int mode, int cap, float *stats) {
    TopkParams p;
    memset(&p, 0, sizeof(p));
    p.cache_R = cache_rows(c, cap);
    p.cap = cap; p.B = c->B; p.H = c->H; p.d = c->d;
    p.bs = block; p.K = topk; p.mode = mode;
    p.sep = separate_gates(c) ? 1 : 0;
    p.nblk = (int)((cap + (long long)block - 1) / block);
    p.stats = stats;
    p.scale_log2 = scale_of(c) * 1.4426950408889634f;
    for (int h = 0; h < c->H; ++h) p.recur[h] = head_recur(c, h) ? 1 : 0;
    return p;
}

}  // namespace

size_t rat_topk_stats_size(const rat_cfg *cfg, int block, int cache_cap) {
    if (check_topk(cfg, block, 0, RAT_TOPK_QUEST, cache_cap) != RAT_OK) return 0;
    const size_t nblk = (size_t)((cache_cap + (long long)block - 1) / block);
    return (size_t)cfg->B * cfg->H * nblk * 2 * cfg->d * sizeof(float);
}

rat_status rat_topk_build_stats(const rat_cfg *cfg, int block, int mode, const void *cache_k, int cache_cap,
                                float *stats, rat_stream_t stream) {
    rat_status st = check_topk(cfg, block, 0, mode, cache_cap);
    if (st != RAT_OK) return st;
    if (cfg->T < 0 || cfg->T > cache_cap) return fail(RAT_ERR_INVALID, "T %d outside [0, cache_cap]", cfg->T);
    if ((size_t)cfg->B * cfg->T == 0) return RAT_OK;
    CHECK_PTR(cache_k, "cache_k"); CHECK_PTR(stats, "stats");
    TopkParams p = topk_params(cfg, block, 0, mode, cache_cap, stats);
    p.cache[0] = const_cast<void *>(cache_k);
    cudaError_t e = launch_topk_stats(p, cfg->T, cfg->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "top-k statistics launch");
    return RAT_OK;
}

rat_status rat_topk_decode_step(const rat_cfg *cfg, int block, int topk, int mode, const void *q, const void *k,
                                const void *v, const void *g, float *state_k, float *state_v, void *cache_k,
                                void *cache_v, int cache_cap, float *stats, const int32_t *pos, void *o,
                                float *lse, int32_t *sel, void *ws, size_t ws_bytes, rat_stream_t stream) {
    rat_status st = check_topk(cfg, block, topk, mode, cache_cap);
    if (st != RAT_OK) return st;
    if (cfg->B == 0) return RAT_OK;
    CHECK_PTR(q, "q"); CHECK_PTR(k, "k"); CHECK_PTR(v, "v"); CHECK_PTR(g, "g");
    CHECK_PTR(state_k, "state_k"); CHECK_PTR(state_v, "state_v");
    CHECK_PTR(cache_k, "cache_k"); CHECK_PTR(cache_v, "cache_v"); CHECK_PTR(stats, "stats");
    CHECK_PTR(pos, "pos"); CHECK_PTR(o, "o"); CHECK_OPT(lse, "lse"); CHECK_OPT(sel, "sel");
    Layout L;
    st = check_ws(cfg, RAT_OP_TOPK_DECODE, cache_cap, ws, ws_bytes, &L);
    if (st != RAT_OK) return st;
    TopkParams p = topk_params(cfg, block, topk, mode, cache_cap, stats);
    p.q = q; p.k = k; p.v = v; p.g = g;
    p.state[0] = state_k; p.state[1] = state_v;
    p.cache[0] = cache_k; p.cache[1] = cache_v;
    p.pos = pos; p.o = o; p.lse = lse; p.sel = sel;
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    cudaError_t e = launch_topk_decode(p, cfg->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "top-k decode launch");
    return RAT_OK;
}

rat_status rat_check_status(void *ws, rat_stream_t stream) {
    if (!ws) return fail(RAT_ERR_INVALID, "workspace is NULL");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int hdr[2] = {0, 0};
    e = cudaMemcpy(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
    if (hdr[0] != 0) {
        const int zero[2] = {0, 0};
        e = cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(clear status)");
        return fail((rat_status)hdr[0], "device reported %s (unit %d)", rat_status_string((rat_status)hdr[0]),
                    hdr[1]);
    }
    return RAT_OK;
}

rat_status rat_debug_set_scan_stall(void *ws, size_t ws_bytes, int64_t ticket, int64_t spin_limit_ns,
                                    rat_stream_t stream) {
    if (!ws || ws_bytes < sizeof(WsHeader)) return fail(RAT_ERR_INVALID, "workspace NULL or too small");
    long long v[2] = {ticket < 0 ? 0LL : (long long)ticket + 1, spin_limit_ns > 0 ? (long long)spin_limit_ns : 0LL};
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemcpy(static_cast<char *>(ws) + offsetof(WsHeader, stall_ticket_plus1), v,
                                         sizeof(v), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "set scan stall");
    return RAT_OK;
}

}  // extern "C"
