/*
 * rat.h -- C ABI of librat.so, the B200 (sm_100a) implementation of the RAT+
 * temporal-mixing operator: a per-channel gated linear recurrence over keys and
 * values, then causal softmax attention over the recurrence-augmented keys and
 * values with dilation D and an optional dense local window W, the two parts
 * merged by log-sum-exp.
 *
 * Sources (page titles and the passages each entry point follows):
 *   "RAT+: Train Dense, Infer Sparse -- Recurrence Augmented Attention for
 *    Dilated Inference": Abstract (dilated attention cuts attention FLOPs and
 *    KV cache by D; optional local windows; hybrid head compositions),
 *    Figure 1(a) (full-sequence recurrence, L = T), Figure 1(c) (dilated
 *    attention with optional local attention), Figure 2 (prefill = scan of the
 *    recurrence + dilated attention; decode = a step update of the recurrence
 *    + attention over the cache), Figure 9 (non-zero initial cell state).
 *   "Augmenting Attention with Exponentially Decaying Memory Improves
 *    Query-Aware KV Sparsity", section 2.1 (key and value states updated with
 *    an input-dependent gate; O(1) extra compute and storage per token).
 *
 * Definitions used by every entry point (the pages give the method at the
 * level of captions; these are the plain readings of them):
 *   recurrence   s_t = a_t * s_{t-1} + (1 - a_t) * x_t per channel, for x = k
 *                and x = v, with a_t = sigmoid(g_t) from one gate tensor g
 *                (one per tensor with RAT_FLAG_SEPARATE_GATES);
 *                s_{-1} = init (zero when not given).  A head with recur = 0
 *                has a = 0: its augmented keys/values are the raw ones.
 *   dilation     query t attends to { j <= t : (t - j) mod D == 0 }.  With
 *                RAT_FLAG_GRID_DILATION it attends instead to the fixed grid
 *                { j <= t : j mod D == D - 1 } plus itself (j = t, once): the
 *                chunk-end keys of the RAT page's Approach (chunk size D),
 *                which a decode can keep in a cache D times smaller.
 *   window       W > 0 adds a second softmax over { max(0, t-W+1) <= j <= t }.
 *   merge        the two softmaxes are merged by log-sum-exp (a key in both
 *                sets counts in both; with RAT_FLAG_DEDUPE, once).
 *   scale        scores are scale * <q_t, k~_j>, scale = 1/sqrt(d) by default.
 *
 * Conventions shared by all calls
 *   - Tensors are dense row-major.  Token tensors are [B, T, H, d] (d fastest);
 *     lse is [B, H, T] fp32; states are [B, H, d] fp32.
 *   - Element type of q/k/v/g/o/kt/vt/cache is cfg->dtype (RAT_BF16 or
 *     RAT_F32).  States, init and lse are always fp32.
 *   - Every device pointer must be 16-byte aligned.
 *   - Ownership: the caller owns every buffer and the stream.  The library
 *     allocates no device memory and may be called from several host threads
 *     on different workspaces.  Its only process-wide state is a launch
 *     counter, a per-thread last-error string, each kernel's shared-memory
 *     limit (raised once per device), and the static scratch of
 *     rat_decode_step_noalloc.  Calls are asynchronous on `stream`; inputs
 *     must stay valid until the stream reaches the call.
 *   - Workspace: `ws` is caller-allocated device memory of at least
 *     rat_workspace_size() bytes, zero-filled once before its first use
 *     (rat_workspace_init does that).  Calls that share a workspace must be
 *     ordered on one stream.
 *   - Errors: argument errors return RAT_ERR_INVALID / RAT_ERR_UNSUPPORTED /
 *     RAT_ERR_WORKSPACE before anything is launched.  A failed launch returns
 *     RAT_ERR_CUDA.  A device-side error (a bounded wait that gave up) is
 *     recorded in the workspace and returned by rat_check_status().
 *     rat_last_error() gives a one-line reason for the calling thread's last
 *     non-OK return.
 */
#ifndef RAT_H
#define RAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbol marker (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define RAT_API __attribute__((visibility("default")))
#else
#define RAT_API
#endif

/* A cudaStream_t (same underlying type); NULL is the legacy default stream. */
typedef struct CUstream_st *rat_stream_t;

typedef enum {
    RAT_OK = 0,
    RAT_ERR_INVALID = 1,     /* null / misaligned pointer, out-of-range size or parameter */
    RAT_ERR_UNSUPPORTED = 2, /* valid request with no kernel in this library (e.g. d not 64/128) */
    RAT_ERR_CUDA = 3,        /* a CUDA runtime call or a kernel launch failed */
    RAT_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (rat_check_status) */
    RAT_ERR_WORKSPACE = 5    /* ws_bytes below rat_workspace_size() */
} rat_status;

typedef enum { RAT_F32 = 0, RAT_BF16 = 1 } rat_dtype;

/* Workspace requests (the `op` argument of rat_workspace_size). */
typedef enum {
    RAT_OP_SCAN = 0,          /* rat_scan_prefill */
    RAT_OP_ATTN = 1,          /* rat_dilated_attn_prefill */
    RAT_OP_MIX = 2,           /* rat_mix_prefill with kt = vt = NULL (K~/V~ kept in ws) */
    RAT_OP_MIX_CALLER_KV = 3, /* rat_mix_prefill with caller-provided kt and vt */
    RAT_OP_DECODE = 4,        /* rat_decode_step */
    RAT_OP_TOPK_DECODE = 5    /* rat_topk_decode_step */
} rat_op;

/*
 * Operator configuration.  The per-head arrays are HOST memory, read during
 * the call only.  Head h uses dilation dil[h] >= 1, window win[h] >= 0 (0 = no
 * window) and recurrence flag recur[h] (0 = no recurrence; NULL = all heads
 * recurrent) -- the hybrid head compositions of the RAT+ Abstract.
 * Limits of this library version: d in {64, 128}; 1 <= H <= 256; B, T >= 0;
 * B*T*H*d < 2^40 elements.
 *
 * Chunked prefill (t0 > 0): a call covers positions t0 .. t0+T-1 of its
 * sequences.  Token inputs (q, k, v, g) and outputs (o, lse) hold those T
 * positions; the augmented keys/values kt, vt are history buffers
 * [B, t_cap, H, d] (t_cap = 0 means t0 + T) whose rows 0 .. t0+T-1 hold
 * positions 0 .. t0+T-1, so one buffer serves every chunk: the scan writes rows t0 ..
 * t0+T-1 (init_k/init_v carry the state after position t0-1) and the
 * attention reads all rows, so the chunks of a prefill give the one-shot
 * result.  Decode-cache rows go to positions t0 + t.  rat_mix_prefill then
 * needs caller kt/vt.  Decode steps ignore t0.  An empty batch or sequence (B*T == 0) launches
 * no kernel; a prefill then only copies init (or zero) to final.
 */
typedef struct {
    int B, T, H, d;
    int dtype;               /* rat_dtype */
    const int32_t *dil;      /* host [H] */
    const int32_t *win;      /* host [H] */
    const uint8_t *recur;    /* host [H] or NULL */
    float scale;             /* <= 0 selects 1/sqrt(d) */
    uint32_t flags;          /* RAT_FLAG_* bits, 0 = the defaults above */
    int t0;                  /* position of this call's first token (chunked prefill), 0 = a whole prefill */
    int t_cap;               /* rows per batch entry of the kt/vt history, >= t0 + T; 0 = t0 + T */
} rat_cfg;

/* Fixed-grid reading of dilation (see "dilation" above) for every head of the
 * call, and the matching decode-cache layout (see rat_cache_rows). */
#define RAT_FLAG_GRID_DILATION 1u
/* A key in both the dilated set and the window counts once: the window part
 * skips the keys the dilated set holds (with D = 1 the window adds nothing). */
#define RAT_FLAG_DEDUPE 2u
/* Separate gates for keys and values: the gate tensor g holds two tensors of
 * the usual shape, g[0] for the key recurrence and g[1] for the value
 * recurrence ([2, B, T, H, d] in a prefill, [2, B, H, d] in a decode step). */
#define RAT_FLAG_SEPARATE_GATES 4u

/* Bytes of workspace `op` needs for `cfg` (cache_cap: decode capacity, else
 * ignored).  Returns 0 when cfg is invalid. */
RAT_API size_t rat_workspace_size(const rat_cfg *cfg, int op, int cache_cap);

/* Zero the workspace header (status word and debug fields). */
RAT_API rat_status rat_workspace_init(void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * Decode cache layout ("dilated KV cache", RAT+ Abstract and Figure 2).
 * A cache tensor is [B, H, R, d] in cfg->dtype with R = rat_cache_rows(cfg,
 * cap).  Position j of head h is stored at row
 *     (j mod D_h) * ceil(cap / D_h) + floor(j / D_h)
 * i.e. residue-major: the rows a decode query at position t reads for its
 * dilated part (all j == t mod D_h, j <= t) form one contiguous slab.
 * With RAT_FLAG_GRID_DILATION a head keeps only its grid: position j with
 * j mod D_h == D_h - 1 at row floor(j / D_h), rows [0, ceil(cap / D_h)).  A
 * head with D_h > 1 and a window W_h > 0 also keeps a ring of its last W_h
 * positions after the grid: position j at row ceil(cap / D_h) + (j mod W_h).
 * R is the largest head's row count in either layout.
 * Returns 0 when cfg or cap is invalid.
 */
RAT_API int64_t rat_cache_rows(const rat_cfg *cfg, int cap);

/*
 * Prefill recurrence (RAT+ Figure 1(a) and Figure 2 "associative scan";
 * Exponentially Decaying Memory section 2.1).
 *   k, v, g          in  [B,T,H,d]  keys, values, gate logits
 *   init_k, init_v   in  [B,H,d] fp32 or NULL (zero initial state; RAT+ Figure 9)
 *   kt, vt           out [B,T,H,d]  augmented keys/values, or NULL when a cache
 *                        is given (recur = 0 heads receive a copy of k / v)
 *   final_k, final_v out [B,H,d] fp32 s_{T-1}, or NULL
 *   cache_k, cache_v out decode cache tensors (layout above) for positions
 *                        0..T-1 (under the fixed grid: the grid rows, and
 *                        the ring rows of positions T-W_h .. T-1), or NULL;
 *                        requires T <= cache_cap
 * At least one of (kt, vt) or (cache_k, cache_v) must be given, as pairs.
 */
RAT_API rat_status rat_scan_prefill(const rat_cfg *cfg, const void *k, const void *v, const void *g,
                            const float *init_k, const float *init_v, void *kt, void *vt,
                            float *final_k, float *final_v, void *cache_k, void *cache_v,
                            int cache_cap, void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * Attention step over augmented keys/values (RAT+ Abstract, Figure 1(c)):
 * dilated causal attention, plus the local window for heads with win > 0,
 * merged by log-sum-exp.
 *   q, kt, vt  in  [B,T,H,d]
 *   o          out [B,T,H,d]
 *   lse        out [B,H,T] fp32 natural-log log-sum-exp of the merged softmax, or NULL
 */
RAT_API rat_status rat_dilated_attn_prefill(const rat_cfg *cfg, const void *q, const void *kt, const void *vt,
                                    void *o, float *lse, void *ws, size_t ws_bytes,
                                    rat_stream_t stream);

/*
 * The whole temporal-mixing operator for a prefill: rat_scan_prefill of k and
 * v followed by rat_dilated_attn_prefill.  kt/vt may be NULL (kept in the
 * workspace, size RAT_OP_MIX) or caller buffers (RAT_OP_MIX_CALLER_KV) that
 * receive the augmented keys/values.  Heads with recur = 0 attend to k and v
 * directly.  final_k/final_v (nullable) receive the recurrent state after
 * token T-1, which a decode continues from.
 */
RAT_API rat_status rat_mix_prefill(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                           const void *g, const float *init_k, const float *init_v, void *o,
                           float *lse, void *kt, void *vt, float *final_k, float *final_v,
                           void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * One decode step for every batch entry (RAT+ Figure 2: "a simple step update"
 * of the recurrence, then attention over the dilated KV cache).  cfg->T is
 * ignored.  For batch entry b the new token is at position t = pos[b]:
 *   1. s <- a*s + (1-a)*x for x = k and v (a = sigmoid(g), a = 0 if recur = 0),
 *      updating state_k / state_v in place (fp32 [B,H,d]);
 *   2. the new augmented key/value (rounded to cfg->dtype) is stored at t's
 *      cache row (under the fixed grid: at its grid row when t is on the
 *      grid, and at its ring row when the head keeps a ring);
 *   3. o[b,h] = merged attention of q over the cache rows j <= t of the
 *      dilated set (and window) of t.
 *   q, k, v, g   in  [B,H,d]
 *   cache_k/v    in/out [B,H,R,d], R = rat_cache_rows(cfg, cache_cap); rows of
 *                positions < pos[b] must hold earlier augmented keys/values
 *                (under the fixed grid: the grid rows below t and the ring
 *                rows of t-W_h+1 .. t-1)
 *   pos          in  DEVICE int32 [B], 0 <= pos[b] < cache_cap (a position out
 *                of range makes the kernel skip that entry and record
 *                RAT_ERR_INVALID for rat_check_status)
 *   o            out [B,H,d];  lse out [B,H] fp32 or NULL
 * Positions may differ between batch entries (a ragged batch).  A step issues
 * one memset (its combine counters) and one kernel on `stream`, and after the
 * first call on a device no other CUDA runtime call, so a step can be captured
 * in a CUDA graph and replayed with the inputs and pos refreshed in place.
 */
RAT_API rat_status rat_decode_step(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                           const void *g, float *state_k, float *state_v, void *cache_k,
                           void *cache_v, int cache_cap, const int32_t *pos, void *o, float *lse,
                           void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * Paged decode cache, for serving engines that hand out KV memory in pages.
 * The logical rows of a (b, h) block -- the layout of rat_cache_rows, in
 * either dilation reading -- live in pages of page_rows rows: logical row r of
 * batch entry b, head h is row (r mod page_rows) of page
 * page_table[b * pages_per_seq + r / page_rows] of the pools, which are
 * [num_pages, H, page_rows, d] in cfg->dtype.  pages_per_seq * page_rows must
 * cover rat_cache_rows(cfg, cache_cap).  Only the pages of the rows a call
 * touches need valid entries; a touched entry outside [0, num_pages) is never
 * dereferenced: the prefill leaves that row unwritten and the decode step
 * skips each (b, h) whose step touches it (o = 0, state unchanged), and either
 * records RAT_ERR_INVALID for rat_check_status.  The caller owns pools and
 * table (device memory).
 */
typedef struct {
    void *pool_k, *pool_v;        /* [num_pages, H, page_rows, d] */
    const int32_t *page_table;    /* device int32 [B, pages_per_seq] */
    int page_rows, pages_per_seq, num_pages;
} rat_paged_cache;

/* rat_scan_prefill writing a paged cache (cache_cap as there). */
RAT_API rat_status rat_scan_prefill_paged(const rat_cfg *cfg, const void *k, const void *v, const void *g,
                                          const float *init_k, const float *init_v, void *kt, void *vt,
                                          float *final_k, float *final_v, const rat_paged_cache *cache,
                                          int cache_cap, void *ws, size_t ws_bytes, rat_stream_t stream);

/* rat_decode_step over a paged cache; the ring's copies split at page ends. */
RAT_API rat_status rat_decode_step_paged(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                                         const void *g, float *state_k, float *state_v,
                                         const rat_paged_cache *cache, int cache_cap, const int32_t *pos,
                                         void *o, float *lse, void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * rat_decode_step without a workspace, for callers that cannot allocate
 * device memory when they decode: a plugin inside an inference engine that
 * owns all device memory and gives its plugins no scratch buffer, or a serving
 * loop whose device-memory budget is fixed at start-up.  The operator paper
 * has no counterpart to this call; it only moves rat_decode_step's scratch.
 * Arguments and results are those of rat_decode_step minus (ws, ws_bytes).
 *   - Scratch: a static 16 MiB device array inside librat.so, held by every
 *     GPU that loads the library until the process exits.  A step needs
 *     about 256 + B * items * (d + 2) * 4 + B * H * 4 bytes, items = sum over
 *     heads of ceil(ceil(cache_cap / D_h) / r), where r = 2048 rows is halved
 *     (down to 256) while B * items < 592; a larger step returns
 *     RAT_ERR_UNSUPPORTED with the sizes in rat_last_error().
 *   - The first call on a device (with that device current) looks up the
 *     array's device address (cudaGetSymbolAddress) and caches it with the
 *     device's current context; make that first call before any stream
 *     capture.  If that context is later destroyed (cudaDeviceReset), the next
 *     call sees a new context and looks the address up again, so it too
 *     should come before any capture.
 *   - Arguments are checked by the same code as rat_decode_step, so a bad
 *     call returns the same status and rat_last_error() text.
 *   - All calls share the one array and it keeps the last call's contents;
 *     each call clears the part that must start at zero (its completion
 *     counters) itself.  Calls whose kernels overlap on a GPU race on it:
 *     order them on one stream.
 *   - Never allocates or frees device memory.  An out-of-range pos[b] still
 *     makes the kernel skip that entry (its o is zero), but is not reported:
 *     there is no workspace for rat_check_status to read.
 */
RAT_API rat_status rat_decode_step_noalloc(const rat_cfg *cfg, const void *q, const void *k, const void *v,
                                           const void *g, float *state_k, float *state_v, void *cache_k,
                                           void *cache_v, int cache_cap, const int32_t *pos, void *o,
                                           float *lse, rat_stream_t stream);

/*
 * Top-k block attention for decoding over the augmented keys/values (RAT+
 * Figure 3 and Tables 17-18; Exponentially Decaying Memory, section 2.2,
 * sparse inference settings).  Keys are grouped in blocks of `block`
 * consecutive positions.  The query at t (block c = t / block) attends, in one
 * softmax, to the rows j <= t of block 0, of block c, and of the `topk` best
 * of blocks 1 .. c-1 (all of them when there are fewer), ranked by
 *   RAT_TOPK_QUEST  sum_ch max(q_ch * kmin_ch, q_ch * kmax_ch) over the block's
 *                   per-channel key range (an upper bound of q.k in the block)
 *   RAT_TOPK_MOBA   q . mean of the block's keys
 * with equal scores going to the lower block.  The cache is the dense layout:
 * every head must have dil = 1 and win = 0 (the sparse selection replaces
 * dilation and window), so position j of a head is row j.
 *
 * Block statistics: `stats` is caller memory of rat_topk_stats_size() bytes,
 * fp32 [B, H, ceil(cache_cap / block), 2, d]: per block the channel minima and
 * maxima (Quest), or the channel sums and zeros (MoBA), of the cached keys.
 * Limits: 1 <= block; 0 <= topk <= 64; ceil(cache_cap / block) <= 16384.
 */
typedef enum { RAT_TOPK_QUEST = 0, RAT_TOPK_MOBA = 1 } rat_topk_mode;

/* Bytes of the block-statistics buffer (0 when an argument is invalid). */
RAT_API size_t rat_topk_stats_size(const rat_cfg *cfg, int block, int cache_cap);

/*
 * Statistics of the blocks of positions 0 .. cfg->T - 1 (the tokens a prefill
 * wrote into cache_k with rat_scan_prefill), in `mode`; a last partial block
 * covers the positions it has.  Blocks at or past cfg->T are left as they are.
 */
RAT_API rat_status rat_topk_build_stats(const rat_cfg *cfg, int block, int mode, const void *cache_k,
                                        int cache_cap, float *stats, rat_stream_t stream);

/*
 * One decode step with top-k block attention.  As rat_decode_step (the state
 * update, the append of the new row at row t = pos[b], ragged positions, the
 * error behaviour), plus: the new key is folded into its block's statistics,
 * which must hold blocks 0 .. c of the positions before t; `sel` (nullable,
 * device int32 [B, H, topk]) receives the selected blocks in selection order,
 * -1 where fewer were available.  ws: rat_workspace_size(cfg,
 * RAT_OP_TOPK_DECODE, cache_cap) bytes.  One kernel per step, no other CUDA
 * call after the first on a device (graph-capturable).
 */
RAT_API rat_status rat_topk_decode_step(const rat_cfg *cfg, int block, int topk, int mode, const void *q,
                                        const void *k, const void *v, const void *g, float *state_k,
                                        float *state_v, void *cache_k, void *cache_v, int cache_cap,
                                        float *stats, const int32_t *pos, void *o, float *lse, int32_t *sel,
                                        void *ws, size_t ws_bytes, rat_stream_t stream);

/*
 * Synchronises `stream`, returns the first device-side error recorded in `ws`
 * since the last check (RAT_OK if none) and clears it.  RAT_ERR_CUDA if the
 * synchronisation itself fails.
 */
RAT_API rat_status rat_check_status(void *ws, rat_stream_t stream);

/* Static string for a status code. */
RAT_API const char *rat_status_string(rat_status s);

/* One-line reason for the calling thread's last non-OK return ("" if none). */
RAT_API const char *rat_last_error(void);

/* ABI version of this header (major * 100 + minor). */
RAT_API int rat_version(void);

/* Number of kernels this library has launched in this process so far. */
RAT_API long long rat_launch_count(void);

/*
 * Failure-injection hooks for tests of the bounded device-side waits.
 * rat_debug_set_scan_stall makes scan chunk `ticket` (0-based launch order;
 * -1 = off) never publish its carry, so the chunks after it must give up after
 * `spin_limit_ns` (0 = the default of one second) and record RAT_ERR_TIMEOUT.
 * Stored in the workspace header; no effect on other workspaces.
 */
RAT_API rat_status rat_debug_set_scan_stall(void *ws, size_t ws_bytes, int64_t ticket, int64_t spin_limit_ns,
                                    rat_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RAT_H */
