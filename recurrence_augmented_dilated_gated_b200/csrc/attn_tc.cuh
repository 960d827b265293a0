// attn_tc.cuh -- parameters of the tensor-core attention kernel (attn_tc.cu).
#pragma once

#include <cuda.h>

#include "rat_internal.cuh"

namespace rat {

constexpr int kTcMaxClasses = 8;
constexpr int kTcRowsQ = 128;   // query rows per sub-tile (Q box height)
constexpr int kTcRowsKV = 128;  // keys per K/V tile (K/V box height)

// Launch kinds: the residue subsequences of the dilated part; the window part
// (merged with the dilated part); the fixed-grid reading of the dilated part
// (every position against the subsequence of residue D-1, plus its own key).
// kTcWindowDedupe is the window part that skips the keys of the dilated set.
constexpr int kTcDilated = 0, kTcWindow = 1, kTcGrid = 2, kTcWindowDedupe = 3;

// Heads of one launch that share a dilation and a K/V source.
struct TcClass {
    int D;       // dilation (1 in the window launch: natural order)
    int n;       // query rows of one group: a residue subsequence (T / D), or T
    int mtiles;  // 256-row work units per group, ceil(n / 256)
    int nheads;  // heads in the class
    int head0;   // first entry of the class in TcParams::heads
    int nres;    // groups per (b, h): residues r0 .. r0+nres-1 (dilated part), else 1
    int kres;    // residue coordinate of K/V relative to Q's in their maps
    int xd;      // dilation of the heads (the dedupe window launch), else 1
    int r0;      // residue of the class's first group (its maps start there)
};

struct TcParams {
    CUtensorMap tq[kTcMaxClasses];  // 5-D maps (d, H, D, T/D, B), box (64, 1, 1, rows, 1), 128B swizzle:
    CUtensorMap tk[kTcMaxClasses];  // Q boxes of kTcRowsQ rows, K and V boxes of kTcRowsKV rows
    CUtensorMap tv[kTcMaxClasses];
    TcClass cls[kTcMaxClasses];     // sorted by mtiles, descending
    long long prefix[kTcMaxClasses + 1];  // prefix[c] = work units of the classes before c
    int ncls;
    int B, T, H;
    int kind;                       // kTcDilated, kTcWindow, kTcGrid or kTcWindowDedupe
    int t0, Tk, Th;                 // chunked prefill: queries at t0 + t; K/V maps cover Tk = t0 + T rows
                                    // of a history with Th rows per batch entry
    int grid;                       // fixed-grid reading (the dedupe window's excluded keys)
    float scale_log2;
    const void *q;                  // [B,T,H,d] bf16 (the grid's own-key score)
    const void *kself[kTcMaxClasses];  // K/V source of each class, [B,T,H,d] bf16
    const void *vself[kTcMaxClasses];
    void *o;                        // [B,T,H,d] bf16
    float *lse_user;                // [B,H,T] or null
    float *lse_dil;                 // [B,H,T] scratch: lse of the dilated part of windowed heads
    WsHeader *hdr;
    unsigned int *ticket;           // work-unit counter of this launch (zero at launch)
    long long total_units;
    unsigned char heads[2 * kMaxHeads];  // class lists (a head with D not dividing T is in two)
    int win[kMaxHeads];
};

size_t attn_tc_smem_bytes(int hd);
cudaError_t launch_attn_tc(const TcParams &p, int hd, cudaStream_t s);
// 5-D TMA map of the first T rows of a [B,Ts,H,d] bf16 tensor (Ts rows per
// batch entry) viewed as (d, H, D, T/D, B), box (64, 1, 1, box_rows, 1);
// requires T % D == 0.
bool encode_map_5d(CUtensorMap *map, const void *base, int B, int T, int Ts, int H, int d, int D, int box_rows);
// 5-D TMA map of residues r0 .. r0+nres-1 of a [B,Ts,H,d] bf16 tensor under
// dilation D, n rows each: element (c, h, r, j, b) is channel c of head h at
// position r0 + r + j*D of batch entry b; box (64, 1, 1, box_rows, 1).  Every
// element of the view must lie inside the tensor (r0 + nres - 1 + (n-1)*D < Ts);
// box rows past n read as zero.
bool encode_map_res(CUtensorMap *map, const void *base, int B, int Ts, int H, int d, int D, int r0, int nres, int n,
                    int box_rows);

}  // namespace rat
