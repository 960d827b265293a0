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
    int nres;    // groups per (b, h): D residues (dilated part), else 1
    int kres;    // residue coordinate of K/V relative to Q's (D - 1 for the grid)
    int xd;      // dilation of the heads (the dedupe window launch), else 1
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
    unsigned char heads[kMaxHeads];
    int win[kMaxHeads];
};

size_t attn_tc_smem_bytes(int hd);
cudaError_t launch_attn_tc(const TcParams &p, int hd, cudaStream_t s);
// 5-D TMA map of the first T rows of a [B,Ts,H,d] bf16 tensor (Ts rows per
// batch entry) viewed as (d, H, D, T/D, B), box (64, 1, 1, box_rows, 1);
// requires T % D == 0.
bool encode_map_5d(CUtensorMap *map, const void *base, int B, int T, int Ts, int H, int d, int D, int box_rows);

}  // namespace rat
