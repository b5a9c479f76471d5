// Split-K work partition shared by the decode kernels.
//
// Every (sequence b, KV head g) pair is a *segment* of keys: the retrieval
// rows or the filled ring slots it reads.  All segments are laid end to end
// in blocks of p.blk tokens and a persistent grid of C CTAs takes C equal
// contiguous ranges of that axis; a CTA walks its range piece by piece (a
// piece = the part of one segment inside the range).  Partial results go to
// workspace slot (segment + CTA), unique because moving along the axis
// crosses either a segment or a CTA boundary.
#pragma once

#include <stdint.h>

#include "duo_internal.cuh"

namespace duo {
namespace {

// Blocks of BLK tokens (16, or a whole tile for paged caches so that no
// tile straddles a page).  BLK is a compile-time constant: a division by a
// run-time 64-bit value is an out-of-line routine, and code first reached
// at a piece boundary while HBM is saturated costs microseconds to fetch.
template <int BLK>
__device__ __forceinline__ int blocks_of(int64_t rows) { return int((rows + BLK - 1) / BLK); }

__device__ __forceinline__ int64_t rows_r(int len, int64_t cap) {
    int64_t r = len < 0 ? 0 : len;
    return r < cap ? r : cap;
}
__device__ __forceinline__ int64_t rows_s(int len, int S, int W) {
    int64_t r = len < 0 ? 0 : len;
    return r < S + W ? r : S + W;
}

// Rows each segment of sequence b reads: retrieval rows [r0, r0 + nr) of its
// cache, streaming slots [0, ns) of its ring.
struct SeqRows {
    int64_t r0, nr, ns;
};

__device__ __forceinline__ SeqRows seq_rows(const DecodeParams& p, int b) {
    SeqRows x;
    if (p.r_end == nullptr) {
        const int L = p.len[b];
        x.r0 = 0;
        x.nr = rows_r(L, p.cap);
        x.ns = rows_s(L, p.S, p.W);
    } else {
        int64_t r0 = p.r_begin ? p.r_begin[b] : 0;
        r0 = r0 < 0 ? 0 : (r0 > p.cap ? p.cap : r0);
        int64_t r1 = p.r_end[b];
        r1 = r1 < r0 ? r0 : (r1 > p.cap ? p.cap : r1);
        x.r0 = r0;
        x.nr = r1 - r0;
        int64_t ns = p.s_len ? p.s_len[b] : 0;
        x.ns = ns < 0 ? 0 : (ns > p.S + p.W ? p.S + p.W : ns);
    }
    return x;
}

// Shared-memory table built once per launch: int32 words
// [0, B]  running count of 16-token blocks per sequence (prefix),
// then three arrays of B: first retrieval row, retrieval rows, ring slots,
// then per KV head: retrieval heads before it (n_kv + 1 words) and its
// rank with the retrieval flag in the sign bit (n_kv words).
// Locating a piece then reads shared memory only: a global read of the
// lengths, or an indexed read of the launch parameters that misses the
// constant cache, costs microseconds while the kernel saturates HBM.
__host__ __device__ constexpr size_t seq_table_bytes(int B, int n_kv) {
    return (size_t(B + 1) + 3 * size_t(B) + 2 * size_t(n_kv) + 1) * 4;
}

// Units a segment of nb blocks takes on the partition axis: its blocks,
// preceded by `weight` blocks that hold no keys when it has any.  The weight
// stands for the fixed cost of starting a piece, so that a CTA whose range
// starts many segments gets fewer keys (0 = partition by keys alone).
__device__ __forceinline__ int seg_units(int nb, int weight) { return nb > 0 ? nb + weight : 0; }

// Fill the table (shared); warp 0 does a chunked shuffle scan.  Caller syncs afterwards.
template <int BLK>
__device__ void build_prefix(const DecodeParams& p, int32_t* bpre) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    int run = 0;
    if (lane == 0) bpre[0] = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        int c = 0;
        if (b < p.B) {
            const SeqRows x = seq_rows(p, b);
            c = p.n_r * seg_units(blocks_of<BLK>(x.nr), p.seg_weight) +
                p.n_s * seg_units(blocks_of<BLK>(x.ns), p.seg_weight);
            int32_t* rows = bpre + p.B + 1;
            rows[b] = int32_t(x.r0);
            rows[p.B + b] = int32_t(x.nr);
            rows[2 * p.B + b] = int32_t(x.ns);
        }
        int x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (b < p.B) bpre[b + 1] = run + x;
        run += __shfl_sync(0xffffffffu, x, 31);
    }
    int32_t* hb = bpre + 4 * p.B + 1;
    int32_t* hr = hb + p.n_kv + 1;
    for (int g = lane; g <= p.n_kv; g += 32) {
        hb[g] = p.r_before[g];
        if (g < p.n_kv) hr[g] = p.rank[g] | (p.is_r[g] ? int32_t(0x80000000u) : 0);
    }
}

// First block index owned by CTA c when `total` blocks are split over n CTAs.
__device__ __forceinline__ int64_t cta_start(int64_t c, int64_t total, int64_t n) { return c * total / n; }
// CTA that owns block gb.
__device__ __forceinline__ int cta_owner(int64_t gb, int64_t total, int64_t n) {
    int64_t c = ((gb + 1) * n - 1) / total;
    return int(c < n - 1 ? c : n - 1);
}

struct Piece {
    int b, g, seg;          // sequence, KV head, segment index b * n_kv + g
    int64_t row0;           // first cache row of the segment (retrieval row ranges)
    int64_t seg_gb;         // first global block of the segment
    int seg_nb;             // blocks in the segment
    int64_t tok0, tok1;     // token rows of this piece inside the segment
    int64_t end_gb;         // global block after the piece
    bool whole;             // the piece is the whole segment
    bool retr;              // KV head g is a retrieval head
    int rank;               // g's index among the layer's retrieval or streaming heads
};

// Locate the piece that starts at global block gb (gb < range end).
template <int BLK>
__device__ __forceinline__ Piece locate(const DecodeParams& p, const int32_t* bpre, int64_t gb,
                                        int64_t range_end) {
    Piece pc;
    // b = last index with bpre[b] <= gb  (binary search over B + 1 entries)
    int lo = 0, hi = p.B;   // invariant: bpre[lo] <= gb < bpre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bpre[mid] <= gb) lo = mid; else hi = mid;
    }
    pc.b = lo;
    const int32_t* tab = bpre + p.B + 1;
    const int64_t r0 = tab[lo], rr = tab[p.B + lo], rs = tab[2 * p.B + lo];
    const int nbr = blocks_of<BLK>(rr), nbs = blocks_of<BLK>(rs);
    const int ur = seg_units(nbr, p.seg_weight), us = seg_units(nbs, p.seg_weight);
    const int64_t local = gb - bpre[lo];
    const int32_t* hb = bpre + 4 * p.B + 1;
    const int32_t* hr = hb + p.n_kv + 1;
    int g = 0;
    int64_t start = 0;
    bool retr = false;
    for (; g < p.n_kv; ++g) {
        start = int64_t(hb[g]) * ur + int64_t(g - hb[g]) * us;
        retr = hr[g] < 0;
        if (local < start + (retr ? ur : us)) break;
    }
    pc.g = g;
    pc.retr = retr;
    pc.rank = hr[g] & 0x7fffffff;
    pc.seg = lo * p.n_kv + g;
    pc.row0 = retr ? r0 : 0;
    pc.seg_nb = retr ? nbr : nbs;
    pc.seg_gb = bpre[lo] + start + (pc.seg_nb > 0 ? p.seg_weight : 0);   // first block with keys
    const int64_t seg_end = pc.seg_gb + pc.seg_nb;
    pc.end_gb = seg_end < range_end ? seg_end : range_end;
    const int64_t rows = retr ? rr : rs;
    pc.tok0 = gb > pc.seg_gb ? (gb - pc.seg_gb) * BLK : 0;
    const int64_t t1 = (pc.end_gb - pc.seg_gb) * BLK;
    pc.tok1 = t1 < rows ? t1 : rows;
    if (pc.tok1 < pc.tok0) pc.tok1 = pc.tok0;   // the range ends before the segment's first key
    pc.whole = (gb <= pc.seg_gb) && (pc.end_gb == seg_end);
    return pc;
}

// The next piece that holds keys, starting at global block gb (advanced
// past it); false when the range has none left.  With a segment weight a
// range may start or end inside a weight, which gives a piece without keys.
template <int BLK>
__device__ __forceinline__ bool next_piece(const DecodeParams& p, const int32_t* bpre, int64_t& gb,
                                           int64_t range_end, Piece& pc) {
    while (gb < range_end) {
        pc = locate<BLK>(p, bpre, gb, range_end);
        gb = pc.end_gb;
        if (pc.tok1 > pc.tok0) return true;
    }
    return false;
}

}  // namespace
}  // namespace duo
