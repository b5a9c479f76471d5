// Chunked-prefill attention on the 5th-generation tensor cores (tcgen05).
//
// A chunk of C query rows that follows P cached tokens: row i sits at
// position P + i and reads keys j <= P + i ("Attention Variants and KV-Cache
// Compression", "When Is Reuse Exact?").  Retrieval heads read all of them
// (dense causal attention: the cached prefix from the retrieval cache, the
// rest from the chunk's own K/V); streaming heads read only the sinks and the
// window (j < S or j >= P + i - W + 1), block-sparse: only the ring's sink
// slots, its window slots (for the first W-1 rows) and the chunk tiles that
// meet the band are visited ("Hardware-Fused Prefill" in the DuoAttention
// guide: dense attention for retrieval heads, a block-sparse sliding-window
// kernel for streaming heads).
//
// Four launches per call:
//  1. convert_v_kernel writes an fp16 copy of every V row the attention can
//     read (cached prefix, ring slots, the chunk) into the caller's workspace,
//     zeroing tile tails; a second, usually empty launch of it rescales the
//     values of any head whose largest |v| reaches 2^15 by a power of two
//     2^-E (undone in the epilogue), so no finite bf16 value overflows fp16.  P is multiplied in fp16 rather than bf16 (rounding
//     P to bf16 alone costs ~1.5e-3 relative error in the output, fp16
//     ~2e-4), and one tcgen05 MMA needs both operands in the same type; this
//     way each V row is converted once per call instead of once per CTA.
//     For FP8 / INT4 or paged caches it also writes bf16 copies of the cached
//     keys (codes as exact values; pages gathered into one range per head).
//  2. prefill_kernel, one CTA per (sequence, query head, 128-row query tile),
//     11 warps:
//       warp 0      TMA: Q once, then K tiles (bf16, 128 keys x 128 dims as
//                   two 128-byte-swizzled slabs) into a 3-stage ring
//       warp 1      allocates TMEM; one lane issues tcgen05.mma:
//                     S_j  = Q K_j^T  (bf16, SS form, M = N = 128, 8 x K16)
//                     O   += P_j V_j  (fp16, TS form: P from TMEM, V MN-major)
//                   S is double-buffered in TMEM so S_{j+1} overlaps softmax_j
//       warp 2      TMA: fp16 V tiles into a 2-stage ring
//       warps 3-10  softmax, two threads per query row (TMEM lane = row, one
//                   64-key half each): masked scores, running max with lazy
//                   rescaling (O rescaled only when the max grows by more
//                   than 2^8), P_j as packed fp16 written to TMEM, O / l.
//
//  3. merge_parts_kernel combines the two halves of every query tile that
//     was split over two CTAs (long retrieval prefixes) by log-sum-exp; rows
//     of unsplit tiles were written directly and are left alone.
//
// Every mbarrier wait is bounded; on a timeout the CTA sets
// DUO_STATUS_WAIT_TIMEOUT, stops, waits (bounded) for its own copies and
// MMAs in flight, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>
#include <string.h>

#include "duo_internal.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kBM = 128;   // query rows per CTA
constexpr int kBN = 128;   // keys per tile
constexpr int kHD = 128;   // head dim (prefill is built for d = 128)
constexpr int kThreads = 352;   // 11 warps: K TMA, MMA, V TMA, 8 softmax
constexpr int kSoftmaxWarp0 = 3;
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kSlab = 128 * 128;        // bytes: 128 rows x 64 16-bit elements
constexpr uint32_t kTile = 2 * kSlab;        // 32 KB: 128 rows x 128 16-bit elements
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256, kTmemP = 384;
constexpr float kNegBig = -1.0e30f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units
// A retrieval query tile with at least this many key tiles is shared by two
// CTAs (the first and the second half of its keys), so that the last wave of
// a launch is made of shorter pieces; their partial outputs are combined by
// log-sum-exp in merge_parts_kernel.
constexpr int kSplitMin = 128;
// CTAs per (head, source) of the value conversion pass.
constexpr int kConvCtas = 64;
// fp16 copies of the values keep |v| * 2^-E below 2^15, E >= 0 a power-of-two
// exponent per (sequence, KV head): far from fp16's 65504 limit, and the
// unnormalised P V sums (P <= 2^8 with lazy rescaling) stay far inside fp32.
constexpr int kV16MaxLog2 = 15;

// Instruction descriptors: S = Q K^T in bf16 (both K-major), O += P V in fp16
// (P from TMEM, V MN-major); M = 128, N = 128.
constexpr uint32_t kIdescQK = idesc_f16(kBM, kBN, true, false, false);
constexpr uint32_t kIdescPV = idesc_f16(kBM, kHD, false, false, true);

struct PrefillParams {
    CUtensorMap tm_q, tm_kc, tm_kr, tm_ks;      // bf16: queries, chunk / retrieval / ring keys
    CUtensorMap tm_kr16, tm_ks16;               // FP8 caches: bf16 copies of the cached keys' codes
    CUtensorMap tm_vc, tm_vr, tm_vs;            // fp16 copies of the values (workspace)
    const int32_t* prefix;
    float* out;
    float* part_o;          // [2][B][hq][C][d] normalised partial outputs of split query tiles
    float* part_lse;        // [2][B][hq][C] their log2-sum-exp (scaled scores)
    int32_t* status;
    const int32_t* vexp;    // [B * n_kv] value exponent E of each head's fp16 copies (out *= 2^E)
    int64_t cap;
    int B, hq, n_kv, G, C, n_qt, S, W, n_r, n_s, LR, LS;
    float scale_log2;
    unsigned long long timeout_ns;
    int fp8;                                    // cached keys / values are E4M3 codes
    int kcopy;                                  // cached keys read from the workspace copies (FP8 or paged)
    int32_t rank[kMaxKvHeads];
    uint8_t is_r[kMaxKvHeads];
    float k_scale[kMaxKvHeads], v_scale[kMaxKvHeads];
};

struct ConvertParams {
    const uint16_t* vr;     // bf16 caches and chunk
    const uint16_t* vs;
    const uint16_t* vc;
    uint16_t* v16r;         // fp16 copies: [B][n_r][LR][d], [B][n_s][LS][d], [B][n_kv][C][d]
    uint16_t* v16s;
    uint16_t* v16c;
    const void* kr;         // cached keys (bf16 or E4M3; retrieval: a contiguous cache or the page pool)
    const void* ks;
    uint16_t* k16r;         // bf16 copies of the cached keys [B][n_r][LR][d], [B][n_s][LS][d]
    uint16_t* k16s;
    int fp8;
    int int4;               // cached codes are packed INT4 (two per byte)
    int page_tokens;        // > 0: retrieval rows live in pages
    int max_pages;
    int64_t num_pages;
    const int32_t* page_table;
    int32_t* status;
    const int32_t* prefix;
    float* vmax;            // [B * n_kv][2][kConvCtas] largest |v| each first-pass CTA converted
    int32_t* vexp;          // [B * n_kv] E: the fp16 copies hold v * 2^-E (read by the attention epilogue)
    int64_t cap;
    int B, n_kv, n_r, n_s, S, W, C, LR, LS;
    int32_t rank[kMaxKvHeads];
    uint8_t is_r[kMaxKvHeads];
};

// ------------------------------------------------------------------ TMA tiles
// One 128-row x 128-dim bf16 tile = two 64-dim slabs (x = 0 and x = 64).
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int row, uint32_t bar) {
    tma_load_2d(dst, map, 0, row, bar);
    tma_load_2d(dst + kSlab, map, 64, row, bar);
}

// ------------------------------------------------------------------ key tiles
enum : int { kSrcCache = 0, kSrcSink = 1, kSrcWindow = 2, kSrcChunk = 3 };

struct KeyTile {
    int src;       // kSrc*
    int row0;      // first row in its source (cache row, ring slot offset, chunk row)
    int nvalid;    // rows of the tile that hold keys
    bool masked;   // needs the element mask
};

// The key tiles one CTA visits, in order.  Computed identically by every role.
struct Plan {
    bool retr;
    int P, i0, i1, C, S, W;
    int n_a;           // cache tiles (retrieval) or sink tiles (streaming)
    int n_w;           // window tiles (streaming)
    int nw_rows;       // filled window slots
    int c0_lo, c0_hi, c1_lo, c1_hi;   // chunk tile ranges (inclusive; empty if lo > hi)
    int n;             // tiles this CTA visits
    int jb;            // index of its first tile in the row's order (split query tiles)

    __device__ void init(bool is_retrieval, int P_, int i0_, int C_, int S_, int W_) {
        retr = is_retrieval;
        P = P_; i0 = i0_; C = C_; S = S_; W = W_;
        i1 = min(i0 + kBM, C);
        const int hi = (i1 - 1) / kBN;
        n_w = 0; nw_rows = 0;
        c1_lo = 1; c1_hi = 0;
        if (retr) {
            n_a = (P + kBN - 1) / kBN;
            c0_lo = 0; c0_hi = hi;
        } else {
            const int sinks = min(S, P);
            n_a = (sinks + kBN - 1) / kBN;
            if (P > S && i0 <= W - 2) {
                nw_rows = min(P - S, W);
                n_w = (nw_rows + kBN - 1) / kBN;
            }
            const int lo = max(0, i0 - W + 1) / kBN;
            if (P < S) {
                const int sc = min((min(S - P, C) - 1) / kBN, hi);
                if (sc + 1 >= lo) { c0_lo = 0; c0_hi = hi; }
                else { c0_lo = 0; c0_hi = sc; c1_lo = lo; c1_hi = hi; }
            } else {
                c0_lo = lo; c0_hi = hi;
            }
        }
        n = n_a + n_w + (c0_hi - c0_lo + 1) + (c1_hi >= c1_lo ? c1_hi - c1_lo + 1 : 0);
        jb = 0;
    }

    // Keep only the first (part 0) or second (part 1) half of the tiles.
    __device__ void take_half(int part) {
        const int h = n / 2;
        jb = part ? h : 0;
        n = part ? n - h : h;
    }

    // Tile j of this CTA holds cached keys (they come first).
    __device__ bool cached(int j) const { return j + jb < n_a + n_w; }

    __device__ KeyTile get(int j) const {
        KeyTile t;
        j += jb;
        if (j < n_a) {
            t.src = retr ? kSrcCache : kSrcSink;
            t.row0 = j * kBN;
            const int lim = retr ? P : min(S, P);
            t.nvalid = min(kBN, lim - t.row0);
            t.masked = t.nvalid < kBN;
            return t;
        }
        j -= n_a;
        if (j < n_w) {
            t.src = kSrcWindow;
            t.row0 = j * kBN;
            t.nvalid = min(kBN, nw_rows - t.row0);
            t.masked = true;
            return t;
        }
        j -= n_w;
        const int n0 = c0_hi - c0_lo + 1;
        const int k = j < n0 ? c0_lo + j : c1_lo + (j - n0);
        t.src = kSrcChunk;
        t.row0 = k * kBN;
        t.nvalid = min(kBN, C - t.row0);
        t.masked = !retr || t.nvalid < kBN || t.row0 + kBN - 1 > i0;
        return t;
    }
};

// Bit c set for every c in [lo, hi] within 0..31.
__device__ __forceinline__ uint32_t range_bits(int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, 31);
    if (lo > hi) return 0u;
    const uint32_t upto = hi == 31 ? 0xffffffffu : ((2u << hi) - 1u);
    return upto & ~((1u << lo) - 1u);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    unsigned long long av = *reinterpret_cast<unsigned long long*>(&a);
    unsigned long long bv = *reinterpret_cast<unsigned long long*>(&b);
    unsigned long long dv;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(dv) : "l"(av), "l"(bv));
    return *reinterpret_cast<float2*>(&dv);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ bool timed_wait(uint32_t bar, uint32_t parity, const PrefillParams& p,
                                           volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, p.timeout_ns)) return true;
    set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Lane 0 waits on the mbarrier for the warp (fewer shared-memory polls).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const PrefillParams& p,
                                          volatile int* abort_flag) {
    // fast path: the phase has completed already (each lane probes it; a
    // phase, once completed, stays so until this warp consumes it)
    if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = timed_wait(bar, parity, p, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Barrier over the 256 softmax threads that also ORs a flag across them, so
// every softmax warp takes the same exit decision.
__device__ __forceinline__ bool softmax_barrier_any(bool flag) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 256, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(out)
        : "r"(uint32_t(flag))
        : "memory");
    return out != 0;
}

// The same over the two softmax warps that share a TMEM lane quarter (the two
// halves of the same 32 query rows): named barrier 4 + quarter, 64 threads.
__device__ __forceinline__ bool pair_barrier_any(int quarter, bool flag) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 64, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(out)
        : "r"(uint32_t(flag)), "r"(4 + quarter)
        : "memory");
    return out != 0;
}

// ------------------------------------------------------------------ V -> fp16 (and FP8 codes -> 16 bits)
// Eight E4M3 codes -> their values as fp16 (exact: every E4M3 value is an
// fp16 value), or as bf16 (also exact).
__device__ __forceinline__ uint4 e4m3x8_to_f16(uint2 c) {
    uint32_t h[4];
    const uint16_t s[4] = {uint16_t(c.x & 0xffff), uint16_t(c.x >> 16), uint16_t(c.y & 0xffff), uint16_t(c.y >> 16)};
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[i]) : "h"(s[i]));
    return make_uint4(h[0], h[1], h[2], h[3]);
}

__device__ __forceinline__ uint4 e4m3x8_to_bf16(uint2 c) {
    const uint4 h = e4m3x8_to_f16(c);
    const uint32_t w[4] = {h.x, h.y, h.z, h.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&w[i]);
        const float2 f = __half22float2(hh);
        const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight INT4 codes (element 2i in the low nibble of byte i) -> their
// integer values as fp16 or bf16 (exact: |c| <= 8).
__device__ __forceinline__ int int4_at(uint32_t w, int i) {
    return int(w << (28 - 4 * i)) >> 28;                  // sign-extend nibble i
}

__device__ __forceinline__ uint4 int4x8_to_f16(uint32_t w) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack_half2(float(int4_at(w, 2 * i)), float(int4_at(w, 2 * i + 1)));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 int4x8_to_bf16(uint32_t w) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(float(int4_at(w, 2 * i)), float(int4_at(w, 2 * i + 1)));
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// One thread per 8 values (16 bytes of output).  blockIdx.y = b * n_kv + g;
// blockIdx.z = 0: the head's cached value rows, 1: its chunk's value rows,
// 2 (quantised caches only): its cached key rows.  Values become fp16; cached
// FP8 or INT4 codes become their (unscaled) values, fp16 for V and bf16 for K -- the
// scales are applied in the attention kernel.  Rows that hold no key (past
// the prefix or the filled ring slots) up to the end of the last tile the
// attention reads are written as zeros, so masked columns always meet
// finite values.
//
// Range of the values.  bf16 reaches 3.4e38, fp16 only 65504, so each head's
// copies hold v * 2^-E with E >= 0 the smallest exponent that keeps every
// |v| * 2^-E below 2^kV16MaxLog2 (a power-of-two scale: exact, apart from
// values that fall into fp16's subnormal range, 2^-24 and below, far under
// the head's largest value); the attention epilogue multiplies by 2^E.  The
// first pass (REDO = false) converts with E = 0 and records the largest |v|
// of every CTA; the second pass (REDO = true, values only) computes E per
// head, writes it for the attention kernel, and leaves at once when E = 0
// (every value already fits) or converts the head's values again with 2^-E.
template <bool REDO>
__global__ void __launch_bounds__(256) convert_v_kernel(const __grid_constant__ ConvertParams c) {
    const int bg = blockIdx.y;
    const int b = bg / c.n_kv, g = bg % c.n_kv;
    const int P = max(c.prefix[b], 0);
    const bool keys = blockIdx.z == 2;
    __shared__ uint32_t red[8];
    float vmul = 1.f;
    if (REDO) {
        uint32_t mx = 0;   // |v| >= 0, so the float bits order as unsigned integers
        for (int t = threadIdx.x; t < 2 * kConvCtas; t += blockDim.x)
            mx = max(mx, __float_as_uint(c.vmax[size_t(bg) * 2 * kConvCtas + t]));
        mx = __reduce_max_sync(0xffffffffu, mx);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        mx = 0;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) mx = max(mx, red[w]);
        const int e = int((mx >> 23) & 0xffu) - 127;        // floor(log2 max |v|)
        const int E = max(0, e - (kV16MaxLog2 - 1));       // <= 114: 2^-E and 2^E are normal floats
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) c.vexp[bg] = E;
        if (E == 0) return;
        vmul = __uint_as_float(uint32_t(127 - E) << 23);
    }
    // bytes per cached row: bf16, E4M3 codes, or INT4 codes two per byte
    const size_t row_bytes = c.int4 ? kHD / 2 : (c.fp8 ? kHD : 2 * kHD);
    const uint8_t* base = nullptr;                        // cached rows (contiguous) or the page pool
    const uint16_t* chunk = nullptr;
    bool paged = false;
    uint16_t* dst;
    int64_t n_conv, n_rows;
    if (blockIdx.z == 1) {
        chunk = c.vc + size_t(bg) * c.C * kHD;
        dst = c.v16c + size_t(bg) * c.C * kHD;
        n_conv = n_rows = c.C;
    } else if (c.is_r[g]) {
        const size_t r = size_t(b) * c.n_r + c.rank[g];
        const uint8_t* pool = static_cast<const uint8_t*>(keys ? c.kr : static_cast<const void*>(c.vr));
        paged = c.page_tokens > 0;
        base = paged ? pool : pool + r * size_t(c.cap) * row_bytes;
        dst = (keys ? c.k16r : c.v16r) + r * size_t(c.LR) * kHD;
        n_conv = min(int64_t(P), c.cap);
        n_rows = (n_conv + kBN - 1) / kBN * kBN;          // tail of the last prefix tile
    } else {
        const size_t r = size_t(b) * c.n_s + c.rank[g];
        base = static_cast<const uint8_t*>(keys ? c.ks : static_cast<const void*>(c.vs)) + r * size_t(c.S + c.W) * row_bytes;
        dst = (keys ? c.k16s : c.v16s) + r * size_t(c.LS) * kHD;
        n_conv = min(P, c.S + c.W);                         // filled slots
        n_rows = c.LS;
    }
    // eight bf16 values -> fp16 of v * vmul, with the largest |v| seen
    auto to_f16 = [vmul](const uint4 w, float& amax) {
        const float2 a = bf2_to_f2(w.x), bb = bf2_to_f2(w.y), cc = bf2_to_f2(w.z), dd = bf2_to_f2(w.w);
        if (!REDO)
            amax = fmaxf(amax, fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(bb.x), fabsf(bb.y))),
                                     fmaxf(fmaxf(fabsf(cc.x), fabsf(cc.y)), fmaxf(fabsf(dd.x), fabsf(dd.y)))));
        return make_uint4(pack_half2(a.x * vmul, a.y * vmul), pack_half2(bb.x * vmul, bb.y * vmul),
                          pack_half2(cc.x * vmul, cc.y * vmul), pack_half2(dd.x * vmul, dd.y * vmul));
    };
    auto scaled_f16 = [vmul](uint4 v) {    // fp16 values (codes) * vmul; only reached when REDO
        uint32_t* x = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x[i]));
            x[i] = pack_half2(f.x * vmul, f.y * vmul);
        }
        return v;
    };
    float amax = 0.f;
    const int64_t pieces = n_rows * (kHD / 8);
    for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < pieces;
         x += int64_t(gridDim.x) * blockDim.x) {
        const int64_t row = x / (kHD / 8);
        const int col8 = int(x % (kHD / 8));              // 8-element chunk of the row
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < n_conv) {
            if (chunk) {
                v = to_f16(*reinterpret_cast<const uint4*>(chunk + x * 8), amax);
            } else {
                const uint8_t* rowp = nullptr;
                if (paged) {
                    const int64_t slot = row / c.page_tokens;
                    const int page = slot < c.max_pages ? c.page_table[size_t(b) * c.max_pages + slot] : -1;
                    if (page >= 0 && page < c.num_pages)
                        rowp = base + ((size_t(page) * c.n_r + c.rank[g]) * size_t(c.page_tokens) +
                                       size_t(row % c.page_tokens)) * row_bytes;
                    else if (col8 == 0 && !REDO)
                        atomicOr(reinterpret_cast<int*>(c.status), DUO_STATUS_NO_PAGE);
                } else {
                    rowp = base + size_t(row) * row_bytes;
                }
                // codes are at most 448 (E4M3) or 8 (INT4) in magnitude: no range to record
                if (rowp && c.int4) {
                    const uint32_t cc = *reinterpret_cast<const uint32_t*>(rowp + col8 * 4);
                    v = keys ? int4x8_to_bf16(cc) : int4x8_to_f16(cc);
                    if (REDO) v = scaled_f16(v);
                } else if (rowp && c.fp8) {
                    const uint2 cc = *reinterpret_cast<const uint2*>(rowp + col8 * 8);
                    v = keys ? e4m3x8_to_bf16(cc) : e4m3x8_to_f16(cc);
                    if (REDO) v = scaled_f16(v);
                } else if (rowp) {
                    const uint4 w = *reinterpret_cast<const uint4*>(rowp + col8 * 16);
                    v = keys ? w : to_f16(w, amax);             // bf16 keys: a copy
                }
            }
        }
        *reinterpret_cast<uint4*>(dst + x * 8) = v;
    }
    if (!REDO && !keys) {
        uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < int(blockDim.x >> 5); ++w) mx = max(mx, red[w]);
            c.vmax[(size_t(bg) * 2 + blockIdx.z) * kConvCtas + blockIdx.x] = __uint_as_float(mx);
        }
    }
}

// ------------------------------------------------------------------ attention
template <bool F8>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_addr(smem);
    const uint32_t sK = sQ + kTile;                    // kKStages tiles
    const uint32_t sV = sK + kKStages * kTile;         // kVStages tiles

    __shared__ __align__(8) uint64_t bar_q, k_full[kKStages], k_empty[kKStages], v_full[kVStages],
        v_empty[kVStages], s_full[2], s_free[2], p_full, o_done, mma_fin;
    __shared__ uint32_t tmem_base_sh;
    __shared__ float red_max[2][2][kBM];   // [tile parity][column half][row]
    __shared__ float red_l[2][kBM];        // [column half][row] final row sums
    __shared__ int abort_sh;
    volatile int* abort_flag = &abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---------------------------------------------------------------- work item
    const int per_qt = p.B * p.hq;
    const int qt = p.n_qt - 1 - int(blockIdx.x) / (2 * per_qt);   // heaviest query tiles first
    const int part = (int(blockIdx.x) / per_qt) & 1;                // share of a split query tile
    const int rem = int(blockIdx.x) % per_qt;
    const int h = rem % p.hq, b = rem / p.hq;
    const int g = h / p.G;
    const int i0 = qt * kBM;
    const int P = p.prefix[b];
    const bool retr = p.is_r[g] != 0;
    Plan plan;
    plan.init(retr, P < 0 ? 0 : P, i0, p.C, p.S, p.W);
    const bool split = retr && plan.n >= kSplitMin;
    if (part == 1 && !split) return;   // the whole CTA leaves before any set-up
    if (split) plan.take_half(part);

    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar_q), 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(smem_addr(&k_full[s]), 1);
            mbar_init(smem_addr(&k_empty[s]), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(smem_addr(&v_full[s]), 1);
            mbar_init(smem_addr(&v_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&s_full[s]), 1);
            mbar_init(smem_addr(&s_free[s]), 8);
        }
        mbar_init(smem_addr(&p_full), 8);
        mbar_init(smem_addr(&o_done), 1);
        mbar_init(smem_addr(&mma_fin), 1);
        abort_sh = (P < 0) ? 1 : 0;
        if (P < 0) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&tmem_base_sh), kTmemCols);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    const int kv_rank = p.rank[g];

    if (warp == 0 || warp == 2) {
        // ============================================================ TMA producers
        if (lane == 0) {
            const bool is_k = warp == 0;
            const int stages = is_k ? kKStages : kVStages;
            uint64_t* full = is_k ? k_full : v_full;
            uint64_t* empty = is_k ? k_empty : v_empty;
            const uint32_t base = is_k ? sK : sV;
            if (is_k) {
                mbar_arrive_expect_tx(smem_addr(&bar_q), kTile);
                tma_tile(sQ, &p.tm_q, (b * p.hq + h) * p.C + i0, smem_addr(&bar_q));
            }
            int issued = 0;
            for (int j = 0; j < plan.n; ++j) {
                const int st = j % stages;
                if (!timed_wait(smem_addr(&empty[st]), ((j / stages) & 1) ^ 1, p, abort_flag)) break;
                const KeyTile kt = plan.get(j);
                const CUtensorMap* map;
                int row;
                // FP8 or paged caches: cached keys come from their bf16 copies (rows LR / LS)
                const bool copy = !is_k || p.kcopy;
                if (kt.src == kSrcCache) {
                    map = is_k ? (p.kcopy ? &p.tm_kr16 : &p.tm_kr) : &p.tm_vr;
                    row = int((int64_t(b) * p.n_r + kv_rank) * (copy ? int64_t(p.LR) : p.cap) + kt.row0);
                } else if (kt.src == kSrcChunk) {
                    map = is_k ? &p.tm_kc : &p.tm_vc;
                    row = (b * p.n_kv + g) * p.C + kt.row0;
                } else {
                    map = is_k ? (p.kcopy ? &p.tm_ks16 : &p.tm_ks) : &p.tm_vs;
                    row = (b * p.n_s + kv_rank) * (copy ? p.LS : p.S + p.W) + (kt.src == kSrcWindow ? p.S : 0) +
                          kt.row0;
                }
                const uint32_t bar = smem_addr(&full[st]);
                mbar_arrive_expect_tx(bar, kTile);
                tma_tile(base + st * kTile, map, row, bar);
                ++issued;
            }
            // do not leave while copies may still land in this CTA's shared memory
            if (is_k) mbar_wait(smem_addr(&bar_q), 0, p.timeout_ns);
            for (int k = 0; k < stages && k < issued; ++k) {
                const int j = issued - 1 - k;
                mbar_wait(smem_addr(&full[j % stages]), (j / stages) & 1, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            bool ok = timed_wait(smem_addr(&bar_q), 0, p, abort_flag);
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int ks = j % kKStages, sb = j & 1;
                if (!timed_wait(smem_addr(&k_full[ks]), (j / kKStages) & 1, p, abort_flag)) return false;
                if (!timed_wait(smem_addr(&s_free[sb]), ((j >> 1) & 1) ^ 1, p, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sk = sK + ks * kTile;
#pragma unroll
                for (int k = 0; k < kHD / 16; ++k) {
                    const uint32_t off = (k >> 2) * kSlab + (k & 3) * 32;
                    umma_f16(tmem + (sb ? kTmemS1 : kTmemS0), smem_desc(sQ + off, 16, 1024),
                             smem_desc(sk + off, 16, 1024), kIdescQK, k > 0);
                }
                umma_commit(smem_addr(&s_full[sb]));
                umma_commit(smem_addr(&k_empty[ks]));
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < plan.n; ++j) {
                if (j + 1 < plan.n && !issue_s(j + 1)) { ok = false; break; }
                const int vs = j % kVStages;
                if (!timed_wait(smem_addr(&p_full), j & 1, p, abort_flag)) { ok = false; break; }
                if (!timed_wait(smem_addr(&v_full[vs]), (j / kVStages) & 1, p, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sv = sV + vs * kTile;
#pragma unroll
                for (int k = 0; k < kBN / 16; ++k) {
                    // A = P_j columns [8k, 8k+8) of the TMEM P region (16 keys, fp16 pairs)
                    umma_f16_ts(tmem + kTmemO, tmem + kTmemP + k * 8, smem_desc(sv + k * 2048, kSlab, 1024),
                                kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(smem_addr(&v_empty[vs]));
                umma_commit(smem_addr(&o_done));
            }
            // all MMAs issued by this thread have completed before TMEM is freed
            umma_commit(smem_addr(&mma_fin));
            mbar_wait(smem_addr(&mma_fin), 0, p.timeout_ns);
        }
    } else {
        // ============================================================ softmax
        // 8 warps, two per scheduler: warp w owns the TMEM lane quarter w % 4
        // (32 query rows) and the column half hf of every S tile (64 keys), of
        // the P tile (32 TMEM columns of fp16 pairs) and of O (64 dims).  The
        // two halves of a row agree on the tile maximum once per tile.
        const int wq = warp & 3;
        const int hf = (warp - kSoftmaxWarp0) >> 2;
        const int r = wq * 32 + lane;            // query row within the tile
        const int i = i0 + r;                    // chunk row
        const int tpos = plan.P + i;             // absolute position
        const int cb = hf * 64;                  // first key column (and O dim) of this half
        const uint32_t lane_off = uint32_t(wq * 32) << 16;
        float m = kNegBig, l = 0.f;
        // FP8 caches: a cached key's tile holds codes, so its scores take the
        // key scale and its probabilities the value scale (the chunk's own
        // keys and values are exact)
        const float ksc = F8 ? p.k_scale[g] : 1.f;
        const float lvs = F8 ? __log2f(p.v_scale[g]) : 0.f, ivs = F8 ? 1.f / p.v_scale[g] : 1.f;
        bool ok = true;
        for (int j = 0; j < plan.n; ++j) {
            const int st = j & 1;
            const bool got = warp_wait(smem_addr(&s_full[st]), (j >> 1) & 1, p, abort_flag);
            float s[64];   // raw scores of this half row, then probabilities
            float mx = -CUDART_INF_F;
            if (got) {
                tc_fence_after();
                uint32_t* u = reinterpret_cast<uint32_t*>(s);
                const uint32_t ta = tmem + lane_off + (st ? kTmemS1 : kTmemS0) + cb;
                tmem_ld32p(ta, u);
                tmem_ld32p(ta + 32, u + 32);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&s_free[st]));

                const KeyTile kt = plan.get(j);
                if (kt.masked) {
                    // Every mask is: c <= hi and (aL <= c <= aH or bL <= c <= bH),
                    // with c the key's column in the tile.
                    int hi = kt.nvalid - 1, aL = 0, aH = kBN, bL = kBN, bH = -1;
                    if (kt.src == kSrcChunk) {
                        // causal (key j <= row i); streaming heads also need j in
                        // the window (j >= i-W+1) or a sink (P + j < S)
                        hi = min(hi, i - kt.row0);
                        if (!plan.retr) {
                            aL = i - p.W + 1 - kt.row0;
                            bL = 0;
                            bH = p.S - plan.P - kt.row0 - 1;
                        }
                    } else if (kt.src == kSrcWindow) {
                        // Window slot k holds the position the append rule gave it:
                        // the ring's newest slot kn = (P-1-S) mod W (nw-1 before it
                        // wraps) holds P-1; positions fall by one per slot going
                        // back and wrap once.  Positions >= t-W+1: two intervals.
                        const bool full = plan.P - p.S >= p.W;
                        const int kn = full ? (plan.P - 1 - p.S) % p.W : plan.nw_rows - 1;
                        aL = (tpos - p.W + 1) - (plan.P - 1) + kn - kt.row0;
                        aH = kn - kt.row0;
                        bL = max(aL + p.W, aH + 1);
                        bH = full ? p.W - 1 - kt.row0 : -1;
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int o = cb + q * 32;
                        const uint32_t keep = (range_bits(aL - o, aH - o) | range_bits(bL - o, bH - o)) &
                                              range_bits(0, hi - o);
#pragma unroll
                        for (int c = 0; c < 32; ++c) s[q * 32 + c] = (keep >> c) & 1u ? s[q * 32 + c] : -CUDART_INF_F;
                    }
                }
                float t8[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) t8[x] = s[x];
#pragma unroll
                for (int c = 8; c < 64; c += 2) t8[(c >> 1) & 7] = fmax3(t8[(c >> 1) & 7], s[c], s[c + 1]);
                mx = fmax3(fmax3(t8[0], t8[1], t8[2]), fmax3(t8[3], t8[4], t8[5]), fmaxf(t8[6], t8[7]));
            }
            // exchange the half-row maxima with the warp that holds the other
            // half of these rows; the barrier also agrees on aborting
            red_max[st][hf][r] = mx;
            if (pair_barrier_any(wq, !got || *abort_flag)) { ok = false; break; }
            mx = fmaxf(red_max[st][0][r], red_max[st][1][r]);

            const bool cached = F8 && plan.cached(j);   // tiles of the cache come first
            const float fs = cached ? p.scale_log2 * ksc : p.scale_log2;   // score factor of this tile
            const float mt = mx * fs;                    // factor > 0 keeps the order
            const bool grow = mt > m + kRescaleThreshold;
            const float m_new = grow ? mt : m;
            const float alpha = fast_exp2(m - m_new);   // 1 when the max is kept
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            uint32_t ph[32];   // probabilities as packed fp16 pairs
            const float2 sc2 = make_float2(fs, fs);
            // cached tiles of an FP8 cache: P times the value scale, via the exponent
            const float off = cached ? lvs - m_new : -m_new;
            const float2 nm2 = make_float2(off, off);
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const float2 x = ffma2(make_float2(s[c], s[c + 1]), sc2, nm2);
                const float2 e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], e);
                ph[c / 2] = pack_half2(e.x, e.y);
            }
            const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
            const float2 at = fadd2(a01, a23);
            l = l * alpha + (at.x + at.y) * (cached ? ivs : 1.f);
            m = m_new;
            // P_j overwrites P_{j-1} in TMEM, and a rescale touches O: both
            // need PV_{j-1} to have completed.
            if (j > 0) {
                if (!warp_wait(smem_addr(&o_done), (j - 1) & 1, p, abort_flag)) continue;   // next barrier exits
                tc_fence_after();
            }
            tmem_st32(tmem + lane_off + kTmemP + hf * 32, *reinterpret_cast<const uint32_t(*)[32]>(ph));
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t u[32];
                    const uint32_t ta = tmem + lane_off + kTmemO + cb + c * 32;
                    tmem_ld32(ta, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(__uint_as_float(u[x]) * alpha);
                    tmem_st32(ta, u);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&p_full));
        }
        // the pairs may have left at different tiles: agree before the epilogue
        ok = !softmax_barrier_any(!ok);
        // epilogue: O / (l of both halves)
        if (ok) {
            const bool got = warp_wait(smem_addr(&o_done), (plan.n - 1) & 1, p, abort_flag);
            red_l[hf][r] = l;
            if (!softmax_barrier_any(!got)) {
                tc_fence_after();
                const float lt = red_l[0][r] + red_l[1][r];
                // the fp16 value copies hold v * 2^-E (E = 0 unless some |v| >= 2^15)
                const float vpow = __uint_as_float(uint32_t(127 + p.vexp[b * p.n_kv + g]) << 23);
                const float inv = lt > 0.f ? vpow / lt : 0.f;
                // a split query tile leaves its normalised half and the row's
                // log2-sum-exp for merge_parts_kernel
                const size_t row = (size_t(split ? part * p.B + b : b) * p.hq + h) * p.C + i;
                float* dst = (split ? p.part_o : p.out) + row * kHD + cb;
                if (split && hf == 0 && i < p.C) p.part_lse[row] = lt > 0.f ? m + __log2f(lt) : -CUDART_INF_F;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tmem + lane_off + kTmemO + cb + c * 32, u);
                    tmem_wait_ld();
                    if (i < p.C) {
#pragma unroll
                        for (int x = 0; x < 32; x += 4)
                            *reinterpret_cast<float4*>(dst + c * 32 + x) =
                                make_float4(__uint_as_float(u[x]) * inv, __uint_as_float(u[x + 1]) * inv,
                                            __uint_as_float(u[x + 2]) * inv, __uint_as_float(u[x + 3]) * inv);
                    }
                }
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

// ------------------------------------------------------------------ split merge
struct MergeParams {
    const float* part_o;
    const float* part_lse;
    float* out;
    const int32_t* prefix;
    int B, hq, G, C, S, W;
    uint8_t is_r[kMaxKvHeads];
};

// One warp per query row of a split query tile: out = sum_p w_p o_p / sum_p w_p
// with w_p = 2^(lse_p - max lse), the log-sum-exp combination of two
// attentions over disjoint key sets.  Rows of unsplit tiles were written by
// the attention kernel and are left alone (the same split rule decides).
__global__ void __launch_bounds__(256) merge_parts_kernel(const __grid_constant__ MergeParams a) {
    const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;   // (b, h, i)
    const int lane = threadIdx.x & 31;
    if (row >= int64_t(a.B) * a.hq * a.C) return;
    const int i = int(row % a.C);
    const int h = int((row / a.C) % a.hq), b = int(row / (int64_t(a.C) * a.hq));
    const bool retr = a.is_r[h / a.G] != 0;
    if (!retr) return;
    const int P = a.prefix[b];
    Plan plan;
    plan.init(true, P < 0 ? 0 : P, i / kBM * kBM, a.C, a.S, a.W);
    if (plan.n < kSplitMin || P < 0) return;
    const size_t r0 = size_t(row), r1 = size_t(a.B) * a.hq * a.C + r0;
    const float l0 = a.part_lse[r0], l1 = a.part_lse[r1];
    const float mx = fmaxf(l0, l1);
    const float w0 = exp2f(l0 - mx), w1 = exp2f(l1 - mx);
    const float inv = 1.f / (w0 + w1);
    const float4 o0 = reinterpret_cast<const float4*>(a.part_o + r0 * kHD)[lane];
    const float4 o1 = reinterpret_cast<const float4*>(a.part_o + r1 * kHD)[lane];
    reinterpret_cast<float4*>(a.out + r0 * kHD)[lane] =
        make_float4((w0 * o0.x + w1 * o1.x) * inv, (w0 * o0.y + w1 * o1.y) * inv, (w0 * o0.z + w1 * o1.z) * inv,
                    (w0 * o0.w + w1 * o1.w) * inv);
}

// ------------------------------------------------------------------ host side
// 2-D map of 16-bit elements over `rows` rows of 128; box 64 x 128 rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, CUtensorMapDataType type) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {uint64_t(kHD), rows < 1 ? 1 : rows};
    cuuint64_t strides[1] = {uint64_t(kHD) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Rows per head of the fp16 value copies (whole tiles plus one spare tile).
int rows_r(int64_t cap) { return int((cap + kBN - 1) / kBN * kBN + kBN); }
int rows_s(int S, int W) { return (S + W + kBN - 1) / kBN * kBN + kBN; }

}  // namespace

size_t prefill_smem_bytes(int S, int W) {
    (void)S;
    (void)W;
    return (1 + kKStages + kVStages) * size_t(kTile) + 1024;
}

size_t prefill_workspace_bytes(int B, int hq, int n_kv, int n_r, int n_s, int64_t cap, int S, int W, int C,
                               bool key_copies) {
    const size_t row = size_t(kHD) * 2;
    const size_t cached = align256(size_t(B) * n_r * rows_r(cap) * row) + align256(size_t(B) * n_s * rows_s(S, W) * row);
    const size_t parts = align256(2 * size_t(B) * hq * C * kHD * 4) + align256(2 * size_t(B) * hq * C * 4);
    const size_t range = align256(size_t(B) * n_kv * 2 * kConvCtas * 4) + align256(size_t(B) * n_kv * 4);
    // V copies, chunk V, key copies, split partials, value ranges
    return cached + align256(size_t(B) * n_kv * C * row) + (key_copies ? cached : 0) + parts + range;
}

int launch_prefill(const PrefillLaunch& a, cudaStream_t s) {
    const int LR = rows_r(a.cap), LS = rows_s(a.S, a.W);
    const size_t row = size_t(kHD) * 2;
    char* ws = static_cast<char*>(a.workspace);
    uint16_t* v16r = reinterpret_cast<uint16_t*>(ws);
    uint16_t* v16s = reinterpret_cast<uint16_t*>(ws + align256(size_t(a.B) * a.n_r * LR * row));
    uint16_t* v16c = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(v16s) +
                                                 align256(size_t(a.B) * a.n_s * LS * row));
    uint16_t* k16r = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(v16c) +
                                                 align256(size_t(a.B) * a.n_kv * a.C * row));
    uint16_t* k16s = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(k16r) +
                                                 align256(size_t(a.B) * a.n_r * LR * row));
    // split partials after the key copies (whose space exists only with key copies)
    const bool kc = a.fp8 || a.page_tokens > 0;
    char* parts = kc ? reinterpret_cast<char*>(k16s) + align256(size_t(a.B) * a.n_s * LS * row)
                     : reinterpret_cast<char*>(k16r);
    float* part_o = reinterpret_cast<float*>(parts);
    float* part_lse = reinterpret_cast<float*>(parts + align256(2 * size_t(a.B) * a.hq * a.C * kHD * 4));
    char* range = reinterpret_cast<char*>(part_lse) + align256(2 * size_t(a.B) * a.hq * a.C * 4);
    float* vmax = reinterpret_cast<float*>(range);
    int32_t* vexp = reinterpret_cast<int32_t*>(range + align256(size_t(a.B) * a.n_kv * 2 * kConvCtas * 4));

    PrefillParams p;
    memset(&p, 0, sizeof p);
    const int SW = a.S + a.W;
    const bool kcopy = a.fp8 || a.page_tokens > 0;
    const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&p.tm_q, a.q, uint64_t(a.B) * a.hq * a.C, BF) ||
        !make_map(&p.tm_kc, a.k_chunk, uint64_t(a.B) * a.n_kv * a.C, BF) ||
        (!kcopy && !make_map(&p.tm_kr, a.kr, uint64_t(a.B) * a.n_r * a.cap, BF)) ||
        (!kcopy && !make_map(&p.tm_ks, a.ks, uint64_t(a.B) * a.n_s * SW, BF)) ||
        (kcopy && !make_map(&p.tm_kr16, k16r, uint64_t(a.B) * a.n_r * LR, BF)) ||
        (kcopy && !make_map(&p.tm_ks16, k16s, uint64_t(a.B) * a.n_s * LS, BF)) ||
        !make_map(&p.tm_vc, v16c, uint64_t(a.B) * a.n_kv * a.C, F16) ||
        !make_map(&p.tm_vr, v16r, uint64_t(a.B) * a.n_r * LR, F16) ||
        !make_map(&p.tm_vs, v16s, uint64_t(a.B) * a.n_s * LS, F16))
        return DUO_ERR_CUDA;
    p.prefix = a.prefix;
    p.out = a.out;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.status = a.status;
    p.vexp = vexp;
    p.cap = a.cap;
    p.B = a.B; p.hq = a.hq; p.n_kv = a.n_kv; p.G = a.hq / a.n_kv; p.C = a.C;
    p.n_qt = (a.C + kBM - 1) / kBM;
    p.S = a.S; p.W = a.W; p.n_r = a.n_r; p.n_s = a.n_s; p.LR = LR; p.LS = LS;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.timeout_ns = a.timeout_ns;
    memcpy(p.rank, a.rank, sizeof p.rank);
    memcpy(p.is_r, a.is_r, sizeof p.is_r);
    p.fp8 = a.fp8;
    p.kcopy = a.fp8 || a.page_tokens > 0;
    memcpy(p.k_scale, a.k_scale, sizeof p.k_scale);
    memcpy(p.v_scale, a.v_scale, sizeof p.v_scale);

    ConvertParams c;
    memset(&c, 0, sizeof c);
    c.vr = static_cast<const uint16_t*>(a.vr);
    c.vs = static_cast<const uint16_t*>(a.vs);
    c.vc = static_cast<const uint16_t*>(a.v_chunk);
    c.v16r = v16r; c.v16s = v16s; c.v16c = v16c;
    c.prefix = a.prefix;
    c.cap = a.cap;
    c.B = a.B; c.n_kv = a.n_kv; c.n_r = a.n_r; c.n_s = a.n_s; c.S = a.S; c.W = a.W; c.C = a.C;
    c.LR = LR; c.LS = LS;
    memcpy(c.rank, a.rank, sizeof c.rank);
    memcpy(c.is_r, a.is_r, sizeof c.is_r);
    c.fp8 = a.fp8;
    c.int4 = a.int4;
    c.kr = a.kr;
    c.ks = a.ks;
    c.k16r = k16r;
    c.k16s = k16s;
    c.page_tokens = a.page_tokens;
    c.max_pages = a.max_pages;
    c.num_pages = a.num_pages;
    c.page_table = a.page_table;
    c.status = a.status;
    c.vmax = vmax;
    c.vexp = vexp;
    if (int64_t(a.B) * a.n_kv > 65535) return DUO_ERR_UNSUPPORTED;
    convert_v_kernel<false><<<dim3(kConvCtas, unsigned(a.B * a.n_kv), p.kcopy ? 3 : 2), 256, 0, s>>>(c);
    if (cudaGetLastError() != cudaSuccess) return DUO_ERR_CUDA;
    // value exponents; a head's values are converted again only when some |v| >= 2^15
    convert_v_kernel<true><<<dim3(kConvCtas, unsigned(a.B * a.n_kv), 2), 256, 0, s>>>(c);
    if (cudaGetLastError() != cudaSuccess) return DUO_ERR_CUDA;

    const size_t smem = prefill_smem_bytes(a.S, a.W);
    const int64_t grid = 2 * int64_t(p.n_qt) * a.B * a.hq;   // two shares per query tile (unsplit: one leaves)
    if (grid > 0x7fffffff) return DUO_ERR_UNSUPPORTED;
    if (a.fp8) {
        if (cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
            cudaSuccess)
            return DUO_ERR_CUDA;
        prefill_kernel<true><<<unsigned(grid), kThreads, smem, s>>>(p);
    } else {
        if (cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
            cudaSuccess)
            return DUO_ERR_CUDA;
        prefill_kernel<false><<<unsigned(grid), kThreads, smem, s>>>(p);
    }
    if (cudaGetLastError() != cudaSuccess) return DUO_ERR_CUDA;
    MergeParams mp;
    memset(&mp, 0, sizeof mp);
    mp.part_o = part_o;
    mp.part_lse = part_lse;
    mp.out = a.out;
    mp.prefix = a.prefix;
    mp.B = a.B; mp.hq = a.hq; mp.G = a.hq / a.n_kv; mp.C = a.C; mp.S = a.S; mp.W = a.W;
    memcpy(mp.is_r, a.is_r, sizeof mp.is_r);
    const int64_t warps = int64_t(a.B) * a.hq * a.C;
    merge_parts_kernel<<<unsigned((warps + 7) / 8), 256, 0, s>>>(mp);
    return cudaGetLastError() == cudaSuccess ? DUO_OK : DUO_ERR_CUDA;
}

}  // namespace duo
