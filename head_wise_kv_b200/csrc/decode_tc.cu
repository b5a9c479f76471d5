// Mixed-head decode attention on the 5th-generation tensor cores (d = 128).
//
// Same work as decode.cu (DuoAttention guide, section 2: retrieval KV heads
// read their full cache, streaming KV heads their sink + window ring) and the
// same split-K partition (decode_sched.cuh), but the two contractions of a
// key tile run as tcgen05 MMAs instead of CUDA-core FMAs:
//
//   S^T = K_tile Q^T      M = 128 keys, N = 16, K = d = 128    (bf16 x bf16)
//   O^T += V_tile^T P^T   M = d = 128,  N = 16, K = 128 keys   (bf16 x bf16)
//
// N = 16 holds the G query heads that share the KV head ("Multi-Query and
// Grouped-Query Attention": one K/V tile feeds all of them).  For the second
// product each probability is split into two bf16 terms, P = P_hi + P_lo
// (columns h and G + h of P^T), so P keeps ~16 significant bits although the
// MMA takes it in bf16; the two output columns are added in the epilogue.
// Decode at G <= 8 is bound by HBM, not by the tensor cores (they run at a
// small fraction of their peak here): moving the dot products off the
// CUDA cores is what lets the kernel stream K/V at the memory's rate, since
// the FMA version issues ~40 warp instructions per 512-byte token.
//
// One persistent CTA per SM, 12 warps:
//   warp 7     stages each piece's q rows into shared memory (K-major,
//              128-byte swizzle), up to two pieces ahead
//   warp 0     one lane issues the TMA loads of the K tiles (3-D tensor
//              maps over [head][row][dim], rows past the cache read as
//              zeros) into a 3-stage ring, L2 evict-first
//   warp 6     the same for the V tiles, into their own ring: a K buffer is
//              released as soon as its S product has completed, a V buffer
//              once its PV product has, so neither waits on the other
//   warp 1     allocates TMEM (S^T double-buffered, O^T) and, one lane,
//              issues the MMAs from an event loop: S_j as soon as K_j and an
//              S buffer are there, PV_j as soon as P_j is, so the softmax of
//              tile j overlaps the products of its neighbours
//   warps 2-5  softmax: thread = TMEM lane = key row of the tile; running max
//              per head in the log2 domain with lazy rescaling (O^T rescaled
//              in TMEM only when a tile's max exceeds it by more than 2^8);
//              P^T written to shared memory; at the end of a piece, the row
//              sums and the max go to the epilogue through shared memory
//   warps 8-11 epilogue (thread = output dim): O^T is double-buffered in TMEM
//              by piece parity, so a piece's tail (its last V tile and PV)
//              never holds up the softmax of the next.  A piece that is a
//              whole segment is written to `out`; otherwise the partial
//              (o, max, sum) goes to the workspace and the last CTA to finish
//              a part of that segment (a per-segment arrival counter, reset
//              by that CTA) merges the parts by log-sum-exp, so no second
//              kernel is launched.
//   warp 7 also writes the output of segments without keys and sets the
//              length status bits.
//   INT4 caches add warps 12-19 (640 threads): the producers bring the packed
//              codes into a staging ring and these warps expand them to E4M3
//              tiles (12-15 K, 16-19 V) for the FP8 arithmetic.
//
// Every mbarrier wait is bounded; on a timeout the CTA sets
// DUO_STATUS_WAIT_TIMEOUT, stops, waits (bounded) for its copies and MMAs in
// flight, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>
#include <string.h>

#include "decode_sched.cuh"
#include "duo_internal.cuh"
#include "tcgen05.cuh"

#include <cuda_fp16.h>

namespace duo {

namespace {

constexpr int kD = 128;                       // head dim
constexpr int kThreads = 384;
constexpr int kSoftWarp0 = 2;              // softmax warps 2-5
constexpr int kVWarp = 6;
constexpr int kQWarp = 7;
constexpr int kEpiWarp0 = 8;               // epilogue warps 8-11
constexpr uint32_t kSlab = 128 * 128;         // 128 rows x 64 bf16: one dim-half of a bf16 tile
constexpr uint32_t kTileBytes = 32768;        // one K or V tile: 128 bf16 rows or 256 FP8 rows
// INT4 caches: the producers bring 256-row tiles of packed codes (64 bytes a
// row) into a staging ring; eight converter warps (12-15 for K, 16-19 for V)
// expand them to E4M3 in the FP8 tile layout, and the rest of the kernel is
// the FP8 one.
constexpr int kConvWarp0 = 12;
constexpr int kThreadsI4 = 640;
constexpr uint32_t kTile4Bytes = 16384;       // one K or V tile of 256 INT4 rows
constexpr float kNegBig = -1.0e30f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units: probabilities stay <= 2^8
// Partition weight of a segment start in 16-token blocks: starting a piece
// (its first tile's latency, the hand-over of the last one) costs about as
// much time as streaming this many blocks.  Measured on the 128K GQA
// workload: 0 -> 193 us, 8 -> 188, 16 -> 183, 24..48 -> 181.5-183, 64 -> 183;
// with the current kernel on one box, 24 -> 182.3-183.6, 32 -> 183.8-184.6,
// 40 -> 184.1-184.3 (layer-step).
#ifndef DUO_DECODE_SEG_WEIGHT
#define DUO_DECODE_SEG_WEIGHT 24
#endif
constexpr int kSegWeight = DUO_DECODE_SEG_WEIGHT;
// FP8 streams twice the keys per byte, so a piece start costs more blocks.
// Measured on the 128K GQA workload (FP8 cache): 32 -> 106.6 us, 48 -> 106.0,
// 64 -> 107.0, 96 -> 109.0, 128 -> 110.2.
#ifndef DUO_DECODE_SEG_WEIGHT_FP8
#define DUO_DECODE_SEG_WEIGHT_FP8 48
#endif
constexpr int kSegWeightF8 = DUO_DECODE_SEG_WEIGHT_FP8;

// Shapes of the two element types.
//   bf16: 128-key tiles; S^T one column per head (q as is); P as hi + lo
//         bf16 terms, so O^T holds two columns per head.
//   FP8:  256-key tiles (two 128-key halves of S^T); q as a sum of four
//         E4M3 terms (~16 significant bits), P rounded to fp16 (11 bits, as
//         the prefill's P) and split into three E4M3 terms, columns
//         term * G + h; the products run as kind::f8f6f4 straight on the
//         cached codes.
template <int G, bool F8>
struct Tr {
    static constexpr int T = F8 ? 256 : 128;                       // keys per tile
    static constexpr int HALVES = T / 128;                         // 128-key blocks of S^T
    static constexpr int QT = F8 ? 4 : 1;                          // q terms
    static constexpr int PT = F8 ? 3 : 2;                          // P terms
    static constexpr int N = F8 ? ((4 * G + 15) / 16) * 16 : 16;   // MMA N (QT * G >= PT * G columns)
    // O^T columns read back: PT * G rounded up to a power of two (the
    // columns past PT * G hold zeros: their P^T rows are never written)
    static constexpr int OL = PT * G <= 2 ? 2 : PT * G <= 4 ? 4 : PT * G <= 8 ? 8 : PT * G <= 16 ? 16 : 32;
    static constexpr uint32_t SB = HALVES * N < 32 ? 32 : HALVES * N;   // TMEM columns of one S buffer
    static constexpr uint32_t OB = N < 32 ? 32 : N;                     // of one O buffer
    static constexpr uint32_t S0 = 0, S1 = SB, O0 = 2 * SB;
    static constexpr uint32_t RAW = 2 * SB + 2 * OB;
    static constexpr uint32_t COLS = RAW <= 32 ? 32 : RAW <= 64 ? 64 : RAW <= 128 ? 128 : RAW <= 256 ? 256 : 512;
    static constexpr uint32_t QB = 4096;                           // bytes of one q operand
    static constexpr uint32_t PB = F8 ? N * 256 : 4096;            // bytes of one P^T operand
    static constexpr uint32_t PHALF = F8 ? N * 128 : 2048;         // P^T bytes per K-half (128 / 64 keys)
    // FP8: P enters the MMA as P' = 2^7 P.  When a tile's max exceeds the
    // running max m by more than 1.75, m moves to that max + 2 (headroom, so
    // that the slowly growing max of a long sequence rarely forces another
    // rescale); hence P' <= 2^8.75 < 448 and the E4M3 grid floor (2^-10
    // after four terms) stays >= 2^-15 below the largest P'.  bf16 terms have
    // no such floor: threshold 2^8, no offset, no headroom.
    static constexpr float THRESH = F8 ? 1.75f : kRescaleThreshold;   // log2 units
    static constexpr float HEAD = F8 ? 2.0f : 0.0f;
    static constexpr float POFF = F8 ? 7.0f : 0.0f;                    // log2 of the P offset
    static constexpr uint32_t IQK = idesc_f16(128, N, !F8, false, false);   // A = K (K-major), B = q
    static constexpr uint32_t IPV = idesc_f16(kD, N, !F8, true, false);     // A = V^T (MN-major), B = P^T
    static_assert(QT * G <= N && PT * G <= N, "terms must fit the MMA N");
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Eight INT4 codes (two's complement nibbles, element i in bits 4i..4i+3)
// -> their eight values as E4M3 bytes (exact: every integer in [-8, 7] is an
// E4M3 value), four per byte permute.  A permute selector with bit 3 set
// yields the sign of the chosen byte replicated, so with the nibble itself
// as the selector:
//   table E4M3(0..7) (signs 0):            the code of c >= 0, else 0x00;
//   nibble xor 8, table E4M3(-8..-1):      the code of c < 0, else 0xFF;
//   bytes whose bit 7 is the sign of each element, replicated: 0xFF for c < 0;
// and code = first | (second & third).  The right shift by 16 runs as a
// multiply-high and the left shift as a multiply, off the integer pipe.
__device__ __forceinline__ uint2 int4x8_to_e4m3(uint32_t w) {
    constexpr uint32_t kPos0 = 0x44403800u, kPos1 = 0x4E4C4A48u;   // E4M3 of 0, 1, ..., 7
    constexpr uint32_t kNeg0 = 0xCACCCED0u, kNeg1 = 0xB8C0C4C8u;   // E4M3 of -8, -7, ..., -1
    const uint32_t hi = __umulhi(w, 0x10000u);                      // w >> 16: elements 4..7
    const uint32_t w4 = w * 16u;                                    // bit 8k+7: sign of element 2k
    const uint32_t wx = w ^ 0x88888888u, hx = hi ^ 0x8888u;
    uint2 r;
    r.x = prmt(kPos0, kPos1, w) | (prmt(kNeg0, kNeg1, wx) & prmt(w4, w, 0xD9C8u));
    r.y = prmt(kPos0, kPos1, hi) | (prmt(kNeg0, kNeg1, hx) & prmt(w4, w, 0xFBEAu));
    return r;
}

// Two values -> two E4M3 codes (round to nearest even, saturating); the
// first operand lands in the upper byte.
__device__ __forceinline__ uint16_t e4m3x2(float hi, float lo) {
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(hi), "f"(lo));
    return c;
}

// Two E4M3 codes -> their values (exact): .x from the low byte.
__device__ __forceinline__ float2 e4m3x2_value(uint16_t c) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return make_float2(__half2float(__ushort_as_half(uint16_t(h2 & 0xffff))),
                       __half2float(__ushort_as_half(uint16_t(h2 >> 16))));
}

// D (TMEM) (+)= A (smem, E4M3) * B (smem, E4M3), fp32 accumulate.
__device__ __forceinline__ void umma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void st_shared_u8(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Byte offset of 16-byte chunk c (0..15, along the 128 dims or keys) of row
// r (0..15) in a 16-row K-major operand with 128-byte swizzle: two 2 KB
// halves (dims / keys 0-63 and 64-127), each two 8-row groups of 1 KB.
__device__ __forceinline__ uint32_t small_off(int r, int c) {
    return uint32_t((c >> 3) * 2048 + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int T>
__device__ __forceinline__ int tiles_of(const Piece& pc) { return int((pc.tok1 - pc.tok0 + T - 1) / T); }

// Position in the CTA's sequence of tiles (T keys each): piece `pi` (pc),
// tile t of its nt; gb is where the search for the next piece starts.
template <int T, int BLK>
struct TileCursor {
    Piece pc;
    int pi, t, nt;
    bool valid;

    int64_t gb;

    __device__ void start(const DecodeParams& p, const int32_t* bpre, int64_t gb_begin, int64_t gb_end) {
        pi = 0;
        t = 0;
        gb = gb_begin;
        valid = next_piece<BLK>(p, bpre, gb, gb_end, pc);
        if (valid) nt = tiles_of<T>(pc);
    }
    __device__ void advance(const DecodeParams& p, const int32_t* bpre, int64_t gb_end) {
        if (++t < nt) return;
        t = 0;
        ++pi;
        valid = next_piece<BLK>(p, bpre, gb, gb_end, pc);
        if (valid) nt = tiles_of<T>(pc);
    }
};

__device__ __forceinline__ bool timed_wait(uint32_t bar, uint32_t parity, const DecodeParams& p,
                                           volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, p.timeout_ns)) return true;
    set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Lane 0 waits (bounded) for the warp; the warp takes its result.
__device__ __forceinline__ bool warp_wait_lead(uint32_t bar, uint32_t parity, const DecodeParams& p,
                                               volatile int* abort_flag) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = timed_wait(bar, parity, p, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// The same with a fast path for a phase that has completed already (each
// lane probes it): for waits that usually find their data there.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DecodeParams& p,
                                          volatile int* abort_flag) {
    if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
    return warp_wait_lead(bar, parity, p, abort_flag);
}

// TMA coordinates of the tile that starts t keys into a piece: (row, head)
// of the [heads][rows] maps; paged retrieval caches address the pool
// [pages * n_r][page_tokens] through the tile's page (a missing page sets
// DUO_STATUS_NO_PAGE and reads as zeros: its coordinate is outside the map).
// A paged tile must start on a page boundary (T divides page_tokens and
// the pieces start on tile boundaries; a row range must start on a
// multiple of 256, else DUO_STATUS_BAD_LENGTH).
template <int T, bool PAGED>
__device__ __forceinline__ void tile_coords(const DecodeParams& p, const Piece& pc, int64_t t, int page, int& y,
                                            int& z) {
    if (PAGED && pc.retr) {
        const uint32_t row = uint32_t(pc.row0 + t);   // < capacity < 2^31: 32-bit arithmetic
        y = int(row % uint32_t(p.page_tokens));
        if (y + T > p.page_tokens) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        if (page < 0 || page >= p.num_pages) {
            set_status(p.status, DUO_STATUS_NO_PAGE);
            z = -1;
        } else {
            z = page * p.n_r + pc.rank;
        }
    } else {
        y = int(pc.row0 + t);
        z = pc.b * (pc.retr ? p.n_r : p.n_s) + pc.rank;
    }
}

// Lane 0 polls for the warp, napping between polls: for waits that span a
// whole piece, so that the poll takes no issue slots from the warps on the
// critical path.
__device__ __forceinline__ bool warp_wait_lazy(uint32_t bar, uint32_t parity, const DecodeParams& p,
                                               volatile int* abort_flag) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) {
        const unsigned long long t0 = global_ns();
        while (!mbar_test_wait(bar, parity)) {
            if (*abort_flag) {
                ok = 0;
                break;
            }
            if (global_ns() - t0 > p.timeout_ns) {
                set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
                *abort_flag = 1;
                ok = 0;
                break;
            }
            __nanosleep(256);
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// CTAs that hold a piece of the segment starting at global block seg_gb
// (seg_nb >= 1 blocks): [c0, c1], of which `n` have a non-empty range.
struct Owners {
    int c0, c1, n;
};

__device__ __forceinline__ Owners owners_of(int64_t seg_gb, int seg_nb, int64_t total, int64_t ctas) {
    Owners o;
    o.c0 = cta_owner(seg_gb, total, ctas);
    o.c1 = cta_owner(seg_gb + seg_nb - 1, total, ctas);
    if (total >= ctas) {
        o.n = o.c1 - o.c0 + 1;   // no CTA range is empty
    } else {
        o.n = 0;
        for (int c = o.c0; c <= o.c1; ++c) o.n += cta_start(c + 1, total, ctas) > cta_start(c, total, ctas);
    }
    return o;
}

// Barrier over 128 threads (named barrier `id`) that ORs a flag across
// them, so that every participating warp takes the same exit decision.
template <int id>
__device__ __forceinline__ bool barrier_any(bool flag) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(out)
        : "r"(uint32_t(flag)), "n"(id)
        : "memory");
    return out != 0;
}
constexpr int kBarSoftmax = 1, kBarEpilogue = 2;

__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

template <int G, bool F8, bool PAGED, bool I4>
__global__ void __launch_bounds__(I4 ? kThreadsI4 : kThreads, 1)
    decode_tc_kernel(const __grid_constant__ DecodeParams p) {
    using C = Tr<G, F8>;
    static_assert(!I4 || F8, "INT4 caches run the FP8 arithmetic");
    constexpr int NT = I4 ? kThreadsI4 : kThreads;
    constexpr int BLK = PAGED ? C::T : 16;   // partition block (tokens)
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nst = p.stages;
    const int ns4 = I4 ? p.stages4 : 0;
    const uint32_t sK = smem_addr(smem);                  // nst K tiles
    const uint32_t sV = sK + nst * kTileBytes;            // nst V tiles
    const uint32_t s4K = sV + nst * kTileBytes;           // INT4: ns4 staged K tiles of codes
    const uint32_t s4V = s4K + ns4 * kTile4Bytes;         //       ns4 staged V tiles
    const uint32_t sQ = s4V + ns4 * kTile4Bytes;          // 2 q operands (piece parity)
    const uint32_t sP = sQ + 2 * C::QB;                   // 2 P^T operands (tile parity)
    int32_t* bpre = reinterpret_cast<int32_t*>(smem + 2 * nst * kTileBytes + 2 * ns4 * kTile4Bytes + 2 * C::QB +
                                               2 * C::PB);
    // paged caches: the pool page of each of this CTA's tiles, in the
    // producers' order (p.pg_cap entries after the sequence table)
    int32_t* pg = bpre + (seq_table_bytes(p.B, p.n_kv) + 15) / 16 * 4;

    constexpr int kMaxStages = 3;
    __shared__ __align__(8) uint64_t full_k[kMaxStages], full_v[kMaxStages], empty_k[kMaxStages],
        empty_v[kMaxStages], q_full[2],
        q_empty[2], s_full[2], s_free[2], p_full[2], p_free[2], o_full[2], o_empty[2], epi_full[2], mma_fin,
        qs_full[4], pg_ready, full4_k[kMaxStages], full4_v[kMaxStages], empty4_k[kMaxStages],
        empty4_v[kMaxStages];
    // FP8: 2^-a of each piece's q prescale, a ring of four (the q warp runs
    // at most three pieces ahead of the softmax, see the q warp)
    __shared__ float q_scale[4];
    __shared__ uint32_t tmem_base_sh;
    __shared__ float red_max[2][4][G];
    __shared__ float red_l[2][4][G];   // [piece parity][softmax warp][head] row sums
    __shared__ float epi_m[2][G];      // [piece parity][head] running max
    __shared__ bool epi_last;          // this CTA is the last owner of the piece's segment
    __shared__ int abort_sh;
    __shared__ bool early_sh;          // step mode: read ahead of the append
    volatile int* abort_flag = &abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            // INT4: an E4M3 tile is full once its four converter warps have arrived
            mbar_init(smem_addr(&full_k[s]), I4 ? 4 : 1);
            mbar_init(smem_addr(&full_v[s]), I4 ? 4 : 1);
            mbar_init(smem_addr(&empty_k[s]), 1);
            mbar_init(smem_addr(&empty_v[s]), 1);
        }
        for (int s = 0; s < ns4; ++s) {
            mbar_init(smem_addr(&full4_k[s]), 1);
            mbar_init(smem_addr(&full4_v[s]), 1);
            mbar_init(smem_addr(&empty4_k[s]), 4);
            mbar_init(smem_addr(&empty4_v[s]), 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&q_full[s]), 1);
            mbar_init(smem_addr(&q_empty[s]), 1);
            mbar_init(smem_addr(&s_full[s]), 1);
            mbar_init(smem_addr(&s_free[s]), 4);
            mbar_init(smem_addr(&p_full[s]), 4);
            mbar_init(smem_addr(&p_free[s]), 1);
            mbar_init(smem_addr(&o_full[s]), 1);
            mbar_init(smem_addr(&o_empty[s]), 4);
            mbar_init(smem_addr(&epi_full[s]), 4);
        }
        mbar_init(smem_addr(&mma_fin), 1);
        for (int s = 0; s < 4; ++s) mbar_init(smem_addr(&qs_full[s]), 1);
        mbar_init(smem_addr(&pg_ready), 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    // q and P^T rows past the heads in use stay zero (their S / O columns are never read)
    for (uint32_t o = threadIdx.x * 16; o < 2 * (C::QB + C::PB); o += NT * 16)
        st_shared_v4(sQ + o, make_uint4(0, 0, 0, 0));
    fence_proxy_async_smem();
    if (warp == 1) tmem_alloc(smem_addr(&tmem_base_sh), C::COLS);
    if (threadIdx.x == 32) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_kr)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_vr)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_ks)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_vs)) : "memory");
    }
    // Launched as a programmatic dependent: everything above overlaps the
    // previous kernel in the stream; nothing it writes is read before this.
    // Step mode (duo_decode_step): the previous kernel is the step's append
    // of one token per sequence, launched once every input of the step was
    // in place.  Until it completes only the newest row of each sequence can
    // be stale (the last row of a retrieval segment, one slot of a streaming
    // ring): the lengths, q and every other tile are read at once, and a
    // producer waits for the append before the first tile that may hold such
    // a row.  Any sequence whose length does not grow by exactly one turns
    // this off for the launch.
    const bool step_mode = p.len_before != nullptr;
    if (!step_mode) asm volatile("griddepcontrol.wait;" ::: "memory");
    build_prefix<BLK>(p, bpre);
    if (step_mode && warp == 2) {
        bool one = true;
        for (int b = lane; b < p.B; b += 32) one = one && p.len_before[b] >= 0 && p.len[b] == p.len_before[b] + 1;
        one = __all_sync(0xffffffffu, one);
        if (lane == 0) early_sh = one;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool early = step_mode && early_sh;
    if (step_mode && !early) asm volatile("griddepcontrol.wait;" ::: "memory");
    // A following kernel launched as a programmatic dependent may be
    // scheduled now; it waits (griddepcontrol.wait) for this grid's writes.
    asm volatile("griddepcontrol.launch_dependents;");
    const uint32_t tmem = tmem_base_sh;

    const int64_t total = bpre[p.B];
    const int64_t n = p.num_ctas;
    const int64_t gb_begin = total > 0 ? cta_start(blockIdx.x, total, n) : 0;
    const int64_t gb_end = total > 0 ? cta_start(blockIdx.x + 1, total, n) : 0;

    if (gb_begin < gb_end) {
        if (warp == 0) {
            // ======================================================== K producer
            if (lane == 0) {
                const uint64_t policy = l2_evict_first_policy();
                uint32_t it = 0;
                bool ahead = early;   // reading ahead of the step's append
                bool ok = !PAGED || timed_wait(smem_addr(&pg_ready), 0, p, abort_flag);
                for (int64_t gb = gb_begin; ok && gb < gb_end;) {
                    Piece pc;
                    if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                    const CUtensorMap* mk = pc.retr ? &p.tm_kr : &p.tm_ks;
                    const bool paged = PAGED && pc.retr;
                    // first tile that may hold the appended row: a retrieval
                    // segment's last tile, any tile of a streaming ring
                    const int64_t t_new = pc.retr ? bpre[2 * p.B + 1 + pc.b] - 1 : 0;
                    for (int64_t t = pc.tok0; t < pc.tok1; t += C::T, ++it) {
                        if (ahead && t + C::T > t_new) {
                            asm volatile("griddepcontrol.wait;" ::: "memory");
                            ahead = false;
                        }
                        // INT4: the staging ring, filled with codes for the converters
                        const int nr = I4 ? ns4 : nst;
                        const int st = int(it % uint32_t(nr));
                        uint64_t* empty = I4 ? &empty4_k[st] : &empty_k[st];
                        if (!timed_wait(smem_addr(empty), ((it / nr) & 1) ^ 1, p, abort_flag)) {
                            ok = false;
                            break;
                        }
                        int y, z;
                        tile_coords<C::T, PAGED>(p, pc, t, paged ? (it < uint32_t(p.pg_cap) ? pg[it] : -1) : 0, y, z);
                        const uint32_t fk = smem_addr(I4 ? &full4_k[st] : &full_k[st]);
                        if constexpr (I4) {
                            mbar_arrive_expect_tx(fk, kTile4Bytes);
                            tma_load_3d(s4K + st * kTile4Bytes, mk, 0, y, z, fk, policy);   // 256 rows x 64 bytes
                        } else if constexpr (F8) {
                            mbar_arrive_expect_tx(fk, kTileBytes);
                            tma_load_3d(sK + st * kTileBytes, mk, 0, y, z, fk, policy);   // 256 rows x 128 codes
                        } else {
                            mbar_arrive_expect_tx(fk, kTileBytes);
                            tma_load_3d(sK + st * kTileBytes, mk, 0, y, z, fk, policy);
                            tma_load_3d(sK + st * kTileBytes + kSlab, mk, 64, y, z, fk, policy);
                        }
                    }
                }
                // do not leave while copies may still land in this CTA's shared memory
                const int nr = I4 ? ns4 : nst;
                for (uint32_t k = 0; k < uint32_t(nr) && k < it; ++k) {
                    const uint32_t last = it - 1 - k;
                    mbar_wait(smem_addr(I4 ? &full4_k[last % nr] : &full_k[last % nr]), (last / nr) & 1, p.timeout_ns);
                }
            }
        } else if (warp == kQWarp) {
            // ======================================================== q staging
            if constexpr (PAGED) {
                // Paged caches: look up the pool page of every retrieval tile
                // now, before HBM is busy (a dependent global read per tile
                // would stall the producers), in the producers' tile order.
                uint32_t idx = 0;
                for (int64_t gb = gb_begin; gb < gb_end;) {
                    Piece pc;
                    if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                    const int nt = tiles_of<C::T>(pc);
                    if (pc.retr)
                        for (int k = lane; k < nt; k += 32) {
                            const uint32_t slot = uint32_t(pc.row0 + pc.tok0 + int64_t(k) * C::T) / uint32_t(p.page_tokens);
                            const int page = slot < uint32_t(p.max_pages) ? p.page_table[size_t(pc.b) * p.max_pages + slot] : -1;
                            if (idx + k < uint32_t(p.pg_cap)) pg[idx + k] = page;
                        }
                    idx += nt;
                }
                if (idx > uint32_t(p.pg_cap) && lane == 0) set_status(p.status, DUO_STATUS_NO_PAGE);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&pg_ready));
            }
            // Runs up to two pieces ahead of the S products (two q buffers).
            int pi = 0;
            for (int64_t gb = gb_begin; gb < gb_end; ++pi) {
                Piece pc;
                if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                if (!warp_wait(smem_addr(&q_empty[pi & 1]), ((pi >> 1) & 1) ^ 1, p, abort_flag)) break;
                const uint16_t* qb = p.q + (size_t(pc.b) * p.hq + size_t(pc.g) * G) * kD;
                const uint32_t qs = sQ + (pi & 1) * C::QB;
                if constexpr (F8) {
                    // q' = q * 2^a (exact) with max |q'| in [128, 256), then four
                    // E4M3 terms, each the code of what the previous ones left:
                    // q' = t0 + t1 + t2 + t3 + r, |r| ~ 2^-16 |q'|.  Row
                    // term * G + h of the operand holds term `term` of head h.
                    constexpr int kItems = (G * 8 + 31) / 32;   // (head, 16-dim chunk) per lane
                    uint4 raw[kItems][2];
                    float amax = 0.f;
#pragma unroll
                    for (int k = 0; k < kItems; ++k) {
                        const int c = lane + 32 * k;
                        raw[k][0] = raw[k][1] = make_uint4(0, 0, 0, 0);
                        if (c < G * 8) {
                            const uint16_t* src = qb + (c >> 3) * kD + (c & 7) * 16;
                            raw[k][0] = *reinterpret_cast<const uint4*>(src);
                            raw[k][1] = *reinterpret_cast<const uint4*>(src + 8);
                        }
                        const uint32_t w[8] = {raw[k][0].x, raw[k][0].y, raw[k][0].z, raw[k][0].w,
                                               raw[k][1].x, raw[k][1].y, raw[k][1].z, raw[k][1].w};
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[i] << 16)),
                                                     fabsf(__uint_as_float(w[i] & 0xffff0000u))));
                    }
                    uint32_t abits;   // non-negative floats order like their bit patterns
                    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(abits) : "r"(__float_as_uint(amax)));
                    const int e = abits ? int((abits >> 23) & 0xff) - 127 : 0;
                    const int a = e > 107 ? -100 : (e < -93 ? 100 : 7 - e);
                    const float up = __uint_as_float(uint32_t(a + 127) << 23);   // 2^a
#pragma unroll
                    for (int k = 0; k < kItems; ++k) {
                        const int c = lane + 32 * k;
                        if (c >= G * 8) continue;
                        const uint32_t w[8] = {raw[k][0].x, raw[k][0].y, raw[k][0].z, raw[k][0].w,
                                               raw[k][1].x, raw[k][1].y, raw[k][1].z, raw[k][1].w};
                        float y[16];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            y[2 * i] = __uint_as_float(w[i] << 16) * up;
                            y[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u) * up;
                        }
#pragma unroll
                        for (int term = 0; term < 4; ++term) {
                            uint32_t pk[4];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const uint16_t c2 = e4m3x2(y[2 * i + 1], y[2 * i]);
                                if (i & 1) pk[i >> 1] |= uint32_t(c2) << 16; else pk[i >> 1] = c2;
                                if (term < 3) {
                                    const float2 v = e4m3x2_value(c2);
                                    y[2 * i] -= v.x;
                                    y[2 * i + 1] -= v.y;
                                }
                            }
                            st_shared_v4(qs + small_off(term * G + (c >> 3), c & 7), make_uint4(pk[0], pk[1], pk[2], pk[3]));
                        }
                    }
                    // factor that turns the S columns' sum into q.k in cache
                    // units times the key scale: 2^-a * k_scale
                    if (lane == 0) q_scale[pi & 3] = __uint_as_float(uint32_t(127 - a) << 23) * p.k_scale[pc.g];
                } else {
                    for (int c = lane; c < G * 16; c += 32) {
                        const int h = c >> 4, c16 = c & 15;
                        st_shared_v4(qs + small_off(h, c16), *reinterpret_cast<const uint4*>(qb + h * kD + c16 * 8));
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_addr(&q_full[pi & 1]));
                    // Ring of four for the softmax: the q warp can stage piece
                    // pi + 3 at most (it needs the last S product of pi + 1,
                    // which needs the softmax past piece pi), so an entry and
                    // its barrier phase are never reused before being read.
                    if constexpr (F8) mbar_arrive(smem_addr(&qs_full[pi & 3]));
                }
            }
        } else if (warp == kVWarp) {
            // ======================================================== V producer
            if (lane == 0) {
                const uint64_t policy = l2_evict_first_policy();
                uint32_t it = 0;
                bool ahead = early;
                bool ok = !PAGED || timed_wait(smem_addr(&pg_ready), 0, p, abort_flag);
                for (int64_t gb = gb_begin; ok && gb < gb_end;) {
                    Piece pc;
                    if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                    const CUtensorMap* mv = pc.retr ? &p.tm_vr : &p.tm_vs;
                    const bool paged = PAGED && pc.retr;
                    const int64_t t_new = pc.retr ? bpre[2 * p.B + 1 + pc.b] - 1 : 0;
                    for (int64_t t = pc.tok0; t < pc.tok1; t += C::T, ++it) {
                        if (ahead && t + C::T > t_new) {
                            asm volatile("griddepcontrol.wait;" ::: "memory");
                            ahead = false;
                        }
                        const int nr = I4 ? ns4 : nst;
                        const int st = int(it % uint32_t(nr));
                        uint64_t* empty = I4 ? &empty4_v[st] : &empty_v[st];
                        if (!timed_wait(smem_addr(empty), ((it / nr) & 1) ^ 1, p, abort_flag)) {
                            ok = false;
                            break;
                        }
                        int y, z;
                        tile_coords<C::T, PAGED>(p, pc, t, paged ? (it < uint32_t(p.pg_cap) ? pg[it] : -1) : 0, y, z);
                        const uint32_t fv = smem_addr(I4 ? &full4_v[st] : &full_v[st]);
                        if constexpr (I4) {
                            mbar_arrive_expect_tx(fv, kTile4Bytes);
                            tma_load_3d(s4V + st * kTile4Bytes, mv, 0, y, z, fv, policy);
                        } else if constexpr (F8) {
                            mbar_arrive_expect_tx(fv, kTileBytes);
                            tma_load_3d(sV + st * kTileBytes, mv, 0, y, z, fv, policy);
                        } else {
                            mbar_arrive_expect_tx(fv, kTileBytes);
                            tma_load_3d(sV + st * kTileBytes, mv, 0, y, z, fv, policy);
                            tma_load_3d(sV + st * kTileBytes + kSlab, mv, 64, y, z, fv, policy);
                        }
                    }
                }
                const int nr = I4 ? ns4 : nst;
                for (uint32_t k = 0; k < uint32_t(nr) && k < it; ++k) {
                    const uint32_t last = it - 1 - k;
                    mbar_wait(smem_addr(I4 ? &full4_v[last % nr] : &full_v[last % nr]), (last / nr) & 1, p.timeout_ns);
                }
            }
        } else if (warp == 1) {
            // ======================================================== MMA issuer
            // An event loop over two cursors: S_j needs K_j and a free S buffer,
            // PV_j needs P_j; whichever is ready goes first, so that PV_j (and
            // with it the release of stage j) never waits on the arrival of
            // K_{j+1}.
            if (lane == 0) {
                TileCursor<C::T, BLK> cq, cv;   // next S tile, next PV tile
                cq.start(p, bpre, gb_begin, gb_end);
                cv.start(p, bpre, gb_begin, gb_end);
                uint32_t jq = 0, jv = 0;
                bool ok = true;
                unsigned long long last = global_ns();
                while (ok && cv.valid) {
                    bool progressed = false;
                    if (cq.valid) {
                        const int st = int(jq % uint32_t(nst));
                        if ((cq.t > 0 || mbar_test_wait(smem_addr(&q_full[cq.pi & 1]), (cq.pi >> 1) & 1)) &&
                            mbar_test_wait(smem_addr(&full_k[st]), (jq / nst) & 1) &&
                            mbar_test_wait(smem_addr(&s_free[jq & 1]), ((jq >> 1) & 1) ^ 1)) {
                            tc_fence_after();
                            const uint32_t sk = sK + st * kTileBytes, sq = sQ + (cq.pi & 1) * C::QB;
                            const uint32_t ts = tmem + ((jq & 1) ? C::S1 : C::S0);
                            if constexpr (F8) {
                                // two 128-key halves; K = d = 128 codes = one swizzled row, 4 x K32
#pragma unroll
                                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                                    for (int k = 0; k < 4; ++k)
                                        umma_f8(ts + hf * C::N, smem_desc(sk + hf * 16384 + k * 32, 16, 1024),
                                                smem_desc(sq + k * 32, 16, 1024), C::IQK, k > 0 ? 1u : 0u);
                            } else {
#pragma unroll
                                for (int k = 0; k < kD / 16; ++k) {
                                    const uint32_t off = (k >> 2) * kSlab + (k & 3) * 32;
                                    const uint32_t qoff = (k >> 2) * 2048 + (k & 3) * 32;
                                    umma_f16(ts, smem_desc(sk + off, 16, 1024), smem_desc(sq + qoff, 16, 1024), C::IQK,
                                             k > 0 ? 1u : 0u);
                                }
                            }
                            umma_commit(smem_addr(&s_full[jq & 1]));
                            umma_commit(smem_addr(&empty_k[st]));
                            if (cq.t == cq.nt - 1) umma_commit(smem_addr(&q_empty[cq.pi & 1]));
                            ++jq;
                            cq.advance(p, bpre, gb_end);
                            progressed = true;
                        }
                    }
                    if (jv < jq) {
                        const int st = int(jv % uint32_t(nst));
                        if (mbar_test_wait(smem_addr(&p_full[jv & 1]), (jv >> 1) & 1) &&
                            mbar_test_wait(smem_addr(&full_v[st]), (jv / nst) & 1) &&
                            (cv.t > 0 || mbar_test_wait(smem_addr(&o_empty[cv.pi & 1]), ((cv.pi >> 1) & 1) ^ 1))) {
                            tc_fence_after();
                            const uint32_t sv = sV + st * kTileBytes, sp = sP + (jv & 1) * C::PB;
                            const uint32_t to = tmem + C::O0 + (cv.pi & 1) * C::OB;
                            if constexpr (F8) {
                                // V^T MN-major: d = 128 codes is one 128-byte atom; 8 x K32 keys
#pragma unroll
                                for (int k = 0; k < 8; ++k)
                                    umma_f8(to, smem_desc(sv + k * 4096, 16, 1024),
                                            smem_desc(sp + (k >> 2) * C::PHALF + (k & 3) * 32, 16, 1024), C::IPV,
                                            (cv.t > 0 || k > 0) ? 1u : 0u);
                            } else {
#pragma unroll
                                for (int k = 0; k < 128 / 16; ++k)
                                    umma_f16(to, smem_desc(sv + k * 2048, kSlab, 1024),
                                             smem_desc(sp + (k >> 2) * C::PHALF + (k & 3) * 32, 16, 1024), C::IPV,
                                             (cv.t > 0 || k > 0) ? 1u : 0u);
                            }
                            umma_commit(smem_addr(&empty_v[st]));
                            umma_commit(smem_addr(&p_free[jv & 1]));
                            if (cv.t == cv.nt - 1) umma_commit(smem_addr(&o_full[cv.pi & 1]));
                            ++jv;
                            cv.advance(p, bpre, gb_end);
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        last = global_ns();
                    } else if (*abort_flag) {
                        ok = false;
                    } else if (global_ns() - last > p.timeout_ns) {
                        set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                    } else {
                        __nanosleep(32);   // leave issue slots to the softmax warp on this scheduler
                    }
                }
                // every MMA issued by this thread has completed before TMEM is freed
                umma_commit(smem_addr(&mma_fin));
                mbar_wait(smem_addr(&mma_fin), 0, p.timeout_ns);
            }
        } else if (I4 && warp >= kConvWarp0) {
            // ======================================================== INT4 -> E4M3
            // Warps 12-15 expand the K tiles, 16-19 the V tiles, in the
            // producers' order.  Thread u of 128 takes the 16-byte pieces u,
            // u + 128, ... of a staged tile (row r = piece / 4, bytes 16 j ..
            // 16 j + 15 = dims 32 j .. 32 j + 31) and writes their 32 codes as
            // the 16-byte chunks 2 j and 2 j + 1 of row r in the layout the FP8
            // tensor map produces (128-byte rows, chunk c of row r stored at
            // position c xor (r mod 8)).
            if constexpr (I4) {
                const bool is_k = warp < kConvWarp0 + 4;
                const int ct = (warp - kConvWarp0) % 4 * 32 + lane;
                const uint32_t src0 = is_k ? s4K : s4V, dst0 = is_k ? sK : sV;
                uint64_t* full4 = is_k ? full4_k : full4_v;
                uint64_t* empty4 = is_k ? empty4_k : empty4_v;
                uint64_t* full8 = is_k ? full_k : full_v;
                uint64_t* empty8 = is_k ? empty_k : empty_v;
                uint32_t it = 0;
                bool ok = true;
                for (int64_t gb = gb_begin; ok && gb < gb_end;) {
                    Piece pc;
                    if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                    for (int64_t t = pc.tok0; t < pc.tok1; t += C::T, ++it) {
                        const int s4 = int(it % uint32_t(ns4)), st = int(it % uint32_t(nst));
                        if (!warp_wait_lead(smem_addr(&full4[s4]), (it / ns4) & 1, p, abort_flag) ||
                            !warp_wait_lead(smem_addr(&empty8[st]), ((it / nst) & 1) ^ 1, p, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t src = src0 + s4 * kTile4Bytes, dst = dst0 + st * kTileBytes;
                        // every code is consumed (stored) before the staging slot is
                        // handed back to the producer
#pragma unroll 2
                        for (int u = ct; u < int(kTile4Bytes / 16); u += 128) {
                            const int r = u >> 2, j = u & 3;
                            const uint4 w = ld_shared_v4(src + u * 16);
                            const uint2 a = int4x8_to_e4m3(w.x), b = int4x8_to_e4m3(w.y);
                            const uint2 c = int4x8_to_e4m3(w.z), d = int4x8_to_e4m3(w.w);
                            const uint32_t row = dst + r * 128, sw = r & 7;
                            st_shared_v4(row + (((2 * j) ^ sw) << 4), make_uint4(a.x, a.y, b.x, b.y));
                            st_shared_v4(row + (((2 * j + 1) ^ sw) << 4), make_uint4(c.x, c.y, d.x, d.y));
                        }
                        fence_proxy_async_smem();   // the tensor cores read the codes through the async proxy
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(smem_addr(&full8[st]));
                            mbar_arrive(smem_addr(&empty4[s4]));
                        }
                    }
                }
            }
        } else if (warp >= kEpiWarp0) {
            // ======================================================== epilogue
            // thread = output dim (TMEM lane of O^T); O^T of piece pi is final
            // once the MMA thread's o_full commit for it has landed.
            const int sub = warp & 3;
            const int d = sub * 32 + lane;
            const uint32_t lane_off = uint32_t(sub * 32) << 16;
            int pi = 0;
            for (int64_t gb = gb_begin; gb < gb_end; ++pi) {
                Piece pc;
                if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                const bool got = warp_wait_lazy(smem_addr(&epi_full[pi & 1]), (pi >> 1) & 1, p, abort_flag) &&
                                 warp_wait_lazy(smem_addr(&o_full[pi & 1]), (pi >> 1) & 1, p, abort_flag);
                if (barrier_any<kBarEpilogue>(!got)) break;
                tc_fence_after();
                uint32_t u[C::OL];
                tmem_ldn<C::OL>(tmem + lane_off + C::O0 + (pi & 1) * C::OB, u);
                tmem_wait_ld();
                float L[G], M[G], o[G];
                const float vs = F8 ? p.v_scale[pc.g] : 1.f;   // FP8: O^T is in value-code units
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = 0.f;
#pragma unroll
                    for (int term = 0; term < C::PT; ++term) x += __uint_as_float(u[term * G + h]);
                    o[h] = x * vs;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    L[h] = red_l[pi & 1][0][h] + red_l[pi & 1][1][h] + red_l[pi & 1][2][h] + red_l[pi & 1][3][h];
                    M[h] = epi_m[pi & 1][h] - C::POFF;   // sums are of P' = 2^POFF P
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&o_empty[pi & 1]));
                if (pc.whole) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const int qh = pc.g * G + h;
                        p.out[(size_t(pc.b) * p.hq + qh) * kD + d] = L[h] > 0.f ? o[h] / L[h] : 0.f;
                        if (d == 0 && p.lse != nullptr)
                            p.lse[size_t(pc.b) * p.hq + qh] =
                                L[h] > 0.f ? (M[h] + __log2f(L[h])) * 0.69314718055994530942f : -CUDART_INF_F;
                    }
                    continue;
                }
                // Part of a segment that other CTAs share: leave the partial in
                // the workspace (slot = segment + CTA); the last of the owners to
                // finish merges them all by log-sum-exp (fence, then count).
                {
                    const size_t slot = size_t(pc.seg) + blockIdx.x;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        p.ws_o[(slot * G + h) * kD + d] = o[h];
                        if (d == 0) {
                            p.ws_ml[(slot * G + h) * 2 + 0] = M[h];
                            p.ws_ml[(slot * G + h) * 2 + 1] = L[h];
                        }
                    }
                }
                __threadfence();
                named_bar_sync(kBarEpilogue, 128);
                const Owners ow = owners_of(pc.seg_gb, pc.seg_nb, total, n);
                if (warp == kEpiWarp0 && lane == 0) {
                    const int before = atomicAdd(&p.seg_count[pc.seg], 1);
                    epi_last = before == ow.n - 1;
                    __threadfence();
                }
                named_bar_sync(kBarEpilogue, 128);
                if (!epi_last) continue;
                float Mx[G], Ls[G], acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    Mx[h] = kNegBig;
                    Ls[h] = 0.f;
                    acc[h] = 0.f;
                }
                if constexpr (I4) {
                    // INT4: 640 threads leave 96 registers each, too few for the
                    // batches below; two passes, one slot at a time
                    for (int c = ow.c0; c <= ow.c1; ++c) {
                        if (total < n && cta_start(c + 1, total, n) == cta_start(c, total, n)) continue;
                        const size_t slot = size_t(pc.seg) + c;
#pragma unroll
                        for (int h = 0; h < G; ++h) Mx[h] = fmaxf(Mx[h], __ldcg(&p.ws_ml[(slot * G + h) * 2]));
                    }
                    for (int c = ow.c0; c <= ow.c1; ++c) {
                        if (total < n && cta_start(c + 1, total, n) == cta_start(c, total, n)) continue;
                        const size_t slot = size_t(pc.seg) + c;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float f = fast_exp2(__ldcg(&p.ws_ml[(slot * G + h) * 2]) - Mx[h]);
                            Ls[h] += __ldcg(&p.ws_ml[(slot * G + h) * 2 + 1]) * f;
                            acc[h] += __ldcg(&p.ws_o[(slot * G + h) * kD + d]) * f;
                        }
                    }
                } else {
                    // One pass over the owners' partials, kB slots at a time: all loads
                    // of a batch are issued before any is used (a segment of one long
                    // sequence spans tens of CTAs, and a round trip to L2 per slot in
                    // turn would cost tens of microseconds), with the log-sum-exp
                    // carried from batch to batch.
                    constexpr int kB = G <= 2 ? 16 : (G == 4 ? 8 : 4);
                    for (int cb = ow.c0; cb <= ow.c1; cb += kB) {
                        float mv[kB][G], lv[kB][G], ov[kB][G];
#pragma unroll
                        for (int k = 0; k < kB; ++k) {
                            const int c = cb + k;
                            const bool use = c <= ow.c1 &&
                                             !(total < n && cta_start(c + 1, total, n) == cta_start(c, total, n));
                            const size_t slot = size_t(pc.seg) + (use ? c : ow.c0);
#pragma unroll
                            for (int h = 0; h < G; ++h) {
                                mv[k][h] = use ? __ldcg(&p.ws_ml[(slot * G + h) * 2]) : kNegBig;
                                lv[k][h] = use ? __ldcg(&p.ws_ml[(slot * G + h) * 2 + 1]) : 0.f;
                                ov[k][h] = use ? __ldcg(&p.ws_o[(slot * G + h) * kD + d]) : 0.f;
                            }
                        }
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            float bm = Mx[h];
#pragma unroll
                            for (int k = 0; k < kB; ++k) bm = fmaxf(bm, mv[k][h]);
                            const float r = fast_exp2(Mx[h] - bm);   // 1 when the max is kept
                            Ls[h] *= r;
                            acc[h] *= r;
                            Mx[h] = bm;
#pragma unroll
                            for (int k = 0; k < kB; ++k) {
                                const float f = fast_exp2(mv[k][h] - bm);   // 0 for unused entries
                                Ls[h] += lv[k][h] * f;
                                acc[h] += ov[k][h] * f;
                            }
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int qh = pc.g * G + h;
                    p.out[(size_t(pc.b) * p.hq + qh) * kD + d] = Ls[h] > 0.f ? acc[h] / Ls[h] : 0.f;
                    if (d == 0 && p.lse != nullptr)
                        p.lse[size_t(pc.b) * p.hq + qh] =
                            Ls[h] > 0.f ? (Mx[h] + __log2f(Ls[h])) * 0.69314718055994530942f : -CUDART_INF_F;
                }
                if (d == 0) p.seg_count[pc.seg] = 0;   // every owner has counted: ready for the next launch
            }
        } else {
            // ======================================================== softmax
            const int sw = warp - kSoftWarp0;              // 0..3
            const int sub = warp & 3;                      // TMEM lane quarter this warp may access
            const int row = sub * 32 + lane;               // key row of each 128-key S^T block
            const uint32_t lane_off = uint32_t(sub * 32) << 16;
            uint32_t j = 0;
            bool ok = true;
            int pi = 0;
            for (int64_t gb = gb_begin; ok && gb < gb_end; ++pi) {
                Piece pc;
                if (!next_piece<BLK>(p, bpre, gb, gb_end, pc)) break;
                const uint32_t tmem_o = tmem + lane_off + C::O0 + (pi & 1) * C::OB;
                float sc = p.scale_log2;   // log2(e) * scale, per score
                if constexpr (F8) {
                    // (on failure the first tile's barrier below agrees on leaving)
                    if (warp_wait(smem_addr(&qs_full[pi & 3]), (pi >> 2) & 1, p, abort_flag)) sc *= q_scale[pi & 3];
                }
                float m[G], l[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    m[h] = kNegBig;
                    l[h] = 0.f;
                }
                const int nt = tiles_of<C::T>(pc);
                const int64_t rows_total = pc.tok1 - pc.tok0;
                for (int t = 0; t < nt; ++t, ++j) {
                    const uint32_t sb = j & 1;
                    const int st = int(j % uint32_t(nst));
                    const bool got = warp_wait(smem_addr(&s_full[sb]), (j >> 1) & 1, p, abort_flag);
                    float s[C::HALVES][G];
                    if (got) {
                        tc_fence_after();
                        uint32_t u[C::HALVES][C::QT * G];
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf)
                            tmem_ldn<C::QT * G>(tmem + lane_off + (sb ? C::S1 : C::S0) + hf * C::N, u[hf]);
                        tmem_wait_ld();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_addr(&s_free[sb]));
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf)
#pragma unroll
                            for (int h = 0; h < G; ++h) {
                                float x = __uint_as_float(u[hf][h]);
#pragma unroll
                                for (int term = 1; term < C::QT; ++term) x += __uint_as_float(u[hf][term * G + h]);
                                s[hf][h] = x;
                            }
                    }
                    const int64_t left = rows_total - int64_t(t) * C::T;
                    const int valid_rows = int(left < C::T ? left : C::T);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float mx = -CUDART_INF_F;
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf) {
                            const bool valid = got && row + 128 * hf < valid_rows;
                            s[hf][h] = valid ? s[hf][h] * sc : -CUDART_INF_F;
                            mx = fmaxf(mx, s[hf][h]);
                        }
                        mx = warp_max_f32(mx);
                        if (lane == 0) red_max[sb][sw][h] = mx;
                    }
                    // the barrier also agrees on aborting
                    if (barrier_any<kBarSoftmax>(!got || *abort_flag)) {
                        ok = false;
                        break;
                    }
                    bool grow_any = false;
                    float alpha[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float mt = fmaxf(fmaxf(red_max[sb][0][h], red_max[sb][1][h]),
                                               fmaxf(red_max[sb][2][h], red_max[sb][3][h]));
                        const bool grow = mt > m[h] + C::THRESH;
                        const float mn = grow ? mt + C::HEAD : m[h];
                        alpha[h] = fast_exp2(m[h] - mn);   // 1 when the max is kept
                        m[h] = mn;
                        l[h] *= alpha[h];
                        grow_any |= grow;
                    }
                    // P^T buffer sb is free once PV_{j-2} has completed
                    if (!warp_wait(smem_addr(&p_free[sb]), ((j >> 1) & 1) ^ 1, p, abort_flag)) continue;
                    if constexpr (F8) {
                        // keys `row` and `row` + 128 of P^T: P' rounded to fp16, then
                        // three E4M3 terms peeled off in fp16 (each residual is exact
                        // in fp16; three 4-bit terms cover its 11 bits); rows term * G + h
                        const uint32_t pb = sP + sb * C::PB + (row & 15);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float r0 = fast_exp2(s[0][h] - m[h] + C::POFF);   // 0 off-piece
                            const float r1 = fast_exp2(s[1][h] - m[h] + C::POFF);
                            l[h] += r0 + r1;
                            uint32_t p16;
                            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(p16) : "f"(r1), "f"(r0));
#pragma unroll
                            for (int term = 0; term < 3; ++term) {
                                uint16_t c2;
                                asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(c2) : "r"(p16));
                                const uint32_t off = small_off(term * G + h, row >> 4);
                                st_shared_u8(pb + off, c2 & 0xffu);
                                st_shared_u8(pb + C::PHALF + off, uint32_t(c2) >> 8);
                                if (term < 2) {
                                    uint32_t dq;
                                    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(dq) : "h"(c2));
                                    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(p16) : "r"(p16), "r"(dq));
                                }
                            }
                        }
                    } else {
                        const uint32_t pb = sP + sb * C::PB + (row & 7) * 2;   // key `row` of P^T
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pr = fast_exp2(s[0][h] - m[h]);   // 0 for rows outside the piece
                            l[h] += pr;
                            const uint16_t hi = bf16_bits(pr);
                            const uint16_t lo = bf16_bits(pr - __uint_as_float(uint32_t(hi) << 16));
                            st_shared_u16(pb + small_off(h, row >> 3), hi);
                            st_shared_u16(pb + small_off(G + h, row >> 3), lo);
                        }
                    }
                    if (valid_rows < C::T) {
                        // Rows past the piece get P = 0; clear their V rows too, so
                        // that whatever the memory there holds adds exactly 0.
                        if (!warp_wait(smem_addr(&full_v[st]), (j / nst) & 1, p, abort_flag)) continue;
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf) {
                            const int kr = row + 128 * hf;
                            if (kr >= valid_rows) {
                                const uint32_t vr = sV + st * kTileBytes + kr * 128;
#pragma unroll
                                for (int c = 0; c < 8; ++c) {
                                    st_shared_v4(vr + c * 16, make_uint4(0, 0, 0, 0));
                                    if constexpr (!F8) st_shared_v4(vr + kSlab + c * 16, make_uint4(0, 0, 0, 0));
                                }
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    if (t > 0 && grow_any) {
                        // rescale O^T (rows = dims) once PV_{j-1} has landed
                        if (!warp_wait(smem_addr(&p_free[(j - 1) & 1]), ((j - 1) >> 1) & 1, p, abort_flag)) continue;
                        tc_fence_after();
                        uint32_t u[C::OL];
                        tmem_ldn<C::OL>(tmem_o, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int term = 0; term < C::PT; ++term)
#pragma unroll
                            for (int h = 0; h < G; ++h)
                                u[term * G + h] = __float_as_uint(__uint_as_float(u[term * G + h]) * alpha[h]);
                        tmem_stn<C::OL>(tmem_o, u);
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&p_full[sb]));
                }
                if (!ok) break;

                // ---- hand the piece to the epilogue warps (per-warp row sums and
                // the max) and go on with the next piece at once
                if (!warp_wait(smem_addr(&o_empty[pi & 1]), ((pi >> 1) & 1) ^ 1, p, abort_flag)) continue;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = l[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                    if (lane == 0) {
                        red_l[pi & 1][sw][h] = x;
                        if (sw == 0) epi_m[pi & 1][h] = m[h];
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&epi_full[pi & 1]));
            }
        }
    }

    if (warp == kQWarp) {
        // Segments without keys (an empty sequence, an empty row range) have
        // no piece: their output is 0 with lse = -inf, which adds nothing to
        // a later merge.  Length checks of the classic form set status bits.
        const int32_t* tab = bpre + p.B + 1;
        const int32_t* hr = bpre + 4 * p.B + 1 + p.n_kv + 1;
        for (int seg = blockIdx.x; seg < p.B * p.n_kv; seg += gridDim.x) {
            const int b = seg / p.n_kv, g = seg % p.n_kv;
            const int32_t rows = hr[g] < 0 ? tab[p.B + b] : tab[2 * p.B + b];
            if (rows == 0) {
                for (int x = lane; x < G * kD; x += 32) p.out[(size_t(b) * p.hq + g * G) * kD + x] = 0.f;
                if (lane < G && p.lse != nullptr) p.lse[size_t(b) * p.hq + g * G + lane] = -CUDART_INF_F;
            }
            if (p.r_end == nullptr && g == 0 && lane == 0) {
                const int L = p.len[b];
                if (L < 0) set_status(p.status, DUO_STATUS_BAD_LENGTH);
                if (int64_t(L) > p.cap && p.n_r > 0) set_status(p.status, DUO_STATUS_OVER_CAPACITY);
                if (L < 1) set_status(p.status, DUO_STATUS_EMPTY_SEQUENCE);
            }
        }
    }

    // step mode: the grid ends after the append it read ahead of
    if (early && threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::COLS);
    }
}

template <int G, bool F8, bool PAGED, bool I4>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t s) {
    using C = Tr<G, F8>;
    DecodeParams q = p;
    // partition: 16-token blocks, or whole tiles for paged caches (no tile
    // straddles a page); the segment weight is a fixed number of keys
    q.blk = PAGED ? C::T : 16;   // the kernel's partition block (kept for the host's bound below)
    q.seg_weight = (F8 ? kSegWeightF8 : kSegWeight) * 16 / q.blk;
    q.pg_cap = 0;
    if (PAGED) {
        // tiles one CTA can see: its share of the largest possible axis, plus
        // one partial tile per piece (at most one piece per segment, plus one)
        const int64_t ur = (p.cap + q.blk - 1) / q.blk + q.seg_weight;
        const int64_t us = (p.S + p.W + q.blk - 1) / q.blk + q.seg_weight;
        const int64_t axis = int64_t(p.B) * (int64_t(p.n_r) * ur + int64_t(p.n_s) * us);
        const int64_t cap = (axis + p.num_ctas - 1) / p.num_ctas + 2 + int64_t(p.B) * p.n_kv;
        if (cap > (1 << 20)) return cudaErrorInvalidConfiguration;
        q.pg_cap = int(cap);
    }
    const size_t fixed = 2 * size_t(C::QB + C::PB) + (seq_table_bytes(p.B, p.n_kv) + 15) / 16 * 16 +
                         size_t(q.pg_cap) * 4 + 1024;
    // INT4: two E4M3 stages fed by a two-deep ring of staged codes
    q.stages = I4 ? 2 : (fixed + 3 * 2 * size_t(kTileBytes) <= size_t(227) * 1024 ? 3 : 2);
    q.stages4 = I4 ? 2 : 0;
    const size_t smem = fixed + size_t(q.stages) * 2 * kTileBytes + size_t(q.stages4) * 2 * kTile4Bytes;
    if (smem > size_t(227) * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<G, F8, PAGED, I4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.num_ctas));
    cfg.blockDim = dim3(I4 ? kThreadsI4 : kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<G, F8, PAGED, I4>, q);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// 3-D map over [heads][rows][128 dims] with 128-byte swizzle: bf16 in boxes
// of 64 dims x 128 rows (two per tile), FP8 codes in boxes of 128 x 256 rows;
// INT4 codes (64 bytes a row) in unswizzled boxes of 64 bytes x 256 rows.
bool make_map3(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads, bool fp8, bool int4) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const uint64_t rb = int4 ? kD / 2 : (fp8 ? kD : 2 * kD);   // bytes per row
    const uint64_t inner = int4 ? rb : uint64_t(kD);           // elements per row in the map's type
    rows = rows < 1 ? 1 : rows;
    cuuint64_t dims[3] = {inner, rows, heads < 1 ? 1 : heads};
    cuuint64_t strides[2] = {rb, rows * rb};
    cuuint32_t box[3] = {int4 ? uint32_t(rb) : (fp8 ? 128u : 64u), fp8 ? 256u : 128u, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               int4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_decode_maps(DecodeMaps* m, const void* kr, const void* vr, const void* ks, const void* vs, int64_t r_heads,
                      int64_t r_rows, int64_t s_heads, int SW, bool fp8, bool int4) {
    return make_map3(&m->kr, kr, uint64_t(r_rows), uint64_t(r_heads), fp8, int4) &&
           make_map3(&m->vr, vr, uint64_t(r_rows), uint64_t(r_heads), fp8, int4) &&
           make_map3(&m->ks, ks, uint64_t(SW), uint64_t(s_heads), fp8, int4) &&
           make_map3(&m->vs, vs, uint64_t(SW), uint64_t(s_heads), fp8, int4);
}

template <bool F8, bool PAGED, bool I4>
cudaError_t launch_group(const DecodeParams& p, int group, cudaStream_t s) {
    switch (group) {
        case 1: return launch_g<1, F8, PAGED, I4>(p, s);
        case 2: return launch_g<2, F8, PAGED, I4>(p, s);
        case 4: return launch_g<4, F8, PAGED, I4>(p, s);
        case 8: return launch_g<8, F8, PAGED, I4>(p, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_tc(const DecodeParams& p, int group, cudaStream_t s) {
    const bool paged = p.page_tokens > 0;
    if (p.int4) return paged ? launch_group<true, true, true>(p, group, s) : launch_group<true, false, true>(p, group, s);
    if (p.fp8) return paged ? launch_group<true, true, false>(p, group, s) : launch_group<true, false, false>(p, group, s);
    return paged ? launch_group<false, true, false>(p, group, s) : launch_group<false, false, false>(p, group, s);
}

}  // namespace duo
