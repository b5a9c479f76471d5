// Mixed-head decode attention (one new query token per sequence).
//
// Retrieval KV heads attend over their full cache, streaming KV heads over
// their sink + window ring (DuoAttention guide, section 2; decode reads
// "Coalesced Autoregressive Reads" under "Zero-Gather Hardware Efficiency").
// Each (sequence b, KV head g) pair is a *segment* of keys: min(len, cap) rows
// of the retrieval cache, or min(len, S + W) filled slots of the ring (slot
// order does not matter to a softmax, and once the token is appended the
// ring holds exactly the sink + window key set of the query).
//
// Work split (split-K, load balanced): all segments are laid end to end in
// units of 16 tokens; a persistent grid of C CTAs takes C equal contiguous
// ranges of that axis.  A CTA walks its range piece by piece (a piece = the
// part of one segment inside the range); pieces that cover a whole segment
// are normalised and written straight to `out`, the others leave an
// unnormalised partial (o, max, sum) in the workspace, slot = segment + CTA
// (unique: moving along the axis crosses either a segment or a CTA boundary).
// A second small kernel merges the partials by log-sum-exp.
//
// Inside a CTA: one producer warp streams K and V tiles of 56 rows into a
// 4-stage shared-memory ring with TMA bulk copies (cp.async.bulk, completion
// on mbarriers, L2 evict-first); 7 consumer warps compute.  GQA packing: a
// KV tile is read once from shared memory and feeds all G query heads of the
// group (the K/V of "Multi-Query and Grouped-Query Attention" reused without
// copies).  A consumer lane group of LPT lanes owns one token per step; each
// lane holds D/LPT dims of q (fp32) for all G heads and of the running output.
// Dot products reduce with xor-shuffles inside the lane group; the softmax
// is online, in the log2 domain, fp32 throughout.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "decode_sched.cuh"
#include "duo_internal.cuh"

namespace duo {

namespace {

// 7 consumer warps + 1 producer warp = 2 warps per SM sub-partition, so each
// thread may hold up to 255 registers (q and the running output of all G
// heads stay in registers).  A tile holds exactly two (four for LPT = 16)
// warp steps of 7 warps x TPW tokens.
constexpr int kTile = 56;        // rows per pipeline stage
constexpr int kStages = 4;
constexpr int kConsumerWarps = 7;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kNegBig = -1.0e30f;   // finite "minus infinity" for running maxima
constexpr float kRescaleThreshold = 8.0f;   // log2 units: probabilities stay <= 2^8

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }

template <int D, int G>
struct Cfg {
    static constexpr int LPT = (D == 128 && G == 8) ? 16 : 8;   // lanes per token
    static constexpr int TPW = 32 / LPT;                         // tokens per warp step
    static constexpr int NCL = D / 8 / LPT;                      // 16-byte chunks per lane
    static constexpr int STEPS = kTile / (TPW * kConsumerWarps);
    static constexpr int ROW_BYTES = D * 2;
    static constexpr int STAGE_BYTES = kTile * ROW_BYTES;        // one of K or V
    static constexpr int RED_STRIDE = D + 4;                     // floats; keeps float4 alignment
    static constexpr int RED_FLOATS = kConsumerWarps * G * RED_STRIDE;
    static constexpr size_t SMEM = size_t(2) * kStages * STAGE_BYTES + RED_FLOATS * 4 + 1024;
    // reduce-scatter of the V = STEPS * G partial dot products of one tile
    // over the LPT lanes of a token group: RS halving rounds leave KEEP
    // complete scores per lane (all-reduce rounds finish when V < LPT)
    static constexpr int V = STEPS * G;
    static constexpr int LOG_LPT = ilog2(LPT);
    static constexpr int LOG_V = ilog2(V);
    static constexpr int RS = LOG_V < LOG_LPT ? LOG_V : LOG_LPT;
    static constexpr int KEEP = V >> RS;
    static_assert(STEPS * TPW * kConsumerWarps == kTile, "tile must be whole warp steps");
    static_assert(STAGE_BYTES % 1024 == 0, "stage buffers stay 1024-byte aligned");
};

// First of the KEEP score indices (step * G + head) lane li of its token group
// holds after the reduce-scatter.
template <class C>
__device__ __forceinline__ int rs_first(int li) {
    int lo = 0;
#pragma unroll
    for (int k = 0; k < C::RS; ++k)
        if (li & (C::LPT >> (k + 1))) lo += C::V >> (k + 1);
    return lo;
}

// Lane (within the token group) holding score index v after the reduce-scatter.
template <class C>
__host__ __device__ constexpr int rs_lane(int v) {
    int lane = 0;
    const int base = v - v % C::KEEP;
    for (int k = 0; k < C::RS; ++k)
        if ((base >> (C::LOG_V - 1 - k)) & 1) lane += C::LPT >> (k + 1);
    return lane;
}

// Sum x[0..V) over the LPT lanes of each token group; lane li keeps the
// complete values of indices rs_first(li) .. + KEEP in x[0..KEEP).
template <class C>
__device__ __forceinline__ void reduce_scatter(float (&x)[C::V], int li) {
#pragma unroll
    for (int k = 0; k < C::RS; ++k) {
        const int o = C::LPT >> (k + 1);
        const int half = C::V >> (k + 1);
        const bool upper = (li & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? x[i] : x[half + i];
            const float keep = upper ? x[half + i] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int k = C::RS; k < C::LOG_LPT; ++k) x[0] += __shfl_xor_sync(0xffffffffu, x[0], C::LPT >> (k + 1));
}

// Every lane of a token group receives all V values the group holds.
template <class C>
__device__ __forceinline__ void gather_group(const float (&held)[C::KEEP], float (&all)[C::V], int group_lane0) {
#pragma unroll
    for (int v = 0; v < C::V; ++v) all[v] = __shfl_sync(0xffffffffu, held[v % C::KEEP], group_lane0 + rs_lane<C>(v));
}

template <int D>
__device__ __forceinline__ void seg_ptrs(const DecodeParams& p, int b, int g, int64_t row0, const uint16_t*& k,
                                         const uint16_t*& v) {
    const int r = p.rank[g];
    if (p.is_r[g]) {
        const size_t off = ((size_t(b) * p.n_r + r) * size_t(p.cap) + size_t(row0)) * D;
        k = p.kr + off;
        v = p.vr + off;
    } else {
        const size_t off = (size_t(b) * p.n_s + r) * size_t(p.S + p.W) * D;
        k = p.ks + off;
        v = p.vs + off;
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    using C = Cfg<D, G>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned carve-up
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sK = smem;
    unsigned char* sV = sK + kStages * C::STAGE_BYTES;
    float* red = reinterpret_cast<float*>(sV + kStages * C::STAGE_BYTES);
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ int abort_flag;

    // the sequence table lives after the reduction buffer; sized by the launcher
    int32_t* bpre = reinterpret_cast<int32_t*>(red + C::RED_FLOATS);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&full_bar[s]), 1);
            mbar_init(smem_addr(&empty_bar[s]), kConsumerWarps);
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    build_prefix<16>(p, bpre);
    __syncthreads();
    // The merge kernel may be scheduled now; it waits (griddepcontrol.wait)
    // for this grid's completion before it reads any partial.
    asm volatile("griddepcontrol.launch_dependents;");

    const int64_t total = bpre[p.B];
    if (total == 0) return;
    const int64_t n = p.num_ctas;
    const int64_t gb_begin = cta_start(blockIdx.x, total, n);
    const int64_t gb_end = cta_start(blockIdx.x + 1, total, n);
    if (gb_begin >= gb_end) return;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t policy = l2_evict_first_policy();
        uint32_t it = 0;
        bool ok = true;
        for (int64_t gb = gb_begin; gb < gb_end && ok;) {
            const Piece pc = locate<16>(p, bpre, gb, gb_end);
            const uint16_t *kp, *vp;
            seg_ptrs<D>(p, pc.b, pc.g, pc.row0, kp, vp);
            for (int64_t t = pc.tok0; t < pc.tok1; t += kTile, ++it) {
                const int rows = int(pc.tok1 - t < kTile ? pc.tok1 - t : kTile);
                const int st = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                if (!mbar_wait(smem_addr(&empty_bar[st]), ph ^ 1, p.timeout_ns) ||
                    *((volatile int*)&abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t bytes = uint32_t(rows) * C::ROW_BYTES;
                mbar_arrive_expect_tx(smem_addr(&full_bar[st]), 2 * bytes);
                bulk_g2s(smem_addr(sK + st * C::STAGE_BYTES), kp + t * D, bytes,
                         smem_addr(&full_bar[st]), policy);
                bulk_g2s(smem_addr(sV + st * C::STAGE_BYTES), vp + t * D, bytes,
                         smem_addr(&full_bar[st]), policy);
            }
            gb = pc.end_gb;
        }
        if (!ok) {
            set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
            atomicExch(&abort_flag, 1);
        }
        // Do not leave while copies issued by this CTA may still land in its
        // shared memory: wait (bounded) for every stage's last issued phase.
        for (uint32_t k = 0; k < kStages && k < it; ++k) {
            const uint32_t last = it - 1 - k;
            mbar_wait(smem_addr(&full_bar[last % kStages]), (last / kStages) & 1, p.timeout_ns);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int grp = lane / C::LPT;          // token slot within the warp step
    const int li = lane % C::LPT;           // lane within the token group
    uint32_t it = 0;
    bool aborted = false;
    const uint32_t sK0 = smem_addr(sK), sV0 = smem_addr(sV);
    const int lo_idx = rs_first<C>(li);   // first (step * G + head) score this lane owns

    for (int64_t gb = gb_begin; gb < gb_end;) {
        const Piece pc = locate<16>(p, bpre, gb, gb_end);
        gb = pc.end_gb;

        // q of the G query heads of this KV head, this lane's dims, fp32
        float2 q2[G][C::NCL * 4];
        {
            const uint16_t* qb = p.q + (size_t(pc.b) * p.hq + size_t(pc.g) * G) * D;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < C::NCL; ++k) {
                    const uint4 v = *reinterpret_cast<const uint4*>(qb + h * D + (li + k * C::LPT) * 8);
                    q2[h][k * 4 + 0] = bf2_to_f2(v.x);
                    q2[h][k * 4 + 1] = bf2_to_f2(v.y);
                    q2[h][k * 4 + 2] = bf2_to_f2(v.z);
                    q2[h][k * 4 + 3] = bf2_to_f2(v.w);
                }
        }
        float2 o2[G][C::NCL * 4];
        float m[G], l[G];
        float mv[C::KEEP];   // m of the head of each score this lane owns
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = kNegBig;
            l[h] = 0.f;
#pragma unroll
            for (int j = 0; j < C::NCL * 4; ++j) o2[h][j] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int e = 0; e < C::KEEP; ++e) mv[e] = kNegBig;

        for (int64_t t = pc.tok0; t < pc.tok1 && !aborted; t += kTile, ++it) {
            const int rows = int(pc.tok1 - t < kTile ? pc.tok1 - t : kTile);
            const int st = it % kStages;
            const uint32_t ph = (it / kStages) & 1;
            if (*((volatile int*)&abort_flag)) {
                aborted = true;
                break;
            }
            if (!mbar_wait(smem_addr(&full_bar[st]), ph, p.timeout_ns)) {
                // Stop consuming; keep taking part in the named barriers below so
                // that no warp of this CTA waits on one forever.
                set_status(p.status, DUO_STATUS_WAIT_TIMEOUT);
                atomicExch(&abort_flag, 1);
                aborted = true;
                break;
            }
            const uint32_t kbase = sK0 + st * C::STAGE_BYTES;
            const uint32_t vbase = sV0 + st * C::STAGE_BYTES;

            // partial dot products of this lane's dims, all steps and heads
            float x[C::V];
#pragma unroll
            for (int s = 0; s < C::STEPS; ++s) {
                const int row = (s * kConsumerWarps + warp) * C::TPW + grp;
                float2 acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < C::NCL; ++k) {
                    const uint4 kv = lds128(kbase + row * C::ROW_BYTES + (li + k * C::LPT) * 16);
                    const float2 k0 = bf2_to_f2(kv.x), k1 = bf2_to_f2(kv.y);
                    const float2 k2 = bf2_to_f2(kv.z), k3 = bf2_to_f2(kv.w);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        acc[h] = ffma2(q2[h][k * 4 + 0], k0, acc[h]);
                        acc[h] = ffma2(q2[h][k * 4 + 1], k1, acc[h]);
                        acc[h] = ffma2(q2[h][k * 4 + 2], k2, acc[h]);
                        acc[h] = ffma2(q2[h][k * 4 + 3], k3, acc[h]);
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) x[s * G + h] = acc[h].x + acc[h].y;
            }
            // complete scores: each lane owns KEEP of the group's (step, head) pairs
            reduce_scatter<C>(x, li);
            float sc[C::KEEP];
            bool need = false;
#pragma unroll
            for (int e = 0; e < C::KEEP; ++e) {
                const int idx = lo_idx + e;
                const int row = ((idx / G) * kConsumerWarps + warp) * C::TPW + grp;
                sc[e] = row < rows ? x[e] * p.scale_log2 : -CUDART_INF_F;
                need |= sc[e] > mv[e] + kRescaleThreshold;
            }
            // Lazy rescaling: the running max only moves when a score exceeds it
            // by more than 2^8 (first tile of a piece, then rarely), so the
            // probabilities stay <= 256 and the common path exchanges nothing.
            if (__any_sync(0xffffffffu, need)) {
                float all[C::V];
                gather_group<C>(sc, all, grp * C::LPT);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float mt = all[h];
#pragma unroll
                    for (int s = 1; s < C::STEPS; ++s) mt = fmaxf(mt, all[s * G + h]);
                    const float mn = fmaxf(m[h], mt);
                    const float a = fast_exp2(m[h] - mn);
                    m[h] = mn;
                    l[h] *= a;
                    const float2 a2 = make_float2(a, a);
#pragma unroll
                    for (int j = 0; j < C::NCL * 4; ++j) o2[h][j] = fmul2(o2[h][j], a2);
                }
#pragma unroll
                for (int e = 0; e < C::KEEP; ++e) {
                    const int hh = (lo_idx + e) % G;
                    float mm = m[0];
#pragma unroll
                    for (int h = 1; h < G; ++h) mm = hh == h ? m[h] : mm;
                    mv[e] = mm;
                }
            }
            float pe[C::KEEP];
#pragma unroll
            for (int e = 0; e < C::KEEP; ++e) pe[e] = fast_exp2(sc[e] - mv[e]);
            float pa[C::V];
            gather_group<C>(pe, pa, grp * C::LPT);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int s = 0; s < C::STEPS; ++s) l[h] += pa[s * G + h];
#pragma unroll
            for (int s = 0; s < C::STEPS; ++s) {
                const int row = (s * kConsumerWarps + warp) * C::TPW + grp;
                if (row < rows) {
#pragma unroll
                    for (int k = 0; k < C::NCL; ++k) {
                        const uint4 vv = lds128(vbase + row * C::ROW_BYTES + (li + k * C::LPT) * 16);
                        const float2 v0 = bf2_to_f2(vv.x), v1 = bf2_to_f2(vv.y);
                        const float2 v2 = bf2_to_f2(vv.z), v3 = bf2_to_f2(vv.w);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float2 pp = make_float2(pa[s * G + h], pa[s * G + h]);
                            o2[h][k * 4 + 0] = ffma2(pp, v0, o2[h][k * 4 + 0]);
                            o2[h][k * 4 + 1] = ffma2(pp, v1, o2[h][k * 4 + 1]);
                            o2[h][k * 4 + 2] = ffma2(pp, v2, o2[h][k * 4 + 2]);
                            o2[h][k * 4 + 3] = ffma2(pp, v3, o2[h][k * 4 + 3]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&empty_bar[st]));
        }

        // -------- merge the token groups of this warp (same lanes li, other grp)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float M = m[h];
#pragma unroll
            for (int o = C::LPT; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            const float f = fast_exp2(m[h] - M);
            float L = l[h] * f;
#pragma unroll
            for (int o = C::LPT; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            m[h] = M;
            l[h] = L;
#pragma unroll
            for (int j = 0; j < C::NCL * 4; ++j) {
                float2 x = make_float2(o2[h][j].x * f, o2[h][j].y * f);
#pragma unroll
                for (int o = C::LPT; o < 32; o <<= 1) {
                    x.x += __shfl_xor_sync(0xffffffffu, x.x, o);
                    x.y += __shfl_xor_sync(0xffffffffu, x.y, o);
                }
                o2[h][j] = x;
            }
        }
        // lanes of token group 0 publish the warp's partial: red[warp][h][o(D), m, l]
        if (grp == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float* dst = red + (warp * G + h) * C::RED_STRIDE;
#pragma unroll
                for (int k = 0; k < C::NCL; ++k) {
                    float4* d4 = reinterpret_cast<float4*>(dst + (li + k * C::LPT) * 8);
                    d4[0] = make_float4(o2[h][k * 4 + 0].x, o2[h][k * 4 + 0].y, o2[h][k * 4 + 1].x,
                                        o2[h][k * 4 + 1].y);
                    d4[1] = make_float4(o2[h][k * 4 + 2].x, o2[h][k * 4 + 2].y, o2[h][k * 4 + 3].x,
                                        o2[h][k * 4 + 3].y);
                }
                if (li == 0) {
                    dst[D] = m[h];
                    dst[D + 1] = l[h];
                }
            }
        }
        named_bar_sync(1, kConsumerWarps * 32);
        // -------- merge the warps and write
        for (int e = threadIdx.x; e < G * D; e += kConsumerWarps * 32) {
            const int h = e / D, x = e % D;
            float M = kNegBig;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[(w * G + h) * C::RED_STRIDE + D]);
            float L = 0.f, acc = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float* src = red + (w * G + h) * C::RED_STRIDE;
                const float f = fast_exp2(src[D] - M);
                L += src[D + 1] * f;
                acc += src[x] * f;
            }
            const int qh = pc.g * G + h;
            if (pc.whole) {
                p.out[(size_t(pc.b) * p.hq + qh) * D + x] = L > 0.f ? acc / L : 0.f;
                if (x == 0 && p.lse != nullptr)
                    p.lse[size_t(pc.b) * p.hq + qh] =
                        L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -CUDART_INF_F;
            } else {
                const size_t slot = size_t(pc.seg) + blockIdx.x;
                p.ws_o[(slot * G + h) * D + x] = acc;
                if (x == 0) {
                    p.ws_ml[(slot * G + h) * 2 + 0] = M;
                    p.ws_ml[(slot * G + h) * 2 + 1] = L;
                }
            }
        }
        named_bar_sync(1, kConsumerWarps * 32);
    }
}

// Merge the partials of segments that more than one CTA touched, and handle
// empty / over-capacity sequences.  One CTA per segment, one warp per query
// head of the group.  Launched as a programmatic dependent of the attention
// kernel: everything before griddepcontrol.wait overlaps its tail.
template <int D, int G>
__global__ void __launch_bounds__(32 * G) merge_kernel(const __grid_constant__ DecodeParams p) {
    extern __shared__ int32_t bpre[];
    build_prefix<16>(p, bpre);
    __syncthreads();
    const int seg = blockIdx.x;
    const int b = seg / p.n_kv, g = seg % p.n_kv;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qh = g * G + h;
    float* out = p.out + (size_t(b) * p.hq + qh) * D;
    const int64_t total = bpre[p.B];
    const SeqRows x = seq_rows(p, b);
    const int nbr = blocks_of<16>(x.nr), nbs = blocks_of<16>(x.ns);
    const int64_t seg_gb = bpre[b] + int64_t(p.r_before[g]) * nbr + int64_t(g - p.r_before[g]) * nbs;
    const int seg_nb = p.is_r[g] ? nbr : nbs;
    const int c0 = seg_nb < 1 ? 0 : cta_owner(seg_gb, total, p.num_ctas);
    const int c1 = seg_nb < 1 ? 0 : cta_owner(seg_gb + seg_nb - 1, total, p.num_ctas);
    const bool dense = total >= p.num_ctas;   // then no CTA range is empty

    // wait for the attention kernel's partials (and its writes of `out`)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (p.r_end == nullptr && threadIdx.x == 0 && g == 0) {
        const int L = p.len[b];
        if (L < 0) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        if (int64_t(L) > p.cap && p.n_r > 0) set_status(p.status, DUO_STATUS_OVER_CAPACITY);
        if (L < 1) set_status(p.status, DUO_STATUS_EMPTY_SEQUENCE);
    }
    if (seg_nb < 1) {   // no key: zero output, lse = -inf (contributes nothing to a merge)
        for (int xx = lane; xx < D; xx += 32) out[xx] = 0.f;
        if (lane == 0 && p.lse != nullptr) p.lse[size_t(b) * p.hq + qh] = -CUDART_INF_F;
        return;
    }
    if (c0 == c1) return;

    // lanes own pieces: max and weighted sum of the (max, sum) pairs.  CTAs
    // with an empty range (fewer blocks than CTAs) wrote nothing: skipped.
    float M = kNegBig;
    for (int c = c0 + lane; c <= c1; c += 32) {
        if (!dense && cta_start(c + 1, total, p.num_ctas) == cta_start(c, total, p.num_ctas)) continue;
        M = fmaxf(M, p.ws_ml[((size_t(seg) + c) * G + h) * 2]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    for (int c = c0 + lane; c <= c1; c += 32) {
        if (!dense && cta_start(c + 1, total, p.num_ctas) == cta_start(c, total, p.num_ctas)) continue;
        const size_t slot = size_t(seg) + c;
        Lsum += p.ws_ml[(slot * G + h) * 2 + 1] * fast_exp2(p.ws_ml[(slot * G + h) * 2] - M);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);

    float acc[D / 32];
#pragma unroll
    for (int j = 0; j < D / 32; ++j) acc[j] = 0.f;
#pragma unroll 4
    for (int c = c0; c <= c1; ++c) {
        if (!dense && cta_start(c + 1, total, p.num_ctas) == cta_start(c, total, p.num_ctas)) continue;
        const size_t slot = size_t(seg) + c;
        const float f = fast_exp2(p.ws_ml[(slot * G + h) * 2] - M);
        const float* src = p.ws_o + (slot * G + h) * D;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) acc[j] += src[lane + 32 * j] * f;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) out[lane + 32 * j] = acc[j] * inv;
    if (lane == 0 && p.lse != nullptr)
        p.lse[size_t(b) * p.hq + qh] =
            Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994530942f : -CUDART_INF_F;
}

template <int D, int G>
cudaError_t launch_merge(const DecodeParams& p, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.B * p.n_kv));
    cfg.blockDim = dim3(32 * G);
    cfg.dynamicSmemBytes = seq_table_bytes(p.B, p.n_kv);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, merge_kernel<D, G>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// d = 128: the tensor-core kernel, which merges its partials itself.
// d = 64: the CUDA-core kernel, then the merge as its programmatic dependent.
template <int D, int G>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
    if constexpr (D == 128) {
        return launch_decode_tc(p, G, s);
    } else {
        using C = Cfg<D, G>;
        const size_t smem = C::SMEM + seq_table_bytes(p.B, p.n_kv);
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        decode_kernel<D, G><<<p.num_ctas, kThreads, smem, s>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_merge<D, G>(p, s);
    }
}

}  // namespace

int decode_ctas_default(int num_sms, int d, int group) {
    (void)d;
    (void)group;
    return num_sms;   // one persistent CTA per SM
}

size_t decode_workspace_bytes(int slots, int d, int group) {
    const size_t o = size_t(slots) * group * d * 4;
    const size_t ml = size_t(slots) * group * 2 * 4;
    return ((o + 255) & ~size_t(255)) + ml;
}

cudaError_t launch_decode(const DecodeParams& p, int d, int group, cudaStream_t s) {
    if (d == 128) {
        switch (group) {
            case 1: return launch_t<128, 1>(p, s);
            case 2: return launch_t<128, 2>(p, s);
            case 4: return launch_t<128, 4>(p, s);
            case 8: return launch_t<128, 8>(p, s);
        }
    } else if (d == 64) {
        switch (group) {
            case 1: return launch_t<64, 1>(p, s);
            case 2: return launch_t<64, 2>(p, s);
            case 4: return launch_t<64, 4>(p, s);
            case 8: return launch_t<64, 8>(p, s);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace duo
