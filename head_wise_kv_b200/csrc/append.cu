// KV append + window eviction for one layer.
//
// Retrieval heads store every token at its own row ("Tokens are stored
// sequentially from step 1 to T", DuoAttention guide, section 2).  Streaming
// heads keep the first S tokens in the sink slots and the most recent W in a
// W-slot ring that overwrites its oldest entry (the guide's simulation,
// append_token; the ring rule of "Attention Variants and Memory Efficiency",
// "Sliding-Window and Mixed Attention").  A bulk append writes only the
// tokens that survive the whole append (p < S or p >= T_new - W), so the
// result equals appending one token at a time and no two threads write the
// same slot.  The position table keeps each slot's original position ("When
// Is Reuse Exact?": positions are not renumbered after eviction).
//
// One row (d bf16 = 128 or 256 bytes) is moved by d/8 threads with 16-byte
// loads and stores; a trailing set of work items resets the position table
// of sequences that start over (len_before == 0).
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include "duo_internal.cuh"

namespace duo {

namespace {

constexpr int kThreads = 256;

// Eight bf16 values (16 bytes) -> their eight E4M3 codes of value / scale:
// IEEE fp32 division, then round-to-nearest-even with saturation (the
// conversion puts its first operand in the upper byte).
__device__ __forceinline__ uint2 e4m3_codes(uint4 x, float scale) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint16_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __fdiv_rn(__uint_as_float(w[i] << 16), scale);
        const float hi = __fdiv_rn(__uint_as_float(w[i] & 0xffff0000u), scale);
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c[i]) : "f"(hi), "f"(lo));
    }
    return make_uint2(uint32_t(c[0]) | (uint32_t(c[1]) << 16), uint32_t(c[2]) | (uint32_t(c[3]) << 16));
}

// Eight bf16 values -> their eight INT4 codes, packed two per byte (element
// 2i in the low nibble of byte i): IEEE fp32 division, round half to even
// (cvt.rni), clamp to [-8, 7].
__device__ __forceinline__ uint32_t int4_codes(uint4 x, float scale) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int lo = __float2int_rn(__fdiv_rn(__uint_as_float(w[i] << 16), scale));
        const int hi = __float2int_rn(__fdiv_rn(__uint_as_float(w[i] & 0xffff0000u), scale));
        const uint32_t cl = uint32_t(min(max(lo, -8), 7)) & 0xFu, ch = uint32_t(min(max(hi, -8), 7)) & 0xFu;
        out |= (cl | (ch << 4)) << (8 * i);
    }
    return out;
}

// Store 8 elements (16 bytes of bf16) at element offset `dst` of a cache:
// as given, as E4M3 codes (8 bytes) or as INT4 codes (4 bytes).
__device__ __forceinline__ void put8(const AppendParams& p, uint16_t* base, size_t dst, uint4 v, float scale) {
    if (p.int4)
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(base) + dst / 2) = int4_codes(v, scale);
    else if (p.fp8)
        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(base) + dst) = e4m3_codes(v, scale);
    else
        *reinterpret_cast<uint4*>(base + dst) = v;
}

template <int D>
__global__ void __launch_bounds__(kThreads) append_kernel(const __grid_constant__ AppendParams p) {
    // Launched as a programmatic dependent: the launch overlaps the tail of
    // the previous kernel, and nothing is read or written before it has
    // completed.  Only then may a decode launched next start (it waits for
    // this grid's writes, or in a decode step reads ahead of them: whatever
    // preceded this append is complete by then).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    constexpr int TPR = D / 8;   // threads per row, 16 bytes each
    const int64_t rows_total = int64_t(p.B) * p.n_kv * p.n_new_max;
    const int64_t item = (int64_t(blockIdx.x) * kThreads + threadIdx.x) / TPR;
    const int part = threadIdx.x % TPR;
    const int SW = p.S + p.W;

    if (item >= rows_total) {
        // position-table reset for sequences that start from empty
        const int64_t r = (item - rows_total) * TPR + part;
        if (r >= int64_t(p.B) * SW) return;
        const int b = int(r / SW), slot = int(r % SW);
        if (p.len_before[b] != 0) return;
        const int nb = p.n_new ? p.n_new[b] : p.n_new_max;
        // slots 0 .. min(nb, S+W)-1 are filled by this append; the rest start empty
        if (slot >= nb) p.pos[size_t(b) * SW + slot] = -1;
        return;
    }

    const int i = int(item % p.n_new_max);
    const int g = int((item / p.n_new_max) % p.n_kv);
    const int b = int(item / (int64_t(p.n_new_max) * p.n_kv));
    const int nb = p.n_new ? p.n_new[b] : p.n_new_max;
    const int lb = p.len_before[b];
    if (lb < 0 || nb < 0 || nb > p.n_new_max) {
        if (part == 0 && i == 0 && g == 0) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        return;
    }
    if (i >= nb) return;
    const int64_t pos = int64_t(lb) + i;
    const int64_t t_new = int64_t(lb) + nb;
    const bool survives = pos < p.S || pos >= t_new - p.W;   // still held once all nb are in
    const int slot = pos < p.S ? int(pos) : p.S + int((pos - p.S) % p.W);
    // one writer per (sequence, slot) of the position table: KV head 0, first thread of the row
    if (g == 0 && part == 0 && survives) p.pos[size_t(b) * SW + slot] = int32_t(pos);

    const size_t src = ((size_t(b) * p.n_kv + g) * p.n_new_max + i) * D + part * 8;
    if (p.is_r[g]) {
        // a cache may hold only a slice [r_pos_begin, r_pos_end) of the
        // positions in its retrieval rows (sequence split over devices)
        const int64_t lo = p.r_pos_begin ? p.r_pos_begin[b] : 0;
        const int64_t hi = p.r_pos_end ? p.r_pos_end[b] : INT64_MAX;
        if (pos < lo || pos >= hi) return;
        const int64_t row = pos - lo;
        if (row >= p.cap) {
            if (part == 0) set_status(p.status, DUO_STATUS_OVER_CAPACITY);
            return;
        }
        size_t dst;
        if (p.page_tokens > 0) {
            // paged: row -> (page from the table, offset in the page); a page
            // holds [n_r][page_tokens][d] for one sequence
            const int64_t slot = row / p.page_tokens;
            const int page = slot < p.max_pages ? p.page_table[size_t(b) * p.max_pages + slot] : -1;
            if (page < 0 || page >= p.num_pages) {
                if (part == 0) set_status(p.status, DUO_STATUS_NO_PAGE);
                return;
            }
            dst = ((size_t(page) * p.n_r + p.rank[g]) * size_t(p.page_tokens) + size_t(row % p.page_tokens)) * D +
                  part * 8;
        } else {
            dst = ((size_t(b) * p.n_r + p.rank[g]) * size_t(p.cap) + row) * D + part * 8;
        }
        const uint4 kv = *reinterpret_cast<const uint4*>(p.k_new + src);
        const uint4 vv = *reinterpret_cast<const uint4*>(p.v_new + src);
        put8(p, p.kr, dst, kv, p.k_scale[g]);
        put8(p, p.vr, dst, vv, p.v_scale[g]);
    } else if (survives) {
        const uint4 kv = *reinterpret_cast<const uint4*>(p.k_new + src);
        const uint4 vv = *reinterpret_cast<const uint4*>(p.v_new + src);
        const size_t dst = ((size_t(b) * p.n_s + p.rank[g]) * SW + slot) * D + part * 8;
        put8(p, p.ks, dst, kv, p.k_scale[g]);
        put8(p, p.vs, dst, vv, p.v_scale[g]);
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int tpr = p.d / 8;
    const int64_t rows = int64_t(p.B) * p.n_kv * p.n_new_max;
    const int64_t reset_items = (int64_t(p.B) * (p.S + p.W) + tpr - 1) / tpr;
    const int64_t threads = (rows + reset_items) * tpr;
    const int64_t blocks = (threads + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (p.d == 128) {
        e = cudaLaunchKernelEx(&cfg, append_kernel<128>, p);
    } else if (p.d == 64) {
        e = cudaLaunchKernelEx(&cfg, append_kernel<64>, p);
    } else {
        return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace duo
