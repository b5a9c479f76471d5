// Prefix sharing: give sequence dst the cache state of sequence src after
// its first `len` tokens, for one layer.
//
// Paged attention lets requests share blocks ("Attention Variants and
// Memory Efficiency", "What the Inference Runtime Can Change": fixed-size
// blocks, prefix sharing prevents duplicate blocks for matching prefixes).
// Retrieval pages that the caller maps to the same pool page for both
// sequences are shared and not touched; every other page of the prefix is
// copied row by row (a copy-on-write of the prefix).  The page holding the
// prefix's last, partly filled block must differ between the two sequences,
// since both will append into it.  Contiguous retrieval caches copy rows
// [0, len).  Streaming heads are small and per sequence: their sink + ring
// rows and the position table are copied whole.
//
// One grid: blockIdx.y strides over the jobs (a retrieval head's page or range, a
// streaming head, the position table); the threads of the row of blocks
// stride over its 16-byte vectors.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "duo_internal.cuh"

namespace duo {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void copy16(uint8_t* dst, const uint8_t* src, int64_t bytes) {
    const int64_t n = bytes / 16;
    for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < n; v += int64_t(gridDim.x) * blockDim.x)
        reinterpret_cast<uint4*>(dst)[v] = reinterpret_cast<const uint4*>(src)[v];
}

__device__ void fork_job(const ForkParams& p, int job) {
    const int r_jobs = p.n_r * p.n_units;
    const int SW = p.S + p.W;
    const bool lead = blockIdx.x == 0 && threadIdx.x == 0;
    if (job < r_jobs) {
        const int r = job / p.n_units, u = job % p.n_units;
        if (p.page_tokens > 0) {
            const int64_t row0 = int64_t(u) * p.page_tokens;
            const int64_t rows = min(int64_t(p.page_tokens), int64_t(p.len) - row0);
            const int ps = p.page_table[size_t(p.src) * p.max_pages + u];
            const int pd = p.page_table[size_t(p.dst) * p.max_pages + u];
            if (ps < 0 || ps >= p.num_pages || pd < 0 || pd >= p.num_pages) {
                if (lead) set_status(p.status, DUO_STATUS_NO_PAGE);
                return;
            }
            if (ps == pd) {
                // shared page: fine when full, a conflict when both sequences append into it
                if (rows < p.page_tokens && lead) set_status(p.status, DUO_STATUS_SHARED_PAGE);
                return;
            }
            const int64_t page_bytes = int64_t(p.page_tokens) * p.row_bytes;
            const int64_t off_s = (int64_t(ps) * p.n_r + r) * page_bytes;
            const int64_t off_d = (int64_t(pd) * p.n_r + r) * page_bytes;
            copy16(p.kr + off_d, p.kr + off_s, rows * p.row_bytes);
            copy16(p.vr + off_d, p.vr + off_s, rows * p.row_bytes);
        } else {
            const int64_t head_bytes = p.cap * p.row_bytes;
            const int64_t off_s = (int64_t(p.src) * p.n_r + r) * head_bytes;
            const int64_t off_d = (int64_t(p.dst) * p.n_r + r) * head_bytes;
            copy16(p.kr + off_d, p.kr + off_s, int64_t(p.len) * p.row_bytes);
            copy16(p.vr + off_d, p.vr + off_s, int64_t(p.len) * p.row_bytes);
        }
    } else if (job < r_jobs + p.n_s) {
        const int s = job - r_jobs;
        const int64_t head_bytes = int64_t(SW) * p.row_bytes;
        const int64_t off_s = (int64_t(p.src) * p.n_s + s) * head_bytes;
        const int64_t off_d = (int64_t(p.dst) * p.n_s + s) * head_bytes;
        copy16(p.ks + off_d, p.ks + off_s, head_bytes);
        copy16(p.vs + off_d, p.vs + off_s, head_bytes);
    } else {
        // position table; the source must hold exactly len tokens: no slot
        // holds a position >= len, and the slot of position len - 1 holds it
        const int32_t* ps = p.pos + size_t(p.src) * SW;
        int32_t* pd = p.pos + size_t(p.dst) * SW;
        bool later = false;
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < SW; i += gridDim.x * blockDim.x) {
            pd[i] = ps[i];
            later |= ps[i] >= p.len;
        }
        if (later) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        if (lead && p.len > 0) {
            const int64_t t = int64_t(p.len) - 1;
            const int slot = t < p.S ? int(t) : p.S + int((t - p.S) % p.W);
            if (ps[slot] != t) set_status(p.status, DUO_STATUS_BAD_LENGTH);
        }
    }
}

__global__ void __launch_bounds__(kThreads) fork_kernel(const __grid_constant__ ForkParams p) {
    const int jobs = p.n_r * p.n_units + p.n_s + 1;
    for (int job = blockIdx.y; job < jobs; job += gridDim.y) fork_job(p, job);
}

}  // namespace

cudaError_t launch_fork(const ForkParams& p, cudaStream_t s) {
    const int jobs = std::min(p.n_r * p.n_units + p.n_s + 1, 65535);
    // enough blocks per job to stream the largest range (a contiguous
    // retrieval head: len rows) at full bandwidth, capped
    const int64_t longest = p.page_tokens > 0 ? int64_t(p.page_tokens) : int64_t(p.len);
    const int64_t vecs = (std::max(longest, int64_t(p.S + p.W)) * p.row_bytes) / 16;
    const int64_t bx = std::min<int64_t>(std::max<int64_t>((vecs + kThreads - 1) / kThreads, 1), 64);
    fork_kernel<<<dim3(unsigned(bx), unsigned(jobs)), kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace duo
