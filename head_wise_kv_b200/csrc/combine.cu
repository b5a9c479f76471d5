// Combining attention results computed over disjoint key sets.
//
// A softmax over the union of key sets K_1 .. K_R is the log-sum-exp weighted
// mix of the softmaxes over each set: with lse_r = log sum_{j in K_r} e^{s_j},
// LSE = log sum_r e^{lse_r} and o = sum_r e^{lse_r - LSE} o_r.  This joins the
// partial results of a sequence split over several devices (each holds a
// slice of a retrieval head's history) and the two key ranges (sinks,
// recent window) of a streaming head read from a full cache.
//
// The blend implements the gated forward of the DuoAttention guide's head
// identification (section 3, item 2): out = alpha_h * FullAttn +
// (1 - alpha_h) * StreamAttn for each query head h.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "duo_internal.cuh"

namespace duo {

namespace {

// One warp per output row; lanes over the head dim.
__global__ void __launch_bounds__(256) lse_merge_kernel(int parts, int rows, int d, const float* __restrict__ part_out,
                                                        const float* __restrict__ part_lse, float* __restrict__ out,
                                                        float* __restrict__ lse) {
    const int row = int(blockIdx.x) * 8 + int(threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float M = -CUDART_INF_F;
    for (int r = 0; r < parts; ++r) M = fmaxf(M, part_lse[size_t(r) * rows + row]);
    if (M == -CUDART_INF_F) {   // no part saw a key
        for (int x = lane; x < d; x += 32) out[size_t(row) * d + x] = 0.f;
        if (lane == 0 && lse) lse[row] = -CUDART_INF_F;
        return;
    }
    float wsum = 0.f;
    for (int r = 0; r < parts; ++r) wsum += __expf(part_lse[size_t(r) * rows + row] - M);
    const float inv = 1.f / wsum;
    for (int x = lane; x < d; x += 32) {
        float acc = 0.f;
        for (int r = 0; r < parts; ++r) {
            const float w = __expf(part_lse[size_t(r) * rows + row] - M);
            if (w > 0.f) acc += w * part_out[(size_t(r) * rows + row) * d + x];
        }
        out[size_t(row) * d + x] = acc * inv;
    }
    if (lane == 0 && lse) lse[row] = M + __logf(wsum);
}

__global__ void __launch_bounds__(256) blend_kernel(int64_t n, int hq, int d, const float* __restrict__ alpha,
                                                    const float* __restrict__ full, const float* __restrict__ strm,
                                                    float* __restrict__ out) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const int h = int((i / d) % hq);
        const float a = alpha[h];
        out[i] = a * full[i] + (1.f - a) * strm[i];
    }
}

}  // namespace

cudaError_t launch_lse_merge(int parts, int rows, int d, const float* part_out, const float* part_lse, float* out,
                             float* lse, cudaStream_t s) {
    lse_merge_kernel<<<unsigned((rows + 7) / 8), 256, 0, s>>>(parts, rows, d, part_out, part_lse, out, lse);
    return cudaGetLastError();
}

cudaError_t launch_blend(int64_t n, int hq, int d, const float* alpha, const float* full, const float* strm,
                         float* out, cudaStream_t s) {
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    blend_kernel<<<unsigned(blocks), 256, 0, s>>>(n, hq, d, alpha, full, strm, out);
    return cudaGetLastError();
}

}  // namespace duo
