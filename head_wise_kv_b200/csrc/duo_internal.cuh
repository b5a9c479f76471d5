// Internal definitions shared by the libduo_kv kernels and host code.
// Not part of the C ABI (include/duo_kv.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "duo_kv.h"

namespace duo {

constexpr int kMaxKvHeads = 64;

// One layer's slice of the caller's device buffer (byte offsets from the base).
struct LayerLayout {
    int n_r = 0, n_s = 0;
    size_t off_kr = 0, off_vr = 0, off_ks = 0, off_vs = 0, off_pos = 0;
    int32_t rank[kMaxKvHeads];      // index among the layer's retrieval or streaming heads
    int32_t r_before[kMaxKvHeads + 1];  // retrieval heads among KV heads 0..g-1
    uint8_t is_r[kMaxKvHeads];
};

// TMA descriptors of one layer's caches for the tensor-core decode
// ([head][row][dim] bf16, 128-row boxes).
struct DecodeMaps {
    CUtensorMap kr, vr, ks, vs;
};

}  // namespace duo

struct duo_kv {
    duo_kv_desc desc;                       // retrieval_mask pointer cleared (not kept)
    std::vector<duo::LayerLayout> layers;
    char* base = nullptr;                   // caller's device buffer
    size_t bytes = 0;
    int32_t* status = nullptr;              // device status word
    int32_t* seg_count = nullptr;           // device [B * n_kv] merge arrival counters (zero between launches)
    int device = 0;
    int num_sms = 0;
    int decode_ctas = 0;                    // 0 = default persistent wave
    int fp8 = 0;                            // caches hold quantised codes (E4M3, or INT4 when int4)
    int int4 = 0;                           // caches hold packed INT4 codes
    int page_tokens = 0;                    // > 0: paged retrieval caches (pools of num_pages pages)
    int64_t num_pages = 0;
    const int32_t* page_table = nullptr;    // device [B][max_pages], caller-owned
    int max_pages = 0;
    std::vector<float> k_scale, v_scale;    // [L][n_kv] (FP8)
    std::vector<duo::DecodeMaps> maps;      // per layer (head_dim 128 only)
};

namespace duo {

// ----------------------------------------------------------------- launch params
struct DecodeParams {
    CUtensorMap tm_kr, tm_vr, tm_ks, tm_vs;   // tensor-core kernel (head_dim 128)
    const uint16_t* kr;
    const uint16_t* vr;
    const uint16_t* ks;
    const uint16_t* vs;
    const uint16_t* q;
    const int32_t* len;       // classic mode: rows = min(len, cap) and min(len, S+W)
    const int32_t* r_begin;   // row-range mode (r_end != null): retrieval rows
    const int32_t* r_end;     //   [r_begin[b], r_end[b]) (r_begin may be null = 0),
    const int32_t* s_len;     //   streaming slots [0, s_len[b]) (null = none)
    float* out;
    float* lse;
    float* ws_o;      // [slots][G][D]  partial outputs (unnormalised)
    float* ws_ml;     // [slots][G][2]  partial (max, sum) in the log2 domain
    int32_t* status;
    int32_t* seg_count;       // tensor-core kernel: per-segment arrival counters for the in-kernel merge
    int64_t cap;
    int B, n_kv, hq, n_r, n_s, S, W;
    int num_ctas;
    int blk;                  // partition block in tokens (16; a whole tile for paged caches)
    int seg_weight;           // partition weight of a segment start, in blocks (0 = none)
    int page_tokens;          // > 0: paged retrieval caches
    int64_t num_pages;
    int max_pages;
    const int32_t* page_table;   // [B][max_pages]
    int pg_cap;                  // tensor-core kernel: entries of its shared page list
    int fp8;                  // caches hold E4M3 codes (tensor-core kernel only)
    int int4;                 // caches hold packed INT4 codes (with fp8 = 1: the same arithmetic)
    int stages;               // tensor-core kernel pipeline depth (set by its launcher)
    int stages4;              // INT4: depth of the staged-code ring (set by the launcher)
    float scale_log2;
    unsigned long long timeout_ns;
    int32_t rank[kMaxKvHeads];
    int32_t r_before[kMaxKvHeads + 1];
    uint8_t is_r[kMaxKvHeads];
    float k_scale[kMaxKvHeads], v_scale[kMaxKvHeads];   // FP8: this layer's scales
    // tensor-core kernel, step mode (duo_decode_step): lengths before the
    // append that precedes this launch in the stream (null otherwise)
    const int32_t* len_before;
};

struct AppendParams {
    const int32_t* r_pos_begin;   // optional: retrieval rows hold positions
    const int32_t* r_pos_end;     //   [r_pos_begin[b], r_pos_end[b]) at rows from 0
    const uint16_t* k_new;
    const uint16_t* v_new;
    const int32_t* len_before;
    const int32_t* n_new;   // may be null
    uint16_t* kr;
    uint16_t* vr;
    uint16_t* ks;
    uint16_t* vs;
    int32_t* pos;
    int32_t* status;
    int64_t cap;
    int B, n_kv, n_r, n_s, S, W, d, n_new_max;
    int fp8;                      // store E4M3 codes of value / scale
    int int4;                     // store packed INT4 codes of value / scale
    int page_tokens;              // > 0: paged retrieval caches
    int64_t num_pages;
    int max_pages;
    const int32_t* page_table;
    int32_t rank[kMaxKvHeads];
    uint8_t is_r[kMaxKvHeads];
    float k_scale[kMaxKvHeads], v_scale[kMaxKvHeads];
};

// Prefix sharing (fork.cu): one layer, sequence src -> dst, first len tokens.
struct ForkParams {
    uint8_t* kr;
    uint8_t* vr;
    uint8_t* ks;
    uint8_t* vs;
    int32_t* pos;
    int32_t* status;
    const int32_t* page_table;    // paged caches
    int64_t cap;                  // contiguous: rows per (sequence, retrieval head)
    int64_t row_bytes;            // d x bytes per element
    int64_t num_pages;
    int src, dst, len;
    int n_r, n_s, S, W;
    int page_tokens, max_pages;
    int n_units;                  // retrieval jobs per head: pages of the prefix, or 1
};

struct PrefillLaunch {
    const void* q;
    const void* k_chunk;
    const void* v_chunk;
    const void* kr;
    const void* vr;
    const void* ks;
    const void* vs;
    const int32_t* prefix;
    float* out;
    int32_t* status;
    void* workspace;        // fp16 value copies (and bf16 key copies of an FP8 prefix), prefill_workspace_bytes(...) bytes
    int64_t cap;
    int B, hq, n_kv, C, S, W, n_r, n_s;
    int fp8;                // cached prefix holds E4M3 codes (or INT4 codes when int4)
    int int4;
    float k_scale[kMaxKvHeads], v_scale[kMaxKvHeads];
    int page_tokens;        // > 0: paged retrieval caches (prefix gathered into the workspace)
    int64_t num_pages;
    int max_pages;
    const int32_t* page_table;
    float scale;
    unsigned long long timeout_ns;
    int32_t rank[kMaxKvHeads];
    uint8_t is_r[kMaxKvHeads];
};

// Host-side launchers (defined in the kernel translation units).
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_fork(const ForkParams& p, cudaStream_t s);
cudaError_t launch_wait_check(int32_t* status, unsigned long long limit_ns, cudaStream_t s);
int decode_ctas_default(int num_sms, int d, int group);
size_t decode_workspace_bytes(int slots, int d, int group);
cudaError_t launch_decode(const DecodeParams& p, int d, int group, cudaStream_t s);
cudaError_t launch_decode_tc(const DecodeParams& p, int group, cudaStream_t s);   // attention only
// Retrieval maps over [B * n_r][cap] rows, or for paged caches over the
// pool [num_pages * n_r][page_tokens] (pass r_heads = num_pages * n_r, r_rows = page_tokens).
bool make_decode_maps(DecodeMaps* m, const void* kr, const void* vr, const void* ks, const void* vs, int64_t r_heads,
                      int64_t r_rows, int64_t s_heads, int SW, bool fp8, bool int4);
cudaError_t launch_lse_merge(int parts, int rows, int d, const float* part_out, const float* part_lse, float* out,
                             float* lse, cudaStream_t s);
cudaError_t launch_blend(int64_t n, int hq, int d, const float* alpha, const float* full, const float* strm,
                         float* out, cudaStream_t s);
size_t prefill_smem_bytes(int S, int W);
size_t prefill_workspace_bytes(int B, int hq, int n_kv, int n_r, int n_s, int64_t cap, int S, int W, int C,
                               bool key_copies);   // key copies: FP8 or paged caches
int launch_prefill(const PrefillLaunch& a, cudaStream_t s);   // returns a DUO_* code

// ----------------------------------------------------------------- device helpers
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of an mbarrier phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the given phase parity of an mbarrier, giving up after limit_ns
// nanoseconds of wall time.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Bulk (TMA engine) copy of `bytes` contiguous bytes global -> shared,
// completing on mbarrier `bar`.  16-byte aligned addresses, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// bf16 pair (low half = element 0) -> two fp32 (exact widening).
__device__ __forceinline__ float2 bf2_to_f2(uint32_t x) {
    float2 r;
    r.x = __uint_as_float(x << 16);
    r.y = __uint_as_float(x & 0xffff0000u);
    return r;
}

// Packed fp32x2 fused multiply-add (sm_100): d = a * b + c, per lane of the pair.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long av = *reinterpret_cast<unsigned long long*>(&a);
    unsigned long long bv = *reinterpret_cast<unsigned long long*>(&b);
    unsigned long long cv = *reinterpret_cast<unsigned long long*>(&c);
    unsigned long long dv;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(dv) : "l"(av), "l"(bv), "l"(cv));
    return *reinterpret_cast<float2*>(&dv);
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    unsigned long long av = *reinterpret_cast<unsigned long long*>(&a);
    unsigned long long bv = *reinterpret_cast<unsigned long long*>(&b);
    unsigned long long dv;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(dv) : "l"(av), "l"(bv));
    return *reinterpret_cast<float2*>(&dv);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t bits) {
    atomicOr(reinterpret_cast<int*>(status), bits);
}
#endif

}  // namespace duo
