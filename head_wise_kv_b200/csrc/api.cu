// Host side of libduo_kv: argument checks, cache layout in the caller's
// buffer, and kernel launches.  No device allocation, no synchronisation
// (except duo_kv_read_status).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>

#include "duo_internal.cuh"

namespace {

constexpr size_t kAlign = 256;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;   // 1 s per pipeline wait

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_desc(const duo_kv_desc* d) {
    if (!d || !d->retrieval_mask) return DUO_ERR_INVALID_ARG;
    if (d->num_layers < 1 || d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1)
        return DUO_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads != 0) return DUO_ERR_INVALID_ARG;
    if (d->sink < 0 || d->window < 1 || d->capacity < 1) return DUO_ERR_INVALID_ARG;
    if (d->capacity > 0x7fffffffLL) return DUO_ERR_INVALID_ARG;       // positions are int32
    if (int64_t(d->sink) + d->window > (1 << 20)) return DUO_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return DUO_ERR_UNSUPPORTED;
    const int g = d->num_q_heads / d->num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return DUO_ERR_UNSUPPORTED;
    if (d->num_kv_heads > duo::kMaxKvHeads) return DUO_ERR_UNSUPPORTED;
    if (d->kv_dtype != DUO_KV_BF16 && d->kv_dtype != DUO_KV_FP8_E4M3 && d->kv_dtype != DUO_KV_INT4)
        return DUO_ERR_INVALID_ARG;
    if (d->page_tokens < 0) return DUO_ERR_INVALID_ARG;
    if (d->page_tokens > 0) {
        if (d->page_tokens % 256 != 0 || d->num_pages < 1) return DUO_ERR_INVALID_ARG;
        if (d->head_dim != 128) return DUO_ERR_UNSUPPORTED;
        // TMA coordinates are int32: pool rows of one page, pages * heads
        if (d->num_pages * int64_t(d->num_kv_heads) >= (int64_t(1) << 31)) return DUO_ERR_UNSUPPORTED;
    }
    if (d->kv_dtype != DUO_KV_BF16) {
        if (d->head_dim != 128) return DUO_ERR_UNSUPPORTED;
        const size_t n = size_t(d->num_layers) * d->num_kv_heads;
        for (const float* s : {d->k_scale, d->v_scale})
            if (s)
                for (size_t i = 0; i < n; ++i)
                    if (!(s[i] > 0.f) || !(s[i] < 3.0e38f)) return DUO_ERR_INVALID_ARG;
    }
    if (d->batch > 65536) return DUO_ERR_UNSUPPORTED;
    return DUO_OK;
}

// Bytes of the head of the buffer: status word, then the decode merge
// counters (one int32 per (sequence, KV head)).
size_t header_bytes(const duo_kv_desc* d) {
    return kAlign + align_up(size_t(d->batch) * d->num_kv_heads * 4);
}

// Layout: [status 256 B][merge counters] then per layer [Kr][Vr][Ks][Vs][pos], each 256-aligned.
size_t plan_layout(const duo_kv_desc* d, std::vector<duo::LayerLayout>* layers, size_t* cache_bytes) {
    size_t off = header_bytes(d);
    size_t cache = 0;
    const size_t D = size_t(d->head_dim), B = size_t(d->batch), SW = size_t(d->sink) + d->window;
    // bytes per cached row: bf16, one E4M3 code per element, or two INT4 codes per byte
    const size_t RB = d->kv_dtype == DUO_KV_INT4 ? D / 2 : (d->kv_dtype == DUO_KV_FP8_E4M3 ? D : 2 * D);
    for (int l = 0; l < d->num_layers; ++l) {
        duo::LayerLayout L;
        memset(L.rank, 0, sizeof L.rank);
        memset(L.r_before, 0, sizeof L.r_before);
        memset(L.is_r, 0, sizeof L.is_r);
        for (int g = 0; g < d->num_kv_heads; ++g) {
            const bool r = d->retrieval_mask[size_t(l) * d->num_kv_heads + g] != 0;
            L.r_before[g] = L.n_r;
            L.is_r[g] = r;
            L.rank[g] = r ? L.n_r++ : L.n_s++;
        }
        L.r_before[d->num_kv_heads] = L.n_r;
        const size_t kr = d->page_tokens > 0 ? size_t(d->num_pages) * L.n_r * size_t(d->page_tokens) * RB
                                             : B * L.n_r * size_t(d->capacity) * RB;
        const size_t ks = B * L.n_s * SW * RB;
        L.off_kr = off; off = align_up(off + kr);
        L.off_vr = off; off = align_up(off + kr);
        L.off_ks = off; off = align_up(off + ks);
        L.off_vs = off; off = align_up(off + ks);
        L.off_pos = off; off = align_up(off + B * SW * 4);
        cache += 2 * kr + 2 * ks;
        if (layers) layers->push_back(L);
    }
    if (cache_bytes) *cache_bytes = cache;
    return off;
}

int cuda_err(cudaError_t e) { return e == cudaSuccess ? DUO_OK : DUO_ERR_CUDA; }

}  // namespace

extern "C" {

int duo_kv_required_bytes(const duo_kv_desc* desc, size_t* total_bytes, size_t* cache_bytes) {
    const int rc = check_desc(desc);
    if (rc) return rc;
    if (!total_bytes) return DUO_ERR_INVALID_ARG;
    *total_bytes = plan_layout(desc, nullptr, cache_bytes);
    return DUO_OK;
}

int duo_kv_alloc(const duo_kv_desc* desc, void* dev_buf, size_t buf_bytes, duo_stream_t stream,
                 duo_kv** out) {
    int rc = check_desc(desc);
    if (rc) return rc;
    if (!out || !dev_buf) return DUO_ERR_INVALID_ARG;
    *out = nullptr;
    if (reinterpret_cast<uintptr_t>(dev_buf) % kAlign) return DUO_ERR_ALIGNMENT;
    duo_kv* h = new (std::nothrow) duo_kv();
    if (!h) return DUO_ERR_INVALID_ARG;
    h->desc = *desc;
    h->desc.retrieval_mask = nullptr;
    h->desc.k_scale = h->desc.v_scale = nullptr;
    h->fp8 = desc->kv_dtype != DUO_KV_BF16;   // quantised: E4M3 or INT4 codes
    h->int4 = desc->kv_dtype == DUO_KV_INT4;
    h->page_tokens = desc->page_tokens;
    h->num_pages = desc->num_pages;
    {
        const size_t n = size_t(desc->num_layers) * desc->num_kv_heads;
        h->k_scale.assign(n, 1.f);
        h->v_scale.assign(n, 1.f);
        for (size_t i = 0; i < n; ++i) {
            if (desc->k_scale) h->k_scale[i] = desc->k_scale[i];
            if (desc->v_scale) h->v_scale[i] = desc->v_scale[i];
        }
    }
    const size_t need = plan_layout(desc, &h->layers, nullptr);
    if (buf_bytes < need) {
        delete h;
        return DUO_ERR_BUFFER_TOO_SMALL;
    }
    h->base = static_cast<char*>(dev_buf);
    h->bytes = need;
    h->status = reinterpret_cast<int32_t*>(h->base);
    h->seg_count = reinterpret_cast<int32_t*>(h->base + kAlign);
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
        delete h;
        return DUO_ERR_CUDA;
    }
    cudaError_t e = cudaMemsetAsync(h->status, 0, header_bytes(desc), stream);
    const size_t SW = size_t(desc->sink) + desc->window;
    for (size_t l = 0; l < h->layers.size() && e == cudaSuccess; ++l)
        e = cudaMemsetAsync(h->base + h->layers[l].off_pos, 0xff, size_t(desc->batch) * SW * 4, stream);
    if (e != cudaSuccess) {
        delete h;
        return DUO_ERR_CUDA;
    }
    if (desc->head_dim == 128) {
        h->maps.resize(h->layers.size());
        for (size_t l = 0; l < h->layers.size(); ++l) {
            const duo::LayerLayout& L = h->layers[l];
            const bool paged = desc->page_tokens > 0;
            if (!duo::make_decode_maps(&h->maps[l], h->base + L.off_kr, h->base + L.off_vr, h->base + L.off_ks,
                                       h->base + L.off_vs,
                                       paged ? desc->num_pages * L.n_r : int64_t(desc->batch) * L.n_r,
                                       paged ? desc->page_tokens : desc->capacity, int64_t(desc->batch) * L.n_s,
                                       int(SW), h->fp8 != 0, h->int4 != 0)) {
                delete h;
                return DUO_ERR_CUDA;
            }
        }
    }
    *out = h;
    return DUO_OK;
}

int duo_kv_free(duo_kv* kv) {
    delete kv;
    return DUO_OK;
}

int duo_kv_layer_view_get(const duo_kv* kv, int32_t layer, duo_kv_layer_view* out) {
    if (!kv || !out || layer < 0 || layer >= kv->desc.num_layers) return DUO_ERR_INVALID_ARG;
    const duo::LayerLayout& L = kv->layers[layer];
    memset(out, 0, sizeof *out);
    out->k_retrieval = reinterpret_cast<uint16_t*>(kv->base + L.off_kr);
    out->v_retrieval = reinterpret_cast<uint16_t*>(kv->base + L.off_vr);
    out->k_streaming = reinterpret_cast<uint16_t*>(kv->base + L.off_ks);
    out->v_streaming = reinterpret_cast<uint16_t*>(kv->base + L.off_vs);
    out->positions = reinterpret_cast<int32_t*>(kv->base + L.off_pos);
    out->n_retrieval = L.n_r;
    out->n_streaming = L.n_s;
    for (int g = 0; g < kv->desc.num_kv_heads; ++g) {
        out->head_rank[g] = L.rank[g];
        out->is_retrieval[g] = L.is_r[g];
    }
    return DUO_OK;
}

static int append_impl(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                       const int32_t* len_before, const int32_t* n_new, int32_t n_new_max,
                       const int32_t* r_pos_begin, const int32_t* r_pos_end, duo_stream_t stream) {
    if (!kv || layer < 0 || layer >= kv->desc.num_layers || n_new_max < 0) return DUO_ERR_INVALID_ARG;
    if (n_new_max == 0) return DUO_OK;
    if (!k_new || !v_new || !len_before) return DUO_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || (reinterpret_cast<uintptr_t>(len_before) & 3) ||
        (reinterpret_cast<uintptr_t>(n_new) & 3))
        return DUO_ERR_ALIGNMENT;
    const duo::LayerLayout& L = kv->layers[layer];
    if ((reinterpret_cast<uintptr_t>(r_pos_begin) & 3) || (reinterpret_cast<uintptr_t>(r_pos_end) & 3))
        return DUO_ERR_ALIGNMENT;
    duo::AppendParams p;
    memset(&p, 0, sizeof p);
    p.r_pos_begin = r_pos_begin;
    p.r_pos_end = r_pos_end;
    p.k_new = k_new;
    p.v_new = v_new;
    p.len_before = len_before;
    p.n_new = n_new;
    p.kr = reinterpret_cast<uint16_t*>(kv->base + L.off_kr);
    p.vr = reinterpret_cast<uint16_t*>(kv->base + L.off_vr);
    p.ks = reinterpret_cast<uint16_t*>(kv->base + L.off_ks);
    p.vs = reinterpret_cast<uint16_t*>(kv->base + L.off_vs);
    p.pos = reinterpret_cast<int32_t*>(kv->base + L.off_pos);
    p.status = kv->status;
    p.cap = kv->desc.capacity;
    p.B = kv->desc.batch;
    p.n_kv = kv->desc.num_kv_heads;
    p.n_r = L.n_r;
    p.n_s = L.n_s;
    p.S = kv->desc.sink;
    p.W = kv->desc.window;
    p.d = kv->desc.head_dim;
    p.n_new_max = n_new_max;
    memcpy(p.rank, L.rank, sizeof p.rank);
    memcpy(p.is_r, L.is_r, sizeof p.is_r);
    p.fp8 = kv->fp8;
    p.int4 = kv->int4;
    for (int g = 0; g < kv->desc.num_kv_heads; ++g) {
        p.k_scale[g] = kv->k_scale[size_t(layer) * kv->desc.num_kv_heads + g];
        p.v_scale[g] = kv->v_scale[size_t(layer) * kv->desc.num_kv_heads + g];
    }
    if (kv->page_tokens > 0) {
        if (!kv->page_table && L.n_r > 0) return DUO_ERR_INVALID_ARG;   // no page table set
        p.page_tokens = kv->page_tokens;
        p.num_pages = kv->num_pages;
        p.max_pages = kv->max_pages;
        p.page_table = kv->page_table;
    }
    return cuda_err(duo::launch_append(p, stream));
}

int duo_kv_append(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                  const int32_t* len_before, const int32_t* n_new, int32_t n_new_max,
                  duo_stream_t stream) {
    return append_impl(kv, layer, k_new, v_new, len_before, n_new, n_new_max, nullptr, nullptr, stream);
}

int duo_kv_append_rows(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                       const int32_t* len_before, const int32_t* n_new, int32_t n_new_max,
                       const int32_t* r_pos_begin, const int32_t* r_pos_end, duo_stream_t stream) {
    if (!r_pos_begin || !r_pos_end) return DUO_ERR_INVALID_ARG;
    return append_impl(kv, layer, k_new, v_new, len_before, n_new, n_new_max, r_pos_begin, r_pos_end, stream);
}

static int decode_slots(const duo_kv* kv) {
    const int ctas = kv->decode_ctas > 0 ? kv->decode_ctas
                                         : duo::decode_ctas_default(kv->num_sms, kv->desc.head_dim,
                                                                    kv->desc.num_q_heads / kv->desc.num_kv_heads);
    return kv->desc.batch * kv->desc.num_kv_heads + ctas;
}

int duo_decode_workspace_bytes(const duo_kv* kv, size_t* bytes) {
    if (!kv || !bytes) return DUO_ERR_INVALID_ARG;
    *bytes = duo::decode_workspace_bytes(decode_slots(kv), kv->desc.head_dim,
                                         kv->desc.num_q_heads / kv->desc.num_kv_heads);
    return DUO_OK;
}

// Checks a decode's arguments and fills its launch parameters.
static int decode_setup(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len, const int32_t* r_begin,
                        const int32_t* r_end, const int32_t* s_len, float scale, float* out, float* lse,
                        void* workspace, size_t workspace_bytes, duo::DecodeParams& p) {
    if (!kv || layer < 0 || layer >= kv->desc.num_layers || !q || (!len && !r_end) || !out)
        return DUO_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(r_begin) & 3) || (reinterpret_cast<uintptr_t>(r_end) & 3) ||
        (reinterpret_cast<uintptr_t>(s_len) & 3))
        return DUO_ERR_ALIGNMENT;
    if (!(scale > 0.f) || scale != scale) return DUO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(len) & 3) ||
        (reinterpret_cast<uintptr_t>(lse) & 3))
        return DUO_ERR_ALIGNMENT;
    const int G = kv->desc.num_q_heads / kv->desc.num_kv_heads;
    const int D = kv->desc.head_dim;
    const int slots = decode_slots(kv);
    const size_t need = duo::decode_workspace_bytes(slots, D, G);
    if (!workspace || workspace_bytes < need) return DUO_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DUO_ERR_ALIGNMENT;
    const duo::LayerLayout& L = kv->layers[layer];
    memset(&p, 0, sizeof p);
    if (!kv->maps.empty()) {
        p.tm_kr = kv->maps[layer].kr;
        p.tm_vr = kv->maps[layer].vr;
        p.tm_ks = kv->maps[layer].ks;
        p.tm_vs = kv->maps[layer].vs;
    }
    p.kr = reinterpret_cast<const uint16_t*>(kv->base + L.off_kr);
    p.vr = reinterpret_cast<const uint16_t*>(kv->base + L.off_vr);
    p.ks = reinterpret_cast<const uint16_t*>(kv->base + L.off_ks);
    p.vs = reinterpret_cast<const uint16_t*>(kv->base + L.off_vs);
    p.q = q;
    p.len = len;
    p.r_begin = r_begin;
    p.r_end = r_end;
    p.s_len = s_len;
    p.out = out;
    p.lse = lse;
    p.ws_o = static_cast<float*>(workspace);
    p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                       ((size_t(slots) * G * D * 4 + 255) & ~size_t(255)));
    p.status = kv->status;
    p.seg_count = kv->seg_count;
    p.cap = kv->desc.capacity;
    p.B = kv->desc.batch;
    p.n_kv = kv->desc.num_kv_heads;
    p.hq = kv->desc.num_q_heads;
    p.n_r = L.n_r;
    p.n_s = L.n_s;
    p.S = kv->desc.sink;
    p.W = kv->desc.window;
    p.num_ctas = slots - p.B * p.n_kv;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = kWaitLimitNs;
    memcpy(p.rank, L.rank, sizeof p.rank);
    memcpy(p.r_before, L.r_before, sizeof p.r_before);
    memcpy(p.is_r, L.is_r, sizeof p.is_r);
    p.fp8 = kv->fp8;
    p.int4 = kv->int4;
    for (int g = 0; g < kv->desc.num_kv_heads; ++g) {
        p.k_scale[g] = kv->k_scale[size_t(layer) * kv->desc.num_kv_heads + g];
        p.v_scale[g] = kv->v_scale[size_t(layer) * kv->desc.num_kv_heads + g];
    }
    p.blk = 16;
    if (kv->page_tokens > 0) {
        if (!kv->page_table && L.n_r > 0) return DUO_ERR_INVALID_ARG;   // no page table set
        p.page_tokens = kv->page_tokens;
        p.num_pages = kv->num_pages;
        p.max_pages = kv->max_pages;
        p.page_table = kv->page_table;
    }
    return DUO_OK;
}

static int decode_impl(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len, const int32_t* r_begin,
                       const int32_t* r_end, const int32_t* s_len, float scale, float* out, float* lse,
                       void* workspace, size_t workspace_bytes, duo_stream_t stream) {
    duo::DecodeParams p;
    const int rc = decode_setup(kv, layer, q, len, r_begin, r_end, s_len, scale, out, lse, workspace,
                                workspace_bytes, p);
    if (rc) return rc;
    const int G = kv->desc.num_q_heads / kv->desc.num_kv_heads;
    return cuda_err(duo::launch_decode(p, kv->desc.head_dim, G, stream));
}

int duo_decode_step(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                    const int32_t* len_before, const uint16_t* q, const int32_t* len, float scale, float* out,
                    float* lse, void* workspace, size_t workspace_bytes, duo_stream_t stream) {
    if (!len || !len_before) return DUO_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(len_before) & 3) return DUO_ERR_ALIGNMENT;
    duo::DecodeParams p;
    int rc = decode_setup(kv, layer, q, len, nullptr, nullptr, nullptr, scale, out, lse, workspace, workspace_bytes,
                          p);
    if (rc) return rc;
    rc = append_impl(kv, layer, k_new, v_new, len_before, nullptr, 1, nullptr, nullptr, stream);
    if (rc) return rc;
    if (kv->desc.head_dim == 128) p.len_before = len_before;   // read ahead of the append
    const int G = kv->desc.num_q_heads / kv->desc.num_kv_heads;
    return cuda_err(duo::launch_decode(p, kv->desc.head_dim, G, stream));
}

int duo_decode_attn(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len, float scale,
                    float* out, float* lse, void* workspace, size_t workspace_bytes,
                    duo_stream_t stream) {
    if (!len) return DUO_ERR_INVALID_ARG;
    return decode_impl(kv, layer, q, len, nullptr, nullptr, nullptr, scale, out, lse, workspace, workspace_bytes,
                       stream);
}

int duo_decode_attn_rows(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* r_begin,
                         const int32_t* r_end, const int32_t* s_len, float scale, float* out, float* lse,
                         void* workspace, size_t workspace_bytes, duo_stream_t stream) {
    if (!r_end) return DUO_ERR_INVALID_ARG;
    return decode_impl(kv, layer, q, nullptr, r_begin, r_end, s_len, scale, out, lse, workspace, workspace_bytes,
                       stream);
}

int duo_lse_merge(int32_t parts, int32_t rows, int32_t d, const float* part_out, const float* part_lse, float* out,
                  float* lse, duo_stream_t stream) {
    if (parts < 1 || rows < 0 || d < 1 || !part_out || !part_lse || !out) return DUO_ERR_INVALID_ARG;
    if (rows == 0) return DUO_OK;
    if ((reinterpret_cast<uintptr_t>(part_out) & 3) || (reinterpret_cast<uintptr_t>(part_lse) & 3) ||
        (reinterpret_cast<uintptr_t>(out) & 3) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return DUO_ERR_ALIGNMENT;
    return cuda_err(duo::launch_lse_merge(parts, rows, d, part_out, part_lse, out, lse, stream));
}

int duo_alpha_blend(int32_t batch, int32_t num_q_heads, int32_t d, const float* alpha, const float* full_out,
                    const float* stream_out, float* out, duo_stream_t stream) {
    if (batch < 0 || num_q_heads < 1 || d < 1 || !alpha || !full_out || !stream_out || !out)
        return DUO_ERR_INVALID_ARG;
    const int64_t n = int64_t(batch) * num_q_heads * d;
    if (n == 0) return DUO_OK;
    if ((reinterpret_cast<uintptr_t>(alpha) & 3) || (reinterpret_cast<uintptr_t>(full_out) & 3) ||
        (reinterpret_cast<uintptr_t>(stream_out) & 3) || (reinterpret_cast<uintptr_t>(out) & 3))
        return DUO_ERR_ALIGNMENT;
    return cuda_err(duo::launch_blend(n, num_q_heads, d, alpha, full_out, stream_out, out, stream));
}

static size_t prefill_ws(const duo_kv* kv, int32_t chunk) {
    int n_r = 0, n_s = 0;
    for (const duo::LayerLayout& L : kv->layers) {
        n_r = std::max(n_r, L.n_r);
        n_s = std::max(n_s, L.n_s);
    }
    const duo_kv_desc& d = kv->desc;
    return duo::prefill_workspace_bytes(d.batch, d.num_q_heads, d.num_kv_heads, n_r, n_s, d.capacity, d.sink, d.window, chunk,
                                        kv->fp8 != 0 || kv->page_tokens > 0);
}

int duo_prefill_workspace_bytes(const duo_kv* kv, int32_t chunk, size_t* bytes) {
    if (!kv || !bytes || chunk < 1) return DUO_ERR_INVALID_ARG;
    *bytes = prefill_ws(kv, chunk);
    return DUO_OK;
}

int duo_prefill_attn(duo_kv* kv, int32_t layer, const uint16_t* q, const uint16_t* k_chunk,
                     const uint16_t* v_chunk, const int32_t* prefix_len, int32_t chunk, float scale,
                     float* out, void* workspace, size_t workspace_bytes, duo_stream_t stream) {
    if (!kv || layer < 0 || layer >= kv->desc.num_layers || !q || !k_chunk || !v_chunk || !prefix_len ||
        !out || chunk < 1)
        return DUO_ERR_INVALID_ARG;
    if (!(scale > 0.f) || scale != scale) return DUO_ERR_INVALID_ARG;
    if (kv->desc.head_dim != 128) return DUO_ERR_UNSUPPORTED;
    const duo_kv_desc& d = kv->desc;
    if (kv->fp8) {
        // the prefix's probabilities are multiplied by the value scale in fp16
        for (int g = 0; g < d.num_kv_heads; ++g) {
            const float vs = kv->v_scale[size_t(layer) * d.num_kv_heads + g];
            if (!(vs >= 1.0f / 256.0f && vs <= 128.0f)) return DUO_ERR_UNSUPPORTED;
        }
    }
    if (duo::prefill_smem_bytes(d.sink, d.window) > 227 * 1024) return DUO_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_chunk) || !aligned16(v_chunk) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(prefix_len) & 3))
        return DUO_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < prefill_ws(kv, chunk)) return DUO_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DUO_ERR_ALIGNMENT;
    const duo::LayerLayout& L = kv->layers[layer];
    const int64_t SW = int64_t(d.sink) + d.window;
    // tile coordinates are 32-bit row indices
    const int64_t rows_max = std::max({int64_t(d.batch) * d.num_q_heads * chunk,
                                       int64_t(d.batch) * d.num_kv_heads * chunk,
                                       int64_t(d.batch) * L.n_r * (d.capacity + 256),
                                       int64_t(d.batch) * L.n_s * (SW + 256)});
    if (rows_max >= (int64_t(1) << 31)) return DUO_ERR_UNSUPPORTED;
    duo::PrefillLaunch a;
    memset(&a, 0, sizeof a);
    a.q = q;
    a.k_chunk = k_chunk;
    a.v_chunk = v_chunk;
    a.kr = kv->base + L.off_kr;
    a.vr = kv->base + L.off_vr;
    a.ks = kv->base + L.off_ks;
    a.vs = kv->base + L.off_vs;
    a.prefix = prefix_len;
    a.out = out;
    a.workspace = workspace;
    a.status = kv->status;
    a.cap = d.capacity;
    a.B = d.batch;
    a.hq = d.num_q_heads;
    a.n_kv = d.num_kv_heads;
    a.C = chunk;
    a.S = d.sink;
    a.W = d.window;
    a.n_r = L.n_r;
    a.n_s = L.n_s;
    a.scale = scale;
    a.timeout_ns = kWaitLimitNs;
    memcpy(a.rank, L.rank, sizeof a.rank);
    memcpy(a.is_r, L.is_r, sizeof a.is_r);
    a.fp8 = kv->fp8;
    a.int4 = kv->int4;
    for (int g = 0; g < d.num_kv_heads; ++g) {
        a.k_scale[g] = kv->k_scale[size_t(layer) * d.num_kv_heads + g];
        a.v_scale[g] = kv->v_scale[size_t(layer) * d.num_kv_heads + g];
    }
    if (kv->page_tokens > 0) {
        if (!kv->page_table && L.n_r > 0) return DUO_ERR_INVALID_ARG;   // no page table set
        a.page_tokens = kv->page_tokens;
        a.num_pages = kv->num_pages;
        a.max_pages = kv->max_pages;
        a.page_table = kv->page_table;
    }
    return duo::launch_prefill(a, stream);
}

int duo_kv_read_status(duo_kv* kv, int32_t* status, int32_t clear, duo_stream_t stream) {
    if (!kv || !status) return DUO_ERR_INVALID_ARG;
    cudaError_t e = cudaMemcpyAsync(status, kv->status, sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(kv->status, 0, sizeof(int32_t), stream);
    // a decode that gave up on a wait may have left merge counters behind
    if (e == cudaSuccess && clear && (*status & DUO_STATUS_WAIT_TIMEOUT))
        e = cudaMemsetAsync(kv->seg_count, 0, size_t(kv->desc.batch) * kv->desc.num_kv_heads * 4, stream);
    return cuda_err(e);
}

int duo_kv_check_wait_timeout(duo_kv* kv, uint64_t limit_ns, duo_stream_t stream) {
    if (!kv || limit_ns == 0 || limit_ns > kWaitLimitNs) return DUO_ERR_INVALID_ARG;
    return cuda_err(duo::launch_wait_check(kv->status, limit_ns, static_cast<cudaStream_t>(stream)));
}

int duo_kv_set_page_table(duo_kv* kv, const int32_t* d_table, int32_t max_pages) {
    if (!kv || kv->page_tokens <= 0 || !d_table || max_pages < 1) return DUO_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_table) & 3) return DUO_ERR_ALIGNMENT;
    kv->page_table = d_table;
    kv->max_pages = max_pages;
    return DUO_OK;
}

int duo_kv_fork(duo_kv* kv, int32_t src, int32_t dst, int32_t len, duo_stream_t stream) {
    if (!kv || src < 0 || dst < 0 || src >= kv->desc.batch || dst >= kv->desc.batch || src == dst)
        return DUO_ERR_INVALID_ARG;
    if (len < 0 || len > kv->desc.capacity) return DUO_ERR_INVALID_ARG;
    const bool paged = kv->page_tokens > 0;
    const int units = paged ? (len + kv->page_tokens - 1) / kv->page_tokens : 1;
    if (paged && len > 0 && (!kv->page_table || units > kv->max_pages)) return DUO_ERR_INVALID_ARG;
    for (int l = 0; l < kv->desc.num_layers; ++l) {
        const duo::LayerLayout& L = kv->layers[l];
        duo::ForkParams p{};
        p.kr = reinterpret_cast<uint8_t*>(kv->base + L.off_kr);
        p.vr = reinterpret_cast<uint8_t*>(kv->base + L.off_vr);
        p.ks = reinterpret_cast<uint8_t*>(kv->base + L.off_ks);
        p.vs = reinterpret_cast<uint8_t*>(kv->base + L.off_vs);
        p.pos = reinterpret_cast<int32_t*>(kv->base + L.off_pos);
        p.status = kv->status;
        p.page_table = kv->page_table;
        p.cap = kv->desc.capacity;
        p.row_bytes = kv->int4 ? kv->desc.head_dim / 2 : int64_t(kv->desc.head_dim) * (kv->fp8 ? 1 : 2);
        p.num_pages = kv->num_pages;
        p.src = src;
        p.dst = dst;
        p.len = len;
        p.n_r = L.n_r;
        p.n_s = L.n_s;
        p.S = kv->desc.sink;
        p.W = kv->desc.window;
        p.page_tokens = kv->page_tokens;
        p.max_pages = kv->max_pages;
        p.n_units = len > 0 ? units : 0;
        const int rc = cuda_err(duo::launch_fork(p, static_cast<cudaStream_t>(stream)));
        if (rc) return rc;
    }
    return DUO_OK;
}

int duo_kv_set_decode_ctas(duo_kv* kv, int32_t ctas) {
    if (!kv || ctas < 0 || ctas > (1 << 20)) return DUO_ERR_INVALID_ARG;
    kv->decode_ctas = ctas;
    return DUO_OK;
}

const char* duo_strerror(int code) {
    switch (code) {
        case DUO_OK: return "ok";
        case DUO_ERR_INVALID_ARG: return "invalid argument";
        case DUO_ERR_UNSUPPORTED: return "unsupported shape (head_dim must be 64 or 128, group 1/2/4/8, <= 64 KV heads)";
        case DUO_ERR_BUFFER_TOO_SMALL: return "device buffer smaller than duo_kv_required_bytes";
        case DUO_ERR_WORKSPACE: return "workspace missing or smaller than required";
        case DUO_ERR_CUDA: return "CUDA runtime error";
        case DUO_ERR_ALIGNMENT: return "misaligned device pointer";
    }
    return "unknown error";
}

}  // extern "C"
