// Decode attention without a caller-provided workspace.
//
// duo_decode_attn needs device scratch for the split-K partials, and the
// usual way to get it is for the caller to allocate a workspace.  Some
// callers cannot do that: a plugin inside a host program that owns all
// device memory and hands the plugin only its input and output buffers; a
// latency-critical serving loop that must not call cudaMalloc (which can
// synchronise the device) or handle an out-of-memory failure in the middle
// of a request.  duo_decode_attn_static_ws serves them: it runs the same
// decode with its scratch in the fixed-size array below, which is part of
// this library's device code, so the call allocates nothing.
//
// The array is DUO_STATIC_WS_BYTES (4 MiB) on every GPU that loads the
// library and stays there until the process exits.  All calls on a device
// share it: two calls whose kernels overlap on the GPU (for example on two
// streams without ordering between them) race on it and produce garbage.
// The decode writes every partial before it reads it, so what a previous
// call left in the array needs no clearing.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "duo_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[DUO_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in;
// the kernel must be given the address cudaGetSymbolAddress returns.
int scratch_address(int device, void** out) {
    if (device < 0 || device >= kMaxDevices) return DUO_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[device]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return DUO_ERR_CUDA;
        g_scratch_ptr[device] = p;
    }
    *out = g_scratch_ptr[device];
    return DUO_OK;
}

}  // namespace

extern "C" int duo_decode_attn_static_ws(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len,
                                         float scale, float* out, float* lse, duo_stream_t stream) {
    if (!kv) return DUO_ERR_INVALID_ARG;
    size_t need = 0;
    int rc = duo_decode_workspace_bytes(kv, &need);
    if (rc) return rc;
    if (need > DUO_STATIC_WS_BYTES) return DUO_ERR_WORKSPACE;   // problem too large for the fixed scratch
    int device = -1;
    if (cudaGetDevice(&device) != cudaSuccess) return DUO_ERR_CUDA;
    if (device != kv->device) return DUO_ERR_INVALID_ARG;       // the handle's device must be current
    void* scratch = nullptr;
    rc = scratch_address(device, &scratch);
    if (rc) return rc;
    return duo_decode_attn(kv, layer, q, len, scale, out, lse, scratch, DUO_STATIC_WS_BYTES, stream);
}
