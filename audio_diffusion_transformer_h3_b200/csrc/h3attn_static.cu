// h3_varlen_attn_fwd_static: the fused RoPE + varlen attention call for
// callers that must not allocate device memory themselves.
//
// Some hosts own every byte of device memory and forbid cudaMalloc from
// inside a plugin (a serving engine with its own arena, a media pipeline that
// allocates only at start-up, a caller holding a fixed memory budget). They
// cannot hand h3_varlen_attn_fwd a workspace of their own. This entry point
// uses a scratch array compiled into the library instead: a file-scope
// __device__ array of H3_STATIC_WORKSPACE_BYTES, which the CUDA driver places
// in device memory when it loads this file's module on a device and keeps
// there until the process exits. Because it lives in its own translation
// unit, the array is only loaded on devices where this entry point is used.
//
// In host code `g_static_ws` names a host-side shadow, not device memory; the
// device address is obtained once per device with cudaGetSymbolAddress (with
// that device current) and only that address is passed to the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "h3attn.h"

namespace {

static __device__ __align__(256) unsigned char g_static_ws[H3_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
void *g_static_ptr[kMaxDevices] = {};
std::mutex g_static_mu;

// Device address of the scratch array on the current device (set-up on the
// first call per device).
h3_status static_workspace(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return H3_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return H3_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || ptr == nullptr)
            return H3_ERR_CUDA;
        g_static_ptr[dev] = ptr;
    }
    *out = g_static_ptr[dev];
    return H3_OK;
}

}  // namespace

extern "C" h3_status h3_varlen_attn_fwd_static(const void *q, const void *k, const void *v,
                                               void *o, float *lse, const int32_t *cu_seqlens,
                                               int32_t nseg, int32_t max_seqlen,
                                               const float *pos, h3_rope_cfg rope, int64_t N,
                                               int32_t H, int32_t D, float softmax_scale,
                                               h3_stream_t stream) {
    // the scratch holds the status block and the rotated keys, bf16 [N, H, D];
    // every other argument is checked by h3_varlen_attn_fwd
    if (h3_workspace_size(N, H, D, nseg) > static_cast<size_t>(H3_STATIC_WORKSPACE_BYTES))
        return H3_ERR_WORKSPACE;
    void *ws = nullptr;
    h3_status st = static_workspace(&ws);
    if (st != H3_OK) return st;
    // h3_varlen_attn_fwd resets the status word on every call and overwrites
    // every rotated-key byte it later reads, so leftovers of an earlier call
    // are never used.
    return h3_varlen_attn_fwd(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos, rope, N, H, D,
                              softmax_scale, ws, static_cast<size_t>(H3_STATIC_WORKSPACE_BYTES),
                              stream);
}
