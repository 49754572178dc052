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
// there until the process exits. Under CUDA's lazy module loading (the
// default, CUDA_MODULE_LOADING=LAZY) the module, and with it the array, is
// loaded only on devices where this entry point is called; with
// CUDA_MODULE_LOADING=EAGER every context that maps the library loads it and
// holds the array, whether or not this entry point is ever used.
//
// In host code `g_static_ws` names a host-side shadow, not device memory. The
// device address is looked up with cudaGetSymbolAddress, with the calling
// device current, on every call (once the module is loaded this is a host-side
// table lookup), and only that address is passed to the kernels. Looking it
// up on every call rather than caching it keeps the entry point valid when
// the primary context is destroyed and recreated (cudaDeviceReset), which
// reloads the module and may place the array at a new address. The first call
// on a device loads the module, so it should come before any stream capture.
#include <cuda_runtime.h>

#include <cstdint>

#include "h3attn.h"

namespace {

static __device__ __align__(256) unsigned char g_static_ws[H3_STATIC_WORKSPACE_BYTES];

// Device address of the scratch array on the current device.
h3_status static_workspace(void **out) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_ws);
    if (e != cudaSuccess || ptr == nullptr) return H3_ERR_CUDA;
    *out = ptr;
    return H3_OK;
}

}  // namespace

extern "C" h3_status h3_varlen_attn_fwd_static(const void *q, const void *k, const void *v,
                                               void *o, float *lse, const int32_t *cu_seqlens,
                                               int32_t nseg, int32_t max_seqlen,
                                               const float *pos, h3_rope_cfg rope, int64_t N,
                                               int32_t H, int32_t D, float softmax_scale,
                                               h3_stream_t stream) {
    // The shape checks of h3_varlen_attn_fwd come first, so that a call that
    // is both malformed and too large reports the same status as there.
    if (N < 0 || N > INT32_MAX - 1 || H < 1 || H > 65535 || nseg < 1 || nseg > 65535)
        return H3_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return H3_ERR_UNSUPPORTED;
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
