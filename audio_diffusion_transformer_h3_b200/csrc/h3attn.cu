// C-ABI entry points of libh3attn (declared in include/h3attn.h).
//
// Host side only: argument validation, the rotary frequency table, TMA
// descriptors, launches on the caller's stream, and the host position
// builder. Every step of the device path runs in the kernels of
// rope.cuh, attn_fwd.cuh, attn_sage.cuh and qkv_gemm.cuh; nothing here computes on the host except
// positions (which the pages place on the host: "MiniMax H3 on Moore Threads
// MUSA", section "MUSA validation").
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "h3attn.h"
#include "attn_fwd.cuh"
#include "attn_sage.cuh"
#include "qkv_gemm.cuh"
#include "rope.cuh"

namespace {

thread_local int32_t g_last_cuda_error = 0;

h3_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int32_t>(e);
    return H3_ERR_CUDA;
}

constexpr size_t kStatusBytes = 256;

// Row tiles of the QKV GEMM that sweep the column tiles together (L2 reuse).
constexpr int32_t kQkvGroupM = 32;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------- driver API

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// Per-device one-time set-up: capability check, SM count, kernel attributes.
struct DeviceInfo {
    bool ready = false;
    bool sm100 = false;
    bool attn_regs_ok = false;
    bool sage_regs_ok = false;
    int sms = 0;
    cudaError_t err = cudaSuccess;
};

template <typename Kernel>
bool attn_regs_cover_split(Kernel kernel, int D) {
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return false;
    using C128 = h3::AttnCfg<128>;
    using C64 = h3::AttnCfg<64>;
    const long long need = D == 128
        ? (C128::THREADS - 128LL) * C128::REGS_SOFTMAX + 128LL * C128::REGS_PRODUCER
        : (C64::THREADS - 128LL) * C64::REGS_SOFTMAX + 128LL * C64::REGS_PRODUCER;
    const int threads = D == 128 ? C128::THREADS : C64::THREADS;
    return static_cast<long long>(a.numRegs) * threads >= need;
}

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

h3_status device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return H3_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        d.sm100 = (major == 10 && minor == 0);
        if (d.sm100) {
            if ((e = cudaFuncSetAttribute(h3::attn_fwd_kernel<128, false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::AttnCfg<128>::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::attn_fwd_kernel<64, false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::AttnCfg<64>::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::attn_fwd_kernel<128, true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::AttnCfg<128>::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::attn_fwd_kernel<64, true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::AttnCfg<64>::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::attn_sage_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::SageCfg::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::qkv_rope_gemm_kernel<128>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::QkvCfg::SMEM_BYTES)) != cudaSuccess ||
                (e = cudaFuncSetAttribute(h3::qkv_rope_gemm_kernel<64>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h3::QkvCfg::SMEM_BYTES)) != cudaSuccess)
                return cuda_fail(e);
            // The attention kernels move registers between warpgroups
            // (setmaxnreg); the raise waits for registers the block holds
            // from launch, so refuse to launch a build whose launch
            // allocation cannot cover the split (it would never return).
            d.attn_regs_ok = attn_regs_cover_split(h3::attn_fwd_kernel<128, false>, 128) &&
                             attn_regs_cover_split(h3::attn_fwd_kernel<128, true>, 128) &&
                             attn_regs_cover_split(h3::attn_fwd_kernel<64, false>, 64) &&
                             attn_regs_cover_split(h3::attn_fwd_kernel<64, true>, 64);
            cudaFuncAttributes a{};
            using S = h3::SageCfg;
            d.sage_regs_ok = cudaFuncGetAttributes(&a, h3::attn_sage_kernel) == cudaSuccess &&
                             static_cast<long long>(a.numRegs) * S::THREADS >=
                                 2LL * 128 * S::REGS_SOFTMAX + 128LL * S::REGS_PRODUCER;
        }
        d.ready = true;
    }
    if (!d.sm100) return H3_ERR_UNSUPPORTED;
    *out = &d;
    return H3_OK;
}

// ------------------------------------------------------------------- helpers

// Inverse frequencies theta^(-2j/d_a) formed in double and rounded to float,
// axis chunks in (t, h, w) order.
bool make_rope_table(const h3_rope_cfg &c, int D, h3::RopeTable *rt) {
    const int dims[3] = {c.d_t, c.d_h, c.d_w};
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 0 || (dims[a] & 1)) return false;
    if (c.d_t + c.d_h + c.d_w != D) return false;
    if (!(c.theta > 0.0f) || !std::isfinite(c.theta)) return false;
    std::memset(rt, 0, sizeof(*rt));
    int pr = 0;
    for (int a = 0; a < 3; ++a)
        for (int j = 0; j < dims[a] / 2; ++j)
            rt->inv_freq[pr++] = static_cast<float>(
                std::pow(static_cast<double>(c.theta), -2.0 * j / static_cast<double>(dims[a])));
    rt->n_t = c.d_t / 2;
    rt->n_th = (c.d_t + c.d_h) / 2;
    return true;
}

// TMA map over a bf16 [N, H, D] tensor: dims (D, H, N), box (64, 1, 128),
// 128-byte swizzle, zero fill out of bounds.
h3_status make_thd_map(CUtensorMap *map, const void *base, int64_t N, int H, int D) {
    EncodeTiledFn enc = encode_tiled();
    if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(H) * D * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return H3_OK;
}

// TMA map over a row-major bf16 [rows, cols] matrix: dims (cols, rows), box
// (64, box_rows), 128-byte swizzle, zero fill out of bounds.
h3_status make_2d_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols,
                      uint32_t box_rows) {
    EncodeTiledFn enc = encode_tiled();
    if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return H3_OK;
}

// TMA map over an e4m3 [N, H, 128] tensor: dims (128, H, N) bytes, box
// (128, 1, 128), 128-byte swizzle, zero fill out of bounds.
h3_status make_u8_thd_map(CUtensorMap *map, const void *base, int64_t N, int H) {
    EncodeTiledFn enc = encode_tiled();
    if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(H) * 128};
    const cuuint32_t box[3] = {128, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return H3_OK;
}

// Byte offsets of the SAGE workspace regions (see h3_sage_workspace_size).
struct SageLayout {
    size_t q8, k8, v8, s_q, s_k, v_amax, s_v, total;
};

SageLayout sage_layout(int64_t N, int32_t H, int32_t nseg) {
    SageLayout L;
    const size_t codes = round_up(static_cast<size_t>(N) * H * 128, 256);
    const size_t scales = round_up(static_cast<size_t>(N) * H * 4, 256);
    const size_t vsc = round_up(static_cast<size_t>(nseg) * H * 128 * 4, 256);
    L.q8 = kStatusBytes;
    L.k8 = L.q8 + codes;
    L.v8 = L.k8 + codes;
    L.s_q = L.v8 + codes;
    L.s_k = L.s_q + scales;
    L.v_amax = L.s_k + scales;
    L.s_v = L.v_amax + vsc;
    L.total = L.s_v + vsc;
    return L;
}

h3_status launch_rope(const void *x, void *out, const float *pos, int64_t N, int H, int D,
                      const h3::RopeTable &rt, int sms, cudaStream_t st) {
    const int64_t tok_blocks = (N + 7) / 8;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    const int grid = static_cast<int>(tok_blocks < cap ? tok_blocks : cap);
    if (D == 128)
        h3::rope_apply_kernel<128><<<grid, 256, 0, st>>>(
            static_cast<const uint4 *>(x), static_cast<uint4 *>(out), pos, N, H, rt);
    else
        h3::rope_apply_kernel<64><<<grid, 256, 0, st>>>(
            static_cast<const uint4 *>(x), static_cast<uint4 *>(out), pos, N, H, rt);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? H3_OK : cuda_fail(e);
}

h3_status attn_call(const void *q, const void *k, const void *v, void *o, float *lse,
                    const int32_t *cu_seqlens, int32_t nseg, int32_t max_seqlen,
                    const float *pos, h3_rope_cfg rope, int64_t N, int32_t H, int32_t D,
                    float softmax_scale, void *workspace, size_t workspace_bytes,
                    h3_stream_t stream, bool skip, float skip_threshold,
                    bool reset_status = true) {
    if (N < 0 || N > INT32_MAX - 1 || H < 1 || H > 65535 || nseg < 1 || nseg > 65535)
        return H3_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return H3_ERR_UNSUPPORTED;
    if (!std::isfinite(softmax_scale) || softmax_scale < 0.0f) return H3_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr) return H3_ERR_INVALID_ARG;
    if (N > 0 && (q == nullptr || k == nullptr || v == nullptr || o == nullptr))
        return H3_ERR_INVALID_ARG;
    if (N > 0 && (max_seqlen < 1 || max_seqlen > N)) return H3_ERR_INVALID_ARG;
    h3::RopeTable rt;
    std::memset(&rt, 0, sizeof(rt));
    if (pos != nullptr && !make_rope_table(rope, D, &rt)) return H3_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(pos, 4) || !aligned(lse, 4) || !aligned(cu_seqlens, 4))
        return H3_ERR_MISALIGNED;
    // without positions there are no rotated keys: the status block suffices
    const size_t need = pos != nullptr ? h3_workspace_size(N, H, D, nseg) : kStatusBytes;
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need)
        return H3_ERR_WORKSPACE;

    DeviceInfo *d = nullptr;
    h3_status st = device_info(&d);
    if (st != H3_OK) return st;
    if (!d->attn_regs_ok) return H3_ERR_UNSUPPORTED;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(workspace);
    // status word (and, for the skip variant, the skipped-block counter at byte 8)
    cudaError_t e = reset_status ? cudaMemsetAsync(status, 0, skip ? 16 : sizeof(int), cs)
                                 : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail(e);
    if (N == 0) return H3_OK;

    // keys rotated once into the workspace (the same rotation the attention
    // kernel applies to each query tile)
    const void *k_src = k;
    if (pos != nullptr) {
        void *k_rot = static_cast<uint8_t *>(workspace) + kStatusBytes;
        st = launch_rope(k, k_rot, pos, N, H, D, rt, d->sms, cs);
        if (st != H3_OK) return st;
        k_src = k_rot;
    }

    CUtensorMap tq, tk, tv;
    if ((st = make_thd_map(&tq, q, N, H, D)) != H3_OK) return st;
    if ((st = make_thd_map(&tk, k_src, N, H, D)) != H3_OK) return st;
    if ((st = make_thd_map(&tv, v, N, H, D)) != H3_OK) return st;

    h3::AttnParams p;
    p.cu_seqlens = cu_seqlens;
    p.pos = pos;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.status = status;
    p.nseg = nseg;
    p.max_seqlen = max_seqlen;
    p.N = static_cast<int32_t>(N);
    p.H = H;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.skip_log2 = skip ? static_cast<float>(std::log2(static_cast<double>(skip_threshold))) : 0.0f;
    p.skip_count = skip ? reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + 8)
                        : nullptr;
    p.rope = rt;

    const dim3 grid(static_cast<unsigned>((max_seqlen + 255) / 256), static_cast<unsigned>(H),
                    static_cast<unsigned>(nseg));
    if (D == 128) {
        if (skip)
            h3::attn_fwd_kernel<128, true><<<grid, h3::AttnCfg<128>::THREADS,
                                             h3::AttnCfg<128>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
        else
            h3::attn_fwd_kernel<128, false><<<grid, h3::AttnCfg<128>::THREADS,
                                              h3::AttnCfg<128>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
    } else {
        if (skip)
            h3::attn_fwd_kernel<64, true><<<grid, h3::AttnCfg<64>::THREADS,
                                            h3::AttnCfg<64>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
        else
            h3::attn_fwd_kernel<64, false><<<grid, h3::AttnCfg<64>::THREADS,
                                             h3::AttnCfg<64>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
    }
    e = cudaGetLastError();
    return e == cudaSuccess ? H3_OK : cuda_fail(e);
}

}  // namespace

// ======================================================================= ABI

extern "C" {

int64_t h3_segment_tokens(const h3_segment_layout *s) {
    if (s == nullptr) return -1;
    const int32_t f[10] = {s->image_refs, s->image_h, s->image_w, s->audio_refs,
                           s->audio_ref_len, s->audio_rate, s->video_t, s->video_h,
                           s->video_w, s->audio_tail};
    for (int i = 0; i < 10; ++i)
        if (f[i] < 0) return -1;
    const int64_t n = static_cast<int64_t>(s->image_refs) * s->image_h * s->image_w +
                      static_cast<int64_t>(s->audio_refs) * s->audio_ref_len +
                      static_cast<int64_t>(s->video_t) * s->video_h * s->video_w +
                      s->audio_tail;
    return n > INT32_MAX ? -1 : n;
}

h3_status h3_build_positions(const h3_segment_layout *segs, int32_t nseg, float *pos,
                             int64_t capacity, int32_t *cu_seqlens) {
    return h3_build_positions_at(segs, nseg, nullptr, pos, capacity, cu_seqlens);
}

h3_status h3_build_positions_at(const h3_segment_layout *segs, int32_t nseg,
                                const double *t_origin, float *pos, int64_t capacity,
                                int32_t *cu_seqlens) {
    if (nseg < 0 || (nseg > 0 && segs == nullptr) || capacity < 0) return H3_ERR_INVALID_ARG;
    if (t_origin != nullptr)
        for (int32_t s = 0; s < nseg; ++s)
            if (!std::isfinite(t_origin[s])) return H3_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int32_t s = 0; s < nseg; ++s) {
        const int64_t n = h3_segment_tokens(&segs[s]);
        if (n < 0) return H3_ERR_INVALID_ARG;
        if (segs[s].audio_refs > 0 && segs[s].audio_ref_len > 0 && segs[s].audio_rate <= 0)
            return H3_ERR_INVALID_ARG;
        total += n;
    }
    if (total > capacity || total > INT32_MAX || (total > 0 && pos == nullptr))
        return H3_ERR_INVALID_ARG;
    int64_t n = 0;
    if (cu_seqlens) cu_seqlens[0] = 0;
    for (int32_t s = 0; s < nseg; ++s) {
        const h3_segment_layout &g = segs[s];
        double t0 = t_origin != nullptr ? t_origin[s] : 0.0;
        auto put = [&](double t, double h, double w) {
            pos[3 * n + 0] = static_cast<float>(t);
            pos[3 * n + 1] = static_cast<float>(h);
            pos[3 * n + 2] = static_cast<float>(w);
            ++n;
        };
        for (int r = 0; r < g.image_refs; ++r) {
            for (int h = 0; h < g.image_h; ++h)
                for (int w = 0; w < g.image_w; ++w) put(t0, h, w);
            t0 = t0 + 1.0;
        }
        for (int r = 0; r < g.audio_refs; ++r) {
            for (int i = 0; i < g.audio_ref_len; ++i)
                put(t0 + static_cast<double>(i) / static_cast<double>(g.audio_rate), 0.0, 0.0);
            if (g.audio_ref_len > 0)
                t0 = t0 + static_cast<double>(g.audio_ref_len) / static_cast<double>(g.audio_rate);
        }
        for (int tau = 0; tau < g.video_t; ++tau)
            for (int h = 0; h < g.video_h; ++h)
                for (int w = 0; w < g.video_w; ++w) put(t0 + static_cast<double>(tau), h, w);
        for (int i = 0; i < g.audio_tail; ++i)
            put(t0 + (static_cast<double>(i) * static_cast<double>(g.video_t)) /
                         static_cast<double>(g.audio_tail),
                0.0, 0.0);
        if (cu_seqlens) cu_seqlens[s + 1] = static_cast<int32_t>(n);
    }
    return H3_OK;
}

h3_status h3_rope_apply(const void *x, void *out, const float *pos, int64_t N, int32_t H,
                        int32_t D, h3_rope_cfg rope, h3_stream_t stream) {
    if (N < 0 || H < 1) return H3_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return H3_ERR_UNSUPPORTED;
    h3::RopeTable rt;
    if (!make_rope_table(rope, D, &rt)) return H3_ERR_INVALID_ARG;
    if (N > 0 && (x == nullptr || out == nullptr || pos == nullptr)) return H3_ERR_INVALID_ARG;
    if (static_cast<double>(N) * H * D >= 1099511627776.0) return H3_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(pos, 4)) return H3_ERR_MISALIGNED;
    if (N == 0) return H3_OK;
    DeviceInfo *d = nullptr;
    h3_status st = device_info(&d);
    if (st != H3_OK) return st;
    return launch_rope(x, out, pos, N, H, D, rt, d->sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t h3_workspace_size(int64_t N, int32_t H, int32_t D, int32_t nseg) {
    (void)nseg;
    if (N < 0 || H < 0 || D < 0) return kStatusBytes;
    return kStatusBytes + round_up(static_cast<size_t>(N) * H * D * 2, 256);
}

h3_status h3_varlen_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                             const int32_t *cu_seqlens, int32_t nseg, int32_t max_seqlen,
                             const float *pos, h3_rope_cfg rope, int64_t N, int32_t H,
                             int32_t D, float softmax_scale, void *workspace,
                             size_t workspace_bytes, h3_stream_t stream) {
    return attn_call(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos, rope, N, H, D,
                     softmax_scale, workspace, workspace_bytes, stream, false, 0.0f);
}

h3_status h3_varlen_attn_fwd_skip(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *cu_seqlens, int32_t nseg,
                                  int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                                  int64_t N, int32_t H, int32_t D, float softmax_scale,
                                  float skip_threshold, void *workspace, size_t workspace_bytes,
                                  h3_stream_t stream) {
    if (!(skip_threshold >= 0.0f && skip_threshold <= 1.0f)) return H3_ERR_INVALID_ARG;
    return attn_call(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos, rope, N, H, D,
                     softmax_scale, workspace, workspace_bytes, stream, true, skip_threshold);
}

h3_status h3_qkv_rope_gemm(const void *x, const void *w, void *q, void *k, void *v,
                           const float *pos, h3_rope_cfg rope, int64_t N, int32_t K,
                           int32_t H, int32_t D, void *workspace, size_t workspace_bytes,
                           h3_stream_t stream) {
    if (N < 0 || N > INT32_MAX - 256 || H < 1 || K < 64 || K > (1 << 20) || (K % 64) != 0)
        return H3_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return H3_ERR_UNSUPPORTED;
    const int64_t HD = static_cast<int64_t>(H) * D;
    if ((HD % 256) != 0 || 3 * HD > (1 << 20)) return H3_ERR_INVALID_ARG;
    if (N > 0 && (x == nullptr || w == nullptr || q == nullptr || k == nullptr || v == nullptr))
        return H3_ERR_INVALID_ARG;
    h3::RopeTable rt;
    std::memset(&rt, 0, sizeof(rt));
    if (pos != nullptr && !make_rope_table(rope, D, &rt)) return H3_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(q, 16) || !aligned(k, 16) ||
        !aligned(v, 16) || !aligned(pos, 4))
        return H3_ERR_MISALIGNED;
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < kStatusBytes)
        return H3_ERR_WORKSPACE;
    DeviceInfo *d = nullptr;
    h3_status st = device_info(&d);
    if (st != H3_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(workspace);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), cs);
    if (e != cudaSuccess) return cuda_fail(e);
    if (N == 0) return H3_OK;

    using C = h3::QkvCfg;
    h3::QkvParams p;
    p.q = static_cast<__nv_bfloat16 *>(q);
    p.k = static_cast<__nv_bfloat16 *>(k);
    p.v = static_cast<__nv_bfloat16 *>(v);
    p.pos = pos;
    p.status = status;
    p.N = static_cast<int32_t>(N);
    p.K = K;
    p.HD = static_cast<int32_t>(HD);
    p.n_row_tiles = static_cast<int32_t>((N + C::BM - 1) / C::BM);
    p.n_col_tiles = static_cast<int32_t>(3 * HD / C::BN);
    const int64_t n_tiles = static_cast<int64_t>(p.n_row_tiles) * p.n_col_tiles;
    if (n_tiles > INT32_MAX) return H3_ERR_INVALID_ARG;
    p.n_tiles = static_cast<int32_t>(n_tiles);
    p.group_m = kQkvGroupM;
    p.rope = rt;

    CUtensorMap tx, tw;
    if ((st = make_2d_map(&tx, x, N, K, C::BM)) != H3_OK) return st;
    if ((st = make_2d_map(&tw, w, 3 * HD, K, C::BN)) != H3_OK) return st;
    const int grid = static_cast<int>(n_tiles < d->sms ? n_tiles : d->sms);
    if (D == 128)
        h3::qkv_rope_gemm_kernel<128><<<grid, C::THREADS, C::SMEM_BYTES, cs>>>(tx, tw, p);
    else
        h3::qkv_rope_gemm_kernel<64><<<grid, C::THREADS, C::SMEM_BYTES, cs>>>(tx, tw, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? H3_OK : cuda_fail(e);
}

h3_status h3_qkv_rope_attn_fwd(const void *x, const void *w, void *q, void *k, void *v,
                               void *o, float *lse, const int32_t *cu_seqlens, int32_t nseg,
                               int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                               int64_t N, int32_t K, int32_t H, int32_t D, float softmax_scale,
                               void *workspace, size_t workspace_bytes, h3_stream_t stream) {
    // the attention's own checks first, so that nothing is launched for a
    // call it would refuse (its pointers are the GEMM's outputs)
    if (N < 0 || N > INT32_MAX - 1 || H < 1 || H > 65535 || nseg < 1 || nseg > 65535)
        return H3_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return H3_ERR_UNSUPPORTED;
    if (!std::isfinite(softmax_scale) || softmax_scale < 0.0f || cu_seqlens == nullptr)
        return H3_ERR_INVALID_ARG;
    if (N > 0 && (o == nullptr || max_seqlen < 1 || max_seqlen > N)) return H3_ERR_INVALID_ARG;
    if (!aligned(o, 16) || !aligned(lse, 4) || !aligned(cu_seqlens, 4)) return H3_ERR_MISALIGNED;
    // q, k, v = x w^T with q and k rotated in the GEMM's epilogue; this call
    // resets the status word
    h3_status st = h3_qkv_rope_gemm(x, w, q, k, v, pos, rope, N, K, H, D, workspace,
                                    workspace_bytes, stream);
    if (st != H3_OK) return st;
    // attention on the rotated q and k (no positions: no key pass and no
    // rotated-key workspace); the status word keeps the GEMM's first error
    return attn_call(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, nullptr, rope, N, H, D,
                     softmax_scale, workspace, workspace_bytes, stream, false, 0.0f, false);
}

size_t h3_sage_workspace_size(int64_t N, int32_t H, int32_t D, int32_t nseg) {
    if (N < 0 || H < 0 || D != 128 || nseg < 0) return 0;
    return sage_layout(N, H, nseg).total;
}

h3_status h3_varlen_attn_fwd_sage(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *cu_seqlens, int32_t nseg,
                                  int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                                  int64_t N, int32_t H, int32_t D, float softmax_scale,
                                  void *workspace, size_t workspace_bytes, h3_stream_t stream) {
    if (N < 0 || N > INT32_MAX - 1 || H < 1 || H > 65535 || nseg < 1 || nseg > 65535)
        return H3_ERR_INVALID_ARG;
    if (D != 128) return H3_ERR_UNSUPPORTED;
    if (!std::isfinite(softmax_scale) || softmax_scale < 0.0f) return H3_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr) return H3_ERR_INVALID_ARG;
    if (N > 0 && (q == nullptr || k == nullptr || v == nullptr || o == nullptr))
        return H3_ERR_INVALID_ARG;
    if (N > 0 && (max_seqlen < 1 || max_seqlen > N)) return H3_ERR_INVALID_ARG;
    h3::RopeTable rt;
    std::memset(&rt, 0, sizeof(rt));
    if (pos != nullptr && !make_rope_table(rope, D, &rt)) return H3_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(pos, 4) || !aligned(lse, 4) || !aligned(cu_seqlens, 4))
        return H3_ERR_MISALIGNED;
    const SageLayout lay = sage_layout(N, H, nseg);
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < lay.total)
        return H3_ERR_WORKSPACE;

    DeviceInfo *d = nullptr;
    h3_status st = device_info(&d);
    if (st != H3_OK) return st;
    if (!d->sage_regs_ok) return H3_ERR_UNSUPPORTED;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), cs);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ws + lay.v_amax, 0, static_cast<size_t>(nseg) * H * 128 * 4, cs);
    if (e != cudaSuccess) return cuda_fail(e);
    if (N == 0) return H3_OK;

    h3::SageQuantParams qp;
    qp.q = static_cast<const __nv_bfloat16 *>(q);
    qp.k = static_cast<const __nv_bfloat16 *>(k);
    qp.v = static_cast<const __nv_bfloat16 *>(v);
    qp.cu_seqlens = cu_seqlens;
    qp.pos = pos;
    qp.q8 = ws + lay.q8;
    qp.k8 = ws + lay.k8;
    qp.v8 = ws + lay.v8;
    qp.s_q = reinterpret_cast<float *>(ws + lay.s_q);
    qp.s_k = reinterpret_cast<float *>(ws + lay.s_k);
    qp.v_amax = reinterpret_cast<unsigned *>(ws + lay.v_amax);
    qp.s_v = reinterpret_cast<float *>(ws + lay.s_v);
    qp.status = status;
    qp.nseg = nseg;
    qp.max_seqlen = max_seqlen;
    qp.N = static_cast<int32_t>(N);
    qp.H = H;
    qp.rope = rt;
    const dim3 qgrid(static_cast<unsigned>((max_seqlen + 127) / 128), static_cast<unsigned>(H),
                     static_cast<unsigned>(nseg));
    const dim3 bgrid(static_cast<unsigned>((max_seqlen + 15) / 16), static_cast<unsigned>(nseg));
    h3::sage_vamax_kernel<<<qgrid, 256, 0, cs>>>(qp);
    h3::sage_quant_kernel<<<bgrid, 256, 0, cs>>>(qp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);

    CUtensorMap tq, tk, tv;
    if ((st = make_u8_thd_map(&tq, qp.q8, N, H)) != H3_OK) return st;
    if ((st = make_u8_thd_map(&tk, qp.k8, N, H)) != H3_OK) return st;
    if ((st = make_u8_thd_map(&tv, qp.v8, N, H)) != H3_OK) return st;
    h3::SageAttnParams ap;
    ap.cu_seqlens = cu_seqlens;
    ap.s_q = qp.s_q;
    ap.s_k = qp.s_k;
    ap.s_v = qp.s_v;
    ap.o = static_cast<__nv_bfloat16 *>(o);
    ap.lse = lse;
    ap.status = status;
    ap.nseg = nseg;
    ap.max_seqlen = max_seqlen;
    ap.N = static_cast<int32_t>(N);
    ap.H = H;
    ap.scale_log2 = softmax_scale * 1.4426950408889634f;
    const dim3 grid(static_cast<unsigned>((max_seqlen + 255) / 256), static_cast<unsigned>(H),
                    static_cast<unsigned>(nseg));
    h3::attn_sage_kernel<<<grid, h3::SageCfg::THREADS, h3::SageCfg::SMEM_BYTES, cs>>>(tq, tk,
                                                                                     tv, ap);
    e = cudaGetLastError();
    return e == cudaSuccess ? H3_OK : cuda_fail(e);
}

h3_status h3_read_skip_count(const void *workspace, h3_stream_t stream, uint64_t *count) {
    if (workspace == nullptr) return H3_ERR_WORKSPACE;
    if (count == nullptr) return H3_ERR_INVALID_ARG;
    unsigned long long host = 0;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&host, static_cast<const uint8_t *>(workspace) + 8,
                                    sizeof(host), cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e);
    *count = static_cast<uint64_t>(host);
    return H3_OK;
}

h3_status h3_selftest_bounded_wait(void *workspace, size_t workspace_bytes,
                                   int64_t limit_cycles, h3_stream_t stream) {
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < kStatusBytes)
        return H3_ERR_WORKSPACE;
    if (limit_cycles < 1 || limit_cycles > 4000000000LL) return H3_ERR_INVALID_ARG;
    DeviceInfo *d = nullptr;
    h3_status st = device_info(&d);
    if (st != H3_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(workspace);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), cs);
    if (e != cudaSuccess) return cuda_fail(e);
    h3::bounded_wait_selftest_kernel<<<1, 32, 0, cs>>>(status, static_cast<long long>(limit_cycles));
    e = cudaGetLastError();
    return e == cudaSuccess ? H3_OK : cuda_fail(e);
}

h3_status h3_read_device_status(const void *workspace, h3_stream_t stream) {
    if (workspace == nullptr) return H3_ERR_WORKSPACE;
    int host = 0;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e);
    return static_cast<h3_status>(host);
}

const char *h3_status_string(h3_status s) {
    switch (s) {
        case H3_OK: return "ok";
        case H3_ERR_INVALID_ARG: return "invalid argument";
        case H3_ERR_UNSUPPORTED: return "unsupported (head dim or device)";
        case H3_ERR_MISALIGNED: return "misaligned pointer";
        case H3_ERR_WORKSPACE: return "workspace missing or too small";
        case H3_ERR_CUDA: return "CUDA error";
        case H3_ERR_DEVICE_TIMEOUT: return "bounded device wait timed out";
        case H3_ERR_BAD_SEQLENS: return "invalid cu_seqlens";
    }
    return "unknown status";
}

int32_t h3_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
