// 3-axis (t, h, w) rotary embedding on the shared audio/video clock.
//
// Operation: "Day 0 Support for MiniMax-H3 on AMD Instinct GPUs", section
// "The diffusion transformer (DiT)" (position encoding: Rotary). Positions
// are fp32 on the device ("MiniMax H3 on Moore Threads MUSA", section "MUSA
// validation": FP64 host metadata cast to FP32 before device arithmetic).
// Pair layout and frequency schedule: the head dim is split into contiguous
// (d_t, d_h, d_w) chunks; pair j of axis a is channels (c_a+2j, c_a+2j+1),
// rotated by pos[a] * theta^(-2j/d_a).
//
// The same device functions rotate q inside the attention kernel and k (or
// any x) in the standalone pass, so both are bit-identical.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace h3 {

// Per-pair inverse frequencies (rounded from double on the host) and the
// pair-index bounds of the t and h chunks. Passed by value as a kernel
// parameter (constant bank).
struct RopeTable {
    float inv_freq[64];
    int32_t n_t;   // pairs [0, n_t) rotate with pos.t
    int32_t n_th;  // pairs [n_t, n_th) with pos.h, [n_th, D/2) with pos.w
};

__device__ __forceinline__ int rope_axis(const RopeTable &rt, int pair) {
    return pair < rt.n_t ? 0 : (pair < rt.n_th ? 1 : 2);
}

// cos and sin of the angle pos * inv_freq (fp32 product, accurate sincosf).
__device__ __forceinline__ void rope_cos_sin(float p, float inv_freq, float &c, float &s) {
    const float phi = __fmul_rn(p, inv_freq);
    sincosf(phi, &s, &c);
}

// (x0, x1) -> (x0 c - x1 s, x0 s + x1 c) with a fixed rounding sequence.
__device__ __forceinline__ void rope_rotate(float x0, float x1, float c, float s, float &y0,
                                            float &y1) {
    y0 = __fmaf_rn(x0, c, -__fmul_rn(x1, s));
    y1 = __fmaf_rn(x0, s, __fmul_rn(x1, c));
}

// Rotates one 32-bit word holding a bf16 pair (low half = even channel).
__device__ __forceinline__ uint32_t rope_word(uint32_t w, float c, float s) {
    const float x0 = __uint_as_float(w << 16);
    const float x1 = __uint_as_float(w & 0xFFFF0000u);
    float y0, y1;
    rope_rotate(x0, x1, c, s, y0, y1);
    __nv_bfloat162 r = __floats2bfloat162_rn(y0, y1);  // .x (low) = y0
    return *reinterpret_cast<uint32_t *>(&r);
}

// Standalone pass: out = RoPE(x, pos), x/out bf16 [N, H, D], pos fp32 [N, 3].
// A block takes TOK tokens at a time: first it computes the TOK x D/2
// (cos, sin) pairs once (shared by all H heads), then it streams the TOK*H*D
// bf16 values as 16-byte vectors, four in flight per thread.
template <int D>
__global__ void __launch_bounds__(256) rope_apply_kernel(const uint4 *x, uint4 *out,
                                                         const float *__restrict__ pos,
                                                         int64_t N, int32_t H,
                                                         const RopeTable rt) {
    constexpr int TOK = 8;
    constexpr int NP = D / 2;        // pairs per head
    constexpr int VPH = D / 8;       // 16-byte vectors per head
    __shared__ float2 cs[TOK][NP];
    const int64_t vpt = static_cast<int64_t>(H) * VPH;  // vectors per token
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * TOK; base < N;
         base += static_cast<int64_t>(gridDim.x) * TOK) {
        for (int i = threadIdx.x; i < TOK * NP; i += blockDim.x) {
            const int t = i / NP, pr = i % NP;
            const int64_t n = base + t;
            float c = 1.f, s = 0.f;
            if (n < N) rope_cos_sin(pos[n * 3 + rope_axis(rt, pr)], rt.inv_freq[pr], c, s);
            cs[t][pr] = make_float2(c, s);
        }
        __syncthreads();
        const int64_t ntok = (N - base) < TOK ? (N - base) : TOK;
        const int64_t total = ntok * vpt;
        const uint4 *src = x + base * vpt;
        uint4 *dst = out + base * vpt;
        for (int64_t i0 = threadIdx.x; i0 < total; i0 += 4 * static_cast<int64_t>(blockDim.x)) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t i = i0 + static_cast<int64_t>(u) * blockDim.x;
                if (i < total) v[u] = src[i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t i = i0 + static_cast<int64_t>(u) * blockDim.x;
                if (i < total) {
                    const int t = static_cast<int>(i / vpt);
                    const int pr0 = static_cast<int>(i % VPH) * 4;  // first pair of the vector
                    const float2 c0 = cs[t][pr0 + 0], c1 = cs[t][pr0 + 1];
                    const float2 c2 = cs[t][pr0 + 2], c3 = cs[t][pr0 + 3];
                    uint4 r;
                    r.x = rope_word(v[u].x, c0.x, c0.y);
                    r.y = rope_word(v[u].y, c1.x, c1.y);
                    r.z = rope_word(v[u].z, c2.x, c2.y);
                    r.w = rope_word(v[u].w, c3.x, c3.y);
                    dst[i] = r;
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace h3
