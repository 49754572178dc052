// SAGE-style FP8 attention (lossy variant of the fused RoPE + packed varlen
// attention), sm_100a, head dim 128.
//
// "MiniMax H3" vLLM-Omni recipe, section "Attention Backends": SAGE
// quantisation with fp8_e4m3 Q/K at q_block_size 1 and k_block_size 16, P and
// V in FP8. Reading used here:
//   Q~ = RoPE(q), K~ = RoPE(k) in fp32;
//   Q: one scale per (token, head): a = max |Q~|, code = e4m3(Q~ * (448 / a)),
//      dequantisation scale s_q = a / 448;
//   K: one scale per (16-key block, head), blocks from the segment start;
//   V: one scale per (segment, head, channel);
//   scores x = (q8 . k8) * s_q * s_k * softmax_scale * log2(e);
//   online softmax over key tiles of 128 with a lazily updated reference max
//   m: m is raised to the running max only when a tile's max exceeds it by
//   more than 2 (log2 units), so 2^(x - m) <= 4; P8 = e4m3(112 * 2^(x - m))
//   (<= 448); the row sum l adds the unquantised 112 * 2^(x - m);
//   O = s_v * (P8 V8) / l. Exponentials: half on MUFU (ex2.approx), half
//   on the FMA pipe (exp2_fma2_deg2: a degree-2 polynomial, relative error
//   below 1.8e-3, well inside e4m3's 2^-3 relative spacing of the P codes;
//   tiles with masked keys use ex2.approx throughout), which shares the load
//   between the two pipes;
//   the scale-and-shift of the scores and the row sums run as packed f32x2
//   FFMA/FADD.
// e4m3 conversions round to nearest even and saturate to +-448
// (cvt.rn.satfinite).
//
// Three launches:
//   sage_vamax_kernel   per (segment, head, channel) max |v| (atomicMax on the
//                       bit patterns of non-negative floats);
//   sage_quant_kernel   RoPE + quantisation of q, k, v into e4m3 codes and
//                       scales; one CTA per 16-token block (all heads, the
//                       block's rotary table computed once), lane = 4 channels;
//   attn_sage_kernel    the attention kernel of attn_fwd.cuh in FP8, with its
//                       earlier schedule (one MMA warp, the two softmax
//                       warpgroups free-running, P released at once; 384
//                       threads, setmaxnreg moving registers to the softmax
//                       warpgroups) and TMEM plan, tcgen05.mma
//                       kind::f8f6f4 for S = Q8 K8^T (A, B K-major in shared
//                       memory) and O += P8 V8 (A = P8 from TMEM, four codes per
//                       32-bit column; B = V8 MN-major), 16 KB tiles in a
//                       three-stage K/V ring.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "attn_fwd.cuh"   // status codes, raise_abort
#include "rope.cuh"
#include "sm100.cuh"

namespace h3 {

constexpr float kE4m3Max = 448.0f;
constexpr float kLazyLog2 = 2.0f;                  // lazy max threshold (log2 units)
constexpr float kLog2PScale = 6.807354922057604f;  // log2(448 / 2^kLazyLog2) = log2(112)

struct SageQuantParams {
    const __nv_bfloat16 *q, *k, *v;   // [N, H, 128]
    const int32_t *cu_seqlens;        // [nseg + 1]
    const float *pos;                 // [N, 3] or nullptr
    uint8_t *q8, *k8, *v8;            // [N, H, 128] e4m3 codes
    float *s_q, *s_k;                 // [H, N] dequantisation scales (s_k per token)
    unsigned *v_amax;                 // [nseg, H, 128] bit patterns of max |v|
    float *s_v;                       // [nseg, H, 128] dequantisation scales
    int *status;
    int32_t nseg, max_seqlen, N, H;
    RopeTable rope;
};

struct SageAttnParams {
    const int32_t *cu_seqlens;
    const float *s_q, *s_k, *s_v;
    __nv_bfloat16 *o;                 // [N, H, 128]
    float *lse;                       // [H, N] or nullptr
    int *status;
    int32_t nseg, max_seqlen, N, H;
    float scale_log2;
};

// (e4m3(lo), e4m3(hi)) in one 16-bit half, lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t e4m3x4(float a0, float a1, float a2, float a3) {
    return e4m3x2(a0, a1) | (e4m3x2(a2, a3) << 16);
}

// The segment's bounds, checked against N and max_seqlen before any access;
// false (and H3_ERR_BAD_SEQLENS in the status word) if they are invalid.
__device__ __forceinline__ bool sage_segment(const int32_t *cu, int seg, int N, int max_seqlen,
                                             int *status, int &a, int &e) {
    a = cu[seg];
    e = cu[seg + 1];
    if (a < 0 || e < a || e > N || e - a > max_seqlen) {
        atomicCAS(status, kStatusOk, kStatusBadSeqlens);
        return false;
    }
    return true;
}

// grid (ceil(max_seqlen / 128), H, nseg), 256 threads: 16 token rows x 16
// chunks of 8 channels; partial maxima reduced through shared memory.
__global__ void __launch_bounds__(256) sage_vamax_kernel(const SageQuantParams p) {
    __shared__ float part[16][128];
    const int seg = blockIdx.z, head = blockIdx.y, tile = blockIdx.x;
    int a, e;
    if (!sage_segment(p.cu_seqlens, seg, p.N, p.max_seqlen, p.status, a, e)) return;
    const int t0 = a + tile * 128;
    if (t0 >= e) return;
    const int t1 = min(e, t0 + 128);
    const int r = threadIdx.x >> 4, c = threadIdx.x & 15;
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.0f;
    for (int t = t0 + r; t < t1; t += 16) {
        const uint4 u = *reinterpret_cast<const uint4 *>(
            p.v + (static_cast<int64_t>(t) * p.H + head) * 128 + c * 8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[2 * i] = fmaxf(m[2 * i], fabsf(__uint_as_float(w[i] << 16)));
            m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) part[r][c * 8 + i] = m[i];
    __syncthreads();
    if (threadIdx.x < 128) {
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = fmaxf(mx, part[i][threadIdx.x]);
        atomicMax(&p.v_amax[(static_cast<int64_t>(seg) * p.H + head) * 128 + threadIdx.x],
                  __float_as_uint(mx));
    }
}

// grid (ceil(max_seqlen / 16), nseg), 256 threads. A CTA takes one 16-token
// block of a segment (the K scale block, counted from the segment start) for
// every head: it first builds the block's (cos, sin) table (16 tokens x 64
// pairs) in shared memory, then warp w quantises heads w, w + 8, ...; lane l
// holds channels 4l .. 4l+3 (rotary pairs 2l and 2l+1). All 48 row fragments
// of a (block, head) are loaded before the first store.
// Two CTAs per SM (at most 128 registers a thread): the second CTA's loads
// overlap the first one's arithmetic (measured 1.13 against 1.54 ms at 78,408
// tokens x 48 heads, codes bit-identical).
__global__ void __launch_bounds__(256, 2) sage_quant_kernel(const SageQuantParams p) {
    __shared__ float4 cs[16][32];   // per token and lane: (cos, sin) of pairs 2l, 2l+1
    const int seg = blockIdx.y, blk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int a, e;
    if (!sage_segment(p.cu_seqlens, seg, p.N, p.max_seqlen, p.status, a, e)) return;
    const int b0 = a + blk * 16;
    if (blk == 0) {
        // per-channel dequantisation scales of V (also for an empty segment)
        for (int i = threadIdx.x; i < p.H * 128; i += 256) {
            const int64_t at = static_cast<int64_t>(seg) * p.H * 128 + i;
            p.s_v[at] = __fdiv_rn(__uint_as_float(p.v_amax[at]), kE4m3Max);
        }
    }
    if (b0 >= e) return;
    const int n = min(16, e - b0);
    for (int i = threadIdx.x; i < 16 * 32; i += 256) {
        const int j = i >> 5, l = i & 31;
        float c0 = 1.0f, s0 = 0.0f, c1 = 1.0f, s1 = 0.0f;
        if (p.pos != nullptr && j < n) {
            const float *pp = p.pos + static_cast<int64_t>(b0 + j) * 3;
            rope_cos_sin(pp[rope_axis(p.rope, 2 * l)], p.rope.inv_freq[2 * l], c0, s0);
            rope_cos_sin(pp[rope_axis(p.rope, 2 * l + 1)], p.rope.inv_freq[2 * l + 1], c1, s1);
        }
        cs[j][l] = make_float4(c0, s0, c1, s1);
    }
    __syncthreads();
    const bool rotate = p.pos != nullptr;
    for (int head = warp; head < p.H; head += 8) {
        auto row = [&](int j) {
            return (static_cast<int64_t>(b0 + j) * p.H + head) * 128 + lane * 4;
        };
        uint2 qraw[16], kraw[16], vraw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const bool in = j < n;
            kraw[j] = in ? __ldg(reinterpret_cast<const uint2 *>(p.k + row(j))) : make_uint2(0, 0);
            qraw[j] = in ? __ldg(reinterpret_cast<const uint2 *>(p.q + row(j))) : make_uint2(0, 0);
            vraw[j] = in ? __ldg(reinterpret_cast<const uint2 *>(p.v + row(j))) : make_uint2(0, 0);
        }
        const int64_t vrow = (static_cast<int64_t>(seg) * p.H + head) * 128 + lane * 4;
        float vinv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float am = __uint_as_float(p.v_amax[vrow + i]);
            vinv[i] = am > 0.0f ? __fdiv_rn(kE4m3Max, am) : 0.0f;
        }
        float kx[16][4];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
#pragma unroll
            for (int i = 0; i < 4; ++i) kx[j][i] = 0.0f;
            if (j >= n) continue;
            const int t = b0 + j;
            const int64_t off = row(j);
            const float4 c = cs[j][lane];
            // Q: rotate, one scale for the token
            {
                const uint2 u = qraw[j];
                float x[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                              __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
                if (rotate) {
                    rope_rotate(x[0], x[1], c.x, c.y, x[0], x[1]);
                    rope_rotate(x[2], x[3], c.z, c.w, x[2], x[3]);
                }
                const float lm = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
                const float am = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(lm)));
                const float inv = am > 0.0f ? __fdiv_rn(kE4m3Max, am) : 0.0f;
                *reinterpret_cast<uint32_t *>(p.q8 + off) =
                    e4m3x4(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv), __fmul_rn(x[2], inv),
                           __fmul_rn(x[3], inv));
                if (lane == 0) p.s_q[static_cast<int64_t>(head) * p.N + t] = __fdiv_rn(am, kE4m3Max);
            }
            // K: rotate, keep for the block scale
            {
                const uint2 u = kraw[j];
                float x[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                              __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
                if (rotate) {
                    rope_rotate(x[0], x[1], c.x, c.y, x[0], x[1]);
                    rope_rotate(x[2], x[3], c.z, c.w, x[2], x[3]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) kx[j][i] = x[i];
            }
            // V: per-channel scales
            {
                const uint2 u = vraw[j];
                const float x[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                                    __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u)};
                *reinterpret_cast<uint32_t *>(p.v8 + off) =
                    e4m3x4(__fmul_rn(x[0], vinv[0]), __fmul_rn(x[1], vinv[1]),
                           __fmul_rn(x[2], vinv[2]), __fmul_rn(x[3], vinv[3]));
            }
        }
        // K block scale over the block's tokens and channels
        float lm = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) lm = fmaxf(lm, fabsf(kx[j][i]));
        const float am = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(lm)));
        const float inv = am > 0.0f ? __fdiv_rn(kE4m3Max, am) : 0.0f;
        const float sk = __fdiv_rn(am, kE4m3Max);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j >= n) continue;
            *reinterpret_cast<uint32_t *>(p.k8 + row(j)) =
                e4m3x4(__fmul_rn(kx[j][0], inv), __fmul_rn(kx[j][1], inv),
                       __fmul_rn(kx[j][2], inv), __fmul_rn(kx[j][3], inv));
        }
        if (lane < n) p.s_k[static_cast<int64_t>(head) * p.N + b0 + lane] = sk;
    }
}

// ------------------------------------------------------------ FP8 attention

// Instruction descriptor of tcgen05.mma kind::f8f6f4: e4m3 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                                      // D format: f32
           | (0u << 7)                                    // A format: e4m3
           | (0u << 10)                                   // B format: e4m3
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f8_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate,
                                             uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

// 2^x for two lanes on the FMA and integer pipes, for P values that are
// rounded to e4m3 next: the split of exp2_fma (x = j + f, j = rint(x) by adding
// and subtracting 1.5 * 2^23, j added to the exponent field) with a degree-2
// polynomial for 2^f on [-1/2, 1/2] instead of degree 3. Its coefficients
// minimise the largest relative error (Lawson's iteratively reweighted least
// squares on a fine grid): below 1.8e-3, against e4m3's relative spacing of
// 2^-3, so a code moves by at most one step and only when the exact value
// lies within 1.8e-3 of a rounding boundary. One FFMA2 fewer than exp2_fma2.
__device__ __forceinline__ void exp2_fma2_deg2(float &y0, float &y1, float x0, float x1) {
    x0 = fmaxf(x0, -126.0f);
    x1 = fmaxf(x1, -126.0f);
    uint32_t t0, t1, p0, p1;
    asm("{\n\t.reg .b64 xa, ta, ra, fa, pa, sh, nsh, nm1, c0, c1, c2;\n\t"
        "mov.b64 xa, {%4, %5};\n\t"
        "mov.b64 sh, {%6, %6};\n\t"
        "mov.b64 nsh, {%7, %7};\n\t"
        "mov.b64 nm1, {%8, %8};\n\t"
        "mov.b64 c0, {%9, %9};\n\t"
        "mov.b64 c1, {%10, %10};\n\t"
        "mov.b64 c2, {%11, %11};\n\t"
        "add.rn.f32x2 ta, xa, sh;\n\t"
        "add.rn.f32x2 ra, ta, nsh;\n\t"
        "fma.rn.f32x2 fa, ra, nm1, xa;\n\t"
        "fma.rn.f32x2 pa, c2, fa, c1;\n\t"
        "fma.rn.f32x2 pa, pa, fa, c0;\n\t"
        "mov.b64 {%0, %1}, ta;\n\t"
        "mov.b64 {%2, %3}, pa;\n\t}"
        : "=r"(t0), "=r"(t1), "=r"(p0), "=r"(p1)
        : "f"(x0), "f"(x1), "f"(12582912.0f), "f"(-12582912.0f), "f"(-1.0f),
          "f"(1.00044296495389f), "f"(0.7034428104994397f), "f"(0.23842570308291403f));
    y0 = __uint_as_float(t0 * 8388608u + p0);
    y1 = __uint_as_float(t1 * 8388608u + p1);
}

__device__ __forceinline__ void umma_f8_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate,
                                             uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

struct SageCfg {
    static constexpr int BM = 128, BN = 128, D = 128;
    static constexpr int TILE_BYTES = 128 * 128;       // one 128-row x 128-byte box
    static constexpr int STAGES = 3;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 384;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;
    // registers per thread: 168 at launch; the producer warpgroup (MMA, TMA
    // and two idle warps) drops to 56 and the softmax warpgroups rise to 224
    // (2 * 128 * 224 + 128 * 56 = 384 * 168)
    static constexpr int REGS_LAUNCH = 168;
    static constexpr int REGS_SOFTMAX = 224;
    static constexpr int REGS_PRODUCER = 56;
    static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_PRODUCER <= THREADS * REGS_LAUNCH,
                  "register split exceeds the launch allocation");
};

enum : int {
    SB_QFULL = 0, SB_KFULL = 1, SB_KEMPTY = 4, SB_VFULL = 7, SB_VEMPTY = 10,
    SB_SFULL = 13, SB_PFULL = 15, SB_OFULL = 17, SB_DRAIN = 19, SB_COUNT = 20
};

__global__ void __launch_bounds__(384, 1)
    attn_sage_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const SageAttnParams p) {
    using C = SageCfg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seg = blockIdx.z, head = blockIdx.y, qpair = blockIdx.x;

    // ---- validate cu_seqlens (every CTA, cooperatively) ----
    int bad = 0;
    for (int i = tid; i <= p.nseg; i += C::THREADS) {
        const int c = p.cu_seqlens[i];
        if (i == 0 && c != 0) bad = 1;
        if (i == p.nseg && c != p.N) bad = 1;
        if (i > 0) {
            const int prev = p.cu_seqlens[i - 1];
            if (c < prev || c - prev > p.max_seqlen) bad = 1;
        }
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0 && seg == 0 && head == 0 && qpair == 0)
            atomicCAS(p.status, kStatusOk, kStatusBadSeqlens);
        return;
    }
    const int seg_start = p.cu_seqlens[seg];
    const int seg_end = p.cu_seqlens[seg + 1];
    const int L = seg_end - seg_start;
    if (qpair * 2 * C::BM >= L) return;
    const int q0 = seg_start + qpair * 2 * C::BM;
    const int n_kv = (L + C::BN - 1) / C::BN;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + SB_COUNT);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    if (tid == 0) {
        mbar_init(&bars[SB_QFULL], 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bars[SB_KFULL + s], 1);
            mbar_init(&bars[SB_KEMPTY + s], 1);
            mbar_init(&bars[SB_VFULL + s], 1);
            mbar_init(&bars[SB_VEMPTY + s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[SB_SFULL + t], 1);
            mbar_init(&bars[SB_PFULL + t], 4);
            mbar_init(&bars[SB_OFULL + t], 1);
        }
        mbar_init(&bars[SB_DRAIN], 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 9 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 10) {
        reg_dealloc<C::REGS_PRODUCER>();   // idle warps of the producer warpgroup
    } else if (warp == 9) {
        // ============================ TMA producer ============================
        reg_dealloc<C::REGS_PRODUCER>();
        const uint32_t leader = elect_one();
        if (leader) {
            mbar_arrive_expect_tx(&bars[SB_QFULL], 2 * C::TILE_BYTES);
            for (int t = 0; t < 2; ++t)
                tma_load_3d(smem + C::OFF_Q + t * C::TILE_BYTES, &tmQ, &bars[SB_QFULL], 0, head,
                            q0 + t * C::BM);
        }
        int last_k = -1, last_v = -1;
        for (int j = 0; j < n_kv; ++j) {
            const int s = j % C::STAGES;
            const uint32_t ph = (j / C::STAGES) & 1;
            const int kv0 = seg_start + j * C::BN;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[SB_KEMPTY + s], ph ^ 1, abort))) {
                if (leader) raise_abort(abort, p.status);
                break;
            }
            if (leader) {
                mbar_arrive_expect_tx(&bars[SB_KFULL + s], C::TILE_BYTES);
                tma_load_3d(smem + C::OFF_K + s * C::TILE_BYTES, &tmK, &bars[SB_KFULL + s], 0,
                            head, kv0);
            }
            last_k = j;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[SB_VEMPTY + s], ph ^ 1, abort))) {
                if (leader) raise_abort(abort, p.status);
                break;
            }
            if (leader) {
                mbar_arrive_expect_tx(&bars[SB_VFULL + s], C::TILE_BYTES);
                tma_load_3d(smem + C::OFF_V + s * C::TILE_BYTES, &tmV, &bars[SB_VFULL + s], 0,
                            head, kv0);
            }
            last_v = j;
        }
        if (*abort) {
            mbar_wait(&bars[SB_QFULL], 0, nullptr);
            for (int j = (last_k >= C::STAGES ? last_k - C::STAGES + 1 : 0); j <= last_k; ++j)
                mbar_wait(&bars[SB_KFULL + j % C::STAGES], (j / C::STAGES) & 1, nullptr);
            for (int j = (last_v >= C::STAGES ? last_v - C::STAGES + 1 : 0); j <= last_v; ++j)
                mbar_wait(&bars[SB_VFULL + j % C::STAGES], (j / C::STAGES) & 1, nullptr);
        }
        __syncwarp();
    } else if (warp == 8) {
        // ============================ MMA issuer ==============================
        reg_dealloc<C::REGS_PRODUCER>();
        const uint32_t leader = elect_one();
        constexpr uint32_t IDESC_S = idesc_e4m3_f32(128, 128, false, false);
        constexpr uint32_t IDESC_O = idesc_e4m3_f32(128, 128, false, true);
        const uint32_t sQ = smem_u32(smem + C::OFF_Q);
        const uint32_t sK = smem_u32(smem + C::OFF_K);
        const uint32_t sV = smem_u32(smem + C::OFF_V);
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[SB_QFULL], 0, abort));
        tc_fence_after();
        for (int j = 0; ok && j <= n_kv; ++j) {
            for (int t = 0; ok && t < 2; ++t) {
                const uint32_t colS = t ? C::COL_S1 : C::COL_S0;
                const uint32_t colO = t ? C::COL_O1 : C::COL_O0;
                if (j > 0) {  // O_t += P8_t(j-1) V8_{j-1}
                    const int jj = j - 1;
                    const int vs = jj % C::STAGES;
                    bool w = mbar_wait(&bars[SB_PFULL + t], jj & 1, abort);
                    if (w && t == 0)
                        w = mbar_wait(&bars[SB_VFULL + vs], (jj / C::STAGES) & 1, abort);
                    ok = __all_sync(0xffffffffu, w);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vbase = sV + vs * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // V8 tile [128 keys][128 channels] is MN-major for B: one
                        // 128-byte atom across N, 8-key groups at SBO = 1024 B;
                        // 32 keys per MMA
                        const uint64_t bdesc = sdesc_sw128(vbase + kk * 4096, 16384, 1024);
                        umma_f8_ts_w(tmem + colO, tmem + colS + kk * 8, bdesc, IDESC_O,
                                     (jj > 0 || kk > 0) ? 1u : 0u, leader);
                    }
                    if (j == n_kv) umma_commit_w(&bars[SB_OFULL + t], leader);
                    if (t == 1) umma_commit_w(&bars[SB_VEMPTY + vs], leader);
                }
                if (j < n_kv) {  // S_t = Q8_t K8_j^T
                    const int ks = j % C::STAGES;
                    if (t == 0) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(&bars[SB_KFULL + ks], (j / C::STAGES) & 1, abort));
                        if (!ok) break;
                        tc_fence_after();
                    }
                    const uint32_t qbase = sQ + t * C::TILE_BYTES;
                    const uint32_t kbase = sK + ks * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 32 channels (bytes) per MMA
                        const uint64_t adesc = sdesc_sw128(qbase + kk * 32, 16, 1024);
                        const uint64_t bdesc = sdesc_sw128(kbase + kk * 32, 16, 1024);
                        umma_f8_ss_w(tmem + colS, adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u, leader);
                    }
                    umma_commit_w(&bars[SB_SFULL + t], leader);
                    if (t == 1) umma_commit_w(&bars[SB_KEMPTY + ks], leader);
                }
            }
        }
        if (!ok) {
            if (leader) raise_abort(abort, p.status);
            umma_commit_w(&bars[SB_DRAIN], leader);
            mbar_wait(&bars[SB_DRAIN], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ============================ softmax / epilogue ======================
        reg_alloc<C::REGS_SOFTMAX>();
        const int t = warp >> 2;
        const int r = tid & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + (t ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_off + (t ? C::COL_O1 : C::COL_O0);
        const int qrow = q0 + t * C::BM + r;
        const bool valid = qrow < seg_end;
        // rows past the segment end get any finite factor (they are not stored)
        const float rowfac =
            valid ? p.s_q[static_cast<int64_t>(head) * p.N + qrow] * p.scale_log2 : 0.0f;
        const float *sk_head = p.s_k + static_cast<int64_t>(head) * p.N;

        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; ok && j < n_kv; ++j) {
            const int kv0 = seg_start + j * C::BN;
            const int kv_valid = seg_end - kv0;
            float cb[8];   // per 16-key block: s_k * s_q * scale * log2(e)
#pragma unroll
            for (int b = 0; b < 8; ++b)
                cb[b] = (16 * b < kv_valid) ? sk_head[kv0 + 16 * b] * rowfac : 0.0f;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[SB_SFULL + t], j & 1, abort));
            if (!ok) break;
            tc_fence_after();
            uint32_t s[128];
            tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
            tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
            tmem_wait_ld();
            const bool partial = kv_valid < C::BN;
            if (partial) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= kv_valid) s[c] = __float_as_uint(-INFINITY);
            }
            // block maxima of the raw scores (8 independent chains), then the
            // scaled tile max: max_c x_c = max_b cb_b * max_{c in b} s_c (cb >= 0)
            float mb[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) mb[b] = __uint_as_float(s[16 * b]);
#pragma unroll
            for (int c = 1; c < 16; ++c)
#pragma unroll
                for (int b = 0; b < 8; ++b) mb[b] = fmaxf(mb[b], __uint_as_float(s[16 * b + c]));
            float xb[8];
#pragma unroll
            for (int b = 0; b < 8; ++b)
                xb[b] = (partial && 16 * b >= kv_valid) ? -INFINITY : mb[b] * cb[b];
            const float mx = fmaxf(fmaxf(fmaxf(xb[0], xb[1]), fmaxf(xb[2], xb[3])),
                                   fmaxf(fmaxf(xb[4], xb[5]), fmaxf(xb[6], xb[7])));
            bool need = false;
            float f = 1.0f;
            if (j == 0) {
                m_used = mx;
            } else if (mx > m_used + kLazyLog2) {
                need = true;
                f = ex2_approx(m_used - mx);
                l *= f;
                m_used = mx;
            }
            const float nm = kLog2PScale - m_used;    // 112 * 2^(x - m) = 2^(x - m + log2 112)
            float lq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            uint32_t pk[32];
            if (partial) {
#pragma unroll
                for (int w = 0; w < 32; ++w) {
                    float pv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = 4 * w + i;
                        pv[i] = (c < kv_valid)
                            ? ex2_approx(fmaf(__uint_as_float(s[c]), cb[c >> 4], nm)) : 0.0f;
                    }
                    lq[w & 3] += (pv[0] + pv[1]) + (pv[2] + pv[3]);
                    pk[w] = e4m3x4(pv[0], pv[1], pv[2], pv[3]);
                }
            } else {
                // packed f32x2 arithmetic: the scale-and-shift of two scores of one
                // 16-key block in one FFMA2, the row sum in FADD2
                const uint64_t n2 = f2_splat(nm);
                uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
                for (int w = 0; w < 32; ++w) {
                    const uint64_t c2 = f2_splat(cb[w >> 2]);
                    float y[4], pv[4];
                    ffma2(y[0], y[1], __uint_as_float(s[4 * w]), __uint_as_float(s[4 * w + 1]), c2, n2);
                    ffma2(y[2], y[3], __uint_as_float(s[4 * w + 2]), __uint_as_float(s[4 * w + 3]), c2,
                          n2);
                    // words 4..7 of every 8 on the FMA pipe, the rest on MUFU
                    if ((w & 7) >= 4) {
                        exp2_fma2_deg2(pv[0], pv[1], y[0], y[1]);
                        exp2_fma2_deg2(pv[2], pv[3], y[2], y[3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) pv[i] = ex2_approx(y[i]);
                    }
                    if (w & 1) {
                        fadd2(acc1, pv[0], pv[1]);
                        fadd2(acc1, pv[2], pv[3]);
                    } else {
                        fadd2(acc0, pv[0], pv[1]);
                        fadd2(acc0, pv[2], pv[3]);
                    }
                    pk[w] = e4m3x4(pv[0], pv[1], pv[2], pv[3]);
                }
                lq[0] += f2_sum(acc0);
                lq[1] += f2_sum(acc1);
            }
            l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
            if (__any_sync(0xffffffffu, need)) {
                // S_t(j) complete implies PV_t(j-1) complete: O_t is at rest
#pragma unroll
                for (int c = 0; c < C::D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(tO + c * 32, o);
                }
            }
            tmem_st32(tS + 0, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[SB_PFULL + t]);
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[SB_OFULL + t], 0, abort));
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float4 *sv = reinterpret_cast<const float4 *>(
                p.s_v + (static_cast<int64_t>(seg) * p.H + head) * C::D);
            uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<int64_t>(qrow) * p.H + head) * C::D);
#pragma unroll
            for (int c = 0; c < C::D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                float g[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 q4 = sv[c * 8 + i];
                    g[4 * i + 0] = q4.x * inv_l;
                    g[4 * i + 1] = q4.y * inv_l;
                    g[4 * i + 2] = q4.z * inv_l;
                    g[4 * i + 3] = q4.w * inv_l;
                }
                tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * g[2 * i],
                                       __uint_as_float(o[2 * i + 1]) * g[2 * i + 1]);
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        orow[c * 4 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            if (valid && p.lse != nullptr)
                p.lse[static_cast<int64_t>(head) * p.N + qrow] =
                    (m_used + log2f(l) - kLog2PScale) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace h3
