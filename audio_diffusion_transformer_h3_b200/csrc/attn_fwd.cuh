// Fused RoPE + packed varlen joint attention, forward, for sm_100a.
//
// Operation (non-causal, one attention document per packed segment):
//   "Day 0 Support for MiniMax-H3 on AMD Instinct GPUs", section "The
//   diffusion transformer (DiT)" -- one joint video+audio token sequence,
//   Rotary position encoding; "MiniMax H3" vLLM-Omni recipe, section "Step
//   execution and continuous batching" -- co-batched requests packed into one
//   sequence with one attention document each (block-diagonal mask from
//   cu_seqlens).
//
// One CTA computes two 128-row query tiles (Q0, Q1) of one (segment, head)
// against every 128-row key/value tile of the segment:
//   warp 9      TMA producer (converged warp, elected lane issues): Q0/Q1
//               once, then K_j and V_j through a
//               two-stage ring (128B-swizzled boxes of 128 rows x 64 cols);
//   warps 0-7   softmax, one thread per query row (warpgroup t owns Q_t and
//               TMEM lanes 0..127): rotate their Q row in shared memory
//               (RoPE fused into the Q tile load), then per KV tile read S_t
//               from TMEM, mask keys past the segment end, keep a running
//               row max m and sum l (online softmax in the log2 domain, the
//               O rescale skipped unless the max grows by more than 2^8),
//               write P_t as bf16 into the same TMEM columns, and finally
//               normalise O_t and store bf16 rows (and the LSE);
//   warp 8      MMA issuer (the whole warp runs the schedule, one elected
//               lane issues): S_t = Q_t K_j^T (A, B from shared
//               memory) and O_t += P_t V_j (A = P from TMEM, B = V from
//               shared memory), ordered PV0(j-1), S0(j), PV1(j-1), S1(j) so
//               the tensor core works on one tile while the other tile's
//               softmax runs.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D) fp32
// columns x 128 lanes. tcgen05.mma operations issued by one thread execute in
// order, so S_t(j) may overwrite P_t(j-1) once PV_t(j-1) has been issued.
// Every wait is bounded: a wait that gives up sets H3_ERR_DEVICE_TIMEOUT in
// the status word, raises a CTA-wide abort flag, and the CTA drains its
// in-flight copies and MMAs (bounded) before releasing TMEM and exiting.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "rope.cuh"
#include "sm100.cuh"

// Column pairs out of every eight whose exponentials run on the FMA pipe
// (exp2_fma) instead of MUFU, and whether the row max uses 3-input max.
#ifndef H3_FMA_EXP2_PAIRS
#define H3_FMA_EXP2_PAIRS 0
#endif
#ifndef H3_MAX3
#define H3_MAX3 0
#endif

namespace h3 {

enum : int { kStatusOk = 0, kStatusTimeout = 6, kStatusBadSeqlens = 7 };

struct AttnParams {
    const int32_t *cu_seqlens;  // [nseg + 1]
    const float *pos;           // [N, 3] or nullptr (q is not rotated)
    __nv_bfloat16 *o;           // [N, H, D]
    float *lse;                 // [H, N] or nullptr
    int *status;                // device status word
    int32_t nseg, max_seqlen, N, H;
    float scale_log2;           // softmax_scale * log2(e)
    float skip_log2;            // log2(skip threshold) (skip-softmax variant only)
    unsigned long long *skip_count;  // skipped (32-row block, key tile) pairs, or nullptr
    RopeTable rope;
};

template <int D>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int BM = 128;                     // query rows per tile
    static constexpr int BN = 128;                     // key rows per tile
    static constexpr int NBOX = D / 64;                // 64-column boxes per row
    static constexpr int BOX_BYTES = 128 * 128;        // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128;
    static constexpr uint32_t COL_O0 = 256, COL_O1 = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 320;
};

// Barrier slots (uint64 each) at OFF_BAR.
enum : int {
    B_QFULL = 0, B_QREADY = 1, B_KFULL = 2, B_KEMPTY = 4, B_VFULL = 6, B_VEMPTY = 8,
    B_SFULL = 10, B_PFULL = 12, B_OFULL = 14, B_DRAIN = 16, B_COUNT = 17
};

__device__ __forceinline__ void raise_abort(volatile int *abort, int *status) {
    *abort = 1;
    atomicCAS(status, kStatusOk, kStatusTimeout);
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing
// arrives on, with a cycle limit, exactly as the attention kernel's waits do;
// when the wait gives up it records H3_ERR_DEVICE_TIMEOUT in the status word
// and the kernel returns normally.
__global__ void __launch_bounds__(32, 1) bounded_wait_selftest_kernel(int *status,
                                                                       long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, nullptr, limit_cycles));
    if (!ok && threadIdx.x == 0) atomicCAS(status, kStatusOk, kStatusTimeout);
}

// SKIP: skip-softmax variant ("MiniMax H3" vLLM-Omni recipe, section
// "Attention Backends", Skip-Softmax). For a 32-row block (one softmax warp)
// and a key tile j > 0, if every row of the block has
// exp(tile max - running max) < threshold (rows past the segment end do not
// vote), the block stores P = 0 without computing exponentials and leaves its
// running state unchanged; if all four blocks of a query tile skip, the MMA
// warp also drops that tile's PV.
template <int D, bool SKIP>
__global__ void __launch_bounds__(320, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = AttnCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
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
    if (qpair * 2 * C::BM >= L) return;  // nothing of this segment for this CTA
    const int q0 = seg_start + qpair * 2 * C::BM;
    const int n_kv = (L + C::BN - 1) / C::BN;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // skip-softmax: per query tile and softmax warp, 1 + the last key tile it skipped
    volatile uint32_t *skipword = reinterpret_cast<volatile uint32_t *>(tmem_slot + 2);

    if (tid == 0) {
        mbar_init(&bars[B_QFULL], 1);
        mbar_init(&bars[B_QREADY], 256);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_KFULL + s], 1);
            mbar_init(&bars[B_KEMPTY + s], 1);
            mbar_init(&bars[B_VFULL + s], 1);
            mbar_init(&bars[B_VEMPTY + s], 1);
            mbar_init(&bars[B_SFULL + s], 1);
            mbar_init(&bars[B_PFULL + s], 4);
            mbar_init(&bars[B_OFULL + s], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort = 0;
        for (int i = 0; i < 8; ++i) skipword[i] = 0;
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

    if (warp == 9) {
        // ============================ TMA producer ============================
        // Converged warp; the elected lane issues the copies and expect_tx.
        const uint32_t leader = elect_one();
        if (leader) mbar_arrive_expect_tx(&bars[B_QFULL], 2 * C::TILE_BYTES);
        for (int t = 0; t < 2; ++t)
            for (int b = 0; b < C::NBOX; ++b)
                if (leader)
                    tma_load_3d(smem + C::OFF_Q + t * C::TILE_BYTES + b * C::BOX_BYTES, &tmQ,
                                &bars[B_QFULL], b * 64, head, q0 + t * C::BM);
        int last_k = -1, last_v = -1;
        for (int j = 0; j < n_kv; ++j) {
            const int s = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            const int kv0 = seg_start + j * C::BN;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_KEMPTY + s], ph ^ 1, abort))) {
                if (leader) raise_abort(abort, p.status);
                break;
            }
            if (leader) {
                mbar_arrive_expect_tx(&bars[B_KFULL + s], C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tma_load_3d(smem + C::OFF_K + s * C::TILE_BYTES + b * C::BOX_BYTES, &tmK,
                                &bars[B_KFULL + s], b * 64, head, kv0);
            }
            last_k = j;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_VEMPTY + s], ph ^ 1, abort))) {
                if (leader) raise_abort(abort, p.status);
                break;
            }
            if (leader) {
                mbar_arrive_expect_tx(&bars[B_VFULL + s], C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tma_load_3d(smem + C::OFF_V + s * C::TILE_BYTES + b * C::BOX_BYTES, &tmV,
                                &bars[B_VFULL + s], b * 64, head, kv0);
            }
            last_v = j;
        }
        if (*abort) {
            // let the copies still in flight land before shared memory is released
            mbar_wait(&bars[B_QFULL], 0, nullptr);
            for (int j = (last_k > 0 ? last_k - 1 : 0); j <= last_k; ++j)
                mbar_wait(&bars[B_KFULL + (j & 1)], (j >> 1) & 1, nullptr);
            for (int j = (last_v > 0 ? last_v - 1 : 0); j <= last_v; ++j)
                mbar_wait(&bars[B_VFULL + (j & 1)], (j >> 1) & 1, nullptr);
        }
        __syncwarp();
    } else if (warp == 8) {
        // ============================ MMA issuer ==============================
        // The whole warp runs this schedule (waits included) so that it stays
        // converged; only the elected lane issues the MMAs and commits.
        const uint32_t leader = elect_one();
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
        const uint32_t sQ = smem_u32(smem + C::OFF_Q);
        const uint32_t sK = smem_u32(smem + C::OFF_K);
        const uint32_t sV = smem_u32(smem + C::OFF_V);
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_QREADY], 0, abort));
        tc_fence_after();
        for (int j = 0; ok && j <= n_kv; ++j) {
            for (int t = 0; ok && t < 2; ++t) {
                const uint32_t colS = t ? C::COL_S1 : C::COL_S0;
                const uint32_t colO = t ? C::COL_O1 : C::COL_O0;
                if (j > 0) {  // O_t += P_t(j-1) V_{j-1}
                    const int jj = j - 1;
                    const int vs = jj & 1;
                    bool w = mbar_wait(&bars[B_PFULL + t], jj & 1, abort);
                    if (w && t == 0) w = mbar_wait(&bars[B_VFULL + vs], (jj >> 1) & 1, abort);
                    ok = __all_sync(0xffffffffu, w);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vbase = sV + vs * C::TILE_BYTES;
                    bool skip_pv = false;
                    if constexpr (SKIP) {
                        const uint32_t tag = static_cast<uint32_t>(jj + 1);
                        skip_pv = skipword[t * 4 + 0] == tag && skipword[t * 4 + 1] == tag &&
                                  skipword[t * 4 + 2] == tag && skipword[t * 4 + 3] == tag;
                    }
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk) {
                        if (skip_pv) break;
                        // V tile [128 keys][D] is MN-major for B: 8 key rows at 128 B,
                        // groups of 8 rows at SBO = 1024 B, 64-col boxes at LBO.
                        const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, C::BOX_BYTES, 1024);
                        umma_ts_w(tmem + colO, tmem + colS + kk * 8, bdesc, IDESC_O,
                                  (jj > 0 || kk > 0) ? 1u : 0u, leader);
                    }
                    if (j == n_kv) umma_commit_w(&bars[B_OFULL + t], leader);
                    if (t == 1) umma_commit_w(&bars[B_VEMPTY + vs], leader);
                }
                if (j < n_kv) {  // S_t = Q_t K_j^T
                    const int ks = j & 1;
                    if (t == 0) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(&bars[B_KFULL + ks], (j >> 1) & 1, abort));
                        if (!ok) break;
                        tc_fence_after();
                    }
                    const uint32_t qbase = sQ + t * C::TILE_BYTES;
                    const uint32_t kbase = sK + ks * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                        const uint64_t adesc = sdesc_sw128(qbase + off, 16, 1024);
                        const uint64_t bdesc = sdesc_sw128(kbase + off, 16, 1024);
                        umma_ss_w(tmem + colS, adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u, leader);
                    }
                    umma_commit_w(&bars[B_SFULL + t], leader);
                    if (t == 1) umma_commit_w(&bars[B_KEMPTY + ks], leader);
                }
            }
        }
        if (!ok) {
            if (leader) raise_abort(abort, p.status);
            umma_commit_w(&bars[B_DRAIN], leader);  // completes once every issued MMA is done
            mbar_wait(&bars[B_DRAIN], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ============================ softmax / epilogue ======================
        const int t = warp >> 2;                 // query tile of this warpgroup
        const int r = tid & 127;                 // row inside the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + (t ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_off + (t ? C::COL_O1 : C::COL_O0);
        const int qrow = q0 + t * C::BM + r;
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_QFULL], 0, abort));

        // RoPE on this thread's Q row, in place in the swizzled tile.
        if (ok && p.pos != nullptr && qrow < p.N) {
            const float pt = p.pos[static_cast<int64_t>(qrow) * 3 + 0];
            const float ph = p.pos[static_cast<int64_t>(qrow) * 3 + 1];
            const float pw = p.pos[static_cast<int64_t>(qrow) * 3 + 2];
            uint8_t *row = smem + C::OFF_Q + t * C::TILE_BYTES + r * 128;
#pragma unroll 1
            for (int c = 0; c < D / 8; ++c) {  // 16-byte chunk c = 4 pairs
                uint4 *ptr = reinterpret_cast<uint4 *>(row + (c >> 3) * C::BOX_BYTES +
                                                       (((c & 7) ^ (r & 7)) << 4));
                uint4 v = *ptr;
                uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int pr = c * 4 + u;
                    const int ax = rope_axis(p.rope, pr);
                    const float pp = ax == 0 ? pt : (ax == 1 ? ph : pw);
                    float cs, sn;
                    rope_cos_sin(pp, p.rope.inv_freq[pr], cs, sn);
                    w[u] = rope_word(w[u], cs, sn);
                }
                *ptr = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_QREADY]);

        float m_used = -INFINITY, l = 0.f;
        float m_run = -INFINITY;  // true running row max (skip-softmax decision)
        const float sl2 = p.scale_log2;
        for (int j = 0; ok && j < n_kv; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_SFULL + t], j & 1, abort));
            if (!ok) break;
            tc_fence_after();
            uint32_t s[128];
            tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
            tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
            tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
            tmem_wait_ld();
            const int kv_valid = seg_end - (seg_start + j * C::BN);
            if (kv_valid < C::BN) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= kv_valid) s[c] = __float_as_uint(-INFINITY);
            }
            // row max over 128 keys in 8 independent chains (ALU throughput, not latency)
            float mq[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mq[i] = __uint_as_float(s[i]);
#if H3_MAX3
#pragma unroll
            for (int c = 8; c < 128; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mq[i] = fmax3(mq[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
#else
#pragma unroll
            for (int c = 8; c < 128; ++c) mq[c & 7] = fmaxf(mq[c & 7], __uint_as_float(s[c]));
#endif
            const float mx = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])),
                                   fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
            const float m_new = mx * sl2;
            if constexpr (SKIP) {
                if (j == 0) {
                    m_run = m_new;
                } else {
                    // rows past the segment end do not vote
                    const bool negligible = qrow >= seg_end || m_new - m_run < p.skip_log2;
                    if (__all_sync(0xffffffffu, negligible)) {
                        uint32_t z[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) z[i] = 0u;
                        tmem_st32(tS + 0, z);
                        tmem_st32(tS + 32, z);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            skipword[t * 4 + (warp & 3)] = static_cast<uint32_t>(j + 1);
                            // blocks with no row inside the segment are not counted
                            if (p.skip_count != nullptr && q0 + t * C::BM + (warp & 3) * 32 < seg_end)
                                atomicAdd(p.skip_count, 1ull);
                            mbar_arrive(&bars[B_PFULL + t]);
                        }
                        continue;
                    }
                    m_run = fmaxf(m_run, m_new);
                }
            }
            bool need = false;
            if (j == 0) {
                m_used = m_new;
            } else if (m_new > m_used + 8.0f) {
                need = true;
            }
            const float f = need ? ex2_approx(m_used - m_new) : 1.0f;
            if (need) {
                l *= f;
                m_used = m_new;
            }
            const float nm = -m_used;
            float lq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            uint32_t pk[64];
            if (kv_valid < C::BN) {
                // keys past the segment end get P = 0 exactly (also when the
                // scale is 0, where -inf * 0 would give NaN)
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float p0 = (2 * c < kv_valid)
                        ? ex2_approx(fmaf(__uint_as_float(s[2 * c]), sl2, nm)) : 0.0f;
                    const float p1 = (2 * c + 1 < kv_valid)
                        ? ex2_approx(fmaf(__uint_as_float(s[2 * c + 1]), sl2, nm)) : 0.0f;
                    lq[c & 3] += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            } else {
                // H3_FMA_EXP2_PAIRS column pairs of every eight on the FMA pipe
                // (exp2_fma), the rest on MUFU (ex2.approx)
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float x0 = fmaf(__uint_as_float(s[2 * c]), sl2, nm);
                    const float x1 = fmaf(__uint_as_float(s[2 * c + 1]), sl2, nm);
                    float p0, p1;
                    if ((c & 7) >= 8 - H3_FMA_EXP2_PAIRS) {
                        p0 = exp2_fma(x0);
                        p1 = exp2_fma(x1);
                    } else {
                        p0 = ex2_approx(x0);
                        p1 = ex2_approx(x1);
                    }
                    lq[c & 3] += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            }
            l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
            if (__any_sync(0xffffffffu, need)) {
                // O_t holds P V up to tile j-1 (S_t(j) completing implies every
                // earlier MMA completed); rescale it before P_t(j) is released.
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(tO + c * 32, o);
                }
            }
            tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PFULL + t]);  // one arrival per warp
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OFULL + t], 0, abort));
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const bool valid = qrow < seg_end;
            uint4 *orow = reinterpret_cast<uint4 *>(
                p.o + (static_cast<int64_t>(qrow) * p.H + head) * D);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                       __uint_as_float(o[2 * i + 1]) * inv_l);
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        orow[c * 4 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            if (valid && p.lse != nullptr)
                p.lse[static_cast<int64_t>(head) * p.N + qrow] =
                    (m_used + log2f(l)) * 0.69314718055994530942f;
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
