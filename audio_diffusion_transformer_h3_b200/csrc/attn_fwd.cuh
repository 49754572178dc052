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
// against every 128-row key/value tile of the segment. 384 threads in three
// warpgroups:
//   warps 0-7   softmax, one thread per query row (warpgroup t owns Q_t and
//               TMEM lanes 0..127): rotate their Q row in shared memory
//               (RoPE fused into the Q tile load), then per KV tile read S_t
//               from TMEM, mask keys past the segment end, keep a running
//               row max m and sum l (online softmax in the log2 domain, the
//               O rescale skipped unless the max grows by more than 2^8),
//               write P_t as bf16 into the first 64 TMEM columns of S_t in
//               two halves of 64 keys, and finally normalise O_t and store
//               bf16 rows (and the LSE). Warps w and w + 4 share an SM
//               sub-partition; they take turns on its exponential unit (tile
//               0 exponentiates key tile j, then tile 1 key tile j, then tile
//               0 key tile j + 1, ...), which keeps the two tiles half a
//               period apart so that one tile's products run while the other
//               exponentiates. Three eighths of the exponentials run as a
//               cubic on the FMA pipe.
//   warp 8      MMA issuer for both query tiles (the whole warp runs the
//               schedule, one elected lane issues): S_t = Q_t K_j^T (A, B
//               from shared memory) and O_t += P_t V_j (A = P from TMEM, B =
//               V from shared memory), in the order the turns produce them:
//               per key tile j, tile 0 then tile 1, each as PV over keys
//               0..63 as soon as the first half of P_t(j) is in TMEM, then
//               PV over keys 64..127 and S_t(j+1) when the second half
//               arrives. One issuing warp keeps the MMA instructions, which
//               take issue slots from the softmax warps of the same
//               sub-partition, on one sub-partition.
//   warp 10     TMA producer (converged warp, elected lane issues): Q0/Q1
//               once, then K_j and V_j through a two-stage ring
//               (128B-swizzled boxes of 128 rows x 64 cols); warps 9 and 11
//               idle.
// The producer warpgroup gives up registers (setmaxnreg) to the two softmax
// warpgroups.
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

// Key pairs out of every eight whose exponentials run on the FMA pipe
// (exp2_fma2, a cubic on the FMA and integer pipes) instead of MUFU: three of
// eight, which shortens each softmax warp's exponential phase (measured: 3 of
// 8 ahead of 0, 1 and 2 of 8; 4 of 8 slower).
#ifndef H3_FMA_EXP2_PAIRS
#define H3_FMA_EXP2_PAIRS 3
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
    static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;  // barriers + alignment slack
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128;
    static constexpr uint32_t COL_O0 = 256, COL_O1 = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;
    // Registers per thread: 168 at launch (384 threads, one CTA per SM);
    // the producer warpgroup (MMA, TMA and two idle warps) drops to
    // REGS_PRODUCER and the two softmax warpgroups rise to REGS_SOFTMAX:
    // 2 * 128 * 224 + 128 * 56 = 384 * 168, so the raise never waits on
    // registers the block does not hold.
    static constexpr int REGS_LAUNCH = 168;
    static constexpr int REGS_SOFTMAX = 224;
    static constexpr int REGS_PRODUCER = 56;
    static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_PRODUCER <= THREADS * REGS_LAUNCH,
                  "register split exceeds the launch allocation");
};

// Barrier slots (uint64 each) at OFF_BAR: per query tile t, S_t full, the
// two halves of P_t written, O_t final; per SM sub-partition the two
// exponential turns (B_TURN + q: tile 1 has finished key tile j there;
// B_TURN + 4 + q: tile 0 has).
enum : int {
    B_QFULL = 0, B_QREADY = 1, B_KFULL = 2, B_KEMPTY = 4, B_VFULL = 6, B_VEMPTY = 8,
    B_SFULL = 10, B_P1 = 12, B_P2 = 14, B_OFULL = 16, B_DRAIN = 18, B_TURN = 19, B_COUNT = 27
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
__global__ void __launch_bounds__(384, 1)
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
            mbar_init(&bars[B_KEMPTY + s], 2);   // one commit per query tile
            mbar_init(&bars[B_VFULL + s], 1);
            mbar_init(&bars[B_VEMPTY + s], 2);   // one commit per query tile
            mbar_init(&bars[B_SFULL + s], 1);
            mbar_init(&bars[B_P1 + s], 4);
            mbar_init(&bars[B_P2 + s], 4);
            mbar_init(&bars[B_OFULL + s], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        for (int i = 0; i < 8; ++i) mbar_init(&bars[B_TURN + i], 1);
        *abort = 0;
        for (int i = 0; i < 8; ++i) skipword[i] = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 10 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 11) {
        // idle warp of the producer warpgroup
        reg_dealloc<C::REGS_PRODUCER>();
    } else if (warp == 10) {
        // ============================ TMA producer ============================
        reg_dealloc<C::REGS_PRODUCER>();
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
    } else if (warp == 9) {
        reg_dealloc<C::REGS_PRODUCER>();
    } else if (warp == 8) {
        reg_dealloc<C::REGS_PRODUCER>();
        const uint32_t leader = elect_one();
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, false, true);
        const uint32_t sQ0 = smem_u32(smem + C::OFF_Q);
        const uint32_t sK = smem_u32(smem + C::OFF_K);
        const uint32_t sV = smem_u32(smem + C::OFF_V);
        const uint64_t dQ = sdesc_sw128(sQ0, 16, 1024);
        const uint64_t dK = sdesc_sw128(sK, 16, 1024);
        const uint64_t dV = sdesc_sw128(sV, C::BOX_BYTES, 1024);
        auto issue_s = [&](int t, int ks) {
            const uint32_t colS = tmem + (t ? C::COL_S1 : C::COL_S0);
            const uint64_t dq = dQ + static_cast<uint64_t>((t * C::TILE_BYTES) >> 4);
            const uint64_t dk = dK + static_cast<uint64_t>((ks * C::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
                umma_ss_w(colS, dq + off, dk + off, IDESC_S, kk > 0 ? 1u : 0u, leader);
            }
        };
        auto issue_pv = [&](int t, int j, int k0, int k1) {
            const uint32_t colS = tmem + (t ? C::COL_S1 : C::COL_S0);
            const uint32_t colO = tmem + (t ? C::COL_O1 : C::COL_O0);
            const uint64_t dv = dV + static_cast<uint64_t>(((j & 1) * C::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = k0; kk < k1; ++kk)
                umma_ts_w(colO, colS + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4),
                          IDESC_O, (j > 0 || kk > 0) ? 1u : 0u, leader);
        };
        auto wait = [&](int bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(&bars[bar], parity, abort));
        };
        bool ok = wait(B_QREADY, 0) && wait(B_KFULL, 0);
        if (ok) {
            tc_fence_after();
            for (int t = 0; t < 2; ++t) {
                issue_s(t, 0);
                umma_commit_w(&bars[B_SFULL + t], leader);
                umma_commit_w(&bars[B_KEMPTY], leader);
            }
        }
        for (int j = 0; ok && j < n_kv; ++j) {
            const bool more = j + 1 < n_kv;
            const int ks = (j + 1) & 1;
            for (int t = 0; ok && t < 2; ++t) {
                ok = wait(B_P1 + t, j & 1) && wait(B_VFULL + (j & 1), (j >> 1) & 1);
                if (!ok) break;
                tc_fence_after();
                bool skip_pv = false;
                if constexpr (SKIP) {
                    const uint32_t tag = static_cast<uint32_t>(j + 1);
                    skip_pv = skipword[t * 4 + 0] == tag && skipword[t * 4 + 1] == tag &&
                              skipword[t * 4 + 2] == tag && skipword[t * 4 + 3] == tag;
                }
                if (!skip_pv) issue_pv(t, j, 0, C::BN / 32);
                ok = wait(B_P2 + t, j & 1);
                if (!ok) break;
                tc_fence_after();
                if (!skip_pv) issue_pv(t, j, C::BN / 32, C::BN / 16);
                umma_commit_w(&bars[B_VEMPTY + (j & 1)], leader);
                if (more) {
                    ok = wait(B_KFULL + ks, ((j + 1) >> 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(t, ks);
                    umma_commit_w(&bars[B_SFULL + t], leader);
                    umma_commit_w(&bars[B_KEMPTY + ks], leader);
                } else {
                    umma_commit_w(&bars[B_OFULL + t], leader);
                }
            }
        }
        if (!ok) {
            if (leader) raise_abort(abort, p.status);
            umma_commit_w(&bars[B_DRAIN], leader);
            mbar_wait(&bars[B_DRAIN], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ============================ softmax / epilogue ======================
        reg_alloc<C::REGS_SOFTMAX>();
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

        // The two query tiles take turns on the exponential unit of each SM
        // sub-partition: warp w of tile 1 exponentiates tile j after warp w of
        // tile 0 has finished tile j, and warp w of tile 0 exponentiates tile
        // j + 1 after warp w of tile 1 has finished tile j (warps w and w + 4
        // share a sub-partition).
        auto take_turn = [&](int j) -> bool {
            if (t == 0 && j == 0) return true;
            const int bar = t == 0 ? B_TURN + (warp & 3) : B_TURN + 4 + (warp & 3);
            const uint32_t par = t == 0 ? static_cast<uint32_t>((j - 1) & 1) : static_cast<uint32_t>(j & 1);
            return __all_sync(0xffffffffu, mbar_wait(&bars[bar], par, abort));
        };
        auto give_turn = [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[t == 0 ? B_TURN + 4 + (warp & 3) : B_TURN + (warp & 3)]);
        };
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
            // row max over 128 keys in 8 independent chains of three-input max
            // (ALU throughput, not latency)
            float mq[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mq[i] = __uint_as_float(s[i]);
#pragma unroll
            for (int c = 8; c < 128; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mq[i] = fmax3(mq[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
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
                        if (!take_turn(j)) { ok = false; break; }
                        give_turn();
                        if (lane == 0) {
                            skipword[t * 4 + (warp & 3)] = static_cast<uint32_t>(j + 1);
                            // blocks with no row inside the segment are not counted
                            if (p.skip_count != nullptr && q0 + t * C::BM + (warp & 3) * 32 < seg_end)
                                atomicAdd(p.skip_count, 1ull);
                            mbar_arrive(&bars[B_P1 + t]);
                            mbar_arrive(&bars[B_P2 + t]);
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
            // P for keys [64 h, 64 h + 64) into pk[32 h .. 32 h + 31]
            auto exp_half = [&](const int h) {
                if (kv_valid < C::BN) {
                    // keys past the segment end get P = 0 exactly (also when the
                    // scale is 0, where -inf * 0 would give NaN)
#pragma unroll
                    for (int c = 32 * h; c < 32 * h + 32; ++c) {
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
                    const uint64_t s2 = f2_splat(sl2), n2 = f2_splat(nm);
                    uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
                    for (int c = 32 * h; c < 32 * h + 32; ++c) {
                        float x0, x1;
                        ffma2(x0, x1, __uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]),
                              s2, n2);
                        float p0, p1;
                        if ((c & 7) >= 8 - H3_FMA_EXP2_PAIRS) {
                            exp2_fma2(p0, p1, x0, x1);
                        } else {
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        if (c & 1) fadd2(acc1, p0, p1); else fadd2(acc0, p0, p1);
                        pk[c] = pack_bf16x2(p0, p1);
                    }
                    lq[0] += f2_sum(acc0);
                    lq[1] += f2_sum(acc1);
                }
            };
            if (!take_turn(j)) { ok = false; break; }
            exp_half(0);
            tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
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
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_P1 + t]);  // one arrival per warp
            exp_half(1);
            give_turn();
            l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
            tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_P2 + t]);
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
