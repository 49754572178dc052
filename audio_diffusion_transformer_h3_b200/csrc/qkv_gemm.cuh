// QKV projection with the rotary embedding fused into its epilogue, sm_100a.
//
// "MiniMax-H3 Reference" Space README, section "AoTI-compiled blocks": the
// norm / rotary / AdaLN epilogues around the block's matmuls; "MiniMax H3"
// vLLM-Omni recipe, section "Online FP8 quantization": the attention's qkv
// projection is one of the DiT linears. Computes Y = X W^T (X [N, K] bf16,
// W [3 H D, K] bf16, fp32 accumulation), splits Y into q, k, v [N, H, D] and
// rotates q and k (same pair layout, frequencies and rounding sequence as
// rope.cuh) before the single rounding to bf16, so the attention takes them
// with no separate rotary pass.
//
// Persistent kernel, one CTA per SM, tiles of 128 x 256 outputs (256 / D heads
// of one of q, k, v) taken in a grouped raster (GROUP_M row tiles sweep the
// column tiles together, so the X rows and W slices in flight stay in L2):
//   warp 4      TMA producer (converged, elected lane): X and W tiles of 64
//               K-elements through a four-stage ring (128-byte swizzle);
//   warp 5      MMA issuer (converged, elected lane): 128x256x16 tcgen05.mma
//               into one of two 256-column fp32 TMEM accumulators;
//   warps 0-3   epilogue, one output row per thread, on the other
//               accumulator: 32 columns at a time, rotate the q/k pairs with
//               the row's (cos, sin) (computed once per 32-column chunk and
//               reused for every head of the tile), round to bf16, store.
// The two accumulators let the epilogue of one tile run under the main loop
// of the next.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "rope.cuh"
#include "sm100.cuh"

namespace h3 {

struct QkvParams {
    __nv_bfloat16 *q, *k, *v;   // [N, H*D] each
    const float *pos;           // [N, 3] or nullptr (no rotation)
    int *status;                // device status word
    int32_t N, K, HD;           // HD = H * D
    int32_t n_row_tiles, n_col_tiles, n_tiles, group_m;
    RopeTable rope;
};

struct QkvCfg {
    static constexpr int BM = 128, BN = 256, BK = 64;
    static constexpr int STAGES = 4;
    static constexpr int A_BYTES = BM * BK * 2;   // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;   // 32 KB
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
    static constexpr int THREADS = 192;
    static constexpr int TMA_WARP = 4, MMA_WARP = 5;
    static constexpr uint32_t ACC_COLS = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

enum : int {
    QB_FULL = 0,        // + stage: X/W tiles landed
    QB_EMPTY = 4,       // + stage: MMAs done reading the stage
    QB_ACC_FULL = 8,    // + buffer: accumulator complete
    QB_ACC_EMPTY = 10,  // + buffer: epilogue done reading the accumulator
    QB_DRAIN = 12,
    QB_COUNT = 13
};

// 2-D tiled bulk tensor load global -> shared; c0 (the K coordinate) is a
// multiple of 64 elements, so c0 * 2 bytes is 16-byte aligned.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map,
                                            uint64_t *bar, int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// Tile index -> (row tile, column tile) in the grouped raster.
__device__ __forceinline__ void qkv_tile_coords(const QkvParams &p, int tile, int &m_tile,
                                                int &n_tile) {
    const int per_group = p.group_m * p.n_col_tiles;
    const int group = tile / per_group;
    const int first_m = group * p.group_m;
    const int rows_left = p.n_row_tiles - first_m;
    const int gm = rows_left < p.group_m ? rows_left : p.group_m;
    const int in_group = tile - group * per_group;
    m_tile = first_m + in_group % gm;
    n_tile = in_group / gm;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    qkv_rope_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmW, const QkvParams p) {
    using C = QkvCfg;
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_k = p.K / C::BK;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + QB_COUNT);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bars[QB_FULL + s], 1);
            mbar_init(&bars[QB_EMPTY + s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[QB_ACC_FULL + b], 1);
            mbar_init(&bars[QB_ACC_EMPTY + b], 4);   // one arrival per epilogue warp
        }
        mbar_init(&bars[QB_DRAIN], 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == C::TMA_WARP && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == C::TMA_WARP) {
        // ============================ TMA producer ============================
        const uint32_t leader = elect_one();
        uint32_t it = 0;   // k-steps issued by this CTA
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x) {
            int mt, nt;
            qkv_tile_coords(p, tile, mt, nt);
            for (int ks = 0; ks < n_k; ++ks) {
                const int st = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[QB_EMPTY + st], ph ^ 1, abort))) {
                    ok = false;
                    break;
                }
                if (leader) {
                    mbar_arrive_expect_tx(&bars[QB_FULL + st], C::A_BYTES + C::B_BYTES);
                    tma_load_2d(smem + C::OFF_A + st * C::A_BYTES, &tmX, &bars[QB_FULL + st],
                                ks * C::BK, mt * C::BM);
                    tma_load_2d(smem + C::OFF_B + st * C::B_BYTES, &tmW, &bars[QB_FULL + st],
                                ks * C::BK, nt * C::BN);
                }
                ++it;
            }
        }
        if (!ok) {
            if (leader) {
                *abort = 1;
                atomicCAS(p.status, 0, 6);
            }
            // copies still in flight land before the CTA leaves
            for (uint32_t j = (it > C::STAGES ? it - C::STAGES : 0); j < it; ++j)
                mbar_wait(&bars[QB_FULL + j % C::STAGES], (j / C::STAGES) & 1, nullptr);
        }
        __syncwarp();
    } else if (warp == C::MMA_WARP) {
        // ============================ MMA issuer ==============================
        const uint32_t leader = elect_one();
        constexpr uint32_t IDESC = idesc_bf16_f32(C::BM, C::BN, false, false);
        const uint32_t sA = smem_u32(smem + C::OFF_A), sB = smem_u32(smem + C::OFF_B);
        uint32_t it = 0;
        int tcount = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++tcount) {
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars[QB_ACC_EMPTY + buf], (use & 1) ^ 1, abort));
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = tmem + static_cast<uint32_t>(buf) * C::ACC_COLS;
            for (int ks = 0; ks < n_k; ++ks, ++it) {
                const int st = it % C::STAGES;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars[QB_FULL + st], (it / C::STAGES) & 1, abort));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C::BK / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(sA + st * C::A_BYTES + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sB + st * C::B_BYTES + kk * 32, 16, 1024);
                    umma_ss_w(acc, ad, bd, IDESC, (ks > 0 || kk > 0) ? 1u : 0u, leader);
                }
                umma_commit_w(&bars[QB_EMPTY + st], leader);
            }
            if (!ok) break;
            umma_commit_w(&bars[QB_ACC_FULL + buf], leader);
        }
        if (!ok) {
            if (leader) {
                *abort = 1;
                atomicCAS(p.status, 0, 6);
            }
            // MMAs in flight complete before the accumulator is released
            umma_commit_w(&bars[QB_DRAIN], leader);
            mbar_wait(&bars[QB_DRAIN], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ============================ epilogue ================================
        constexpr int HEADS = C::BN / D;               // heads in one tile
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++tcount) {
            const int buf = tcount & 1;
            const uint32_t use = static_cast<uint32_t>(tcount >> 1);
            int mt, nt;
            qkv_tile_coords(p, tile, mt, nt);
            const int grow = mt * C::BM + tid;         // output row = TMEM lane
            const int n0 = nt * C::BN;
            const int section = n0 / p.HD;             // 0 q, 1 k, 2 v (HD % 256 == 0)
            const int hd0 = n0 - section * p.HD;
            __nv_bfloat16 *out = section == 0 ? p.q : (section == 1 ? p.k : p.v);
            const bool rotate = section < 2 && p.pos != nullptr;
            float pt = 0.f, ph = 0.f, pw = 0.f;
            if (rotate && grow < p.N) {
                pt = p.pos[static_cast<int64_t>(grow) * 3 + 0];
                ph = p.pos[static_cast<int64_t>(grow) * 3 + 1];
                pw = p.pos[static_cast<int64_t>(grow) * 3 + 2];
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[QB_ACC_FULL + buf], use & 1, abort))) {
                if (lane == 0) {
                    *abort = 1;
                    atomicCAS(p.status, 0, 6);
                }
                break;
            }
            tc_fence_after();
            const uint32_t acc = tmem + lane_off + static_cast<uint32_t>(buf) * C::ACC_COLS;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {         // 32 columns = 16 pairs of one head
                float cs[16], sn[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    cs[i] = 1.0f;
                    sn[i] = 0.0f;
                    if (rotate) {
                        const int pr = c * 16 + i;
                        const int ax = rope_axis(p.rope, pr);
                        rope_cos_sin(ax == 0 ? pt : (ax == 1 ? ph : pw), p.rope.inv_freq[pr],
                                     cs[i], sn[i]);
                    }
                }
#pragma unroll 1
                for (int hh = 0; hh < HEADS; ++hh) {
                    const int col = hh * D + c * 32;
                    uint32_t a[32];
                    tmem_ld32(acc + col, a);
                    tmem_wait_ld();
                    uint32_t wv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float y0 = __uint_as_float(a[2 * i]), y1 = __uint_as_float(a[2 * i + 1]);
                        if (rotate) rope_rotate(y0, y1, cs[i], sn[i], y0, y1);
                        wv[i] = pack_bf16x2(y0, y1);
                    }
                    if (grow < p.N) {
                        uint4 *dst = reinterpret_cast<uint4 *>(
                            out + static_cast<int64_t>(grow) * p.HD + hd0 + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2],
                                                wv[4 * i + 3]);
                    }
                }
            }
            // accumulator reads done -> the MMA warp may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[QB_ACC_EMPTY + buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace h3
