/*
 * h3attn -- packed variable-length joint video+audio self-attention with a
 * 3-axis (t, h, w) rotary embedding on the shared audio/video clock, for
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (sources are the public pages on MiniMax-H3):
 *   - "Day 0 Support for MiniMax-H3 on AMD Instinct GPUs", section "The
 *     diffusion transformer (DiT)": the DiT flattens the video latent and the
 *     audio latent into one token sequence and attends over it jointly; its
 *     position encoding is Rotary (RoPE); heads are 128 wide.
 *   - "MiniMax H3" vLLM-Omni recipe, section "Step execution and continuous
 *     batching": co-batched requests are packed into one sequence that keeps
 *     one attention document per request (a block-diagonal mask given by
 *     cu_seqlens); section "Attention Backends": packed varlen backends.
 *   - "MiniMax-H3 Reference" Space README, section "References": the order of
 *     the references advances the shared audio/video rotary clock.
 *   - "MiniMax H3 on Moore Threads MUSA", section "MUSA validation": position
 *     metadata is FP64 on the host and is cast to FP32 before device
 *     arithmetic.
 *
 * Conventions for every call:
 *   - Tensors q, k, v, o are bf16, layout [N, H, D] ("THD"), contiguous, token
 *     stride H*D elements. N = total packed tokens, H = heads, D = head dim.
 *   - pos is fp32 [N, 3] = (t, h, w) per token, contiguous.
 *   - cu_seqlens is int32 [nseg + 1]: cu[0] = 0, non-decreasing, cu[nseg] = N.
 *     Segment s holds tokens [cu[s], cu[s+1]); zero-length segments are legal.
 *   - The caller owns every buffer. No call allocates device memory, and no
 *     call synchronises the stream except h3_read_device_status.
 *   - Device calls are asynchronous on `stream` and report argument errors
 *     through the return value before anything is enqueued. Errors never
 *     abort or throw across this boundary.
 *   - Device pointers must point to memory of the current CUDA device.
 */
#ifndef H3ATTN_H
#define H3ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. NULL is the legacy default stream. */
typedef struct CUstream_st *h3_stream_t;

typedef enum h3_status {
    H3_OK = 0,
    H3_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad rotary split */
    H3_ERR_UNSUPPORTED = 2,    /* head dim other than 64 or 128, no sm_100 device */
    H3_ERR_MISALIGNED = 3,     /* q/k/v/o/x/out not 16-byte aligned, pos/lse not 4-byte aligned */
    H3_ERR_WORKSPACE = 4,      /* workspace null or smaller than h3_workspace_size() */
    H3_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed; see h3_last_cuda_error() */
    H3_ERR_DEVICE_TIMEOUT = 6, /* a bounded in-kernel wait gave up (device status only) */
    H3_ERR_BAD_SEQLENS = 7     /* cu_seqlens invalid on the device (device status only) */
} h3_status;

/* Rotary split of the head dimension into contiguous (t, h, w) chunks.
 * Each width is even and d_t + d_h + d_w = D. Inside the chunk of axis a
 * (width d_a, first channel c_a), pair j (j < d_a/2) is channels
 * (c_a + 2j, c_a + 2j + 1) and is rotated by the angle
 * pos[a] * theta^(-2j/d_a):  (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
 * The inverse frequencies are formed in double on the host and rounded to
 * float; angles, cos and sin are fp32 on the device. */
typedef struct h3_rope_cfg {
    int32_t d_t, d_h, d_w;
    float theta;
} h3_rope_cfg;

/* Composition of one packed segment (one attention document), in token
 * order: `image_refs` single-frame reference grids of image_h x image_w
 * tokens, then `audio_refs` audio-reference runs of audio_ref_len tokens,
 * then the video latent grid video_t x video_h x video_w (row-major t, h, w),
 * then `audio_tail` audio tokens spread over the video grid's frames.
 * Source: "MiniMax-H3 Reference" Space README, sections "References" and
 * "AoTI-compiled blocks" (reference rows packed in front of generated rows,
 * their order advancing the shared clock). */
typedef struct h3_segment_layout {
    int32_t image_refs, image_h, image_w;
    int32_t audio_refs, audio_ref_len, audio_rate; /* audio_rate: tokens per clock unit */
    int32_t video_t, video_h, video_w;
    int32_t audio_tail;
} h3_segment_layout;

/* Number of tokens of one segment layout, or -1 if a field is negative or
 * the count overflows int32. Host only. */
int64_t h3_segment_tokens(const h3_segment_layout *seg);

/* Host-side position build for `nseg` packed segments (host memory only,
 * no CUDA call). Writes pos[n] = (t, h, w) as float for every token and, if
 * cu_seqlens is not NULL, the nseg+1 segment boundaries. Each segment's clock
 * starts at t0 = 0. Image reference: tokens (t0, h, w), then t0 += 1. Audio
 * reference: token i at (t0 + i/audio_rate, 0, 0), then
 * t0 += audio_ref_len/audio_rate. Video grid: (t0 + tau, h, w). Audio tail
 * token i of n: (t0 + (i*video_t)/n, 0, 0). Every value is formed in double
 * in the order written and rounded once to float ("MiniMax H3 on Moore
 * Threads MUSA", section "MUSA validation").
 * pos: host float [capacity, 3]. Returns H3_ERR_INVALID_ARG on a null
 * pointer, a bad layout (negative field, audio_rate <= 0 with audio refs) or
 * if the total exceeds `capacity`. */
h3_status h3_build_positions(const h3_segment_layout *segs, int32_t nseg, float *pos,
                             int64_t capacity, int32_t *cu_seqlens);

/* h3_build_positions with a clock origin per segment: segment s starts at
 * t0 = t_origin[s] instead of 0 (every other rule unchanged), which places a
 * long-video continuation chunk on the global temporal RoPE clock ("MiniMax
 * H3" vLLM-Omni recipe, section "Long video and driving audio": latent
 * continuation with global temporal RoPE positions). The attention calls need
 * no change: positions are their input.
 *   t_origin: host double [nseg], finite, or NULL (all 0, h3_build_positions).
 * Returns H3_ERR_INVALID_ARG for a non-finite origin and as h3_build_positions
 * otherwise. Host only. */
h3_status h3_build_positions_at(const h3_segment_layout *segs, int32_t nseg,
                                const double *t_origin, float *pos, int64_t capacity,
                                int32_t *cu_seqlens);

/* Standalone rotary pass: out = RoPE(x, pos). "Day 0 Support for MiniMax-H3
 * on AMD Instinct GPUs", section "The diffusion transformer (DiT)".
 *   x, out : device bf16 [N, H, D], 16-byte aligned; out may equal x
 *            (in place); other overlap is undefined.
 *   pos    : device fp32 [N, 3], 4-byte aligned.
 *   N >= 0 (N = 0 is a no-op), 1 <= H, D in {64, 128}, H*D*N < 2^40.
 * Results are rounded to bf16 (round to nearest even). Bit-identical to the
 * rotation that h3_varlen_attn_fwd applies to q and k. One kernel launch. */
h3_status h3_rope_apply(const void *x, void *out, const float *pos, int64_t N, int32_t H,
                        int32_t D, h3_rope_cfg rope, h3_stream_t stream);

/* Bytes of device workspace h3_varlen_attn_fwd needs: a 256-byte status
 * block plus, for the rotated keys, N*H*D*2 bytes rounded up to 256. */
size_t h3_workspace_size(int64_t N, int32_t H, int32_t D, int32_t nseg);

/* Fused RoPE + packed varlen joint attention, forward, non-causal.
 * For every segment s and head h, with Q~ = RoPE(q), K~ = RoPE(k) when pos is
 * not NULL (else Q~ = q, K~ = k):
 *     O = softmax(softmax_scale * Q~ K~^T) V     over the segment's rows only,
 *     LSE = row log-sum-exp of softmax_scale * Q~ K~^T (natural log).
 * Sources: see the file header (joint sequence, RoPE, packed documents).
 *   q, k, v    : device bf16 [N, H, D], 16-byte aligned, unrotated.
 *   o          : device bf16 [N, H, D], 16-byte aligned; must not overlap inputs.
 *   lse        : device fp32 [H, N] or NULL (not written).
 *   cu_seqlens : device int32 [nseg + 1]; validated on the device: a
 *                violation (cu[0] != 0, decreasing, cu[nseg] != N, or a
 *                segment longer than max_seqlen) makes the kernel skip the
 *                work and set H3_ERR_BAD_SEQLENS in the workspace status.
 *   max_seqlen : upper bound on every segment length, 1 <= max_seqlen <= N.
 *   pos        : device fp32 [N, 3] or NULL (no rotary embedding).
 *   N, H, D    : 0 <= N < 2^31 (N = 0 is a no-op), 1 <= H <= 65535,
 *                D in {64, 128}; 1 <= nseg <= 65535.
 *   softmax_scale : finite, >= 0 (0 gives the mean of V over the segment).
 *   workspace  : device, 256-byte aligned, >= h3_workspace_size(N, H, D, nseg)
 *                bytes (>= 256 bytes when pos is NULL: no rotated keys are
 *                stored); owned by the caller, must not be shared by calls
 *                that run concurrently. Its status word is reset by every call.
 * Accumulation is fp32; P is rounded to bf16 before the PV product; O is
 * rounded to bf16. Results are deterministic run to run. Launches: one
 * rotary kernel for k (when pos is not NULL) and one attention kernel. */
h3_status h3_varlen_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                             const int32_t *cu_seqlens, int32_t nseg, int32_t max_seqlen,
                             const float *pos, h3_rope_cfg rope, int64_t N, int32_t H,
                             int32_t D, float softmax_scale, void *workspace,
                             size_t workspace_bytes, h3_stream_t stream);

/* Skip-Softmax variant of h3_varlen_attn_fwd (lossy). "MiniMax H3" vLLM-Omni
 * recipe, section "Attention Backends": Skip-Softmax sparse attention skips
 * tiles whose softmax contribution is below a direct threshold (0.05 in the
 * pages' example; which denoising steps stay dense is the caller's choice).
 * Reading used here: keys are taken in tiles of 128 from the segment start,
 * query rows in blocks of 32 inside 128-row tiles from the segment start. A
 * block skips key tile j > 0 when, for every row of the block,
 * exp(tile's max score - row's running max score) < skip_threshold (scores
 * include softmax_scale; skipped tiles never raise the running max). The
 * result is softmax attention over the keys of the kept tiles.
 *   skip_threshold: 0 <= t <= 1 (0 never skips), else H3_ERR_INVALID_ARG.
 *   workspace: as for h3_varlen_attn_fwd; bytes [8, 16) receive the number of
 *              skipped (32-row block, key tile) pairs (h3_read_skip_count).
 * All other arguments, results and errors are those of h3_varlen_attn_fwd. */
h3_status h3_varlen_attn_fwd_skip(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *cu_seqlens, int32_t nseg,
                                  int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                                  int64_t N, int32_t H, int32_t D, float softmax_scale,
                                  float skip_threshold, void *workspace, size_t workspace_bytes,
                                  h3_stream_t stream);

/* Bytes of device workspace h3_varlen_attn_fwd_sage needs (0 if D != 128 or
 * a size is negative). Layout, each region starting on a 256-byte boundary
 * in this order: the 256-byte status block; q8, k8, v8 (e4m3 codes, [N, H,
 * 128] bytes each, regions of round_up(N*H*128, 256)); s_q, s_k (fp32
 * dequantisation scales [H, N], s_k repeated for every token of its 16-key
 * block; regions of round_up(N*H*4, 256)); v_amax (fp32 [nseg, H, 128], max
 * |v| per segment, head and channel) and s_v (fp32 [nseg, H, 128], v_amax /
 * 448; regions of round_up(nseg*H*128*4, 256)). A call leaves its quantised
 * tensors and scales there. */
size_t h3_sage_workspace_size(int64_t N, int32_t H, int32_t D, int32_t nseg);

/* SAGE-style FP8 variant of h3_varlen_attn_fwd (lossy). "MiniMax H3"
 * vLLM-Omni recipe, section "Attention Backends": Q and K in fp8_e4m3 with
 * q_block_size 1 and k_block_size 16, P and V in FP8. Reading used here
 * (conversions to e4m3 round to nearest even and saturate to +-448):
 *   Q~ = RoPE(q), K~ = RoPE(k) in fp32 (pos NULL: no rotation);
 *   Q: per (token, head) a = max|Q~|, codes e4m3(Q~ * (448/a)), s_q = a/448;
 *   K: per (16-key block from the segment start, head), same formulas;
 *   V: per (segment, head, channel), same formulas over the segment's tokens;
 *   scores x = (q8.k8) s_q s_k softmax_scale log2(e); online softmax over key
 *   tiles of 128 from the segment start, the running max m raised whenever a
 *   tile raises it; P8 = e4m3(448 * 2^(x - m)); the row sum l adds the
 *   unquantised 448 * 2^(x - m); O = s_v (P8 V8) / l, rounded to bf16;
 *   LSE = (m + log2(l / 448)) ln 2.
 * Arguments as h3_varlen_attn_fwd except: D must be 128 (else
 * H3_ERR_UNSUPPORTED) and the workspace is >= h3_sage_workspace_size bytes.
 * Launches: a V max pass, a quantisation pass (RoPE fused), the FP8 attention
 * kernel. Invalid cu_seqlens set H3_ERR_BAD_SEQLENS without any access
 * outside [0, N). Deterministic. */
h3_status h3_varlen_attn_fwd_sage(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *cu_seqlens, int32_t nseg,
                                  int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                                  int64_t N, int32_t H, int32_t D, float softmax_scale,
                                  void *workspace, size_t workspace_bytes, h3_stream_t stream);

/* Waits for `stream`, then writes to *count the number of (32-row block, key
 * tile) pairs the last h3_varlen_attn_fwd_skip call on `workspace` skipped.
 * H3_ERR_WORKSPACE / H3_ERR_INVALID_ARG on null pointers, H3_ERR_CUDA if the
 * copy fails. */
h3_status h3_read_skip_count(const void *workspace, h3_stream_t stream, uint64_t *count);

/* QKV projection with the rotary embedding fused into its epilogue: the step
 * that produces this path's q, k, v inside a DiT block. "MiniMax-H3
 * Reference" Space README, section "AoTI-compiled blocks" (rotary epilogues
 * around the block's matmuls); "MiniMax H3" vLLM-Omni recipe, section "Online
 * FP8 quantization" (the attention's qkv projection is one of the DiT
 * linears; BF16 here). Computes, with HD = H*D,
 *     Y = x w^T                                   (fp32 accumulation)
 *     q = RoPE(Y[:, 0:HD]),  k = RoPE(Y[:, HD:2HD]),  v = Y[:, 2HD:3HD]
 * with RoPE as in h3_rope_apply (same table, pair layout and rounding
 * sequence) but applied to the fp32 accumulator, each output rounded once to
 * bf16 (round to nearest even). With pos NULL no rotation is applied and
 * `rope` is ignored.
 *   x        : device bf16 [N, K] row-major, 16-byte aligned.
 *   w        : device bf16 [3*H*D, K] row-major (the linear layer's weight:
 *              rows [0, HD) make q, [HD, 2HD) k, [2HD, 3HD) v), 16-byte aligned.
 *   q, k, v  : device bf16 [N, H, D] each, 16-byte aligned, overlapping
 *              neither each other nor x, w.
 *   pos      : device fp32 [N, 3] or NULL.
 *   N >= 0 (N = 0 is a no-op), N < 2^31; K a multiple of 64, 64 <= K <= 2^20;
 *   D in {64, 128}; H >= 1 with H*D a multiple of 256 and 3*H*D <= 2^20.
 *   workspace: device, 256-byte aligned, >= 256 bytes (its status word, which
 *              a timed-out bounded wait sets to H3_ERR_DEVICE_TIMEOUT; read
 *              it with h3_read_device_status). Reset by every call.
 * One persistent kernel launch (one CTA per SM), deterministic. */
h3_status h3_qkv_rope_gemm(const void *x, const void *w, void *q, void *k, void *v,
                           const float *pos, h3_rope_cfg rope, int64_t N, int32_t K,
                           int32_t H, int32_t D, void *workspace, size_t workspace_bytes,
                           h3_stream_t stream);

/* The QKV projection with RoPE in its epilogue, chained into the attention:
 * h3_qkv_rope_gemm(x, w -> q, k, v, rotating q and k by pos), then
 * h3_varlen_attn_fwd on q, k, v with pos = NULL. The keys reach the attention
 * already rotated, so no rotary pass over k runs and no rotated-key workspace
 * is needed; each rotation happens once, in the projection's epilogue
 * ("MiniMax-H3 Reference" Space README, section "AoTI-compiled blocks":
 * rotary epilogues around the block's matmuls).
 *   x, w, pos, rope, N, K, H, D : as for h3_qkv_rope_gemm (pos may be NULL:
 *              no rotation anywhere).
 *   q, k, v    : device bf16 [N, H, D], written by the projection and read
 *              by the attention (the caller owns them and may read them).
 *   o, lse, cu_seqlens, nseg, max_seqlen, softmax_scale : as for
 *              h3_varlen_attn_fwd.
 *   workspace  : device, 256-byte aligned, >= 256 bytes: one status word
 *              for both launches, reset once at the start; a bounded wait
 *              that times out in either kernel, or invalid cu_seqlens found
 *              by the attention kernel, leaves its code there
 *              (h3_read_device_status).
 * Errors: the attention's argument checks run before anything is launched,
 * then those of h3_qkv_rope_gemm; the first failing check's status is
 * returned. Two kernel launches (projection, attention), asynchronous on
 * `stream`; deterministic. */
h3_status h3_qkv_rope_attn_fwd(const void *x, const void *w, void *q, void *k, void *v,
                               void *o, float *lse, const int32_t *cu_seqlens, int32_t nseg,
                               int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                               int64_t N, int32_t K, int32_t H, int32_t D, float softmax_scale,
                               void *workspace, size_t workspace_bytes, h3_stream_t stream);

/* Bytes of the scratch array compiled into the library for
 * h3_varlen_attn_fwd_static: a 256-byte status block plus room for the
 * rotated keys of N*H*D <= 2^25 elements (64 MiB of bf16). */
#define H3_STATIC_WORKSPACE_BYTES (256u + (64u << 20))

/* h3_varlen_attn_fwd for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment convenience. Hosts
 * that own all device memory (their own arena or a fixed budget, allocation
 * only at start-up) cannot give h3_varlen_attn_fwd a workspace; this call
 * allocates nothing and uses a scratch array compiled into the library
 * instead (H3_STATIC_WORKSPACE_BYTES of device memory, held until the
 * process exits: under CUDA's default lazy module loading only on devices
 * where this call is used; with CUDA_MODULE_LOADING=EAGER on every device
 * whose context maps the library). Arguments and results are those of
 * h3_varlen_attn_fwd without the workspace pair.
 *   Check order: N, H, nseg out of range -> H3_ERR_INVALID_ARG and D not in
 *          {64, 128} -> H3_ERR_UNSUPPORTED (as h3_varlen_attn_fwd); then
 *          N*H*D*2 + 256 > H3_STATIC_WORKSPACE_BYTES (N*H*D > 2^25) ->
 *          H3_ERR_WORKSPACE; then every check of h3_varlen_attn_fwd. Nothing
 *          is enqueued on any of these errors.
 *   Set-up: every call looks up the array's device address on the current
 *          device (cudaGetSymbolAddress), so the call stays valid after the
 *          context is reset. The first call on a device also loads the
 *          array's module; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array. Calls that can run
 *          concurrently on the GPU (different streams, no ordering) race on
 *          it and must be serialised by the caller. Each call resets the
 *          status word and rewrites all of the scratch it reads.
 *   Device status: the array's status word is not exposed; a caller that
 *          needs H3_ERR_BAD_SEQLENS / H3_ERR_DEVICE_TIMEOUT from the device
 *          uses h3_varlen_attn_fwd with its own workspace. */
h3_status h3_varlen_attn_fwd_static(const void *q, const void *k, const void *v, void *o,
                                    float *lse, const int32_t *cu_seqlens, int32_t nseg,
                                    int32_t max_seqlen, const float *pos, h3_rope_cfg rope,
                                    int64_t N, int32_t H, int32_t D, float softmax_scale,
                                    h3_stream_t stream);

/* Failure-detection self-test (no counterpart on the pages): one warp runs the
 * same bounded mbarrier wait the attention kernel uses, on a barrier that
 * nothing arrives on, giving up after `limit_cycles` SM clock cycles
 * (1 .. 4e9; the attention kernel's own limit is 2e9, about one second). The
 * kernel then writes H3_ERR_DEVICE_TIMEOUT to the status word of `workspace`
 * (>= 256 bytes, 256-byte aligned) and returns normally, so the CUDA context
 * stays usable; read it with h3_read_device_status. Asynchronous on `stream`. */
h3_status h3_selftest_bounded_wait(void *workspace, size_t workspace_bytes,
                                   int64_t limit_cycles, h3_stream_t stream);

/* Waits for `stream`, then returns the device status word of the last call
 * that used `workspace` (H3_OK, H3_ERR_BAD_SEQLENS or H3_ERR_DEVICE_TIMEOUT),
 * or H3_ERR_CUDA if the copy fails. */
h3_status h3_read_device_status(const void *workspace, h3_stream_t stream);

/* Static description of a status code. Never NULL. */
const char *h3_status_string(h3_status status);

/* cudaError_t value of the most recent H3_ERR_CUDA on the calling thread
 * (0 if none). */
int32_t h3_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* H3ATTN_H */
