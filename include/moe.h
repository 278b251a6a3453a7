/*
 * moe.h -- C ABI of the B200 (sm_100a) library for the LongCat-Flash MoE layer with
 * zero-computation experts.
 *
 * What the layer computes ("衝上熱搜！美團大模型，靠「快」火了", section 零計算專家): the expert
 * pool holds N SwiGLU FFN experts and Z zero-computation experts (E = N + Z).  A softmax router
 * R scores all E experts for each token x_t; a per-expert bias b_i is added to the router
 * probability for the top-K selection only; the gate g_i is the (unbiased, not renormalised)
 * probability; the output is y_t = sum over the K selected experts of g_i * E_i(x_t), where an
 * FFN expert is E(x) = W_d (silu(W_g x) * (W_u x)) and a zero expert returns x_t unchanged.
 * A PID controller on the biases (same page, last paragraph of that section) holds the mean
 * number of FFN experts per token near a set-point.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller owns every buffer.
 *     The library never allocates or frees device memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t passed as void*; every call only enqueues work on it and
 *     returns without synchronising (except moe_last_device_error).  Calls on one stream are
 *     ordered; calls sharing a workspace must not run concurrently on different streams.
 *   - bf16 tensors are arrays of uint16_t bit patterns (moe_bf16).  Layouts are row-major and
 *     contiguous.  Shapes use the dims struct: T tokens, d model width, N FFN experts of
 *     intermediate width I, Z zero experts, K experts per token.
 *   - Limits: T >= 0; d and I positive multiples of 64; N >= 0, Z >= 0, 1 <= N + Z <= 1024;
 *     1 <= K <= min(N + Z, 32); T * K < 2^31; flags a combination of the MOE_* flags below.
 *     Violations return MOE_ERR_SHAPE.
 *   - Every tensor pointer must be 16-byte aligned (MOE_ERR_ALIGN otherwise); a workspace
 *     must be 256-byte aligned.  A NULL required pointer returns MOE_ERR_ARG.
 *   - Errors are reported by the return code before anything is enqueued; a launch failure
 *     returns MOE_ERR_CUDA.  Kernels never trap: a device-side check that fails (a bounded wait
 *     that gave up, an expert id or row index out of range) records a code in the workspace's
 *     status word, skips the offending access and lets the kernel finish; read it with
 *     moe_last_device_error.  No call aborts the process.
 *   - T == 0 is valid: outputs are left as described per call (counts zeroed where written),
 *     and every token-sized pointer (x, y, top-K, dispatch and grouped-row buffers) may then be
 *     NULL.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16; /* bf16 bit pattern */

typedef struct {
    int32_t T; /* tokens in the batch */
    int32_t d; /* model width */
    int32_t N; /* FFN experts (ids 0 .. N-1) */
    int32_t Z; /* zero-computation experts (ids N .. N+Z-1) */
    int32_t K; /* experts selected per token */
    int32_t I; /* intermediate width of each SwiGLU FFN expert */
    uint32_t flags; /* variant switches (MOE_RENORMALIZE_GATES, MOE_FP8_ACTIVATIONS,
                       MOE_FUSED_COMBINE); 0 = the layer as defined */
} moe_dims;

/* Gates renormalised over the selected set: g_i = p_i / sum of p over the K selected experts
 * (zero experts included), instead of the layer's unrenormalised p_i.  An optional variant;
 * it changes moe_route's topk_gate and hence everything downstream, not the selection. */
#define MOE_RENORMALIZE_GATES 1u

/* FP8 activations, for the FP8-weight entry points only (moe_expert_ffn_fp8, moe_forward_fp8;
 * the bf16 ones return MOE_ERR_ARG when it is set): the inputs of both expert GEMMs -- the token
 * rows and h -- are quantised to E4M3 with one power-of-two scale per token per 128 channels
 * (the activation side of the DeepSeek-V3 block scheme that "衝上熱搜！美團大模型，靠「快」火了",
 * §系統級優化 names; scale rule and rounding as in moe_quantize_fp8, see moe_quantize_fp8_rows),
 * and the tensor cores multiply E4M3 by E4M3 with fp32 sums, each 128-long block of the
 * reduction scaled by its weight and activation scales.  Requires d and I multiples of 128
 * (MOE_ERR_SHAPE otherwise); the codes and scales of x_perm and h live in the workspace scratch
 * (moe_scratch_size grows by about T*K*(d + I)*1.03 bytes). */
#define MOE_FP8_ACTIVATIONS 2u

/* The combine fused into the down projection, for moe_forward / moe_forward_timed with bf16
 * weights only (every other entry point returns MOE_ERR_ARG when it is set): the down
 * projection's epilogue counts, per token and feature block, the FFN rows it has stored; the
 * tile completing a token's count sums that block of y_t from the token's rows in slot order
 * with the combine's arithmetic, so y is bit-identical to the unfused layer whichever tile
 * finishes last; tokens without an FFN slot are written by a zero-only combine pass.  The down
 * projection then runs on single CTAs, and the workspace grows by T * 4 * ceil(d / 256) * 4
 * bytes of counters (set by the call).  An optional variant after the CSDN codearts article
 * on LongCat-Flash, §二、训练优化 (tiles accumulated in a deterministic order, the fp32 addition
 * fused into the GEMM epilogue instead of written back and re-read). */
#define MOE_FUSED_COMBINE 4u

/* PID gains and set-point: target = desired mean number of FFN experts per token.
 * balance_gamma: step of the per-expert balancing term (see moe_bias_update); 0 = off. */
typedef struct {
    float target;
    float kp;
    float ki;
    float kd;
    float balance_gamma;
} moe_pid_params;

enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,       /* NULL pointer or invalid parameter value */
    MOE_ERR_SHAPE = 2,     /* dims outside the supported limits */
    MOE_ERR_ALIGN = 3,     /* pointer not 16-byte (tensor) / 256-byte (workspace) aligned */
    MOE_ERR_WORKSPACE = 4, /* ws_bytes smaller than required */
    MOE_ERR_CUDA = 5,      /* a CUDA runtime call or kernel launch failed */
    MOE_ERR_DEVICE = 6,    /* a device-side check failed (see moe_last_device_error) */
    MOE_ERR_ARCH = 7       /* the current device is not sm_100 (B200-class) */
};

/* Device-side status codes reported by moe_last_device_error (0 = none). */
enum {
    MOE_DEV_OK = 0,
    MOE_DEV_WAIT_TIMEOUT = 0x100, /* a pipeline wait in the grouped GEMM gave up (bounded) */
    MOE_DEV_BAD_EXPERT = 0x200,   /* an expert id outside [0, N+Z) was met */
    MOE_DEV_BAD_ROWS = 0x300      /* group offsets not monotone or beyond T*K rows */
};

/* Human-readable text for a return code (host only; never NULL). */
const char *moe_strerror(int code);

/* Workspace bytes needed by moe_forward for these dims (0 for invalid dims).  The workspace
 * holds the status word, router logits, top-K results, dispatch tables, the grouped
 * activations x_perm [T*K, d], the SwiGLU activations h [T*K, I] and the expert outputs
 * y_perm [T*K, d]; about (2d + I) * 2 * T * K bytes plus small tables.  The flags add their
 * regions: MOE_FP8_ACTIVATIONS the codes and block scales of the token rows and of h (in the
 * scratch part, about (d + I) * 1.03 * T * K bytes), MOE_FUSED_COMBINE one counter per token
 * and 64-feature block (T * 4 * ceil(d / 256) * 4 bytes). */
size_t moe_workspace_size(const moe_dims *dims);

/* Scratch bytes needed by the staged calls (moe_route, moe_dispatch, moe_expert_ffn): the
 * status word, split-K router logits and per-chunk histograms.  Always <= the above. */
size_t moe_scratch_size(const moe_dims *dims);

/* Router R and biased top-K ("衝上熱搜！美團大模型，靠「快」火了", §零計算專家: softmax
 * router over all N+Z experts; b_i shifts the selection score only).
 *   x        [T, d] bf16            tokens
 *   W_r      [N+Z, d] bf16          router weights; logits l = x W_r^T (fp32 accumulation on
 *                                   tensor cores)
 *   b        [N+Z] fp32             per-expert selection bias
 *   topk_idx [T, K] int32   (out)   selected expert ids, ascending
 *   topk_gate[T, K] fp32    (out)   g_i = softmax(l)_i of the selected ids (not renormalised;
 *                                   with MOE_RENORMALIZE_GATES divided by their fp32 sum)
 *   gap      [T] fp32       (out, nullable)  s_(K) - s_(K+1) with s = softmax(l) + b
 *                                   (+inf when K == N+Z); a small gap marks a near-tie
 * Exact score ties go to the lower expert id. */
int moe_route(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r, const float *b,
              int32_t *topk_idx, float *topk_gate, float *gap, void *ws, size_t ws_bytes,
              void *stream);

/* The router logits l = x W_r^T (same section: the scores the softmax router R normalises)
 * that the last moe_route or moe_forward with these dims computed into workspace `ws`, summed
 * over the router GEMM's split-K partials in the same fixed order the top-K kernel sums them,
 * so they are bit-identical to the logits the selection used.  For inspecting the router's
 * fp32 accuracy; calls on the same stream after that routing call see its logits.
 *   ws      the workspace given to that call (>= moe_scratch_size(dims) bytes)
 *   logits  [T, N+Z] fp32 (out) */
int moe_router_logits(const moe_dims *dims, const void *ws, size_t ws_bytes, float *logits,
                      void *stream);

/* Dispatch: group the FFN slots by expert (zero-expert slots are never copied).  Stable
 * counting sort with key (expert id, token), deterministic.
 *   x         [T, d] bf16, topk_idx/topk_gate [T, K] as produced by moe_route (ids in
 *             ascending order per token, each in [0, N+Z))
 *   counts    [N+Z] int32   (out)   slots per expert (zero experts included)
 *   offsets   [N+1] int32   (out)   row offset of each FFN expert's group; offsets[N] = A,
 *                                   the number of FFN slots
 *   perm_tok  [T*K] int32   (out)   token of grouped row r (r < A)
 *   perm_gate [T*K] fp32    (out)   gate of grouped row r
 *   slot_pos  [T, K] int32  (out)   grouped row of slot (t, k), -1 for a zero-expert slot
 *   x_perm    [T*K, d] bf16 (out, nullable)  x_perm[r] = x[perm_tok[r]] for r < A; NULL skips
 *                                   the copy (moe_expert_ffn_gather reads x directly)
 * Rows r >= A of the [T*K]-sized outputs are left untouched. */
int moe_dispatch(const moe_dims *dims, const moe_bf16 *x, const int32_t *topk_idx,
                 const float *topk_gate, int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                 float *perm_gate, int32_t *slot_pos, moe_bf16 *x_perm, void *ws,
                 size_t ws_bytes, void *stream);

/* moe_dispatch for callers that cannot provide a workspace.  The pages have no counterpart;
 * this exists for library users, not for the layer's definition.  Some callers cannot give
 * the library device memory: a plugin whose host process owns all device memory through its
 * own pool, or a deployment whose memory budget forbids allocations after start-up.  This
 * variant takes the same arguments as moe_dispatch minus the workspace and produces the same
 * outputs; its scratch is a fixed 1 MiB array inside the library image (present on every GPU
 * that loads the library, until the process exits).
 *   - needs ceil(T/256) * (N+Z) <= 262144; larger requests return MOE_ERR_WORKSPACE;
 *   - calls share that array: two calls whose kernels overlap on the GPU race on it;
 *   - device-side checks still skip bad accesses but have no status word to report to;
 *   - the first call on a device looks up the array's device address with that device
 *     current; make that first call before any stream capture.
 * It allocates and frees nothing. */
int moe_dispatch_noalloc(const moe_dims *dims, const moe_bf16 *x, const int32_t *topk_idx,
                         const float *topk_gate, int32_t *counts, int32_t *offsets,
                         int32_t *perm_tok, float *perm_gate, int32_t *slot_pos,
                         moe_bf16 *x_perm, void *stream);

/* The FFN experts on the grouped rows (grouped GEMMs on tcgen05 tensor cores):
 *   h[r]      = silu(x_perm[r] W_g[e]^T) * (x_perm[r] W_u[e]^T)       bf16 [T*K, I]
 *   y_perm[r] = perm_gate[r] * (h[r] W_d[e]^T)                          bf16 [T*K, d]
 * for every row r in [offsets[e], offsets[e+1]) of FFN expert e (gate applied in fp32 before
 * the bf16 rounding).  Weights in their natural layouts: W_g, W_u [N, I, d]; W_d [N, d, I].
 * offsets must be non-decreasing with offsets[N] <= T*K (checked on the device). */
int moe_expert_ffn(const moe_dims *dims, const moe_bf16 *x_perm, const int32_t *offsets,
                   const float *perm_gate, const moe_bf16 *W_g, const moe_bf16 *W_u,
                   const moe_bf16 *W_d, moe_bf16 *h, moe_bf16 *y_perm, void *ws,
                   size_t ws_bytes, void *stream);

/* moe_expert_ffn with the dispatch gather fused into the up-projection: grouped row r's
 * token row is read straight from x[perm_tok[r]] by the GEMM's own loads, so no x_perm copy is
 * written or read: T*K*d*2 bytes of memory saved, at some cost in speed at large T (the
 * row-by-row copies; moe_forward keeps the copy).  A perm_tok value outside [0, T) is
 * reported as MOE_DEV_BAD_ROWS and row 0 is read instead.  Arguments as moe_expert_ffn, with
 *   x        [T, d] bf16      the tokens (as given to moe_dispatch)
 *   perm_tok [T*K] int32      token of each grouped row, from moe_dispatch (values in [0, T))
 * in place of x_perm.  h and y_perm are bit-identical to moe_expert_ffn on the gathered
 * x_perm. */
int moe_expert_ffn_gather(const moe_dims *dims, const moe_bf16 *x, const int32_t *perm_tok,
                          const int32_t *offsets, const float *perm_gate, const moe_bf16 *W_g,
                          const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *h,
                          moe_bf16 *y_perm, void *ws, size_t ws_bytes, void *stream);

/* Dense SwiGLU FFN, y = W_d (silu(W_g x) * (W_u x)) for every token: the shortcut branch of
 * ScMoE ("衝上熱搜！美團大模型，靠「快」火了", §快捷連接 MoE: the previous block's dense FFN runs
 * in parallel with the current MoE layer, which on one GPU means on a second stream beside
 * moe_forward; the MoE layer and this call share no buffers, so they may overlap).  Uses the
 * experts' grouped GEMMs with one group of T rows and gate 1.  Only dims->T, d and I are read
 * (I = the dense intermediate width; d and I positive multiples of 64).
 *   x [T, d] bf16; W_g, W_u [I, d] bf16; W_d [d, I] bf16
 *   h [T, I] bf16 (out, scratch)    y [T, d] bf16 (out)
 *   ws: a workspace of at least 256 bytes, first 256 zero (its status word is used); do not
 *   share it with a concurrent moe_forward. */
int moe_dense_ffn(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_g,
                  const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *h, moe_bf16 *y, void *ws,
                  size_t ws_bytes, void *stream);

/* Combine / un-permute: y_t = sum over FFN slots k (ascending expert id) of y_perm[slot_pos]
 * + (sum of the zero-expert gates of t) * x_t, accumulated in fp32 in that fixed order and
 * rounded once to bf16.  Zero experts are identities ("衝上熱搜！美團大模型，靠「快」火了",
 * §零計算專家), so they cost one fused scalar-times-row term and no copy.
 *   y  [T, d] bf16 (out).
 *   ws a workspace of at least 256 bytes whose status word (its first 4 bytes, zero before the
 *      first call) records MOE_DEV_BAD_ROWS when an FFN slot's slot_pos lies outside
 *      [0, T*K); that slot's term is skipped.  Any workspace of the other calls will do. */
int moe_combine(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *y_perm,
                const int32_t *topk_idx, const float *topk_gate, const int32_t *slot_pos,
                moe_bf16 *y, void *ws, size_t ws_bytes, void *stream);

/* PID update of the FFN experts' biases from one batch's counts (same page and section, last
 * paragraph; the law is a reading, the pages give no equation):
 *   m = sum_{i<N} counts[i] / T;  e = (target - m) / K;  integral += e;
 *   u = kp*e + ki*integral + kd*(e - e_prev);  e_prev = e;  b[i] += u for i < N.
 * fp32, one rounding per operation in that order (bit-reproducible on the host).
 * Then, when params->balance_gamma != 0, the per-expert term of the aux-loss-free bias scheme
 * that the PID refines (same section: the expert-specific bias follows recent expert usage;
 * the rule is that scheme's published one): b[i] += balance_gamma * sign(mean - counts[i]) for
 * i < N, mean = sum_{i<N} counts[i] / N, the sign taken exactly from the integers
 * (sign(total - N*counts[i])).  balance_gamma must be finite (MOE_ERR_ARG otherwise).
 *   counts    [N+Z] int32 (as written by moe_dispatch / moe_forward)
 *   b         [N+Z] fp32  (in/out)  zero-expert biases are not changed
 *   pid_state [2] fp32    (in/out)  {integral, e_prev}; zero-initialise before the first step
 * T == 0 changes nothing. */
int moe_bias_update(const moe_dims *dims, const int32_t *counts, float *b, float *pid_state,
                    const moe_pid_params *params, void *stream);

/* The whole layer in one call: moe_route, moe_dispatch, moe_expert_ffn and moe_combine on
 * buffers carved from the workspace, with no host synchronisation.
 *   y      [T, d] bf16 (out)
 *   counts [N+Z] int32 (out, nullable)  per-expert slot counts of this batch, for
 *          moe_bias_update
 *   ws     >= moe_workspace_size(dims) bytes. */
int moe_forward(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r, const float *b,
                const moe_bf16 *W_g, const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *y,
                int32_t *counts, void *ws, size_t ws_bytes, void *stream);

/* moe_forward with timing hooks: when stage_events is not NULL it must hold
 * MOE_NUM_STAGE_EVENTS created cudaEvent_t handles (passed as void*); event i is recorded on
 * `stream` right before stage i is enqueued and the last one after the final stage:
 *   0 router logits GEMM   1 softmax + biased top-K   2 dispatch (histogram, scan, permute,
 *   gather)   3 FFN up-projection GEMM with SwiGLU   4 FFN down-projection GEMM   5 combine
 *   6 end.
 * Stages are enqueued exactly as by moe_forward; only the event records are added. */
#define MOE_NUM_STAGE_EVENTS 7
int moe_forward_timed(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r,
                      const float *b, const moe_bf16 *W_g, const moe_bf16 *W_u,
                      const moe_bf16 *W_d, moe_bf16 *y, int32_t *counts, void *ws,
                      size_t ws_bytes, void *const *stage_events, void *stream);

/* ---------------------------------------------------------------- FP8 expert weights
 * Block-wise FP8 quantisation ("衝上熱搜！美團大模型，靠「快」火了", §系統級優化: the same
 * fine-grained block-wise scheme as DeepSeek-V3, one scale per 128 x 128 weight block).  For
 * each of G matrices w[g] [R, C] and each 128 x 128 block: e = the smallest integer with
 * max|w| <= 448 * 2^e (e >= -126; 0 for an all-zero block), scale = 2^e, and
 * q = E4M3(w / 2^e), rounded to nearest with ties to even and saturated at +-448 (E4M3: 1 sign,
 * 4 exponent bits biased by 7, 3 mantissa bits, S.1111.111 = NaN, largest finite 448).  The
 * element format and the power-of-two scale are readings; with them q * scale is exact in
 * bf16.
 *   w     [G, R, C] bf16            R and C multiples of 128 (MOE_ERR_SHAPE otherwise)
 *   q     [G, R, C] uint8 (out)     E4M3 codes
 *   scale [G, R/128, C/128] fp32 (out)
 * Expert weights: W_g and W_u with G = N, R = I, C = d; W_d with G = N, R = d, C = I. */
int moe_quantize_fp8(const moe_bf16 *w, int64_t G, int64_t R, int64_t C, uint8_t *q,
                     float *scale, void *stream);

/* Block-wise FP8 of activation rows (the MOE_FP8_ACTIVATIONS variant): for each row r of
 * x [R, C] bf16 and each 1 x 128 block of it, e = the smallest integer with max|x| <= 448 * 2^e
 * (e >= -126; 0 for an all-zero block) and q = E4M3(x / 2^e), nearest, ties to even (the rule
 * of moe_quantize_fp8 on 1 x 128 blocks).
 *   x     [R, C] bf16                C a multiple of 128 (MOE_ERR_SHAPE otherwise)
 *   q     [R, C] uint8 (out)         E4M3 codes
 *   scale [C/128, R] fp32 (out)      block-major: scale[(c / 128) * R + r] = 2^e
 * All pointers 16-byte aligned. */
int moe_quantize_fp8_rows(const moe_bf16 *x, int64_t R, int64_t C, uint8_t *q, float *scale,
                          void *stream);

/* moe_expert_ffn with block-quantised expert weights (from moe_quantize_fp8): each weight
 * tile is read as E4M3 codes (half the bytes of bf16) and turned into the exact bf16 weights
 * q * scale in shared memory; activations, accumulation and outputs are as in moe_expert_ffn,
 * so the result equals moe_expert_ffn on the dequantised weights.  d and I must be multiples
 * of 128.  With MOE_FP8_ACTIVATIONS in dims->flags the activations are quantised too and the
 * tensor cores read E4M3 on both sides (see the flag); h is then unused (may be NULL) and the
 * quantised h stays in the workspace. */
int moe_expert_ffn_fp8(const moe_dims *dims, const moe_bf16 *x_perm, const int32_t *offsets,
                       const float *perm_gate, const uint8_t *q_g, const float *s_g,
                       const uint8_t *q_u, const float *s_u, const uint8_t *q_d,
                       const float *s_d, moe_bf16 *h, moe_bf16 *y_perm, void *ws,
                       size_t ws_bytes, void *stream);

/* moe_forward with block-quantised expert weights (the router weights stay bf16);
 * stage_events as in moe_forward_timed, or NULL.  With MOE_FP8_ACTIVATIONS the token rows are
 * quantised straight from x through the dispatch permutation (no bf16 copy of them is made) and
 * both expert GEMMs multiply E4M3 by E4M3; the workspace is moe_workspace_size of those dims. */
int moe_forward_fp8(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r,
                    const float *b, const uint8_t *q_g, const float *s_g, const uint8_t *q_u,
                    const float *s_u, const uint8_t *q_d, const float *s_d, moe_bf16 *y,
                    int32_t *counts, void *ws, size_t ws_bytes, void *const *stage_events,
                    void *stream);

/* Synchronises `stream`, returns the device status word of the workspace (MOE_DEV_* code,
 * 0 if none) and clears it.  Returns a negative value if the synchronisation itself failed. */
int moe_last_device_error(void *ws, void *stream);

/* Testing hook for the failure path of the grouped GEMMs (moe_route's router GEMM, the expert
 * FFN GEMMs, moe_dense_ffn): sets, for launches enqueued afterwards by this process, the SM
 * clock cycles after which one pipeline wait gives up; 0 restores the default of 2^32 cycles.
 * With a limit shorter than a real wait (e.g. 64 cycles: no tile completes that fast) the
 * kernel records MOE_DEV_WAIT_TIMEOUT, unwinds every role, waits (bounded) for its copies and
 * MMAs in flight, frees its tensor memory and exits, so the context stays usable.  Not for
 * production use.  Returns MOE_ERR_ARG for a negative value. */
int moe_debug_set_wait_limit(int64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
