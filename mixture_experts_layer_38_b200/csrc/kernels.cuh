// kernels.cuh -- host-side launchers of the library's kernels (internal C++ interface between
// the C ABI in moe_api.cu and the kernel files).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ------------------------------------------------------------------ grouped GEMM (tcgen05)
// Output tile = 2 x (128 weight rows) x (<= 128 or 256 activation rows); see gemm.cu.
enum EpiKind : int {
  kEpiSwiGLU = 0,  // h = silu(A0 x) * (A1 x)           -> bf16 [rows, M]
  kEpiGated = 1,   // y = row_scale[r] * (A x)          -> bf16 [rows, M]
  kEpiF32 = 2,     // logits (split-K partials)         -> fp32 [splits][rows, M]
  kEpiGatedCombine = 3  // kEpiGated, then the layer's combine fused in: the last tile to store
                        // a token's rows of a feature block sums that block of y (gemm.cu)
};

struct GemmArgs {
  CUtensorMap map_a0;    // weight rows (box 64 x 128)
  CUtensorMap map_a1;    // W_u for SwiGLU, the same tensor as map_a0 otherwise
  CUtensorMap map_a01;   // map_a0's tensor in 64 x 256 boxes: both 128-row blocks at once when
                         // they are adjacent rows (down projection, router)
  // The same three weight maps for tiles that read their weights exactly once (Tile::once):
  // 256-byte L2 promotion, so each 128-byte row segment a stage requests also brings the next
  // k-slice's segment into L2, doubling the bytes in flight of a weight-streaming tile.
  CUtensorMap map_s0, map_s1, map_s01;
  CUtensorMap map_b[4];  // activation rows, boxes of 128 / 64 / 32 / 16 rows x 64 columns
  CUtensorMap map_b256;  // activation rows, boxes of 256 rows
  const int32_t *group_offsets;  // [num_groups + 1] activation-row offsets, or nullptr
  int num_groups;                // groups (experts); 1 when group_offsets == nullptr
  int rows;                      // activation rows available (bound for group_offsets)
  int M;                         // weight rows per group that produce outputs
  int K;                         // reduction length, a multiple of 64
  int k_splits;                  // split-K factor (kEpiF32 only)
  void *out;
  int out_ld;                    // elements per output row
  long long split_stride;        // elements between split-K partial outputs
  const float *row_scale;        // kEpiGated: per-row gate (NULL: 1)
  int *status;                   // device status word
  // Row gather (up-projection only): when row_index is set, activation row r is row
  // row_index[r] of the row-major bf16 matrix gather_src (K columns), copied by loader warps;
  // map_b / map_b256 are then unused.
  const int *row_index;
  const void *gather_src;
  int gather_rows;               // rows of gather_src; row indices outside are reported, not read
  // FP8 weights (launch_grouped_gemm_fp8): map_a0 / map_a1 cover E4M3 codes (64 x 128 boxes,
  // no swizzle); the scale of the 128 x 128 block holding weight row r, column k is
  // scale_a0/1[(r / 128) * scale_ld + k / 128].
  const float *scale_a0;
  const float *scale_a1;
  int scale_ld;
  // Cycles after which one pipeline wait gives up (set by the launchers; see
  // gemm_set_wait_limit).
  long long wait_limit;
  // E4M3 activations (launch_grouped_gemm_e4m3): the scale of activation row r, columns
  // [128 kb, 128 kb + 128) is act_scale[kb * rows + r]; with kEpiSwiGLU the kernel writes h as
  // E4M3 codes (out, [rows, M] bytes) and their scales to out_scale[(f / 128) * rows + r].
  const float *act_scale;
  float *out_scale;
  // kEpiGatedCombine: the combine of the MoE layer (see launch_combine) fused into the down
  // projection.  cmb_count [T, cmb_blocks] holds each token's FFN-slot count at launch
  // (launch_combine_counters); cmb_blocks = 4 * m-tiles.
  const uint16_t *cmb_x;        // [T, M] token inputs
  const int32_t *cmb_perm_tok;  // [rows] token of each grouped row
  const int32_t *cmb_idx;       // [T, K] selected expert ids, ascending
  const float *cmb_gate;        // [T, K] gates
  const int32_t *cmb_slot;      // [T, K] grouped row of each FFN slot
  int *cmb_count;
  uint16_t *cmb_y;              // [T, M] layer output
  int cmb_K, cmb_N, cmb_blocks;
};

// Grouped GEMM block: warp 0 issues TMA loads, warp 1 allocates TMEM and issues MMAs, and
// kGemmEpiWarps warps (a multiple of 4: one per TMEM lane quarter, per group) drain TMEM.
// Eight shortened the MMA thread's waits for a free accumulator at 256-token tiles but were no
// faster: those tiles run at the board's power limit, where idle tensor cycles cost no time.
constexpr int kGemmEpiWarps = 4;
constexpr int kGemmThreads = 64 + 32 * kGemmEpiWarps;
cudaError_t gemm_prepare(int device);  // sets the kernels' shared-memory limit once per device
// Wait limit in SM cycles for grouped-GEMM launches enqueued from now on (0: the default,
// kWaitLimitCycles).  A testing hook for the timeout path.
void gemm_set_wait_limit(long long cycles);
// Token-tile width (128 or 256) for `rows` activation rows over `groups` groups, reduction K.
int gemm_tile_tokens(long long rows, int groups, int K);
cudaError_t launch_grouped_gemm(int epi, const GemmArgs &args, int grid, int tile_tokens,
                                cudaStream_t stream);
// SwiGLU or gated grouped GEMM on CTA pairs (clusters of two SMs, pair MMAs of 256 weight
// rows) running two pipelines per pair at once: full 224-token tiles (and tails over 32 rows)
// beside tails of at most 32 rows, so tensor work and weight streaming overlap within each SM.
// Needs M a multiple of 256 (SwiGLU) or 512 (gated), group row counts within gemm_dual_fits;
// `pairs` = the persistent pairs to launch (gemm_max_dual_pairs caps it).
cudaError_t launch_grouped_gemm_dual(int epi, const GemmArgs &args, int pairs,
                                     cudaStream_t stream);
int gemm_max_dual_pairs(int device);  // co-resident pairs on the device (gemm_prepare queries it)
bool gemm_dual_fits(long long rows, int groups);
// SwiGLU or gated grouped GEMM with E4M3 weights AND E4M3 activations (tcgen05.mma
// kind::f8f6f4): map_a0 / map_a1 cover weight codes and map_b[1..3] activation codes in
// 128-byte-swizzled boxes of 128 columns (64 / 32 / 16 rows for the tokens); scale_a0/1 and
// act_scale as described in GemmArgs.  K and M multiples of 128.
cudaError_t launch_grouped_gemm_e4m3(int epi, const GemmArgs &args, int grid,
                                     cudaStream_t stream);
cudaError_t gemm_e4m3_prepare();  // sets the kernels' shared-memory limit (gemm_prepare calls it)
long long gemm_wait_limit();      // the current gemm_set_wait_limit value (0: the default)
// SwiGLU or gated grouped GEMM with E4M3 block-quantised weights, 128-token tiles.
cudaError_t launch_grouped_gemm_fp8(int epi, const GemmArgs &args, int grid,
                                    cudaStream_t stream);

// Block-wise E4M3 of G matrices [R, C] bf16 (R, C multiples of 128): codes and one power-of-two
// scale per 128 x 128 block.
cudaError_t launch_quantize_fp8(const uint16_t *w, long long G, long long R, long long C,
                                uint8_t *q, float *scale, cudaStream_t stream);

// FP8 activations: rows of the bf16 matrix x [R, C] (C a multiple of 128) -> E4M3 codes q
// [R, C] and one power-of-two scale per 1 x 128 block, stored block-major:
// scale_t[(c / 128) * R + r].  Rows from *live_rows on are skipped (live_rows may be NULL).
// With row_index, output row r quantises row row_index[r] of x ([src_rows, C]); indices outside
// that range are reported (MOE_DEV_BAD_ROWS on status) and their rows skipped.
cudaError_t launch_quantize_fp8_rows(const uint16_t *x, long long R, int C, const int *live_rows,
                                     uint8_t *q, float *scale_t, cudaStream_t stream,
                                     const int32_t *row_index = nullptr, long long src_rows = 0,
                                     int *status = nullptr);

// ------------------------------------------------------------------ routing
// logits [splits][T][E] fp32 -> softmax, biased top-K, ascending ids.
// renormalize: gates divided by their sum over the K selected experts.
cudaError_t launch_route_topk(const float *logits, int splits, int T, int E, int K,
                              const float *b, bool renormalize, int32_t *topk_idx,
                              float *topk_gate, float *gap, int *status, cudaStream_t stream);

// logits [splits][T][ld] fp32 partials -> l [T][E] fp32, summed in the top-K kernels' order.
cudaError_t launch_router_logits(const float *partial, int splits, int T, int E, float *out,
                                 int num_sms, cudaStream_t stream);

// ------------------------------------------------------------------ dispatch
constexpr int kDispatchChunk = 256;  // tokens per histogram chunk (8 warps x 32)
inline int dispatch_chunks(int T) { return (T + kDispatchChunk - 1) / kDispatchChunk; }
cudaError_t launch_dispatch(const uint16_t *x, const int32_t *topk_idx, const float *topk_gate,
                            int T, int d, int N, int E, int K, int32_t *chunk_counts,
                            int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                            float *perm_gate, int32_t *slot_pos, uint16_t *x_perm, int *status,
                            int num_sms, cudaStream_t stream);

// ------------------------------------------------------------------ combine and PID
// zero_only: write only the tokens with no FFN slot (the others come from the fused combine).
cudaError_t launch_combine(const uint16_t *x, const uint16_t *y_perm, const int32_t *topk_idx,
                           const float *topk_gate, const int32_t *slot_pos, int T, int d, int N,
                           int K, int rows, uint16_t *y, int *status, cudaStream_t stream,
                           bool zero_only = false);
// Fused combine: count[t * blocks + b] = number of FFN slots of token t, for every block b.
cudaError_t launch_combine_counters(const int32_t *topk_idx, int T, int K, int N, int blocks,
                                    int *count, cudaStream_t stream);
// PID step on the FFN biases, then (gamma != 0) the per-expert balancing term.
cudaError_t launch_pid(const int32_t *counts, int N, int K, int T, float *b, float *state,
                       float target, float kp, float ki, float kd, float gamma,
                       cudaStream_t stream);

}  // namespace moe
