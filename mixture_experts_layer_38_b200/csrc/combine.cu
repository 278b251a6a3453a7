// combine.cu -- weighted combine / un-permute with the zero experts fused in, and the PID
// bias update.
//
// "衝上熱搜！美團大模型，靠「快」火了", §零計算專家:
//   y_t = sum over the K selected experts of g_i * E_i(x_t), and a zero-computation expert returns
//   x_t unchanged.  The FFN terms g_i * E_i(x_t) arrive as bf16 rows of y_perm (gate already
//   applied in fp32); the zero-expert terms collapse to (sum of their gates) * x_t, so no
//   identity copy exists anywhere.  Per token: fp32 accumulation of the FFN rows in ascending
//   expert id, then the zero term, one bf16 rounding.
// Same section, last paragraph: a PID controller tunes the expert biases from recent expert
//   usage so the activated amount per token holds near a target (law: see moe_bias_update in
//   the public header).  Optionally followed by the per-expert term of the aux-loss-free
//   scheme the PID refines: b_i += gamma * sign(mean load - load_i), sign from integers.
#include <algorithm>

#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kCombineThreads = 128;
constexpr int kCombineMinBlocks = 1184;  // 8 blocks per SM of a B200
constexpr int kMaxK = 32;

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint4 *__restrict__ x, const uint4 *__restrict__ y_perm,
                   const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_gate,
                   const int32_t *__restrict__ slot_pos, int T, int d16, int N, int K, int rows,
                   uint4 *__restrict__ y, int *status, bool zero_only) {
  __shared__ int s_pos[kMaxK];
  __shared__ float s_zsum;
  __shared__ int s_nffn;
  const int t = blockIdx.x;
  if (threadIdx.x == 0) {
    float zsum = 0.f;
    int n = 0;
    for (int k = 0; k < K; ++k) {
      const long long slot = (long long)t * K + k;
      const int e = __ldg(topk_idx + slot);
      const int r = __ldg(slot_pos + slot);
      if (e >= N) {
        zsum += __ldg(topk_gate + slot);
      } else if (r >= 0 && r < rows) {
        s_pos[n++] = r;
      } else {
        record_status(status, MOE_DEV_BAD_ROWS);
      }
    }
    s_zsum = zsum;
    s_nffn = n;
  }
  __syncthreads();
  const float zsum = s_zsum;
  const int nffn = s_nffn;
  if (zero_only && nffn > 0) return;  // written by the combine fused into the down projection
  // Block (t, s) covers slice s of the token's row (one slice unless the batch is small).
  const int per = (d16 + (int)gridDim.y - 1) / (int)gridDim.y;
  const int i_end = min(d16, ((int)blockIdx.y + 1) * per);
  for (int i = (int)blockIdx.y * per + threadIdx.x; i < i_end; i += kCombineThreads) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int n = 0; n < nffn; ++n) combine_add8(acc, __ldg(y_perm + (long long)s_pos[n] * d16 + i));
    y[(long long)t * d16 + i] = combine_finish8(acc, zsum, __ldg(x + (long long)t * d16 + i));
  }
}

// Counters of the combine fused into the down projection: every feature block of token t
// starts at t's number of FFN slots.
__global__ void __launch_bounds__(256)
    combine_counters_kernel(const int32_t *__restrict__ topk_idx, int T, int K, int N,
                            int blocks, int *__restrict__ count) {
  const int t = blockIdx.x * 256 + threadIdx.x;
  if (t >= T) return;
  int nffn = 0;
  for (int k = 0; k < K; ++k) nffn += __ldg(topk_idx + (long long)t * K + k) < N;
  for (int b = 0; b < blocks; ++b) count[(long long)t * blocks + b] = nffn;
}

__global__ void __launch_bounds__(256)
    pid_kernel(const int32_t *__restrict__ counts, int N, int K, int T, float *b, float *state,
               float target, float kp, float ki, float kd, float gamma) {
  __shared__ long long part[256];
  __shared__ float s_u;
  long long sum = 0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) sum += counts[i];
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // One rounding per operation, in the order of the documented law (no contraction).
    const float m = __fdiv_rn(__ll2float_rn(part[0]), __int2float_rn(T));
    const float e = __fdiv_rn(__fsub_rn(target, m), __int2float_rn(K));
    const float integral = __fadd_rn(state[0], e);
    const float p_term = __fmul_rn(kp, e);
    const float i_term = __fmul_rn(ki, integral);
    const float d_term = __fmul_rn(kd, __fsub_rn(e, state[1]));
    s_u = __fadd_rn(__fadd_rn(p_term, i_term), d_term);
    state[0] = integral;
    state[1] = e;
  }
  __syncthreads();
  const float u = s_u;
  const long long total = part[0];
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    float bi = __fadd_rn(b[i], u);
    if (gamma != 0.f) {
      const long long diff = total - (long long)N * counts[i];
      bi = __fadd_rn(bi, diff > 0 ? gamma : (diff < 0 ? -gamma : 0.f));
    }
    b[i] = bi;
  }
}

}  // namespace

cudaError_t launch_combine(const uint16_t *x, const uint16_t *y_perm, const int32_t *topk_idx,
                           const float *topk_gate, const int32_t *slot_pos, int T, int d, int N,
                           int K, int rows, uint16_t *y, int *status, cudaStream_t stream,
                           bool zero_only) {
  if (T == 0) return cudaSuccess;
  // Small batches: split each token's row over several blocks (at least ~1184 blocks, slices of
  // at least 128 16-byte pieces) so the row loads of a few tokens spread over every SM.
  const int d16 = d / 8;
  const int max_slices = std::max(1, d16 / kCombineThreads);
  const int slices = std::min(max_slices, std::max(1, (kCombineMinBlocks + T - 1) / T));
  combine_kernel<<<dim3(T, slices), kCombineThreads, 0, stream>>>(
      reinterpret_cast<const uint4 *>(x), reinterpret_cast<const uint4 *>(y_perm), topk_idx,
      topk_gate, slot_pos, T, d / 8, N, K, rows, reinterpret_cast<uint4 *>(y), status,
      zero_only);
  return cudaGetLastError();
}

cudaError_t launch_combine_counters(const int32_t *topk_idx, int T, int K, int N, int blocks,
                                    int *count, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  combine_counters_kernel<<<(T + 255) / 256, 256, 0, stream>>>(topk_idx, T, K, N, blocks, count);
  return cudaGetLastError();
}

cudaError_t launch_pid(const int32_t *counts, int N, int K, int T, float *b, float *state,
                       float target, float kp, float ki, float kd, float gamma,
                       cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  pid_kernel<<<1, 256, 0, stream>>>(counts, N, K, T, b, state, target, kp, ki, kd, gamma);
  return cudaGetLastError();
}

}  // namespace moe
