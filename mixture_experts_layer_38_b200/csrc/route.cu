// route.cu -- softmax router R and biased top-K selection: one thread block per token, or one
// warp per token for pools of up to 256 experts.
//
// "衝上熱搜！美團大模型，靠「快」火了", §零計算專家: R is a softmax router over the N FFN experts
// and Z zero-computation experts; a per-expert bias b_i adjusts the routing score used to pick
// the K experts while the gate stays the router's output.  Per token t:
//   l   = sum of the split-K partial logits (fixed order), fp32
//   p   = exp(l - max l) / sum exp(l - max l)
//   s   = p + b;  the K largest s are selected, an exact tie going to the lower expert id
//   out = selected ids in ascending order, gates g = p (not renormalised), gap = s_(K) - s_(K+1)
//   (variant: g = p / sum of the K selected p, summed in a fixed shuffle order)
// Thread i of the 256-thread block holds experts i, i+256, i+512, i+768 in registers, so the
// split-K partial sums, exp and bias are spread over 8 warps; each of the K+1 selection rounds
// is a block-wide argmax of one 64-bit key per thread, and the result does not depend on
// thread timing.
#include <math.h>

#include <algorithm>

#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

// Selection key of expert id with score s:
// (order-preserving bits of s) << 32 | (0xffffffff - id)  ->  larger score, then lower id.
constexpr int kBlockThreads = 256;
constexpr int kWarps = kBlockThreads / 32;
constexpr int kMaxPerThread = 4;  // E <= 1024

__device__ __forceinline__ uint64_t score_key(float s, int id) {
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | (0xffffffffu - static_cast<uint32_t>(id));
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
    v = o > v ? o : v;
  }
  return v;
}

__device__ __forceinline__ float block_reduce(float v, bool is_max, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kBlockThreads / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  __syncthreads();
  return r;
}

// kPerThread experts per thread (E <= 256 * kPerThread).  With three, at most 64 registers so
// that four blocks share an SM.
template <int kPerThread>
__global__ void __launch_bounds__(kBlockThreads, kPerThread <= 3 ? 4 : 3)
    route_topk_block_kernel(const float *__restrict__ logits, int splits, int T, int E, int ld,
                            int K, const float *__restrict__ b, bool renormalize,
                            int32_t *__restrict__ topk_idx, float *__restrict__ topk_gate,
                            float *__restrict__ gap, int *status) {
  __shared__ float red[kBlockThreads / 32];
  __shared__ uint64_t wbest[2][kWarps];
  __shared__ int sel_id[33];
  __shared__ float sel_p[33];
  __shared__ float sel_s[33];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const long long split_stride = (long long)T * ld;
  float l[kPerThread];
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    const int e = tid + kBlockThreads * j;
    float v = -INFINITY;
    if (e < E) {
      const float *src = logits + (long long)t * ld + e;
      v = src[0];
      for (int sp = 1; sp < splits; ++sp) v += src[sp * split_stride];
    }
    l[j] = v;
  }
  float m = l[0];
#pragma unroll
  for (int j = 1; j < kPerThread; ++j) m = fmaxf(m, l[j]);
  m = block_reduce(m, true, red);
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    const int e = tid + kBlockThreads * j;
    l[j] = (e < E) ? expf(l[j] - m) : 0.f;  // now exp(l - max)
    z += l[j];
  }
  z = block_reduce(z, false, red);
  float p[kPerThread];
  uint64_t key[kPerThread];
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    const int e = tid + kBlockThreads * j;
    p[j] = __fdiv_rn(l[j], z);
    key[j] = (e < E) ? score_key(__fadd_rn(p[j], __ldg(b + e)), e) : 0ull;
  }
  const int rounds = K < E ? K + 1 : K;
  // One barrier per round: the warp maxima alternate between two buffers, so round k + 2
  // cannot overwrite what a slow thread still reads from round k (every thread passes round
  // k + 1's barrier first).
  for (int k = 0; k < rounds; ++k) {
    uint64_t *wb = wbest[k & 1];
    uint64_t best = key[0];
#pragma unroll
    for (int j = 1; j < kPerThread; ++j) best = key[j] > best ? key[j] : best;
    best = warp_max_u64(best);
    if ((tid & 31) == 0) wb[tid >> 5] = best;
    __syncthreads();
    uint64_t win = wb[tid & (kWarps - 1)];  // lane i takes warp i % 8's maximum
#pragma unroll
    for (int off = 1; off < kWarps; off <<= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, win, off);
      win = o > win ? o : win;
    }
    const int id = (int)(0xffffffffu - (uint32_t)(win & 0xffffffffu));
    if (win == 0ull) {  // nothing left that is selectable (non-finite scores): flag, skip
      if (tid == 0) {
        record_status(status, MOE_DEV_BAD_EXPERT);
        sel_id[k] = 0x7fffffff;
        sel_p[k] = 0.f;
      }
    } else if (id % kBlockThreads == tid) {
      const int j = id / kBlockThreads;
#pragma unroll
      for (int jj = 0; jj < kPerThread; ++jj) {
        if (jj == j) {
          sel_id[k] = id;
          sel_p[k] = p[jj];
          sel_s[k] = __fadd_rn(p[jj], __ldg(b + id));
          key[jj] = 0ull;
        }
      }
    }
  }
  __syncthreads();  // the selections of the last round are written
  if (tid < 32) {
    const int lane = tid;
    const int my_id = lane < K ? sel_id[lane] : 0x7fffffff;
    int rank = 0;
    for (int k2 = 0; k2 < K; ++k2) {
      const int other = __shfl_sync(0xffffffffu, my_id, k2);
      rank += other < my_id;
    }
    float g = lane < K ? sel_p[lane] : 0.f;
    if (renormalize) {
      float sum = g;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
      g = __fdiv_rn(g, sum);
    }
    if (lane < K) {
      topk_idx[(long long)t * K + rank] = my_id;
      topk_gate[(long long)t * K + rank] = g;
    }
    if (gap != nullptr && lane == 0)
      gap[t] = (K < E) ? __fsub_rn(sel_s[K - 1], sel_s[K]) : INFINITY;
  }
}

// One warp per token (8 tokens per block), lane i holding experts i, i + 32, ... (kWarpPer of
// them: E <= 32 * kWarpPer); the same keys and K+1 argmax rounds as above, with warp shuffles
// only.  Used for small pools (a 96-expert pool would leave most of a 256-thread block idle)
// and for large batches of any pool (no block barrier per round, about a fifth of the block
// kernel's instructions per token); a small batch of a large pool keeps the block kernel,
// whose 8 warps per token spread a short batch over more SMs.
template <int kWarpPer>
__global__ void __launch_bounds__(256, kWarpPer <= 8 ? 1 : 2)
    route_topk_warp_kernel(const float *__restrict__ logits, int splits, int T, int E, int ld,
                           int K, const float *__restrict__ b, bool renormalize,
                           int32_t *__restrict__ topk_idx, float *__restrict__ topk_gate,
                           float *__restrict__ gap, int *status) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  const long long split_stride = (long long)T * ld;
  float p[kWarpPer];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < kWarpPer; ++j) {
    const int e = lane + 32 * j;
    float v = -INFINITY;
    if (e < E) {
      const float *src = logits + (long long)t * ld + e;
      v = src[0];
      for (int sp = 1; sp < splits; ++sp) v += src[sp * split_stride];
    }
    p[j] = v;
    m = fmaxf(m, v);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < kWarpPer; ++j) {
    p[j] = (lane + 32 * j < E) ? expf(p[j] - m) : 0.f;
    z += p[j];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  // Scores as order-preserving 32-bit patterns (0 = taken or not an expert; every real score
  // maps above 0); the id of slot j of this lane is lane + 32 j, so the 64-bit key of the
  // selection order (score, then the lower id) is formed only for the warp-wide maximum.
  uint32_t sk[kWarpPer];
#pragma unroll
  for (int j = 0; j < kWarpPer; ++j) {
    const int e = lane + 32 * j;
    p[j] = __fdiv_rn(p[j], z);
    sk[j] = (e < E) ? (uint32_t)(score_key(__fadd_rn(p[j], __ldg(b + e)), e) >> 32) : 0u;
  }
  const int rounds = K < E ? K + 1 : K;
  int my_id = 0x7fffffff;  // lane k keeps the k-th selected expert
  float my_p = 0.f, s_k1 = 0.f, s_k = 0.f;
  for (int k = 0; k < rounds; ++k) {
    uint32_t bs = sk[0];
    int bj = 0;
#pragma unroll
    for (int j = 1; j < kWarpPer; ++j) {  // strict: among equal scores the lower id (lower j)
      if (sk[j] > bs) {
        bs = sk[j];
        bj = j;
      }
    }
    const uint64_t mine = bs == 0u ? 0ull
                                   : ((uint64_t)bs << 32) |
                                         (0xffffffffu - (uint32_t)(lane + 32 * bj));
    const uint64_t best = warp_max_u64(mine);
    if (best == 0ull) {  // nothing left that is selectable (non-finite scores): flag, skip
      if (lane == 0) record_status(status, MOE_DEV_BAD_EXPERT);
      continue;
    }
    const int id = (int)(0xffffffffu - (uint32_t)(best & 0xffffffffu));
    const int owner = id & 31, jo = id >> 5;
    float pv = 0.f;
    if (lane == owner) {
#pragma unroll
      for (int j = 0; j < kWarpPer; ++j) {
        if (j == jo) {
          pv = p[j];
          sk[j] = 0u;
        }
      }
    }
    pv = __shfl_sync(0xffffffffu, pv, owner);
    const float sv = __fadd_rn(pv, __ldg(b + id));
    if (lane == k) {
      my_id = id;
      my_p = pv;
    }
    if (k == K - 1) s_k1 = sv;
    if (k == K) s_k = sv;
  }
  int rank = 0;
  for (int k2 = 0; k2 < K; ++k2) {
    const int other = __shfl_sync(0xffffffffu, my_id, k2);
    rank += other < my_id;
  }
  float g = lane < K ? my_p : 0.f;
  if (renormalize) {
    float sum = g;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
    g = __fdiv_rn(g, sum);
  }
  if (lane < K) {
    topk_idx[(long long)t * K + rank] = my_id;
    topk_gate[(long long)t * K + rank] = g;
  }
  if (gap != nullptr && lane == 0) gap[t] = (K < E) ? __fsub_rn(s_k1, s_k) : INFINITY;
}

// Tokens from which a pool of more than 256 experts goes to the warp-per-token kernel.
constexpr int kWarpTopkMinTokens = 2048;

}  // namespace

// l[t, e] = sum of the split-K partial logits in split order, the same fixed order as the
// top-K kernels above, so the result is bit-identical to the logits they select from.
__global__ void __launch_bounds__(256)
    router_logits_kernel(const float *__restrict__ partial, int splits, int T, int E, int ld,
                         float *__restrict__ out) {
  const long long n = (long long)T * E;
  const long long split_stride = (long long)T * ld;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
    const int t = (int)(i / E), e = (int)(i % E);
    const float *src = partial + (long long)t * ld + e;
    float v = src[0];
    for (int sp = 1; sp < splits; ++sp) v += src[sp * split_stride];
    out[i] = v;
  }
}

cudaError_t launch_router_logits(const float *partial, int splits, int T, int E, float *out,
                                 int num_sms, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const long long n = (long long)T * E;
  const long long blocks = std::min<long long>((n + 255) / 256, 8ll * num_sms);
  router_logits_kernel<<<(int)blocks, 256, 0, stream>>>(partial, splits, T, E, (E + 3) & ~3, out);
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const float *logits, int splits, int T, int E, int K,
                              const float *b, bool renormalize, int32_t *topk_idx,
                              float *topk_gate, float *gap, int *status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int ld = (E + 3) & ~3;
  const int blocks = (T + 7) / 8;
  if (E <= 256)
    route_topk_warp_kernel<8><<<blocks, 256, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  else if (T >= kWarpTopkMinTokens && E <= 512)
    route_topk_warp_kernel<16><<<blocks, 256, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  else if (T >= kWarpTopkMinTokens && E <= 768)
    route_topk_warp_kernel<24><<<blocks, 256, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  else if (T >= kWarpTopkMinTokens)
    route_topk_warp_kernel<32><<<blocks, 256, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  else if (E <= 3 * kBlockThreads)
    route_topk_block_kernel<3><<<T, kBlockThreads, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  else
    route_topk_block_kernel<kMaxPerThread><<<T, kBlockThreads, 0, stream>>>(
        logits, splits, T, E, ld, K, b, renormalize, topk_idx, topk_gate, gap, status);
  return cudaGetLastError();
}

}  // namespace moe
