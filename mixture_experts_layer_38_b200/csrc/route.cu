// route.cu -- softmax router R and biased top-K selection, one warp per token.
//
// "衝上熱搜！美團大模型，靠「快」火了", §零計算專家: R is a softmax router over the N FFN experts
// and Z zero-computation experts; a per-expert bias b_i adjusts the routing score used to pick
// the K experts while the gate stays the router's output.  Per token t:
//   l   = sum of the split-K partial logits (fixed order), fp32
//   p   = exp(l - max l) / sum exp(l - max l)
//   s   = p + b;  the K largest s are selected, an exact tie going to the lower expert id
//   out = selected ids in ascending order, gates g = p (not renormalised), gap = s_(K) - s_(K+1)
// Lane j holds experts j, j+32, j+64, ... in registers; each of the K+1 selection rounds is a
// local scan plus a 5-step butterfly argmax over (score desc, id asc), so the result does not
// depend on thread timing.
#include <math.h>

#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

struct Cand {
  float s;  // biased score
  float p;  // router probability
  int id;
};

__device__ __forceinline__ bool better(const Cand &a, const Cand &b) {
  return a.s > b.s || (a.s == b.s && a.id < b.id);
}

template <int PER>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float *__restrict__ logits, int splits, int T, int E, int ld, int K,
                      const float *__restrict__ b, int32_t *__restrict__ topk_idx,
                      float *__restrict__ topk_gate, float *__restrict__ gap, int *status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const long long split_stride = (long long)T * ld;

  float l[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    float v = -INFINITY;
    if (e < E) {
      const float *src = logits + (long long)t * ld + e;
      v = src[0];
      for (int sp = 1; sp < splits; ++sp) v += src[sp * split_stride];
    }
    l[j] = v;
  }
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < PER; ++j) m = fmaxf(m, l[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    l[j] = (e < E) ? expf(l[j] - m) : 0.f;  // l now holds exp(l - max)
    z += l[j];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);

  float p[PER], s[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    p[j] = __fdiv_rn(l[j], z);
    s[j] = (e < E) ? __fadd_rn(p[j], __ldg(b + e)) : -INFINITY;
  }

  uint32_t chosen = 0;
  int my_id = 0x7fffffff;  // lane k (< K) keeps the k-th selected expert
  float my_gate = 0.f;
  float kth = INFINITY, next = -INFINITY;
  for (int k = 0; k <= K && k < E; ++k) {
    Cand c{-INFINITY, 0.f, 0x7fffffff};
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      const Cand o{s[j], p[j], e};
      if (e < E && !((chosen >> j) & 1u) && (c.id == 0x7fffffff || better(o, c))) c = o;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      Cand o;
      o.s = __shfl_xor_sync(0xffffffffu, c.s, off);
      o.p = __shfl_xor_sync(0xffffffffu, c.p, off);
      o.id = __shfl_xor_sync(0xffffffffu, c.id, off);
      if (o.id != 0x7fffffff && (c.id == 0x7fffffff || better(o, c))) c = o;
    }
    if (c.id == 0x7fffffff) {  // only non-finite scores were left: flag, never index with it
      if (lane == 0) record_status(status, MOE_DEV_BAD_EXPERT);
      break;
    }
    if (k == K) { next = c.s; break; }
    if (lane == (c.id & 31)) chosen |= 1u << (c.id >> 5);
    if (lane == k) { my_id = c.id; my_gate = c.p; }
    kth = c.s;
  }

  // Ascending-id order: rank of my id among the K selected ids (all distinct).
  int rank = 0;
  for (int k2 = 0; k2 < K; ++k2) {
    const int other = __shfl_sync(0xffffffffu, my_id, k2);
    rank += other < my_id;
  }
  if (lane < K) {
    topk_idx[(long long)t * K + rank] = my_id;
    topk_gate[(long long)t * K + rank] = my_gate;
  }
  if (gap != nullptr && lane == 0) gap[t] = (K < E) ? __fsub_rn(kth, next) : INFINITY;
}

template <int PER>
void launch_per(const float *logits, int splits, int T, int E, int ld, int K, const float *b,
                int32_t *idx, float *gate, float *gap, int *status, cudaStream_t stream) {
  const int grid = (T + kRouteWarps - 1) / kRouteWarps;
  route_topk_kernel<PER><<<grid, kRouteWarps * 32, 0, stream>>>(logits, splits, T, E, ld, K, b,
                                                                 idx, gate, gap, status);
}

}  // namespace

cudaError_t launch_route_topk(const float *logits, int splits, int T, int E, int K,
                              const float *b, int32_t *topk_idx, float *topk_gate, float *gap,
                              int *status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int ld = (E + 3) & ~3;
  const int per = (E + 31) / 32;
  if (per <= 1) launch_per<1>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else if (per <= 2) launch_per<2>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else if (per <= 4) launch_per<4>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else if (per <= 8) launch_per<8>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else if (per <= 16) launch_per<16>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else if (per <= 24) launch_per<24>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  else launch_per<32>(logits, splits, T, E, ld, K, b, topk_idx, topk_gate, gap, status, stream);
  return cudaGetLastError();
}

}  // namespace moe
