// dispatch.cu -- group the FFN slots by expert: deterministic histogram, exclusive scans and a
// stable token permutation, then a 16-byte-vectorised copy of each token row to its slots.
//
// Zero-computation experts return their input ("衝上熱搜！美團大模型，靠「快」火了", §零計算專家), so
// only slots whose expert id is < N are grouped and copied; zero-expert slots are counted (for
// the PID controller) and get slot_pos = -1.
//
// Order is the stable counting sort with key (expert id, token).  Tokens are cut into chunks of
// 256 (8 warps x 32 tokens).  In a chunk, each warp builds one 32-bit token mask per expert with
// atomicOr (the final mask does not depend on timing), so the rank of a slot among the same
// expert's slots is: slots in earlier chunks (column scan of the per-chunk histogram) + slots in
// earlier warps of the chunk (popcounts) + earlier lanes of the warp (popcount of the lower mask
// bits).  No float atomics, no spin waits: four plain kernels (one block for the tables when
// the batch is a single chunk), the last copying each token's row to its slots' rows.
#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = kDispatchChunk / 32;

// Masks of the chunk's tokens per (warp, expert) in shared memory: masks[w * E + e].
__device__ __forceinline__ void build_masks(const int32_t *__restrict__ topk_idx, int T, int K,
                                            int E, uint32_t *masks, int *status) {
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kDispatchChunk + threadIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      const int e = __ldg(topk_idx + (long long)t * K + k);
      if (e < 0 || e >= E) {
        record_status(status, MOE_DEV_BAD_EXPERT);
        continue;
      }
      atomicOr(&masks[w * E + e], 1u << lane);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kDispatchChunk)
    dispatch_hist_kernel(const int32_t *__restrict__ topk_idx, int T, int K, int E,
                         int32_t *__restrict__ chunk_counts, int *status) {
  extern __shared__ uint32_t masks[];
  build_masks(topk_idx, T, K, E, masks, status);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += __popc(masks[w * E + e]);
    chunk_counts[(long long)blockIdx.x * E + e] = c;
  }
}

// One block of 1024 threads (E <= 1024): column scan of the chunk histogram (in place, turning
// counts into the chunk's starting rank per expert), expert totals, and the exclusive scan of
// the FFN experts' totals into row offsets.
__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int32_t *__restrict__ chunk_counts, int nchunks, int N, int E,
                         int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
  __shared__ int warp_tot[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      int32_t *p = chunk_counts + (long long)c * E + e;
      const int v = *p;
      *p = total;
      total += v;
    }
    counts[e] = total;
  }
  const int v = (e < N) ? total : 0;
  const int lane = e & 31, warp = e >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  if (e < N) offsets[e + 1] = base + incl;
  if (e == 0) offsets[0] = 0;
}

__global__ void __launch_bounds__(kDispatchChunk)
    dispatch_permute_kernel(const int32_t *__restrict__ topk_idx,
                            const float *__restrict__ topk_gate, int T, int K, int N, int E,
                            const int32_t *__restrict__ chunk_base,
                            const int32_t *__restrict__ offsets, int32_t *__restrict__ perm_tok,
                            float *__restrict__ perm_gate, int32_t *__restrict__ slot_pos,
                            int *status) {
  extern __shared__ uint32_t masks[];
  build_masks(topk_idx, T, K, E, masks, status);
  const int t = blockIdx.x * kDispatchChunk + threadIdx.x;
  if (t >= T) return;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lower = (1u << lane) - 1u;
  for (int k = 0; k < K; ++k) {
    const long long slot = (long long)t * K + k;
    const int e = __ldg(topk_idx + slot);
    if (e < 0 || e >= N) {  // zero expert (or an invalid id, already flagged)
      slot_pos[slot] = -1;
      continue;
    }
    int rank = __ldg(chunk_base + (long long)blockIdx.x * E + e);
    for (int w2 = 0; w2 < w; ++w2) rank += __popc(masks[w2 * E + e]);
    rank += __popc(masks[w * E + e] & lower);
    const int r = __ldg(offsets + e) + rank;
    perm_tok[r] = t;
    perm_gate[r] = __ldg(topk_gate + slot);
    slot_pos[slot] = r;
  }
}

// A batch of one chunk (T <= 256): histogram, scans and permutation in one block -- the same
// masks, the same ranks and the same tables as the three kernels above, without their two
// extra launches and second mask build (decode-sized batches are launch- and latency-bound).
// Thread i owns experts [i * P, i * P + P), P = ceil(E / 256), so the exclusive scan over
// experts is a block scan of per-thread sums.
__global__ void __launch_bounds__(kDispatchChunk)
    dispatch_small_kernel(const int32_t *__restrict__ topk_idx,
                          const float *__restrict__ topk_gate, int T, int K, int N, int E,
                          int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                          int32_t *__restrict__ perm_tok, float *__restrict__ perm_gate,
                          int32_t *__restrict__ slot_pos, int *status) {
  extern __shared__ uint32_t masks[];  // [kWarps * E] masks, then [E] first rows
  int *first = reinterpret_cast<int *>(masks + kWarps * E);
  __shared__ int warp_tot[kWarps];
  build_masks(topk_idx, T, K, E, masks, status);
  const int P = (E + kDispatchChunk - 1) / kDispatchChunk;  // <= 4
  const int e0 = threadIdx.x * P;
  int c[4];
  int mine = 0;  // this thread's FFN rows, in expert order
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    c[j] = 0;
    const int e = e0 + j;
    if (j < P && e < E) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) c[j] += __popc(masks[w * E + e]);
      counts[e] = c[j];
      if (e < N) mine += c[j];
    }
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < wid; ++w) run += warp_tot[w];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + j;
    if (j < P && e < N) {
      first[e] = run;
      run += c[j];
      offsets[e + 1] = run;
    }
  }
  if (threadIdx.x == 0) offsets[0] = 0;
  __syncthreads();
  const int t = threadIdx.x;
  if (t >= T) return;
  const uint32_t lower = (1u << lane) - 1u;
  for (int k = 0; k < K; ++k) {
    const long long slot = (long long)t * K + k;
    const int e = __ldg(topk_idx + slot);
    if (e < 0 || e >= N) {  // zero expert (or an invalid id, already flagged)
      slot_pos[slot] = -1;
      continue;
    }
    int rank = 0;
    for (int w2 = 0; w2 < wid; ++w2) rank += __popc(masks[w2 * E + e]);
    rank += __popc(masks[wid * E + e] & lower);
    const int r = first[e] + rank;
    perm_tok[r] = t;
    perm_gate[r] = __ldg(topk_gate + slot);
    slot_pos[slot] = r;
  }
}

// x_perm[slot_pos[t, k]] = x[t] for every FFN slot (t, k): one warp per token reads the token's
// row once and writes it to each of its FFN slots' rows (16-byte accesses, four in flight per
// lane).  Token-major on purpose: a gather over the grouped rows visits a token once per slot,
// in expert order, and when x exceeds the L2 (prefill: 201 MB) each visit is a DRAM read; with
// x in the L2, the gather below has the parallelism (a warp per row, not per token).
constexpr int kScatterWarps = 8;

__global__ void __launch_bounds__(32 * kScatterWarps)
    scatter_rows_kernel(const uint4 *__restrict__ x, int d16, int T, int K,
                        const int32_t *__restrict__ slot_pos, int rows,
                        uint4 *__restrict__ x_perm, int *status) {
  __shared__ int dst_row[kScatterWarps][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = gridDim.x * kScatterWarps;
  for (int t = blockIdx.x * kScatterWarps + w; t < T; t += warps) {
    int r = -1;
    if (lane < K) {
      r = __ldg(slot_pos + (long long)t * K + lane);
      if (r < -1 || r >= rows) {  // -1: a zero-expert slot
        record_status(status, MOE_DEV_BAD_ROWS);
        r = -1;
      }
    }
    const uint32_t slots = __ballot_sync(0xffffffffu, r >= 0);
    dst_row[w][lane] = r;
    __syncwarp();
    if (slots != 0u) {
      const uint4 *src = x + (long long)t * d16;
      for (int i0 = lane; i0 < d16; i0 += 128) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i0 + 32 * u < d16) v[u] = __ldg(src + i0 + 32 * u);
        for (uint32_t m = slots; m != 0u; m &= m - 1) {
          uint4 *dst = x_perm + (long long)dst_row[w][__ffs(m) - 1] * d16;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (i0 + 32 * u < d16) dst[i0 + 32 * u] = v[u];
        }
      }
    }
    __syncwarp();
  }
}

// x_perm[r] = x[perm_tok[r]] for r < A = offsets[N]; one warp per row, 16-byte accesses: more
// warps than tokens, the better choice while x stays in the L2 (decode, mid).
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4 *__restrict__ x, int d16, int T,
                       const int32_t *__restrict__ perm_tok, const int32_t *__restrict__ a_rows,
                       uint4 *__restrict__ x_perm, int *status) {
  const int A = __ldg(a_rows);
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < A; r += warps) {
    const int t = __ldg(perm_tok + r);
    if (t < 0 || t >= T) {
      if ((threadIdx.x & 31) == 0) record_status(status, MOE_DEV_BAD_ROWS);
      continue;
    }
    const uint4 *src = x + (long long)t * d16;
    uint4 *dst = x_perm + (long long)r * d16;
    int i = threadIdx.x & 31;
    for (; i + 96 < d16; i += 128) {
      const uint4 v0 = __ldg(src + i), v1 = __ldg(src + i + 32), v2 = __ldg(src + i + 64),
                  v3 = __ldg(src + i + 96);
      dst[i] = v0;
      dst[i + 32] = v1;
      dst[i + 64] = v2;
      dst[i + 96] = v3;
    }
    for (; i < d16; i += 32) dst[i] = __ldg(src + i);
  }
}

// Token rows of at least this many bytes in all (about half the L2) are copied token-major.
constexpr long long kScatterMinBytes = 64ll << 20;

cudaError_t copy_rows(const uint16_t *x, int T, int d, int K, int N, const int32_t *perm_tok,
                      const int32_t *offsets, const int32_t *slot_pos, uint16_t *x_perm,
                      int *status, int num_sms, cudaStream_t stream) {
  if ((long long)T * d * 2 >= kScatterMinBytes)
    scatter_rows_kernel<<<num_sms * 8, 32 * kScatterWarps, 0, stream>>>(
        reinterpret_cast<const uint4 *>(x), d / 8, T, K, slot_pos, T * K,
        reinterpret_cast<uint4 *>(x_perm), status);
  else
    gather_rows_kernel<<<num_sms * 8, 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(x), d / 8, T, perm_tok, offsets + N,
        reinterpret_cast<uint4 *>(x_perm), status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch(const uint16_t *x, const int32_t *topk_idx, const float *topk_gate,
                            int T, int d, int N, int E, int K, int32_t *chunk_counts,
                            int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                            float *perm_gate, int32_t *slot_pos, uint16_t *x_perm, int *status,
                            int num_sms, cudaStream_t stream) {
  const int nchunks = dispatch_chunks(T);
  const size_t mask_bytes = sizeof(uint32_t) * kWarps * E;
  if (nchunks == 1) {  // one block does the histogram, the scans and the permutation
    dispatch_small_kernel<<<1, kDispatchChunk, mask_bytes + sizeof(int) * E, stream>>>(
        topk_idx, topk_gate, T, K, N, E, counts, offsets, perm_tok, perm_gate, slot_pos, status);
    if (x_perm != nullptr)
      return copy_rows(x, T, d, K, N, perm_tok, offsets, slot_pos, x_perm, status, num_sms,
                       stream);
    return cudaGetLastError();
  }
  if (nchunks > 0) {
    dispatch_hist_kernel<<<nchunks, kDispatchChunk, mask_bytes, stream>>>(topk_idx, T, K, E,
                                                                          chunk_counts, status);
  }
  dispatch_scan_kernel<<<1, 1024, 0, stream>>>(chunk_counts, nchunks, N, E, counts, offsets);
  if (nchunks > 0) {
    dispatch_permute_kernel<<<nchunks, kDispatchChunk, mask_bytes, stream>>>(
        topk_idx, topk_gate, T, K, N, E, chunk_counts, offsets, perm_tok, perm_gate, slot_pos,
        status);
    if (x_perm != nullptr)  // NULL: the up-projection gathers the rows itself
      return copy_rows(x, T, d, K, N, perm_tok, offsets, slot_pos, x_perm, status, num_sms,
                       stream);
  }
  return cudaGetLastError();
}

}  // namespace moe
