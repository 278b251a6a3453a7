// quant.cu -- block-wise FP8 (E4M3) quantisation of expert weights (128 x 128 blocks) and of
// activation rows (1 x 128 blocks, the FP8-activation variant).
//
// "衝上熱搜！美團大模型，靠「快」火了", §系統級優化: LongCat-Flash quantises with the same
// fine-grained block-wise scheme as DeepSeek-V3, one scale per 128 x 128 block of a weight
// matrix.  Per block: e = the smallest integer with max|w| <= 448 * 2^e (448 is the largest
// finite E4M3 value; e >= -126, e = 0 for an all-zero block), scale = 2^e, and each weight
// becomes E4M3(w / 2^e), rounded to nearest with ties to even and saturated at +-448.  A
// power-of-two scale makes w / 2^e and the dequantised q * 2^e exact, so the grouped GEMM's
// bf16 weights are exactly q * scale.
#include <cuda_fp8.h>

#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kChunks = 128 * 128 / 8 / kQuantThreads;  // 16-byte chunks of 8 weights per thread

// One CTA per 128 x 128 block; thread t owns chunks t, t + 256, ... (16 chunks of 8 columns per
// row), so every load and store instruction is coalesced.
__global__ void __launch_bounds__(kQuantThreads)
    quantize_fp8_kernel(const uint16_t *__restrict__ w, long long R, long long C,
                        uint8_t *__restrict__ q, float *__restrict__ scale) {
  __shared__ float red[kQuantThreads / 32];
  const long long RB = R / 128, CB = C / 128;
  const long long blk = blockIdx.x;
  const long long g = blk / (RB * CB), rb = (blk / CB) % RB, cb = blk % CB;
  const uint16_t *src = w + (g * R + rb * 128) * C + cb * 128;
  uint8_t *dst = q + (g * R + rb * 128) * C + cb * 128;
  uint4 v[kChunks];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    const int c = threadIdx.x + kQuantThreads * j, row = c >> 4, col = (c & 15) * 8;
    v[j] = *reinterpret_cast<const uint4 *>(src + row * C + col);
    const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(__uint_as_float(u[i] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(u[i] & 0xffff0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < kQuantThreads / 32; ++i) amax = fmaxf(amax, red[i]);
  const int e = fp8_scale_exponent(amax);
  if (threadIdx.x == 0) scale[blk] = exp2_int(e);
  const float inv = exp2_int(-e);  // 2^-e, exact (e <= 120 for finite input)
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    const int c = threadIdx.x + kQuantThreads * j, row = c >> 4, col = (c & 15) * 8;
    const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(u[i] << 16) * inv;
      const float hi = __uint_as_float(u[i] & 0xffff0000u) * inv;
      const uint32_t b0 = __nv_cvt_float_to_fp8(lo, __NV_SATFINITE, __NV_E4M3);
      const uint32_t b1 = __nv_cvt_float_to_fp8(hi, __NV_SATFINITE, __NV_E4M3);
      o[i >> 1] |= (b0 | (b1 << 8)) << (16 * (i & 1));
    }
    *reinterpret_cast<uint2 *>(dst + row * C + col) = make_uint2(o[0], o[1]);
  }
}

// FP8 activations: one scale per 1 x 128 block of a row, by the same rule.  One warp per row
// and pair of blocks: lanes 0-15 take block 2p, lanes 16-31 block 2p + 1, eight values (16
// bytes) per lane, so each half-warp reads one 256-byte block segment.  Rows from *live_rows on
// (when given) are skipped: grouped rows past the last expert's hold nothing.  With row_index,
// output row r is the quantised row row_index[r] of x (src_rows rows): the dispatch gather and
// the quantisation in one pass; an index outside [0, src_rows) is reported and its row skipped.
constexpr int kRowQuantThreads = 256;

__global__ void __launch_bounds__(kRowQuantThreads)
    quantize_rows_fp8_kernel(const uint16_t *__restrict__ x, long long R, int C,
                             const int *__restrict__ live_rows,
                             const int32_t *__restrict__ row_index, long long src_rows,
                             uint8_t *__restrict__ q, float *__restrict__ scale_t, int *status) {
  const int lane = threadIdx.x & 31;
  const int CB = C / 128, pairs = (CB + 1) / 2;
  const long long gw = (long long)blockIdx.x * (kRowQuantThreads / 32) + (threadIdx.x >> 5);
  const long long r = gw / pairs;
  const int cb = (int)(gw % pairs) * 2 + (lane >> 4);
  long long rows = R;
  if (live_rows != nullptr) rows = min(rows, (long long)max(__ldg(live_rows), 0));
  if (r >= rows) return;  // uniform over the warp
  long long src = r;
  if (row_index != nullptr) {
    src = __ldg(row_index + r);
    if (src < 0 || src >= src_rows) {
      if (lane == 0) record_status(status, MOE_DEV_BAD_ROWS);
      return;
    }
  }
  const bool active = cb < CB;
  const long long col = (long long)cb * 128 + (lane & 15) * 8;
  const long long off = r * C + col;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (active) v = *reinterpret_cast<const uint4 *>(x + src * C + col);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    amax = fmaxf(amax, fabsf(__uint_as_float(u[i] << 16)));
    amax = fmaxf(amax, fabsf(__uint_as_float(u[i] & 0xffff0000u)));
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = fp8_scale_exponent(amax);
  const float inv = exp2_int(-e);
  uint32_t o[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t b0 =
        __nv_cvt_float_to_fp8(__uint_as_float(u[i] << 16) * inv, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b1 = __nv_cvt_float_to_fp8(__uint_as_float(u[i] & 0xffff0000u) * inv,
                                              __NV_SATFINITE, __NV_E4M3);
    o[i >> 1] |= (b0 | (b1 << 8)) << (16 * (i & 1));
  }
  if (!active) return;
  *reinterpret_cast<uint2 *>(q + off) = make_uint2(o[0], o[1]);
  if ((lane & 15) == 0) scale_t[(long long)cb * R + r] = exp2_int(e);
}

}  // namespace

cudaError_t launch_quantize_fp8_rows(const uint16_t *x, long long R, int C, const int *live_rows,
                                     uint8_t *q, float *scale_t, cudaStream_t stream,
                                     const int32_t *row_index, long long src_rows, int *status) {
  if (R == 0 || C == 0) return cudaSuccess;
  const long long warps = R * ((C / 128 + 1) / 2);
  const long long blocks = (warps + kRowQuantThreads / 32 - 1) / (kRowQuantThreads / 32);
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  quantize_rows_fp8_kernel<<<(unsigned)blocks, kRowQuantThreads, 0, stream>>>(
      x, R, C, live_rows, row_index, src_rows, q, scale_t, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp8(const uint16_t *w, long long G, long long R, long long C,
                                uint8_t *q, float *scale, cudaStream_t stream) {
  const long long blocks = G * (R / 128) * (C / 128);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  quantize_fp8_kernel<<<(unsigned)blocks, kQuantThreads, 0, stream>>>(w, R, C, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
