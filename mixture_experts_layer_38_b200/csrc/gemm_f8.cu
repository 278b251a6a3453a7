// gemm_f8.cu -- grouped GEMM with E4M3 operands on both sides for the FP8-activation variant of
// the expert FFN: the tensor cores read the FP8 codes themselves (tcgen05.mma kind::f8f6f4).
//
// "衝上熱搜！美團大模型，靠「快」火了", §系統級優化: LongCat-Flash quantises with the block-wise
// scheme of DeepSeek-V3.  Weights carry one power-of-two scale per 128 x 128 block, activations
// (the token rows x, then h) one per token per 128 channels, so the product of a weight row w
// and a token row x is
//     sum_kb  s_w(kb) * s_x(kb) * sum_{k in block kb} q_w[k] * q_x[k],
// with one scale pair per 128-long block of the reduction.  A stage of this kernel is exactly one
// such block: the MMA thread accumulates the block's 128 products in a fresh TMEM partial sum
// (four K = 32 MMAs per weight sub-tile), and the epilogue warps promote it, scaled by the
// block's two scales, into fp32 registers (the promotion DeepSeek-V3 describes, here once per
// block).  Four partial-sum buffers in TMEM let the MMAs run up to four blocks ahead of the
// promotion.
//
// Tiles: as the bf16 kernel's 128-token tiles (weights on M, tokens on N, two 128-row weight
// sub-tiles sharing one token tile; gemm_common.cuh's schedule), with at most kF8BN = 64 tokens
// so the promoted sums fit in registers (2 x 64 per thread).  This variant is made for
// weight-streaming (decode-sized) batches, where a tile's weights cross HBM once at one byte
// per weight and the promotion hides under the stream.
//
// Epilogues:
//   kEpiSwiGLU  h = silu(a) * u per (feature, token); then h is quantised for the down
//               projection: the tile's 128 features of a token are exactly one 1 x 128 block of
//               h, so its scale comes from a maximum over the four epilogue warps (column maxima
//               within each warp by a halving shuffle exchange, then shared memory), and the
//               codes are rounded once from fp32 and stored as [rows, I] bytes.
//   kEpiGated   y_perm = gate * (down-projection), bf16, as the bf16 kernel's gated epilogue.
//
// Warp roles (224 threads, one CTA per SM, persistent): warp 0 TMA producer, warp 1 TMEM
// allocator and MMA issuer, warps 2-5 promotion and epilogue (warp w reads TMEM lane quarter
// w mod 4), warp 6 loads each block's scales (s_x per token times s_w per sub-tile) into a
// shared-memory slot per partial-sum buffer, up to four blocks ahead of the promotion, so the
// promotion never waits on a global load.  Every wait is bounded; on timeout the kernel
// records MOE_DEV_WAIT_TIMEOUT and all roles unwind (the epilogue warps agree on stopping before
// their shared barriers, so none is left waiting at one), in-flight copies and MMAs are drained
// and TMEM is freed.
#include <cuda_fp8.h>

#include "device.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kF8BK = 128;                            // reduction elements (= bytes) per stage
constexpr int kF8BN = 64;                             // token rows per tile, at most
constexpr int kF8TileA = kBM * kF8BK;                 // 16 KB of codes per weight sub-tile
constexpr int kF8Stage = 2 * kF8TileA + kF8BN * kF8BK;  // 40 KB
constexpr int kF8Stages = 5;
constexpr int kF8Parts = kTmemCols / (2 * kF8BN);     // TMEM partial-sum buffers
constexpr int kF8PartCols = 2 * kF8BN;                // sub-tile 0 | sub-tile 1
constexpr int kF8EpiWarps = 4;
constexpr int kF8ScaleWarp = 2 + kF8EpiWarps;         // warp 6: block-scale loader
constexpr int kF8Threads = 32 * (kF8ScaleWarp + 1);
constexpr int kF8StageBytes = 2048;                   // per epilogue warp: output staging
constexpr int kF8GateBytes = kF8BN * 4;               // per epilogue warp: the tile's gates
constexpr int kF8EpiBytes = kF8StageBytes + kF8GateBytes;
constexpr int kF8SlotFloats = 2 * kF8BN;              // per partial sum: s_x * s_w0, s_x * s_w1
constexpr int kF8ScaleRing = kF8Parts * kF8SlotFloats * 4;
constexpr int kF8Shared = 4 * kF8BN * 4 + kF8BN * 4 + 16;  // column maxima, exponents, stop flag
constexpr int kF8Prefix = 2 * (kMaxGroups + 4) * 4;
constexpr int kF8NumBars = 2 * kF8Stages + 4 * kF8Parts + 1;
constexpr int kF8Smem = 1024 + kF8Stages * kF8Stage + kF8EpiWarps * kF8EpiBytes + kF8ScaleRing +
                        kF8Shared + kF8Prefix + kF8NumBars * 8 + 16;
static_assert(kF8Parts * kF8PartCols <= kTmemCols, "TMEM holds 512 columns");
static_assert(kF8Smem <= 232448, "shared memory per block");
static_assert(kF8Stage % 1024 == 0 && kF8TileA % 1024 == 0, "1024-byte-aligned operand tiles");
static_assert(kF8EpiWarps == 4, "one epilogue warp per TMEM lane quarter");

// Lane l of the warp returns the maximum over the warp's 32 lanes of |v[l]| (column l of the
// 32 x 32 block held one row per lane): five exchange steps that each halve the columns a lane
// keeps, 31 shuffles in all.
__device__ __forceinline__ float warp_column_absmax(const float (&v)[32], int lane) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool hi = (lane & 16) != 0;
    const float keep = fabsf(hi ? v[i + 16] : v[i]);
    const float send = fabsf(hi ? v[i] : v[i + 16]);
    a[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    const bool hi = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = hi ? a[i + w] : a[i];
      const float send = hi ? a[i] : a[i + w];
      a[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, w));
    }
  }
  return a[0];
}

template <int EPI>
__global__ void __launch_bounds__(kF8Threads, 1)
    grouped_gemm_e4m3_kernel(const __grid_constant__ GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint8_t *epi = smem + kF8Stages * kF8Stage;
  float *scale_ring = reinterpret_cast<float *>(epi + kF8EpiWarps * kF8EpiBytes);
  float *colmax = scale_ring + kF8Parts * kF8SlotFloats;                        // [4][64]
  int *bexp = reinterpret_cast<int *>(colmax + 4 * kF8BN);                     // [64]
  volatile int *stop_flag = reinterpret_cast<volatile int *>(bexp + kF8BN);
  int *hpre = reinterpret_cast<int *>(epi + kF8EpiWarps * kF8EpiBytes + kF8ScaleRing +
                                     kF8Shared);
  int *lpre = hpre + kMaxGroups + 4;
  uint64_t *bars = reinterpret_cast<uint64_t *>(hpre + 2 * (kMaxGroups + 4));
  uint64_t *full_bar = bars;
  uint64_t *empty_bar = bars + kF8Stages;
  uint64_t *pfull_bar = bars + 2 * kF8Stages;
  uint64_t *pempty_bar = pfull_bar + kF8Parts;
  uint64_t *sfull_bar = pempty_bar + kF8Parts;   // the slot's block scales are written
  uint64_t *sempty_bar = sfull_bar + kF8Parts;   // the epilogue has used them
  uint64_t *drain_bar = sempty_bar + kF8Parts;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kF8NumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int unit = (int)blockIdx.x;
  const int units = (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF8Stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < kF8Parts; ++b) {
      mbar_init(&pfull_bar[b], 1);
      mbar_init(&pempty_bar[b], kF8EpiWarps);
      mbar_init(&sfull_bar[b], 1);
      mbar_init(&sempty_bar[b], kF8EpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *stop_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.map_a0);
    tma_prefetch_desc(&args.map_a1);
#pragma unroll
    for (int i = 1; i < 4; ++i) tma_prefetch_desc(&args.map_b[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  Schedule sched;
  build_schedule<kF8BN>(args, hpre, lpre, reinterpret_cast<int *>(colmax), sched);
  sched.m_tiles = m_tiles_of<EPI>(args.M);
  sched.splits = 1;
  sched.total = sched.total * sched.m_tiles;
  const int KB = args.K / kF8BK;
  const long long wlim = args.wait_limit > 0 ? args.wait_limit : kWaitLimitCycles;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_w_reused = l2_policy_evict_normal();
      const uint64_t pol_w_once = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < sched.total; tile += units) {
        const Tile t = decode_tile<EPI, kF8BN>(args, sched, tile);
        const uint32_t bytes = kF8TileA * (t.has_a1 ? 2 : 1) + t.nb * kF8BK;
        const uint64_t pol_w = t.once ? pol_w_once : pol_w_reused;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, wlim)) {
            signal_abort(args, abort_flag);
            ok = false;
            break;
          }
          uint8_t *sa0 = ring + stage * kF8Stage;
          uint8_t *sb = sa0 + 2 * kF8TileA;
          const int kc = kb * kF8BK;  // a multiple of 128 bytes
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          tma_load_2d(sa0, &args.map_a0, &full_bar[stage], kc, t.a0_row, pol_w);
          if (t.has_a1)
            tma_load_2d(sa0 + kF8TileA, &args.map_a1, &full_bar[stage], kc, t.a1_row, pol_w);
          int r = 0;  // token rows in boxes of 64 / 32 / 16
#pragma unroll
          for (int i = 1; i < 4; ++i) {
            const int box = 128 >> i;
            if (t.nb - r >= box) {
              tma_load_2d(sb + r * kF8BK, &args.map_b[i], &full_bar[stage], kc, t.row0 + r,
                          pol_x);
              r += box;
            }
          }
          ++issued;
          if (++stage == kF8Stages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        for (long long i = 1; i <= issued && i <= kF8Stages; ++i) {
          const long long idx = issued - i;
          const int s = (int)(idx % kF8Stages);
          const uint32_t par = (uint32_t)((idx / kF8Stages) & 1);
          const long long t0 = clock64();
          while (!mbar_try_wait(&full_bar[s], par) && clock64() - t0 < kDrainLimitCycles) {}
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long n = 0;  // partial sums issued
      bool ok = true;
      bool any = false;
      for (int tile = unit; ok && tile < sched.total; tile += units) {
        const Tile t = decode_tile<EPI, kF8BN>(args, sched, tile);
        const uint32_t idesc = idesc_e4m3_f32(kBM, t.nb);
        for (int kb = 0; kb < KB; ++kb, ++n) {
          const int pb = (int)(n % kF8Parts);
          const uint32_t use = (uint32_t)(n / kF8Parts);
          if (!mbar_wait(&pempty_bar[pb], (use & 1) ^ 1, abort_flag, wlim) ||
              !mbar_wait(&full_bar[stage], phase, abort_flag, wlim)) {
            signal_abort(args, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + pb * kF8PartCols;
          const uint32_t abase = smem_u32(ring + stage * kF8Stage);
          const uint32_t bbase = abase + 2 * kF8TileA;
#pragma unroll
          for (int k = 0; k < kF8BK / 32; ++k) {
            const uint64_t bdesc = sw128_kmajor_desc(bbase + k * 32);
            const uint32_t acc = k > 0 ? 1u : 0u;
            umma_e4m3(d0, sw128_kmajor_desc(abase + k * 32), bdesc, idesc, acc);
            if (t.has_a1)
              umma_e4m3(d0 + kF8BN, sw128_kmajor_desc(abase + kF8TileA + k * 32), bdesc, idesc,
                        acc);
          }
          any = true;
          umma_commit(&empty_bar[stage]);
          umma_commit(&pfull_bar[pb]);
          if (++stage == kF8Stages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok && any) {  // wait (bounded) for the MMAs in flight before TMEM is freed
        umma_commit(drain_bar);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain_bar, 0) && clock64() - t0 < kDrainLimitCycles) {}
      }
    }
  } else if (warp == kF8ScaleWarp) {
    // ---------------------------------------------------------------- block-scale loader
    long long n = 0;
    bool ok = true;
    for (int tile = unit; ok && tile < sched.total; tile += units) {
      const Tile t = decode_tile<EPI, kF8BN>(args, sched, tile);
      const float *ws0 = args.scale_a0 + (long long)(t.a0_row / 128) * args.scale_ld;
      const float *ws1 = args.scale_a1 + (long long)(t.a1_row / 128) * args.scale_ld;
      for (int kb = 0; kb < KB; ++kb, ++n) {
        const float sw0 = __ldg(ws0 + kb);
        const float sw1 = t.has_a1 ? __ldg(ws1 + kb) : 0.f;
        const float *sx = args.act_scale + (long long)kb * args.rows + t.row0;
        float xs[kF8BN / 32];
#pragma unroll
        for (int i = 0; i < kF8BN / 32; ++i)
          xs[i] = i * 32 + lane < t.n_valid ? __ldg(sx + i * 32 + lane) : 0.f;
        const int pb = (int)(n % kF8Parts);
        const uint32_t use = (uint32_t)(n / kF8Parts);
        if (!warp_wait(&sempty_bar[pb], (use & 1) ^ 1, abort_flag, wlim)) {
          if (lane == 0) signal_abort(args, abort_flag);
          ok = false;
          break;
        }
        float *slot = scale_ring + pb * kF8SlotFloats;
#pragma unroll
        for (int i = 0; i < kF8BN / 32; ++i) {
          slot[i * 32 + lane] = xs[i] * sw0;
          slot[kF8BN + i * 32 + lane] = xs[i] * sw1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfull_bar[pb]);
      }
    }
  } else {
    // ---------------------------------------------------------------- promotion + epilogue
    const int q = warp & 3;
    const int ew = warp - 2;
    uint8_t *stage_bytes = epi + ew * kF8EpiBytes;
    float *gates = reinterpret_cast<float *>(stage_bytes + kF8StageBytes);  // [64]
    long long n = 0;
    bool ok = true;
    for (int tile = unit; tile < sched.total; tile += units) {
      const Tile t = decode_tile<EPI, kF8BN>(args, sched, tile);
      const int chunks = (t.nb + 31) / 32;
      float acc0[kF8BN], acc1[kF8BN];
#pragma unroll
      for (int j = 0; j < kF8BN; ++j) {
        acc0[j] = 0.f;
        acc1[j] = 0.f;
      }
      for (int kb = 0; kb < KB; ++kb, ++n) {
        const int pb = (int)(n % kF8Parts);
        const uint32_t use = (uint32_t)(n / kF8Parts);
        // This block's scales s_x(token) * s_w(sub-tile) (0 past the tile's rows), then the sums.
        if (!warp_wait(&sfull_bar[pb], use & 1, abort_flag, wlim) ||
            !warp_wait(&pfull_bar[pb], use & 1, abort_flag, wlim)) {
          if (lane == 0) signal_abort(args, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const float *sc = scale_ring + pb * kF8SlotFloats;
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + pb * kF8PartCols;
#pragma unroll
        for (int c = 0; c < kF8BN / 32; ++c) {
          if (c < chunks) {
            uint32_t p0[32], p1[32];
            tmem_ld_32x32b_x32(tb + c * 32, p0);
            tmem_ld_32x32b_x32(tb + kF8BN + c * 32, p1);
            tmem_ld_wait();
            if (c == chunks - 1) {  // the buffer is free once its last columns are read
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&pempty_bar[pb]);
            }
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 s0 = reinterpret_cast<const float4 *>(sc)[c * 8 + j4];
              const float4 s1 = reinterpret_cast<const float4 *>(sc + kF8BN)[c * 8 + j4];
              const int j = c * 32 + j4 * 4;
              acc0[j] = fmaf(__uint_as_float(p0[j4 * 4]), s0.x, acc0[j]);
              acc0[j + 1] = fmaf(__uint_as_float(p0[j4 * 4 + 1]), s0.y, acc0[j + 1]);
              acc0[j + 2] = fmaf(__uint_as_float(p0[j4 * 4 + 2]), s0.z, acc0[j + 2]);
              acc0[j + 3] = fmaf(__uint_as_float(p0[j4 * 4 + 3]), s0.w, acc0[j + 3]);
              acc1[j] = fmaf(__uint_as_float(p1[j4 * 4]), s1.x, acc1[j]);
              acc1[j + 1] = fmaf(__uint_as_float(p1[j4 * 4 + 1]), s1.y, acc1[j + 1]);
              acc1[j + 2] = fmaf(__uint_as_float(p1[j4 * 4 + 2]), s1.z, acc1[j + 2]);
              acc1[j + 3] = fmaf(__uint_as_float(p1[j4 * 4 + 3]), s1.w, acc1[j + 3]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty_bar[pb]);
      }

      if (EPI == kEpiSwiGLU) {
        // h, then its E4M3 codes: the four warps agree on stopping before their barriers.
        if (lane == 0 && (!ok || *abort_flag)) *stop_flag = 1;
#pragma unroll
        for (int c = 0; c < kF8BN / 32; ++c) {
          if (c < chunks) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              acc0[c * 32 + j] = silu(acc0[c * 32 + j]) * acc1[c * 32 + j];
              v[j] = acc0[c * 32 + j];
            }
            colmax[ew * kF8BN + c * 32 + lane] = warp_column_absmax(v, lane);
          }
        }
        named_bar_sync(1, 32 * kF8EpiWarps);
        const bool stop = *stop_flag != 0;
        if (!stop && ew == 0) {
          for (int c = 0; c < chunks; ++c) {
            const int col = c * 32 + lane;
            const float amax = fmaxf(fmaxf(colmax[col], colmax[kF8BN + col]),
                                     fmaxf(colmax[2 * kF8BN + col], colmax[3 * kF8BN + col]));
            const int e = fp8_scale_exponent(amax);
            bexp[col] = e;
            if (col < t.n_valid)
              args.out_scale[(long long)(t.m0 / 128) * args.rows + t.row0 + col] = exp2_int(e);
          }
        }
        named_bar_sync(1, 32 * kF8EpiWarps);
        if (stop) break;
        // Codes of token j land in row j of the warp's staging area (32 bytes: this warp's 32
        // features), then each lane stores 16-byte halves of rows.
#pragma unroll
        for (int c = 0; c < kF8BN / 32; ++c) {
          if (c < chunks) {
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const int4 e4 = reinterpret_cast<const int4 *>(bexp)[c * 8 + j4];
              const int ee[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = c * 32 + j4 * 4 + i;
                stage_bytes[j * 32 + lane] = static_cast<uint8_t>(
                    __nv_cvt_float_to_fp8(acc0[j] * exp2_int(-ee[i]), __NV_SATFINITE, __NV_E4M3));
              }
            }
          }
        }
        __syncwarp();
        uint8_t *out = reinterpret_cast<uint8_t *>(args.out);
#pragma unroll
        for (int i = 0; i < kF8BN / 16; ++i) {
          const int p = i * 32 + lane, j = p >> 1, half = p & 1;
          if (j < t.n_valid)
            *reinterpret_cast<uint4 *>(out + (long long)(t.row0 + j) * args.out_ld + t.m0 +
                                       q * 32 + half * 16) =
                *reinterpret_cast<const uint4 *>(stage_bytes + j * 32 + half * 16);
        }
        __syncwarp();
      } else {
        if (!ok) break;
        // Gates of the tile's tokens, then bf16 rows of both sub-tiles.
#pragma unroll
        for (int i = 0; i < kF8BN / 32; ++i) {
          const int j = i * 32 + lane;
          gates[j] = j >= t.n_valid ? 0.f : (args.row_scale ? __ldg(args.row_scale + t.row0 + j)
                                                            : 1.f);
        }
        __syncwarp();
        uint32_t *stg = reinterpret_cast<uint32_t *>(stage_bytes);
        uint16_t *out = reinterpret_cast<uint16_t *>(args.out);
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          if (sub == 1 && !t.has_a1) break;
#pragma unroll
          for (int c = 0; c < kF8BN / 32; ++c) {
            if (c < chunks) {
              float y[32];
#pragma unroll
              for (int j4 = 0; j4 < 8; ++j4) {
                const float4 g4 = reinterpret_cast<const float4 *>(gates)[c * 8 + j4];
                const int j = c * 32 + j4 * 4;
                y[j4 * 4] = (sub == 0 ? acc0[j] : acc1[j]) * g4.x;
                y[j4 * 4 + 1] = (sub == 0 ? acc0[j + 1] : acc1[j + 1]) * g4.y;
                y[j4 * 4 + 2] = (sub == 0 ? acc0[j + 2] : acc1[j + 2]) * g4.z;
                y[j4 * 4 + 3] = (sub == 0 ? acc0[j + 3] : acc1[j + 3]) * g4.w;
              }
              store_rows_bf16(out, args.out_ld, t.row0, c * 32, t.n_valid,
                              t.m0 + sub * kBM + q * 32, args.M, lane, y, stg);
            }
          }
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t gemm_e4m3_prepare() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_e4m3_kernel<kEpiSwiGLU>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kF8Smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_e4m3_kernel<kEpiGated>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kF8Smem);
}

cudaError_t launch_grouped_gemm_e4m3(int epi, const GemmArgs &args_in, int grid,
                                     cudaStream_t stream) {
  GemmArgs args = args_in;
  args.wait_limit = gemm_wait_limit();
  if (args.K % kF8BK != 0 || args.M % kBM != 0 || grid <= 0) return cudaErrorInvalidValue;
  if (epi == kEpiSwiGLU)
    grouped_gemm_e4m3_kernel<kEpiSwiGLU><<<grid, kF8Threads, kF8Smem, stream>>>(args);
  else if (epi == kEpiGated)
    grouped_gemm_e4m3_kernel<kEpiGated><<<grid, kF8Threads, kF8Smem, stream>>>(args);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace moe
