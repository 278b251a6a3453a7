// gemm.cu -- persistent grouped GEMM on the sm_100a tensor cores (tcgen05.mma, TMEM
// accumulators, TMA-fed multi-stage shared-memory ring).
//
// Used three ways by the MoE layer with zero-computation experts ("衝上熱搜！美團大模型，靠「快」
// 火了", §零計算專家 and §系統級優化):
//   router logits   l = x W_r^T                       (one group, fp32 split-K partials)
//   FFN up          h = silu(x_perm W_g^T) * (x_perm W_u^T)    (one group per FFN expert)
//   FFN down        y_perm = g * (h W_d^T)                     (one group per FFN expert)
//
// Orientation: the pages' serving stack puts the weights on the MMA's M side and the tokens on
// N ("SwapAB"), because N may be small and irregular.  The same holds for tcgen05: with M = 128,
// N may be any multiple of 16 up to 256, so a tile is 2 x (128 weight rows) x (n <= 128 or 256
// tokens, see Cfg): two accumulators share one token tile.  For the up-projection the two weight
// sub-tiles are 128 rows of W_g and the same 128 rows of W_u, so each TMEM lane (thread) holds
// the gate and the up value of one feature and SwiGLU needs no data exchange.  For the down
// projection and the router they are 256 consecutive output rows.
//
// At large batches the FFN GEMMs run on CTA pairs instead (dual_gemm_kernel, second half of this
// file): a cluster of two CTAs on two SMs issues pair MMAs of M = 256 weight rows, each CTA
// holding half the weight rows and half the token rows of a stage, and each pair runs two
// pipelines at once, full tiles beside the lightly used experts' weight-streaming tails.
//
// Warp roles of the single-CTA kernel (64 + 32 x kGemmEpiWarps = 192 threads, one CTA per SM,
// persistent over a static tile schedule; the two-pipeline pair kernel has two such sets):
//   warp 0      TMA producer: A0/A1 weight tiles (128 x 64) and the token tile (n x 64, issued
//               as 256/128/64/32/16-row boxes) into a 192 KB ring of 48 KB or 64 KB stages
//   warp 1      TMEM allocator (512 columns: 2 buffers x 2 x 128, or 1 x 2 x 256) and MMA issuer
//   warps 2-5   epilogue: tcgen05.ld from TMEM, fused SwiGLU / gate scaling / fp32 store via a
//               per-warp shared-memory transpose and coalesced row stores.  A warp may only
//               read the TMEM lane quarter (warp id mod 4); with more than four epilogue warps
//               the warps of a quarter take alternate 32-token chunks of the tile.
//   warps 6-13  FP8-weight instantiations only: converters (E4M3 codes -> bf16 slots, see Cfg)
//   warps 6-9   row-gather instantiation only: token-row loaders (cp.async, see Cfg)
// Token tiles come in two kinds: full tiles of BN rows (compute-bound) and each expert's partial
// tail tile (for the many lightly loaded experts: weight streaming).  The static schedule
// interleaves the two lists in proportion, and within a token tile the weight tiles come
// fastest, so the CTAs in flight share token tiles and walk one expert's weights together (L2
// reuse) while the tensor cores and HBM stay busy at the same time.
//
// Every wait is bounded (device.cuh): on timeout the kernel records MOE_DEV_WAIT_TIMEOUT, all
// roles unwind, in-flight copies and MMAs are drained (again bounded) and TMEM is freed.
#include <cuda_fp8.h>

#include <atomic>

#include "device.cuh"
#include "kernels.cuh"
#include "gemm_common.cuh"

namespace moe {
namespace {

// Adjacent 128-row weight blocks and full 256-token tiles are fetched as single 256-row boxes
// (fewer TMA operations for the one producer thread to issue).
constexpr bool kWideBoxes = true;
constexpr int kEpiWarps = kGemmEpiWarps;
constexpr int kEpiGroups = kEpiWarps / 4;    // warps sharing one TMEM lane quarter
static_assert(kEpiWarps % 4 == 0, "epilogue warps come in groups of four lane quarters");
constexpr int kSmemStaging = kEpiWarps * kStagingFloats * 4;
constexpr int kSmemPrefix = 2 * (kMaxGroups + 4) * 4;  // full-tile and tail-tile prefixes

// Two tile widths.  BN = 128 tokens: 48 KB stages, 4 in a 192 KB ring (128 KB of weights in
// flight, which weight-streaming tiles need), TMEM double-buffered (2 x 2 x 128 columns) so the
// epilogue overlaps the next tile.  BN = 256: 64 KB stages, 3 in the ring, one 2 x 256-column
// accumulator; every MMA and token load does twice the work, which is what compute-bound
// tiles need (the issuing threads, not the tensor cores, limit 128-wide tiles).
//
// FP8 weights (WQ, used with BN = 128): a stage holds the two weight blocks as E4M3 codes
// (2 x 8 KB, half the bytes, so twice the weights in flight per byte of ring) and the token
// rows; eight converter warps (four per weight block) turn the codes into bf16
// (times the block's power-of-two scale: exact) in a separate ring of two 32 KB bf16 slots,
// which is what the MMA reads.  A stage is free again once the converters have read its
// codes and the MMA its token rows; a slot once the MMA has read it.
constexpr int kQTile = kBM * kBK;            // 8 KB of E4M3 codes per weight block
constexpr int kConvWarps = 8;
// Row gather (GA): four loader warps copy the token rows of each stage from x[row_index[r]]
// with 16-byte cp.async into the swizzled token tile; the stage barrier expects one arrival
// per loader thread besides the producer's.
constexpr int kLoadWarps = 4;
constexpr int kLoadThreads = 32 * kLoadWarps;

template <int BN, bool WQ = false, bool GA = false>
struct Cfg {
  static constexpr int kAccBufs = BN <= 128 ? 2 : 1;
  static constexpr int kStage = (WQ ? 2 * kQTile : 2 * kTileA) + BN * kBK * 2;
  static constexpr int kCSlots = WQ ? 2 : 0;              // bf16 weight slots
  static constexpr int kCRing = kCSlots * 2 * kTileA;
  static constexpr int kStages = (192 * 1024 - kCRing) / kStage;
  static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 1 + 2 * kCSlots;
  static constexpr int kThreads =
      64 + 32 * kEpiWarps + (WQ ? 32 * kConvWarps : 0) + (GA ? kLoadThreads : 0);
  static constexpr int kSmemBytes = 1024 + kStages * kStage + kCRing + kSmemStaging +
                                    kSmemPrefix + kNumBars * 8 + 16;
  static_assert(kAccBufs * 2 * BN <= kTmemCols, "TMEM holds 512 columns");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};


// Thread `lane` of the epilogue warp with TMEM lane quarter q owns output feature (q*32 + lane)
// of each 128-row sub-tile.
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs &a, const Tile &t, uint32_t tcol,
                                               int chunk, int q, int lane, float *stage) {
  const int tok0 = chunk * 32;
  if (EPI == kEpiSwiGLU) {
    uint32_t g[32], u[32];
    tmem_ld_32x32b_x32(tcol, g);
    tmem_ld_32x32b_x32(tcol + BN, u);
    tmem_ld_wait();
    float h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) h[j] = silu(__uint_as_float(g[j])) * __uint_as_float(u[j]);
    store_rows_bf16(reinterpret_cast<uint16_t *>(a.out), a.out_ld, t.row0, tok0, t.n_valid,
                    t.m0 + q * 32, a.M, lane, h, reinterpret_cast<uint32_t *>(stage));
  } else if (EPI == kEpiGated || EPI == kEpiGatedCombine) {
    // The chunk's 32 gates, read by every lane as broadcast vector loads from the warp's
    // staging area (one store per lane, eight loads) instead of 32 shuffles.
    const int tok = tok0 + lane;
    stage[lane] = tok >= t.n_valid ? 0.f : (a.row_scale ? __ldg(a.row_scale + t.row0 + tok) : 1.f);
    __syncwarp();
    float gate[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 g4 = reinterpret_cast<const float4 *>(stage)[i];
      gate[4 * i] = g4.x;
      gate[4 * i + 1] = g4.y;
      gate[4 * i + 2] = g4.z;
      gate[4 * i + 3] = g4.w;
    }
    __syncwarp();
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
      if (sub == 1 && !t.has_a1) break;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tcol + sub * BN, v);
      tmem_ld_wait();
      float y[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(v[j]) * gate[j];
      store_rows_bf16(reinterpret_cast<uint16_t *>(a.out), a.out_ld, t.row0, tok0, t.n_valid,
                      t.m0 + sub * kBM + q * 32, a.M, lane, y, reinterpret_cast<uint32_t *>(stage));
    }
  } else {
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
      if (sub == 1 && !t.has_a1) break;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tcol + sub * BN, v);
      tmem_ld_wait();
      const int fbase = t.m0 + sub * kBM + q * 32;
      {  // kEpiF32: two passes of 16 tokens through the staging buffer
        const int f = fbase + (lane & 7) * 4;
        float *out = reinterpret_cast<float *>(a.out) + (long long)t.split * a.split_stride;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int j = 0; j < 16; ++j) stage[j * 32 + lane] = __uint_as_float(v[half * 16 + j]);
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int r = it * 4 + (lane >> 3);
            const int tok = tok0 + half * 16 + r;
            if (tok < t.n_valid && f < a.M) {
              const float4 val =
                  *reinterpret_cast<const float4 *>(stage + r * 32 + (lane & 7) * 4);
              *reinterpret_cast<float4 *>(out + (long long)(t.row0 + tok) * a.out_ld + f) = val;
            }
          }
          __syncwarp();
        }
      }
    }
  }
}

// ------------------------------------------------------------------ combine fused into GEMM2
// kEpiGatedCombine (the MoE layer's combine in the down projection's epilogue, deterministic):
// warp q of a tile owns feature block (tile's m-range, q) = features m0 + q*32 + [0, 32) and
// m0 + 128 + q*32 + [0, 32).  Each token's counter of each block starts at the token's number of
// FFN slots (launch_combine_counters).  After storing a 32-token chunk of y_perm rows, the warp
// makes the stores visible device-wide and counts one arrival down per token; the arrival that
// reaches zero belongs to the last tile holding one of the token's rows for that block, and that
// warp then sums the block of y for the token from y_perm in slot order -- the combine kernel's
// arithmetic (combine_add8 / combine_finish8), so the result does not depend on which tile
// finishes last.  Tokens with no FFN slot are left to launch_combine's zero-only pass.

// Counts the arrivals of the tile's tokens (after all of the warp's stores of the tile, one
// fence): one atomic per token, all issued before any result is used.  fin[c] gets the lanes
// (tokens c * 32 + lane) this warp completes.
template <int NC>
__device__ __forceinline__ void combine_count(const GemmArgs &a, const Tile &t, int chunks, int q,
                                              int lane, uint32_t (&fin)[NC]) {
  __threadfence();  // release: this lane's y_perm stores before its arrivals
  __syncwarp();
  const int blk = (t.m0 / (2 * kBM)) * 4 + q;
  int old[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    old[c] = 0;
    const int j = c * 32 + lane;
    if (c < chunks && j < t.n_valid) {
      const long long tok = __ldg(a.cmb_perm_tok + t.row0 + j);
      old[c] = atomicSub(a.cmb_count + tok * a.cmb_blocks + blk, 1);
    }
  }
  __threadfence();  // acquire: a lane that completed a count orders it before the warp's vote
#pragma unroll
  for (int c = 0; c < NC; ++c) fin[c] = __ballot_sync(0xffffffffu, old[c] == 1);
}

// Sums the completed tokens' blocks of y, four tokens at a time (eight lanes, 16 bytes each).
__device__ __forceinline__ void combine_finish(const GemmArgs &a, const Tile &t, int tok0,
                                               uint32_t fin, int q, int lane) {
  __threadfence();  // the rows of the tiles whose arrivals preceded ours, for every lane
  const int g = lane >> 3, i = lane & 7;
  const int f = t.m0 + (i < 4 ? 0 : kBM) + q * 32 + (i & 3) * 8;
  const uint16_t *y_perm = reinterpret_cast<const uint16_t *>(a.out);
  while (fin != 0u) {
    uint32_t m = fin;
    for (int s = 0; s < g && m != 0u; ++s) m &= m - 1;  // the g-th lowest remaining token
    if (m != 0u && f < a.M) {
      const long long tok = __ldg(a.cmb_perm_tok + t.row0 + tok0 + __ffs(m) - 1);
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      float zsum = 0.f;
      // Eight slots at a time: their loads are independent, the sums stay in slot order.
      constexpr int kB = 8;
      for (int k0 = 0; k0 < a.cmb_K; k0 += kB) {
        int e[kB], r[kB];
        float gv[kB];
        uint4 v[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const long long slot = tok * a.cmb_K + k0 + u;
          const bool in = k0 + u < a.cmb_K;
          e[u] = in ? __ldg(a.cmb_idx + slot) : a.cmb_N;
          r[u] = in ? __ldg(a.cmb_slot + slot) : 0;
          gv[u] = in ? __ldg(a.cmb_gate + slot) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (e[u] < a.cmb_N && r[u] >= 0 && r[u] < a.rows)
            v[u] = __ldcg(reinterpret_cast<const uint4 *>(y_perm + (long long)r[u] * a.out_ld +
                                                          f));
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (k0 + u >= a.cmb_K) break;
          if (e[u] >= a.cmb_N)
            zsum += gv[u];
          else if (r[u] >= 0 && r[u] < a.rows)
            combine_add8(acc, v[u]);
          else
            record_status(a.status, MOE_DEV_BAD_ROWS);
        }
      }
      const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(a.cmb_x + tok * a.M + f));
      *reinterpret_cast<uint4 *>(a.cmb_y + tok * a.M + f) = combine_finish8(acc, zsum, xv);
    }
    for (int s = 0; s < 4 && fin != 0u; ++s) fin &= fin - 1;
  }
}

// E4M3 block (128 rows x 64 codes, row-major) -> bf16 block in the 128-byte-swizzled K-major
// layout the MMA descriptors read, times `scale` (a power of two: exact).  `ct` in [0, 128):
// each thread converts one 16-code chunk of a row per pass; consecutive threads read
// consecutive 16-byte chunks, and each warp's stores cover all 32 banks four times.
__device__ __forceinline__ void convert_fp8_block(const uint8_t *q, uint8_t *dst, float scale,
                                                  int ct) {
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int r = pass * 32 + (ct >> 2), c = ct & 3;
    const uint4 v = *reinterpret_cast<const uint4 *>(q + r * kBK + c * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * h)) & 0xffffu), __NV_E4M3);
        const float2 f = __half22float2(__half2(hr));
        const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
        o[2 * i + h] = *reinterpret_cast<const uint32_t *>(&b);
      }
    }
    uint8_t *row = dst + r * (kBK * 2);
    const int j0 = 2 * c, sw = r & 7;
    *reinterpret_cast<uint4 *>(row + ((j0 ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4 *>(row + (((j0 + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

template <int EPI, int BN, bool WQ, bool GATHER>
__global__ void __launch_bounds__(Cfg<BN, WQ, GATHER>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs args) {
  using C = Cfg<BN, WQ, GATHER>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  constexpr int kRing = C::kStages * C::kStage + C::kCRing;
  uint8_t *cring = smem + C::kStages * C::kStage;  // WQ: bf16 weight slots (2 x 16 KB each)
  float *staging = reinterpret_cast<float *>(smem + kRing);
  int *hpre = reinterpret_cast<int *>(smem + kRing + kSmemStaging);
  int *lpre = hpre + kMaxGroups + 4;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kRing + kSmemStaging + kSmemPrefix);
  uint64_t *full_bar = bars;
  uint64_t *empty_bar = bars + C::kStages;
  uint64_t *tfull_bar = bars + 2 * C::kStages;
  uint64_t *tempty_bar = bars + 2 * C::kStages + C::kAccBufs;
  uint64_t *drain_bar = bars + 2 * C::kStages + 2 * C::kAccBufs;
  uint64_t *cfull_bar = drain_bar + 1;           // WQ: slot holds converted weights
  uint64_t *cempty_bar = cfull_bar + C::kCSlots;  // WQ: the MMA has read the slot
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int unit = (int)blockIdx.x;
  const int units = (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], GATHER ? 1 + kLoadThreads : 1);
      mbar_init(&empty_bar[s], WQ ? 1 + kConvWarps : 1);  // WQ: the converters read it too
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    for (int c = 0; c < C::kCSlots; ++c) {
      mbar_init(&cfull_bar[c], kConvWarps);
      mbar_init(&cempty_bar[c], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.map_a0);
    tma_prefetch_desc(&args.map_a1);
    tma_prefetch_desc(&args.map_a01);
    tma_prefetch_desc(&args.map_s0);
    tma_prefetch_desc(&args.map_s1);
    tma_prefetch_desc(&args.map_s01);
    tma_prefetch_desc(&args.map_b256);
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&args.map_b[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  Schedule sched;
  build_schedule<BN>(args, hpre, lpre, reinterpret_cast<int *>(staging), sched);
  sched.m_tiles = m_tiles_of<EPI>(args.M);
  sched.splits = EPI == kEpiF32 ? args.k_splits : 1;
  sched.total = sched.total * sched.m_tiles * sched.splits;
  const long long wlim = args.wait_limit > 0 ? args.wait_limit : kWaitLimitCycles;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Lane 0 issues the weight loads and the tiled token loads (in gather mode the loader warps
    // fetch the token rows instead).
    if (lane == 0) {
      // Weights of a group with a single token tile are read once: stream them past L2
      // (evict-first) so they do not push out the tiles other CTAs are still re-reading.
      const uint64_t pol_w_reused = l2_policy_evict_normal();
      const uint64_t pol_w_once = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < sched.total; tile += units) {
        const Tile t = decode_tile<EPI, BN>(args, sched, tile);
        const uint32_t bytes = (WQ ? kQTile : kTileA) * (t.has_a1 ? 2 : 1) +
                               (GATHER ? 0 : t.nb * kBK * 2);
        const uint64_t pol_w = t.once ? pol_w_once : pol_w_reused;
        const CUtensorMap *map_w0 = t.once ? &args.map_s0 : &args.map_a0;
        const CUtensorMap *map_w1 = t.once ? &args.map_s1 : &args.map_a1;
        const CUtensorMap *map_w01 = t.once ? &args.map_s01 : &args.map_a01;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, wlim)) {
            signal_abort(args, abort_flag);
            ok = false;
            break;
          }
          uint8_t *sa0 = ring + stage * C::kStage;
          uint8_t *sa1 = sa0 + kTileA;
          uint8_t *sb = sa0 + (WQ ? 2 * kQTile : 2 * kTileA);
          const int kc = kb * kBK;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          if (WQ) {  // E4M3 codes of both weight blocks at the start of the stage
            tma_load_2d(sa0, map_w0, &full_bar[stage], kc, t.a0_row, pol_w);
            if (t.has_a1)
              tma_load_2d(sa0 + kQTile, map_w1, &full_bar[stage], kc, t.a1_row, pol_w);
          } else if (kWideBoxes && EPI != kEpiSwiGLU && t.has_a1) {
            tma_load_2d(sa0, map_w01, &full_bar[stage], kc, t.a0_row, pol_w);
          } else {
            tma_load_2d(sa0, map_w0, &full_bar[stage], kc, t.a0_row, pol_w);
            if (t.has_a1)
              tma_load_2d(sa1, map_w1, &full_bar[stage], kc, t.a1_row, pol_w);
          }
          if (!GATHER) {
            // Token rows in boxes of 256 / 128 (as many as needed), then 64 / 32 / 16.
            int r = 0;
            if (kWideBoxes && t.nb == 256) {
              tma_load_2d(sb, &args.map_b256, &full_bar[stage], kc, t.row0, pol_x);
              r = 256;
            }
            for (; t.nb - r >= 128; r += 128)
              tma_load_2d(sb + r * (kBK * 2), &args.map_b[0], &full_bar[stage], kc, t.row0 + r,
                          pol_x);
#pragma unroll
            for (int i = 1; i < 4; ++i) {
              const int box = 128 >> i;
              if (t.nb - r >= box) {
                tma_load_2d(sb + r * (kBK * 2), &args.map_b[i], &full_bar[stage], kc,
                            t.row0 + r, pol_x);
                r += box;
              }
            }
          }
          ++issued;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Drain the copies that may still be landing in the ring (bounded).
        for (long long i = 1; i <= issued && i <= C::kStages; ++i) {
          const long long idx = issued - i;
          const int s = (int)(idx % C::kStages);
          const uint32_t par = (uint32_t)((idx / C::kStages) & 1);
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
      int cslot = 0;            // WQ: bf16 slot of the current k-step
      uint32_t cphase = 0;
      int it = 0;
      bool ok = true;
      bool any = false;
      for (int tile = unit; ok && tile < sched.total; tile += units, ++it) {
        const Tile t = decode_tile<EPI, BN>(args, sched, tile);
        const int buf = it % C::kAccBufs;
        const uint32_t use = (uint32_t)(it / C::kAccBufs);
        if (!mbar_wait(&tempty_bar[buf], (use & 1) ^ 1, abort_flag, wlim)) {
          signal_abort(args, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * (2 * BN);
        const uint32_t d1 = d0 + BN;
        const uint32_t idesc = idesc_bf16_f32(kBM, t.nb);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, wlim) ||
              (WQ && !mbar_wait(&cfull_bar[cslot], cphase, abort_flag, wlim))) {
            signal_abort(args, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          // Gathered token rows were written through the generic proxy (cp.async): order them
          // before the tensor cores' async-proxy reads.
          if (GATHER) fence_proxy_async_shared();
          const uint32_t sbase = smem_u32(ring + stage * C::kStage);
          const uint32_t abase = WQ ? smem_u32(cring + cslot * (2 * kTileA)) : sbase;
          const uint32_t bbase = sbase + (WQ ? 2 * kQTile : 2 * kTileA);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = sw128_kmajor_desc(bbase + k * 32);
            const uint32_t acc = (kb > t.kb0 || k > 0) ? 1u : 0u;
            umma_bf16(d0, sw128_kmajor_desc(abase + k * 32), bdesc, idesc, acc);
            if (t.has_a1)
              umma_bf16(d1, sw128_kmajor_desc(abase + kTileA + k * 32), bdesc, idesc, acc);
          }
          any = true;
          umma_commit(&empty_bar[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
          if (WQ) {
            umma_commit(&cempty_bar[cslot]);
            if (++cslot == C::kCSlots) { cslot = 0; cphase ^= 1; }
          }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[buf]);
      }
      if (!ok && any) {
        umma_commit(drain_bar);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain_bar, 0) && clock64() - t0 < kDrainLimitCycles) {}
      }
    }
  } else if (GATHER && warp >= 2 + kEpiWarps) {
    // ---------------------------------------------------------------- row-gather loaders
    // Thread g copies the 16-byte chunk j = g % 8 of rows g / 8, g / 8 + 16, ... of each
    // stage's token tile, so every warp moves whole 128-byte row segments; the chunk lands at
    // its 128-byte-swizzled place (chunk j of row r at (j ^ (r % 8)) * 16).
    const int g = (int)threadIdx.x - (2 + kEpiWarps) * 32;
    const int j = g & 7, r0 = g >> 3, sw = r0 & 7;
    const uint16_t *src = reinterpret_cast<const uint16_t *>(args.gather_src);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = unit; ok && tile < sched.total; tile += units) {
      const Tile t = decode_tile<EPI, BN>(args, sched, tile);
      const int nrow = t.nb >> 4;  // rows of this thread: r0 + 16 * i, i < nrow (<= 16)
      int rix[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        int v = i < nrow ? __ldg(args.row_index + t.row0 + min(r0 + 16 * i, t.n_valid - 1)) : 0;
        if (v < 0 || v >= args.gather_rows) {  // a bad index: report it, read row 0 instead
          record_status(args.status, MOE_DEV_BAD_ROWS);
          v = 0;
        }
        rix[i] = v;
      }
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!warp_wait(&empty_bar[stage], phase ^ 1, abort_flag, wlim)) {
          if (lane == 0) signal_abort(args, abort_flag);
          ok = false;
          break;
        }
        uint8_t *sb = ring + stage * C::kStage + 2 * kTileA;
        const uint16_t *col = src + kb * kBK + j * 8;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < nrow)
            cp_async_16(sb + (r0 + 16 * i) * (kBK * 2) + ((j ^ sw) << 4),
                        col + (long long)rix[i] * args.K);
        cp_async_mbar_arrive_noinc(&full_bar[stage]);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
  } else if (WQ && warp >= 2 + kEpiWarps) {
    // ---------------------------------------------------------------- converters (FP8)
    // Warps 0-3 of the converters handle weight block 0 of each k-step, warps 4-7 block 1.
    const int ct = (int)threadIdx.x - (2 + kEpiWarps) * 32;
    const int half = ct >> 7, lt = ct & 127;
    int stage = 0, cslot = 0;
    uint32_t phase = 0, cphase = 0;
    bool ok = true;
    for (int tile = unit; ok && tile < sched.total; tile += units) {
      const Tile t = decode_tile<EPI, BN>(args, sched, tile);
      const int row = half ? t.a1_row : t.a0_row;
      const float *scales = (half ? args.scale_a1 : args.scale_a0) + (row / 128) * args.scale_ld;
      const bool mine = half == 0 || t.has_a1;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!warp_wait(&full_bar[stage], phase, abort_flag, wlim) ||
            !warp_wait(&cempty_bar[cslot], cphase ^ 1, abort_flag, wlim)) {
          if (lane == 0) signal_abort(args, abort_flag);
          ok = false;
          break;
        }
        if (mine) {
          const uint8_t *q = ring + stage * C::kStage + half * kQTile;
          uint8_t *dst = cring + cslot * (2 * kTileA) + half * kTileA;
          convert_fp8_block(q, dst, __ldg(scales + (kb * kBK) / 128), lt);
          fence_proxy_async_shared();  // generic-proxy stores -> visible to the tensor cores
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&cfull_bar[cslot]);
          mbar_arrive(&empty_bar[stage]);  // this warp is done reading the stage's codes
        }
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        if (++cslot == C::kCSlots) { cslot = 0; cphase ^= 1; }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int group = (warp - 2) >> 2;   // the warps of a quarter take alternate 32-token chunks
    float *stage = staging + (warp - 2) * kStagingFloats;
    int it = 0;
    for (int tile = unit; tile < sched.total; tile += units, ++it) {
      const Tile t = decode_tile<EPI, BN>(args, sched, tile);
      const int buf = it % C::kAccBufs;
      const uint32_t use = (uint32_t)(it / C::kAccBufs);
      if (!warp_wait(&tfull_bar[buf], use & 1, abort_flag, wlim)) {
        if (lane == 0) signal_abort(args, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * (2 * BN);
      const int chunks = (t.n_valid + 31) / 32;
      if (EPI == kEpiGatedCombine) {
        // Stores and arrivals first, then the accumulator is released, then the sums.
        static_assert(EPI != kEpiGatedCombine || kEpiGroups == 1, "one warp per quarter");
        uint32_t fin[BN / 32];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
          if (c < chunks) epilogue_chunk<EPI, BN>(args, t, tcol + c * 32, c, q, lane, stage);
        combine_count(args, t, chunks, q, lane, fin);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[buf]);
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
          if (c < chunks && fin[c] != 0u) combine_finish(args, t, c * 32, fin[c], q, lane);
      } else {
        for (int c = group; c < chunks; c += kEpiGroups)
          epilogue_chunk<EPI, BN>(args, t, tcol + c * 32, c, q, lane, stage);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[buf]);
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

// ==================================================================== dual-pipeline CTA pairs
// Each CTA pair runs two independent pipelines at once, each with its own shared-memory ring,
// barriers, TMA producer, MMA issuer, four epilogue warps and TMEM columns:
//   F  full token tiles of kDualBNF = 224 rows, and the tail of an expert when it holds more than
//      kDualBNL rows (compute-bound: 3 stages of 2 x 16 KB weights + 112 token rows per CTA,
//      2 x 224 accumulator columns);
//   L  an expert's tail of at most kDualBNL = 32 rows (weight streaming: 2 stages of 2 x 16 KB
//      weights + 16 token rows per CTA, 2 x 32 accumulator columns).
// With one pipeline per SM every SM alternated between streaming a lightly used expert's weights
// (tensor pipe idle) and a heavily used expert's compute-bound tiles; here both kinds of tile are
// in flight on every SM, so HBM streaming and tensor work overlap within each SM.  Items of each
// list are dealt round-robin over the pairs; within a token tile the weight tiles come fastest.
constexpr int kDualBNF = 224;
constexpr int kDualBNL = 32;
constexpr int kDualStagesF = 3;
constexpr int kDualStagesL = 2;
constexpr int kDualStageF = 2 * kTileA + (kDualBNF / 2) * kBK * 2;  // 46 KB
constexpr int kDualStageL = 2 * kTileA + (kDualBNL / 2) * kBK * 2;  // 34 KB
constexpr int kDualEpiWarps = 4;                                     // per pipeline
constexpr int kDualThreads = 32 * 2 * (2 + kDualEpiWarps);           // 384
constexpr int kDualRing = kDualStagesF * kDualStageF + kDualStagesL * kDualStageL;
constexpr int kDualStaging = 2 * kDualEpiWarps * kStagingFloats * 4;
// uint16 prefixes of F and L tiles per group, sized per launch for the groups present (the
// maximum group count does not fit beside the rings).
__host__ __device__ constexpr int dual_prefix_len(int groups) { return (groups + 4 + 7) & ~7; }
constexpr int kDualBarsPerPipe = 2 * kDualStagesF + 3;
constexpr int kDualSmemFixed = 1024 + kDualRing + kDualStaging + 2 * kDualBarsPerPipe * 8 + 16;
constexpr int kDualSmemLimit = 232448;  // shared memory per block
__host__ __device__ constexpr int dual_smem_bytes(int groups) {
  return kDualSmemFixed + 2 * dual_prefix_len(groups) * 2;
}
static_assert(kDualStageF % 1024 == 0 && kDualStageL % 1024 == 0, "1024-byte-aligned stages");
// Most groups whose prefixes fit: 512 + 256 experts need 512.
constexpr int kDualMaxGroups = 960;
static_assert(dual_smem_bytes(kDualMaxGroups) <= kDualSmemLimit, "shared memory per block");
static_assert(2 * kDualBNF + 2 * kDualBNL <= kTmemCols, "TMEM holds 512 columns");

struct DualSchedule {
  const uint16_t *fpre;  // [G + 1] prefix of F tiles per group
  const uint16_t *lpre;  // [G + 1] prefix of L tiles per group
  int G;
  int F, L;              // tiles of each list
  int m_tiles;
};

__device__ __forceinline__ int find_group16(const uint16_t *pre, int G, int v) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int)pre[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// F and L tile counts per group (rows c): F = floor(c / BNF) + (c % BNF > BNL), L = (0 < c % BNF
// <= BNL).  The host guarantees the totals fit 16 bits (gemm_dual_fits).  Records
// MOE_DEV_BAD_ROWS and schedules nothing if the offsets are not monotone or exceed the rows.
__device__ void build_dual_schedule(const GemmArgs &a, uint16_t *fpre, uint16_t *lpre,
                                    int *scratch, DualSchedule &s) {
  const int G = a.num_groups;
  const int per = (G + (int)blockDim.x - 1) / (int)blockDim.x;
  const int g_begin = min(G, (int)threadIdx.x * per);
  const int g_end = min(G, g_begin + per);
  int nf = 0, nl = 0;
  bool bad = false;
  for (int g = g_begin; g < g_end; ++g) {
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    if (lo < 0 || hi < lo || hi > a.rows) { bad = true; continue; }
    const int c = hi - lo, r = c % kDualBNF;
    nf += c / kDualBNF + (r > kDualBNL ? 1 : 0);
    nl += (r > 0 && r <= kDualBNL) ? 1 : 0;
  }
  int F = 0, L = 0;
  int frun = block_exclusive_scan(nf, scratch, F);
  int lrun = block_exclusive_scan(nl, scratch, L);
  for (int g = g_begin; g < g_end; ++g) {
    fpre[g] = (uint16_t)frun;
    lpre[g] = (uint16_t)lrun;
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    if (!(lo < 0 || hi < lo || hi > a.rows)) {
      const int c = hi - lo, r = c % kDualBNF;
      frun += c / kDualBNF + (r > kDualBNL ? 1 : 0);
      lrun += (r > 0 && r <= kDualBNL) ? 1 : 0;
    }
  }
  if (threadIdx.x == 0) {
    fpre[G] = (uint16_t)F;
    lpre[G] = (uint16_t)L;
  }
  const bool any_bad = __syncthreads_or(bad);
  if (any_bad && threadIdx.x == 0) record_status(a.status, MOE_DEV_BAD_ROWS);
  s.fpre = fpre;
  s.lpre = lpre;
  s.G = G;
  s.F = any_bad ? 0 : F;
  s.L = any_bad ? 0 : L;
}

// Work item `item` of list F (full) or L (tail): weight tile fastest.
template <int EPI, bool FULL>
__device__ __forceinline__ Tile decode_dual(const GemmArgs &a, const DualSchedule &s, int item,
                                           uint32_t rank) {
  Tile t;
  const int mt = item % s.m_tiles;
  const int pos = item / s.m_tiles;
  int g;
  if (FULL) {
    g = find_group16(s.fpre, s.G, pos);
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    t.row0 = lo + (pos - (int)s.fpre[g]) * kDualBNF;
    t.n_valid = min(kDualBNF, hi - t.row0);
    t.once = (hi - lo) <= kDualBNF;  // the group's only tile
  } else {
    g = find_group16(s.lpre, s.G, pos);
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    t.row0 = lo + ((hi - lo) / kDualBNF) * kDualBNF;
    t.n_valid = hi - t.row0;
    t.once = (hi - lo) < kDualBNF;
  }
  t.nb = (t.n_valid + 31) & ~31;  // a pair MMA splits N in two halves of 16k rows
  if (EPI == kEpiSwiGLU) {
    t.m0 = mt * 2 * kBM + (int)rank * kBM;
    t.a0_row = g * a.M + t.m0;
    t.a1_row = t.a0_row;
  } else {
    t.m0 = mt * 4 * kBM + (int)rank * 2 * kBM;
    t.a0_row = g * a.M + t.m0;
    t.a1_row = t.a0_row + kBM;
  }
  t.has_a1 = true;
  t.kb0 = 0;
  t.kb1 = a.K / kBK;
  t.split = 0;
  return t;
}

// TMA producer of one pipeline (lane 0 of its warp, both CTAs).  Each CTA loads its 128 weight
// rows of both sub-tiles and its half of the token rows; the bytes of both CTAs complete on the
// even CTA's stage barrier.
template <int EPI, bool FULL, int BN, int STAGES>
__device__ void dual_producer(const GemmArgs &args, const DualSchedule &s, uint8_t *ring,
                              uint64_t *full_bar, uint64_t *empty_bar, volatile int *abort_flag,
                              long long wlim, int unit, int units, uint32_t rank) {
  constexpr int kStage = 2 * kTileA + (BN / 2) * kBK * 2;
  const int total = (FULL ? s.F : s.L) * s.m_tiles;
  const uint64_t pol_w_reused = l2_policy_evict_normal();
  const uint64_t pol_w_once = l2_policy_evict_first();
  const uint64_t pol_x = l2_policy_evict_last();
  int stage = 0;
  uint32_t phase = 0;
  long long issued = 0;
  bool ok = true;
  for (int item = unit; ok && item < total; item += units) {
    const Tile t = decode_dual<EPI, FULL>(args, s, item, rank);
    const uint32_t bytes = 2u * (2 * kTileA + (t.nb / 2) * kBK * 2);
    const uint64_t pol_w = t.once ? pol_w_once : pol_w_reused;
    const CUtensorMap *map_w0 = t.once ? &args.map_s0 : &args.map_a0;
    const CUtensorMap *map_w1 = t.once ? &args.map_s1 : &args.map_a1;
    const CUtensorMap *map_w01 = t.once ? &args.map_s01 : &args.map_a01;
    for (int kb = t.kb0; kb < t.kb1; ++kb) {
      if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, wlim)) {
        signal_abort(args, abort_flag);
        ok = false;
        break;
      }
      uint8_t *sa0 = ring + stage * kStage;
      uint8_t *sa1 = sa0 + kTileA;
      uint8_t *sb = sa0 + 2 * kTileA;
      const int kc = kb * kBK;
      const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
      if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], bytes);
      if (EPI != kEpiSwiGLU) {
        tma_load_2d_pair(sa0, map_w01, fb, kc, t.a0_row, pol_w);
      } else {
        tma_load_2d_pair(sa0, map_w0, fb, kc, t.a0_row, pol_w);
        tma_load_2d_pair(sa1, map_w1, fb, kc, t.a1_row, pol_w);
      }
      const int half = t.nb >> 1, brow = t.row0 + (int)rank * half;
      int r = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int box = 128 >> i;
        if (half - r >= box) {
          tma_load_2d_pair(sb + r * (kBK * 2), &args.map_b[i], fb, kc, brow + r, pol_x);
          r += box;
        }
      }
      ++issued;
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
  }
  if (!ok && rank == 0) {
    // Drain the copies that may still be landing in the ring (bounded; the even CTA's
    // barriers count both CTAs' copies).
    for (long long i = 1; i <= issued && i <= STAGES; ++i) {
      const long long idx = issued - i;
      const int st = (int)(idx % STAGES);
      const uint32_t par = (uint32_t)((idx / STAGES) & 1);
      const long long t0 = clock64();
      while (!mbar_try_wait(&full_bar[st], par) && clock64() - t0 < kDrainLimitCycles) {}
    }
  }
}

// MMA issuer of one pipeline (lane 0 of its warp, even CTA): pair MMAs (M = 256 weight rows,
// N = the tile's rows rounded to 32) into the pipeline's two accumulators at TMEM column `col`.
template <int EPI, bool FULL, int BN, int STAGES>
__device__ void dual_mma(const GemmArgs &args, const DualSchedule &s, uint8_t *ring,
                         uint64_t *full_bar, uint64_t *empty_bar, uint64_t *tfull_bar,
                         uint64_t *tempty_bar, uint64_t *drain_bar, volatile int *abort_flag,
                         long long wlim, int unit, int units, uint32_t tmem_base, int col) {
  constexpr int kStage = 2 * kTileA + (BN / 2) * kBK * 2;
  const int total = (FULL ? s.F : s.L) * s.m_tiles;
  int stage = 0;
  uint32_t phase = 0;
  int it = 0;
  bool ok = true;
  bool any = false;
  for (int item = unit; ok && item < total; item += units, ++it) {
    const Tile t = decode_dual<EPI, FULL>(args, s, item, 0);
    if (!mbar_wait(tempty_bar, (it & 1) ^ 1, abort_flag, wlim)) {
      signal_abort(args, abort_flag);
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d0 = tmem_base + col;
    const uint32_t d1 = d0 + BN;
    const uint32_t idesc = idesc_bf16_f32(2 * kBM, t.nb);
    for (int kb = t.kb0; kb < t.kb1; ++kb) {
      if (!mbar_wait(&full_bar[stage], phase, abort_flag, wlim)) {
        signal_abort(args, abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t abase = smem_u32(ring + stage * kStage);
      const uint32_t bbase = abase + 2 * kTileA;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        const uint64_t bdesc = sw128_kmajor_desc(bbase + k * 32);
        const uint32_t acc = (kb > t.kb0 || k > 0) ? 1u : 0u;
        umma_bf16_pair(d0, sw128_kmajor_desc(abase + k * 32), bdesc, idesc, acc);
        umma_bf16_pair(d1, sw128_kmajor_desc(abase + kTileA + k * 32), bdesc, idesc, acc);
      }
      any = true;
      umma_commit_pair(&empty_bar[stage], 0x3);  // frees the stage in both CTAs
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
    if (!ok) break;
    umma_commit_pair(tfull_bar, 0x3);
  }
  if (!ok && any) {
    umma_commit_pair(drain_bar, 0x1);
    const long long t0 = clock64();
    while (!mbar_try_wait(drain_bar, 0) && clock64() - t0 < kDrainLimitCycles) {}
  }
}

// Epilogue warp of one pipeline (both CTAs): drains its lane quarter of the accumulators at TMEM
// column `col` and releases them on the even CTA's barrier.
template <int EPI, bool FULL, int BN>
__device__ void dual_epilogue(const GemmArgs &args, const DualSchedule &s, uint64_t *tfull_bar,
                              uint64_t *tempty_bar, volatile int *abort_flag, long long wlim,
                              int unit, int units, uint32_t rank, uint32_t tmem_base, int col,
                              int q, int lane, float *stage) {
  const int total = (FULL ? s.F : s.L) * s.m_tiles;
  int it = 0;
  for (int item = unit; item < total; item += units, ++it) {
    const Tile t = decode_dual<EPI, FULL>(args, s, item, rank);
    if (!warp_wait(tfull_bar, it & 1, abort_flag, wlim)) {
      if (lane == 0) signal_abort(args, abort_flag);
      break;
    }
    tc_fence_after();
    const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col;
    const int chunks = (t.n_valid + 31) / 32;
    for (int c = 0; c < chunks; ++c)
      epilogue_chunk<EPI, BN>(args, t, tcol + c * 32, c, q, lane, stage);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(tempty_bar), 0));
  }
}

template <int EPI>
__global__ void __launch_bounds__(kDualThreads, 1)
    dual_gemm_kernel(const __grid_constant__ GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring_f = smem;
  uint8_t *ring_l = smem + kDualStagesF * kDualStageF;
  float *staging = reinterpret_cast<float *>(smem + kDualRing);
  uint16_t *fpre = reinterpret_cast<uint16_t *>(smem + kDualRing + kDualStaging);
  const int pfx = dual_prefix_len(args.num_groups);
  uint16_t *lpre = fpre + pfx;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kDualRing + kDualStaging + 2 * pfx * 2);
  // per pipeline p: full[kDualStagesF], empty[kDualStagesF], tfull, tempty, drain
  uint64_t *bf = bars, *bl = bars + kDualBarsPerPipe;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kDualBarsPerPipe);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int unit = (int)(blockIdx.x >> 1);
  const int units = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int p = 0; p < 2; ++p) {
      uint64_t *b = p ? bl : bf;
      const int stages = p ? kDualStagesL : kDualStagesF;
      for (int i = 0; i < stages; ++i) {
        mbar_init(&b[i], 1);
        mbar_init(&b[kDualStagesF + i], 1);
      }
      mbar_init(&b[2 * kDualStagesF], 1);                       // tfull
      mbar_init(&b[2 * kDualStagesF + 1], 2 * kDualEpiWarps);   // tempty: both CTAs' epilogues
      mbar_init(&b[2 * kDualStagesF + 2], 1);                   // drain
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.map_a0);
    tma_prefetch_desc(&args.map_a1);
    tma_prefetch_desc(&args.map_a01);
    tma_prefetch_desc(&args.map_s0);
    tma_prefetch_desc(&args.map_s1);
    tma_prefetch_desc(&args.map_s01);
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&args.map_b[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  DualSchedule sched;
  build_dual_schedule(args, fpre, lpre, reinterpret_cast<int *>(staging), sched);
  // Weight rows per pair tile: 2 x 128 features (gate and up rows of each) for the
  // up-projection, 2 x 2 x 128 output rows for the down-projection.
  sched.m_tiles = (args.M + (EPI == kEpiSwiGLU ? 2 : 4) * kBM - 1) / ((EPI == kEpiSwiGLU ? 2 : 4) * kBM);
  const long long wlim = args.wait_limit > 0 ? args.wait_limit : kWaitLimitCycles;
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  constexpr int kColF = 0, kColL = 2 * kDualBNF;

  const int role = warp % 6;           // 0 producer, 1 MMA, 2-5 epilogue
  const bool full = warp < 6;
  uint64_t *b = full ? bf : bl;
  if (role == 0) {
    if (lane == 0) {
      if (full)
        dual_producer<EPI, true, kDualBNF, kDualStagesF>(args, sched, ring_f, b, b + kDualStagesF,
                                                         abort_flag, wlim, unit, units, rank);
      else
        dual_producer<EPI, false, kDualBNL, kDualStagesL>(args, sched, ring_l, b,
                                                          b + kDualStagesF, abort_flag, wlim,
                                                          unit, units, rank);
    }
  } else if (role == 1) {
    if (lane == 0 && rank == 0) {
      if (full)
        dual_mma<EPI, true, kDualBNF, kDualStagesF>(
            args, sched, ring_f, b, b + kDualStagesF, b + 2 * kDualStagesF,
            b + 2 * kDualStagesF + 1, b + 2 * kDualStagesF + 2, abort_flag, wlim, unit, units,
            tmem_base, kColF);
      else
        dual_mma<EPI, false, kDualBNL, kDualStagesL>(
            args, sched, ring_l, b, b + kDualStagesF, b + 2 * kDualStagesF,
            b + 2 * kDualStagesF + 1, b + 2 * kDualStagesF + 2, abort_flag, wlim, unit, units,
            tmem_base, kColL);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    float *stage = staging + (warp - (full ? 2 : 4)) * kStagingFloats;
    if (full)
      dual_epilogue<EPI, true, kDualBNF>(args, sched, b + 2 * kDualStagesF,
                                         b + 2 * kDualStagesF + 1, abort_flag, wlim, unit, units,
                                         rank, tmem_base, kColF, q, lane, stage);
    else
      dual_epilogue<EPI, false, kDualBNL>(args, sched, b + 2 * kDualStagesF,
                                          b + 2 * kDualStagesF + 1, abort_flag, wlim, unit,
                                          units, rank, tmem_base, kColL, q, lane, stage);
  }

  tc_fence_before();
  __syncwarp();    // lanes 1-31 of the producer and MMA warps skipped the role loops: reconverge
  cluster_sync();  // no CTA leaves while its peer may still touch its barriers or memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int EPI, int BN, bool WQ = false, bool GATHER = false>
cudaError_t set_smem_limit() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<EPI, BN, WQ, GATHER>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<BN, WQ, GATHER>::kSmemBytes);
}

// Wait limit applied to launches (0: kWaitLimitCycles); only the timeout-path tests change it.
std::atomic<long long> g_wait_limit{0};

GemmArgs with_limit(const GemmArgs &args) {
  GemmArgs a = args;
  a.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  return a;
}

constexpr int kMaxDevices = 64;
int g_max_dual_pairs[kMaxDevices] = {0};

// Clusters of two CTAs (one CTA pair per cluster) of the two-pipeline kernel.
cudaLaunchConfig_t dual_config(int pairs, int groups, cudaStream_t stream,
                               cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kDualThreads, 1, 1);
  cfg.dynamicSmemBytes = dual_smem_bytes(groups);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int EPI>
cudaError_t prepare_dual(int device) {
  cudaError_t e = cudaFuncSetAttribute(dual_gemm_kernel<EPI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kDualSmemLimit);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = dual_config(1, kDualMaxGroups, nullptr, attr);
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, dual_gemm_kernel<EPI>, &cfg);
  if (e != cudaSuccess) return e;
  if (clusters <= 0) return cudaErrorInvalidConfiguration;
  if (g_max_dual_pairs[device] == 0 || clusters < g_max_dual_pairs[device])
    g_max_dual_pairs[device] = clusters;
  return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(int epi, const GemmArgs &args_in, int grid, cudaStream_t stream) {
  const GemmArgs args = with_limit(args_in);
  constexpr int smem = Cfg<BN>::kSmemBytes;
  constexpr int threads = Cfg<BN>::kThreads;
  switch (epi) {
    case kEpiSwiGLU:
      if (args.row_index != nullptr)
        grouped_gemm_kernel<kEpiSwiGLU, BN, false, true>
            <<<grid, Cfg<BN, false, true>::kThreads, smem, stream>>>(args);
      else
        grouped_gemm_kernel<kEpiSwiGLU, BN, false, false><<<grid, threads, smem, stream>>>(args);
      break;
    case kEpiGated:
      grouped_gemm_kernel<kEpiGated, BN, false, false><<<grid, threads, smem, stream>>>(args);
      break;
    case kEpiGatedCombine:
      grouped_gemm_kernel<kEpiGatedCombine, BN, false, false>
          <<<grid, threads, smem, stream>>>(args);
      break;
    default:
      grouped_gemm_kernel<kEpiF32, BN, false, false><<<grid, threads, smem, stream>>>(args);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_prepare(int device) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaError_t e;
  if ((e = prepare_dual<kEpiSwiGLU>(device)) != cudaSuccess) return e;
  if ((e = prepare_dual<kEpiGated>(device)) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiSwiGLU, 128>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiGated, 128>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiGatedCombine, 128>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiGatedCombine, 256>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiF32, 128>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiSwiGLU, 256>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiGated, 256>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiSwiGLU, 128, false, true>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiSwiGLU, 256, false, true>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiSwiGLU, 128, true>()) != cudaSuccess) return e;
  if ((e = set_smem_limit<kEpiGated, 128, true>()) != cudaSuccess) return e;
  if ((e = gemm_e4m3_prepare()) != cudaSuccess) return e;
  return set_smem_limit<kEpiF32, 256>();
}

void gemm_set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed);
}

long long gemm_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

int gemm_tile_tokens(long long rows, int groups, int K) {
  // 256-token tiles need enough rows per group to fill them (mean rows per group, an upper
  // bound since zero-expert slots are counted too) and a long reduction, over which the
  // single accumulator buffer's epilogue stall is amortised.  Otherwise 128.
  return (rows >= 128ll * groups && K >= 4096) ? 256 : 128;
}

int gemm_max_dual_pairs(int device) {
  return (device >= 0 && device < kMaxDevices) ? g_max_dual_pairs[device] : 0;
}

bool gemm_dual_fits(long long rows, int groups) {
  // Per-group tile prefixes are 16-bit (F tiles <= rows / BNF + groups, L tiles <= groups) and
  // sized to the groups present, within the shared memory beside the rings.
  return groups <= kDualMaxGroups && rows / kDualBNF + groups + 8 < 65536;
}

cudaError_t launch_grouped_gemm_dual(int epi, const GemmArgs &args_in, int pairs,
                                     cudaStream_t stream) {
  if (pairs <= 0) return cudaErrorInvalidConfiguration;
  const GemmArgs args = with_limit(args_in);
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = dual_config(pairs, args.num_groups, stream, attr);
  switch (epi) {
    case kEpiSwiGLU: return cudaLaunchKernelEx(&cfg, dual_gemm_kernel<kEpiSwiGLU>, args);
    case kEpiGated: return cudaLaunchKernelEx(&cfg, dual_gemm_kernel<kEpiGated>, args);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_grouped_gemm(int epi, const GemmArgs &args, int grid, int tile_tokens,
                                cudaStream_t stream) {
  return tile_tokens == 256 ? launch_bn<256>(epi, args, grid, stream)
                            : launch_bn<128>(epi, args, grid, stream);
}

cudaError_t launch_grouped_gemm_fp8(int epi, const GemmArgs &args_in, int grid,
                                    cudaStream_t stream) {
  using C = Cfg<128, true>;
  const GemmArgs args = with_limit(args_in);
  if (epi == kEpiSwiGLU)
    grouped_gemm_kernel<kEpiSwiGLU, 128, true, false>
        <<<grid, C::kThreads, C::kSmemBytes, stream>>>(args);
  else if (epi == kEpiGated)
    grouped_gemm_kernel<kEpiGated, 128, true, false>
        <<<grid, C::kThreads, C::kSmemBytes, stream>>>(args);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace moe
