// gemm_common.cuh -- pieces shared by the grouped-GEMM kernel files (gemm.cu, gemm_f8.cu): the
// token-tile schedule over groups, tile decoding, bounded warp waits and the packed bf16 row
// store of the epilogues.  Everything here has internal linkage (an anonymous namespace), so
// each kernel file compiles its own copy.
#pragma once

#include "device.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;                      // reduction elements per stage (128-byte rows)
constexpr int kBM = 128;                     // weight rows per MMA
constexpr int kTileA = kBM * kBK * 2;        // 16 KB per weight block
constexpr int kStagingFloats = 16 * 32;      // 2 KB per epilogue warp: 32 x 32 bf16 or 16 x 32 fp32
constexpr int kMaxGroups = 1024;
constexpr int kTmemCols = 512;
constexpr long long kDrainLimitCycles = 1ll << 30;

struct Tile {
  int row0;     // first activation row
  int n_valid;  // activation rows in this tile (1..128)
  int nb;       // rows loaded / MMA N: n_valid rounded up to 16
  int a0_row;   // first weight row of sub-tile 0 in map_a0
  int a1_row;   // first weight row of sub-tile 1 in map_a1
  int m0;       // first output feature of the tile
  bool has_a1;  // sub-tile 1 exists
  bool once;    // the group's only token tile: its weight tiles are read exactly once
  int kb0, kb1; // reduction blocks [kb0, kb1)
  int split;
};

// Token tiles of a group (expert) with c rows: floor(c/BN) full BN-row tiles ("heavy":
// compute-bound at d = 6144) and, if c % BN != 0, one partial tail tile ("light": for the many
// experts with a handful of tokens it only streams the expert's weights).  The schedule merges
// the two lists so the tiles in flight at any moment mix both kinds and the tensor cores and
// HBM are busy together: of the first p+1 merged positions, floor((p+1) L / (H+L)) are light.
// Work items (token tile, weight tile, split) are dealt round-robin to the persistent units
// (CTAs, or CTA pairs).  Every SM therefore streams some of the time: one SM keeps only ~128 KB
// of weights in flight, about 45-60 GB/s, so HBM needs most SMs streaming at once (measured:
// dedicating a subset of units to the tail tiles and the rest to full tiles was slower for
// every split tried, the tail side never reaching the bandwidth the interleaving gets).
struct Schedule {
  const int *hpre;  // [G + 1] prefix of full tiles per group (shared memory)
  const int *lpre;  // [G + 1] prefix of tail tiles per group
  int G;
  int H, L;         // total full / tail tiles
  int m_tiles;
  int splits;
  int total;        // work items
};

__device__ __forceinline__ int group_off(const GemmArgs &a, int g) {
  if (a.group_offsets == nullptr) return g == 0 ? 0 : a.rows;
  return __ldg(a.group_offsets + g);
}

// Largest g in [0, G) with pre[g] <= v (pre non-decreasing, pre[0] = 0 <= v).
__device__ __forceinline__ int find_group(const int *pre, int G, int v) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int EPI, int BN>
__device__ __forceinline__ Tile decode_tile(const GemmArgs &a, const Schedule &s, int tile) {
  Tile t;
  const int mt = tile % s.m_tiles;
  const int rest = tile / s.m_tiles;
  t.split = rest % s.splits;
  const int pos = rest / s.splits;
  const long long P = (long long)s.H + s.L;
  const int light_upto = (int)(((long long)pos + 1) * s.L / P);
  const int light_before = (int)((long long)pos * s.L / P);
  int g;
  if (light_upto > light_before) {  // the (light_upto-1)-th tail tile
    g = find_group(s.lpre, s.G, light_upto - 1);
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    t.row0 = lo + ((hi - lo) / BN) * BN;
    t.n_valid = hi - t.row0;
    t.once = (hi - lo) < BN;
  } else {  // the (pos - light_before)-th full tile
    const int i = pos - light_before;
    g = find_group(s.hpre, s.G, i);
    t.row0 = group_off(a, g) + (i - s.hpre[g]) * BN;
    t.n_valid = BN;
    t.once = false;
  }
  t.nb = (t.n_valid + 15) & ~15;
  if (EPI == kEpiSwiGLU) {
    t.m0 = mt * kBM;
    t.a0_row = g * a.M + t.m0;
    t.a1_row = t.a0_row;
    t.has_a1 = true;
  } else {
    t.m0 = mt * 2 * kBM;
    t.a0_row = g * a.M + t.m0;
    t.a1_row = t.a0_row + kBM;
    t.has_a1 = (t.m0 + kBM) < a.M;
  }
  const int kblocks = a.K / kBK;
  t.kb0 = (int)(((long long)kblocks * t.split) / s.splits);
  t.kb1 = (int)(((long long)kblocks * (t.split + 1)) / s.splits);
  return t;
}

// Exclusive block-wide scan of one int per thread; returns the thread's exclusive prefix and
// the block total.  `scratch` holds one int per warp.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int base = 0;
  total = 0;
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
    if (w < warp) base += scratch[w];
    total += scratch[w];
  }
  __syncthreads();
  return base + incl - v;
}

// Full-tile and tail-tile prefixes over groups, computed by all threads of the block.  Returns
// false (and records MOE_DEV_BAD_ROWS) if the offsets are not monotone or exceed the rows.
template <int BN>
__device__ bool build_schedule(const GemmArgs &a, int *hpre, int *lpre, int *scratch,
                               Schedule &s) {
  const int G = a.group_offsets ? a.num_groups : 1;
  const int per = (G + (int)blockDim.x - 1) / (int)blockDim.x;
  const int g_begin = min(G, (int)threadIdx.x * per);
  const int g_end = min(G, g_begin + per);
  int nh = 0, nl = 0;
  bool bad = false;
  for (int g = g_begin; g < g_end; ++g) {
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    if (lo < 0 || hi < lo || hi > a.rows) { bad = true; continue; }
    nh += (hi - lo) / BN;
    nl += ((hi - lo) % BN) != 0;
  }
  int H = 0, L = 0;
  int hrun = block_exclusive_scan(nh, scratch, H);
  int lrun = block_exclusive_scan(nl, scratch, L);
  for (int g = g_begin; g < g_end; ++g) {
    hpre[g] = hrun;
    lpre[g] = lrun;
    const int lo = group_off(a, g), hi = group_off(a, g + 1);
    if (!(lo < 0 || hi < lo || hi > a.rows)) {
      hrun += (hi - lo) / BN;
      lrun += ((hi - lo) % BN) != 0;
    }
  }
  if (threadIdx.x == 0) {
    hpre[G] = H;
    lpre[G] = L;
  }
  const bool any_bad = __syncthreads_or(bad);
  if (any_bad && threadIdx.x == 0) record_status(a.status, MOE_DEV_BAD_ROWS);
  s.hpre = hpre;
  s.lpre = lpre;
  s.G = G;
  s.H = any_bad ? 0 : H;
  s.L = any_bad ? 0 : L;
  s.total = s.H + s.L;  // token tiles; times m_tiles and splits by the caller
  return !any_bad;
}

template <int EPI>
__device__ __forceinline__ int m_tiles_of(int M) {
  const int rows = EPI == kEpiSwiGLU ? kBM : 2 * kBM;
  return (M + rows - 1) / rows;
}

// Bounded wait by lane 0 of a warp, result broadcast so the warp stays converged.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          long long limit) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, limit) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void signal_abort(const GemmArgs &a, volatile int *abort) {
  record_status(a.status, MOE_DEV_WAIT_TIMEOUT);
  *abort = 1;
}

// silu(z) = z / (1 + e^-z) with the fast division: a few ulp in fp32, far below the bf16 rounding
// of h that follows; for z below about -87 it returns 0 (the true value is under 1e-36).  The
// epilogue runs between tiles on the MMA thread's critical path, and with the IEEE division's
// longer sequence the up-projection took ~7% longer.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// ------------------------------------------------------------------ epilogue, one 32-token chunk
// Stores a 32 x 32 block held one feature per lane (v[j] = feature f0 + lane of token tok0 + j)
// as bf16 token rows.  Lanes 2i and 2i+1 trade one value per pair of tokens, so lane 2i holds
// features (f0 + 2i, f0 + 2i + 1) of token j and lane 2i + 1 the same two features of token
// j + 1: one packed conversion and one 4-byte shared-memory store per two values, each store
// instruction filling two 64-byte rows of the warp's 2 KB staging area without bank conflicts;
// then each lane copies 16 bytes of a row to global memory (four 16-byte stores per lane).
// Every value is rounded to nearest once.
__device__ __forceinline__ void store_rows_bf16(uint16_t *out, long long ld, int row0, int tok0,
                                                int n_valid, int f0, int M, int lane,
                                                const float (&v)[32], uint32_t *stage) {
  const bool odd = (lane & 1) != 0;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float mine = odd ? v[j + 1] : v[j];
    const float theirs = __shfl_xor_sync(0xffffffffu, odd ? v[j] : v[j + 1], 1);
    stage[(j + (odd ? 1 : 0)) * 16 + (lane >> 1)] =
        odd ? pack_bf16x2(theirs, mine) : pack_bf16x2(mine, theirs);
  }
  __syncwarp();
  const int f = f0 + (lane & 3) * 8;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = it * 8 + (lane >> 2);
    const int tok = tok0 + r;
    if (tok < n_valid && f < M) {
      const uint4 val = *reinterpret_cast<const uint4 *>(stage + r * 16 + (lane & 3) * 4);
      *reinterpret_cast<uint4 *>(out + (long long)(row0 + tok) * ld + f) = val;
    }
  }
  __syncwarp();
}

}  // namespace
}  // namespace moe
