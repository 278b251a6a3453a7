// moe_api.cu -- the C ABI declared in include/moe.h: argument checks, workspace layout, TMA
// descriptors and the launch sequence of the MoE layer with zero-computation experts.
//
// Every check happens on the host before anything is enqueued; nothing here synchronises
// except moe_last_device_error, and nothing allocates device memory.
#include <cmath>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kernels.cuh"
#include "../../include/moe.h"

namespace moe {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxExperts = 1024;
constexpr int kMaxK = 32;
constexpr int kNominalSms = 148;  // B200; sizes the router's split-K from the dims alone
constexpr size_t kAlign = 256;

struct DeviceInfo {
  bool ready = false;
  int status = MOE_OK;
  int sms = 0;
  int dual_pairs = 0;  // persistent CTA pairs of the pair GEMMs (co-resident, <= sms / 2)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

int device_info(const DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo &di = g_dev[dev];
  if (!di.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      return MOE_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
      di.status = MOE_ERR_ARCH;
    } else if (gemm_prepare(dev) != cudaSuccess) {
      return MOE_ERR_CUDA;
    } else {
      di.status = MOE_OK;
    }
    di.sms = sms;
    di.dual_pairs = di.status == MOE_OK ? std::min(gemm_max_dual_pairs(dev), sms / 2) : 0;
    di.ready = true;
  }
  *out = &di;
  return di.status;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in boxes of 64 columns x box_rows rows, 128-byte
// swizzle (the layout the tcgen05 descriptors expect), zero fill outside the matrix.
// L2 promotion: each box row is a 128-byte segment; promoting misses to 256 bytes fetches the
// next k-slice early, which helps weight streaming (128-token tiles: decode 8% faster) but at
// 256-token tiles the promoted halves are often evicted before use and fetched again (prefill
// DRAM traffic 10% higher), so those launches promote to 128 bytes.
bool make_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
              uint32_t box_rows, bool promote256 = true) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            promote256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Row-major E4M3 codes [rows, cols] in boxes of 64 columns (64 bytes) x 128 rows, no swizzle
// (the converter warps read them row by row).
bool make_map_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Row-major E4M3 codes [rows, cols] in boxes of 128 columns (128 bytes) x box_rows rows with the
// 128-byte swizzle: the operand layout the kind::f8f6f4 MMAs read (FP8 activations).
bool make_map_e4m3(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Block-quantised expert weights: E4M3 codes in the bf16 weights' layouts and one fp32
// power-of-two scale per 128 x 128 block ([N][rows / 128][cols / 128]).
struct Fp8Weights {
  const uint8_t *q_g, *q_u, *q_d;
  const float *s_g, *s_u, *s_d;
};

bool make_act_maps(GemmArgs &a, const void *base, uint64_t rows, uint64_t cols,
                   bool promote256 = true) {
  for (int i = 0; i < 4; ++i)
    if (!make_map(&a.map_b[i], base, rows, cols, 128u >> i, promote256)) return false;
  return make_map(&a.map_b256, base, rows, cols, 256, promote256);
}

// Weight maps for tiles that read their weights once: the given maps themselves when they
// already promote to 256 bytes (or hold FP8 codes), else the same tensors with 256-byte
// promotion (GemmArgs::map_s0).
bool make_stream_maps(GemmArgs &a, const void *w0, const void *w1, uint64_t rows,
                      uint64_t cols, bool promote256) {
  if (promote256) {
    a.map_s0 = a.map_a0;
    a.map_s1 = a.map_a1;
    a.map_s01 = a.map_a01;
    return true;
  }
  return make_map(&a.map_s0, w0, rows, cols, 128, true) &&
         make_map(&a.map_s1, w1, rows, cols, 128, true) &&
         make_map(&a.map_s01, w0, rows, cols, 256, true);
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool dims_ok(const moe_dims *d) {
  if (d == nullptr) return false;
  const long long E = (long long)d->N + d->Z;
  if (d->T < 0 || d->N < 0 || d->Z < 0) return false;
  if (d->d <= 0 || d->d % 64 != 0 || d->I <= 0 || d->I % 64 != 0) return false;
  if (E < 1 || E > kMaxExperts) return false;
  if (d->K < 1 || d->K > kMaxK || d->K > E) return false;
  if ((long long)d->T * d->K >= (1ll << 31)) return false;
  if ((long long)d->N * d->I >= (1ll << 31) || (long long)d->N * d->d >= (1ll << 31)) return false;
  if ((d->flags & ~(MOE_RENORMALIZE_GATES | MOE_FP8_ACTIVATIONS | MOE_FUSED_COMBINE)) != 0)
    return false;
  // FP8 activations are scaled per 128 channels (and need FP8 weights, whose blocks are 128).
  if ((d->flags & MOE_FP8_ACTIVATIONS) && (d->d % 128 != 0 || d->I % 128 != 0)) return false;
  return true;
}

// The FP8 weight path scales 128 x 128 blocks: both GEMMs' dims must be whole blocks.
bool fp8_dims_ok(const moe_dims &d) { return d.d % 128 == 0 && d.I % 128 == 0; }

bool fp8_act(const moe_dims &d) { return (d.flags & MOE_FP8_ACTIVATIONS) != 0; }
bool fused_combine(const moe_dims &d) { return (d.flags & MOE_FUSED_COMBINE) != 0; }
// Feature blocks of the fused combine: four per 256-feature m-tile of the down projection.
int combine_blocks(const moe_dims &d) { return 4 * ((d.d + 255) / 256); }

int router_splits(const moe_dims &d) {
  const int E = d.N + d.Z;
  const long long tiles = (long long)((d.T + 127) / 128) * ((E + 255) / 256);
  const int kblocks = d.d / 64;
  long long s = tiles > 0 ? kNominalSms / tiles : 1;
  if (s < 1) s = 1;
  if (s > 16) s = 16;
  if (s > kblocks) s = kblocks;
  return (int)s;
}

struct Layout {
  int splits;
  int epad;
  size_t status, logits, chunk, xq, sx, hq, sh, scratch_end;
  size_t topk_idx, topk_gate, gap, counts, offsets, perm_tok, perm_gate, slot_pos;
  size_t x_perm, h, y_perm, cmb_count, total;
};

Layout layout_of(const moe_dims &d) {
  Layout L{};
  const size_t T = (size_t)d.T, E = (size_t)(d.N + d.Z), K = (size_t)d.K;
  const size_t rows = T * K;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes > 0 ? bytes : 1, kAlign);
    return o;
  };
  L.splits = router_splits(d);
  L.epad = (int)align_up(E, 4);
  L.status = take(kAlign);
  L.logits = take((size_t)L.splits * T * L.epad * 4);
  L.chunk = take((size_t)dispatch_chunks(d.T) * E * 4);
  if (d.flags & MOE_FP8_ACTIVATIONS) {  // E4M3 codes and block scales of x_perm and h
    L.xq = take(rows * (size_t)d.d);
    L.sx = take(rows * (size_t)(d.d / 128) * 4);
    L.hq = take(rows * (size_t)d.I);
    L.sh = take(rows * (size_t)(d.I / 128) * 4);
  }
  L.scratch_end = off;
  L.topk_idx = take(rows * 4);
  L.topk_gate = take(rows * 4);
  L.gap = take(T * 4);
  L.counts = take(E * 4);
  L.offsets = take(((size_t)d.N + 1) * 4);
  L.perm_tok = take(rows * 4);
  L.perm_gate = take(rows * 4);
  L.slot_pos = take(rows * 4);
  L.x_perm = take(rows * (size_t)d.d * 2);
  L.h = take(rows * (size_t)d.I * 2);
  L.y_perm = take(rows * (size_t)d.d * 2);
  if (d.flags & MOE_FUSED_COMBINE) L.cmb_count = take(T * (size_t)combine_blocks(d) * 4);
  L.total = off;
  return L;
}

template <typename P>
bool aligned16(P p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

#define MOE_REQUIRE(cond, code) \
  do {                          \
    if (!(cond)) return (code); \
  } while (0)

#define MOE_CHECK_PTR(p)                      \
  do {                                        \
    MOE_REQUIRE((p) != nullptr, MOE_ERR_ARG); \
    MOE_REQUIRE(aligned16(p), MOE_ERR_ALIGN); \
  } while (0)

// Token-sized buffers may be NULL when the batch is empty (an empty tensor has no storage).
#define MOE_CHECK_TOKEN_PTR(p, T)               \
  do {                                          \
    if ((T) > 0 || (p) != nullptr) MOE_CHECK_PTR(p); \
  } while (0)

int check_ws(const void *ws, size_t ws_bytes, size_t need) {
  MOE_REQUIRE(ws != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) == 0, MOE_ERR_ALIGN);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_WORKSPACE);
  return MOE_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

int to_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------- stage bodies (checked args)
int record(void *const *events, int i, cudaStream_t stream);

int do_route(const moe_dims &d, const DeviceInfo &di, const Layout &L, const moe_bf16 *x,
             const moe_bf16 *W_r, const float *b, int32_t *topk_idx, float *topk_gate, float *gap,
             void *ws, cudaStream_t stream, void *const *events = nullptr) {
  if (d.T == 0) return record(events, 1, stream);
  const int E = d.N + d.Z;
  int *status = at<int>(ws, L.status);
  float *logits = at<float>(ws, L.logits);
  GemmArgs a{};
  const int router_tile = gemm_tile_tokens(d.T, 1, d.d);
  const bool p256 = router_tile != 256;
  if (!make_map(&a.map_a0, W_r, (uint64_t)E, (uint64_t)d.d, 128, p256) ||
      !make_map(&a.map_a1, W_r, (uint64_t)E, (uint64_t)d.d, 128, p256) ||
      !make_map(&a.map_a01, W_r, (uint64_t)E, (uint64_t)d.d, 256, p256) ||
      !make_act_maps(a, x, (uint64_t)d.T, (uint64_t)d.d, p256) ||
      !make_stream_maps(a, W_r, W_r, (uint64_t)E, (uint64_t)d.d, true)) {
    return MOE_ERR_CUDA;
  }
  a.group_offsets = nullptr;
  a.num_groups = 1;
  a.rows = d.T;
  a.M = E;
  a.K = d.d;
  a.k_splits = L.splits;
  a.out = logits;
  a.out_ld = L.epad;
  a.split_stride = (long long)d.T * L.epad;
  a.row_scale = nullptr;
  a.status = status;
  const long long tiles = (long long)((d.T + 127) / 128) * ((E + 255) / 256) * L.splits;
  const int grid = (int)(tiles < di.sms ? tiles : di.sms);
  cudaError_t e = launch_grouped_gemm(kEpiF32, a, grid, router_tile, stream);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (record(events, 1, stream) != MOE_OK) return MOE_ERR_CUDA;
  return to_status(
      launch_route_topk(logits, L.splits, d.T, E, d.K, b, (d.flags & MOE_RENORMALIZE_GATES) != 0,
                        topk_idx, topk_gate, gap, status, stream));
}

int do_dispatch(const moe_dims &d, const DeviceInfo &di, const Layout &L, const moe_bf16 *x,
                const int32_t *topk_idx, const float *topk_gate, int32_t *counts,
                int32_t *offsets, int32_t *perm_tok, float *perm_gate, int32_t *slot_pos,
                moe_bf16 *x_perm, void *ws, cudaStream_t stream) {
  return to_status(launch_dispatch(x, topk_idx, topk_gate, d.T, d.d, d.N, d.N + d.Z, d.K,
                                   at<int32_t>(ws, L.chunk), counts, offsets, perm_tok,
                                   perm_gate, slot_pos, x_perm, at<int>(ws, L.status), di.sms,
                                   stream));
}

int record(void *const *events, int i, cudaStream_t stream) {
  if (events == nullptr) return MOE_OK;
  return to_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream));
}

int do_expert_ffn(const moe_dims &d, const DeviceInfo &di, const Layout &L,
                  const moe_bf16 *x_perm, const int32_t *offsets, const float *perm_gate,
                  const moe_bf16 *W_g, const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *h,
                  moe_bf16 *y_perm, void *ws, cudaStream_t stream,
                  void *const *events = nullptr, const moe_bf16 *x = nullptr,
                  const int32_t *perm_tok = nullptr, const Fp8Weights *fw = nullptr,
                  const GemmArgs *cmb = nullptr) {
  if (d.T == 0 || d.N == 0) return record(events, 4, stream);
  const uint64_t rows = (uint64_t)d.T * d.K;
  int *status = at<int>(ws, L.status);
  GemmArgs up{};
  // Token rows: the grouped copy x_perm, or (perm_tok given) gathered from x by the GEMM.
  const bool gather = perm_tok != nullptr;
  const int tile_tokens = gemm_tile_tokens((long long)rows, d.N, d.d);
  const bool p256 = fw != nullptr || tile_tokens != 256;  // L2 promotion, see make_map
  // Wide tiles run on CTA pairs (two pipelines per pair: full and tail tiles side by side)
  // where the weight rows split into whole pair tiles; otherwise on single CTAs.
  const bool dual = fw == nullptr && !gather && tile_tokens == 256 && di.dual_pairs > 0 &&
                    d.I % 256 == 0 && d.d % 512 == 0 &&
                    gemm_dual_fits((long long)rows, d.N);
  const bool ok_w = fw != nullptr
      ? make_map_u8(&up.map_a0, fw->q_g, (uint64_t)d.N * d.I, (uint64_t)d.d) &&
            make_map_u8(&up.map_a1, fw->q_u, (uint64_t)d.N * d.I, (uint64_t)d.d) &&
            make_map_u8(&up.map_a01, fw->q_g, (uint64_t)d.N * d.I, (uint64_t)d.d)
      : make_map(&up.map_a0, W_g, (uint64_t)d.N * d.I, (uint64_t)d.d, 128, p256) &&
            make_map(&up.map_a1, W_u, (uint64_t)d.N * d.I, (uint64_t)d.d, 128, p256) &&
            make_map(&up.map_a01, W_g, (uint64_t)d.N * d.I, (uint64_t)d.d, 256, p256);
  if (!ok_w ||
      !make_act_maps(up, gather ? x : x_perm, gather ? (uint64_t)d.T : rows, (uint64_t)d.d,
                     p256) ||
      !make_stream_maps(up, W_g, W_u, (uint64_t)d.N * d.I, (uint64_t)d.d,
                        p256 || fw != nullptr)) {
    return MOE_ERR_CUDA;
  }
  up.row_index = perm_tok;
  up.gather_src = x;
  up.gather_rows = d.T;
  up.group_offsets = offsets;
  up.num_groups = d.N;
  up.rows = (int)rows;
  up.M = d.I;
  up.K = d.d;
  up.k_splits = 1;
  up.out = h;
  up.out_ld = d.I;
  up.split_stride = 0;
  up.row_scale = nullptr;
  up.status = status;
  if (fw != nullptr) {
    up.scale_a0 = fw->s_g;
    up.scale_a1 = fw->s_u;
    up.scale_ld = d.d / 128;
  }
  if ((fw != nullptr ? launch_grouped_gemm_fp8(kEpiSwiGLU, up, di.sms, stream)
       : dual        ? launch_grouped_gemm_dual(kEpiSwiGLU, up, di.dual_pairs, stream)
                     : launch_grouped_gemm(kEpiSwiGLU, up, di.sms, tile_tokens, stream)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (record(events, 4, stream) != MOE_OK) return MOE_ERR_CUDA;

  GemmArgs down{};
  const bool ok_wd = fw != nullptr
      ? make_map_u8(&down.map_a0, fw->q_d, (uint64_t)d.N * d.d, (uint64_t)d.I) &&
            make_map_u8(&down.map_a1, fw->q_d, (uint64_t)d.N * d.d, (uint64_t)d.I) &&
            make_map_u8(&down.map_a01, fw->q_d, (uint64_t)d.N * d.d, (uint64_t)d.I)
      : make_map(&down.map_a0, W_d, (uint64_t)d.N * d.d, (uint64_t)d.I, 128, p256) &&
            make_map(&down.map_a1, W_d, (uint64_t)d.N * d.d, (uint64_t)d.I, 128, p256) &&
            make_map(&down.map_a01, W_d, (uint64_t)d.N * d.d, (uint64_t)d.I, 256, p256);
  if (!ok_wd || !make_act_maps(down, h, rows, (uint64_t)d.I, p256) ||
      !make_stream_maps(down, W_d, W_d, (uint64_t)d.N * d.d, (uint64_t)d.I,
                        p256 || fw != nullptr)) {
    return MOE_ERR_CUDA;
  }
  down.group_offsets = offsets;
  down.num_groups = d.N;
  down.rows = (int)rows;
  down.M = d.d;
  down.K = d.I;
  down.k_splits = 1;
  down.out = y_perm;
  down.out_ld = d.d;
  down.split_stride = 0;
  down.row_scale = perm_gate;
  down.status = status;
  if (fw != nullptr) {
    down.scale_a0 = fw->s_d;
    down.scale_a1 = fw->s_d;
    down.scale_ld = d.I / 128;
    return to_status(launch_grouped_gemm_fp8(kEpiGated, down, di.sms, stream));
  }
  if (cmb != nullptr) {  // the combine fused into the down projection (single CTAs)
    down.cmb_x = cmb->cmb_x;
    down.cmb_perm_tok = cmb->cmb_perm_tok;
    down.cmb_idx = cmb->cmb_idx;
    down.cmb_gate = cmb->cmb_gate;
    down.cmb_slot = cmb->cmb_slot;
    down.cmb_count = cmb->cmb_count;
    down.cmb_y = cmb->cmb_y;
    down.cmb_K = cmb->cmb_K;
    down.cmb_N = cmb->cmb_N;
    down.cmb_blocks = cmb->cmb_blocks;
    if (launch_combine_counters(down.cmb_idx, d.T, d.K, d.N, down.cmb_blocks, down.cmb_count,
                                stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return to_status(launch_grouped_gemm(kEpiGatedCombine, down, di.sms, tile_tokens, stream));
  }
  if (dual) return to_status(launch_grouped_gemm_dual(kEpiGated, down, di.dual_pairs, stream));
  return to_status(launch_grouped_gemm(kEpiGated, down, di.sms, tile_tokens, stream));
}

// The expert FFN with FP8 weights and FP8 activations: x_perm's rows are quantised (1 x 128
// blocks) into the workspace, the up-projection reads the codes on the tensor cores and writes
// h as codes and scales, and the down projection reads those.
// x_perm NULL: the token rows are quantised straight from x through perm_tok (no bf16 copy).
int do_expert_ffn_e4m3(const moe_dims &d, const DeviceInfo &di, const Layout &L,
                       const moe_bf16 *x_perm, const int32_t *offsets, const float *perm_gate,
                       const Fp8Weights &fw, moe_bf16 *y_perm, void *ws, cudaStream_t stream,
                       void *const *events = nullptr, const moe_bf16 *x = nullptr,
                       const int32_t *perm_tok = nullptr) {
  if (d.T == 0 || d.N == 0) return record(events, 4, stream);
  const uint64_t rows = (uint64_t)d.T * d.K;
  int *status = at<int>(ws, L.status);
  uint8_t *xq = at<uint8_t>(ws, L.xq);
  float *sx = at<float>(ws, L.sx);
  uint8_t *hq = at<uint8_t>(ws, L.hq);
  float *sh = at<float>(ws, L.sh);
  // Only the rows of the FFN experts' groups (offsets[N] of them) are quantised.
  const cudaError_t qe =
      x_perm != nullptr
          ? launch_quantize_fp8_rows(x_perm, (long long)rows, d.d, offsets + d.N, xq, sx, stream)
          : launch_quantize_fp8_rows(x, (long long)rows, d.d, offsets + d.N, xq, sx, stream,
                                     perm_tok, d.T, status);
  if (qe != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs up{};
  bool ok = make_map_e4m3(&up.map_a0, fw.q_g, (uint64_t)d.N * d.I, (uint64_t)d.d, 128) &&
            make_map_e4m3(&up.map_a1, fw.q_u, (uint64_t)d.N * d.I, (uint64_t)d.d, 128);
  for (int i = 1; i < 4 && ok; ++i)
    ok = make_map_e4m3(&up.map_b[i], xq, rows, (uint64_t)d.d, 128u >> i);
  if (!ok) return MOE_ERR_CUDA;
  up.group_offsets = offsets;
  up.num_groups = d.N;
  up.rows = (int)rows;
  up.M = d.I;
  up.K = d.d;
  up.k_splits = 1;
  up.out = hq;
  up.out_ld = d.I;
  up.status = status;
  up.scale_a0 = fw.s_g;
  up.scale_a1 = fw.s_u;
  up.scale_ld = d.d / 128;
  up.act_scale = sx;
  up.out_scale = sh;
  if (launch_grouped_gemm_e4m3(kEpiSwiGLU, up, di.sms, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (record(events, 4, stream) != MOE_OK) return MOE_ERR_CUDA;

  GemmArgs down{};
  ok = make_map_e4m3(&down.map_a0, fw.q_d, (uint64_t)d.N * d.d, (uint64_t)d.I, 128) &&
       make_map_e4m3(&down.map_a1, fw.q_d, (uint64_t)d.N * d.d, (uint64_t)d.I, 128);
  for (int i = 1; i < 4 && ok; ++i)
    ok = make_map_e4m3(&down.map_b[i], hq, rows, (uint64_t)d.I, 128u >> i);
  if (!ok) return MOE_ERR_CUDA;
  down.group_offsets = offsets;
  down.num_groups = d.N;
  down.rows = (int)rows;
  down.M = d.d;
  down.K = d.I;
  down.k_splits = 1;
  down.out = y_perm;
  down.out_ld = d.d;
  down.row_scale = perm_gate;
  down.status = status;
  down.scale_a0 = fw.s_d;
  down.scale_a1 = fw.s_d;
  down.scale_ld = d.I / 128;
  down.act_scale = sh;
  return to_status(launch_grouped_gemm_e4m3(kEpiGated, down, di.sms, stream));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument (NULL pointer or bad parameter)";
    case MOE_ERR_SHAPE: return "unsupported dims (see the limits in moe.h)";
    case MOE_ERR_ALIGN: return "pointer not aligned (16 bytes for tensors, 256 for workspaces)";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime or launch error";
    case MOE_ERR_DEVICE: return "device-side check failed";
    case MOE_ERR_ARCH: return "current device is not sm_100 (B200 class)";
    default: return "unknown error code";
  }
}

size_t moe_workspace_size(const moe_dims *dims) {
  if (!dims_ok(dims)) return 0;
  return layout_of(*dims).total;
}

size_t moe_scratch_size(const moe_dims *dims) {
  if (!dims_ok(dims)) return 0;
  return layout_of(*dims).scratch_end;
}

int moe_route(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r, const float *b,
              int32_t *topk_idx, float *topk_gate, float *gap, void *ws, size_t ws_bytes,
              void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(x, dims->T);
  MOE_CHECK_PTR(W_r);
  MOE_CHECK_PTR(b);
  MOE_CHECK_TOKEN_PTR(topk_idx, dims->T);
  MOE_CHECK_TOKEN_PTR(topk_gate, dims->T);
  if (gap != nullptr) MOE_REQUIRE(aligned16(gap), MOE_ERR_ALIGN);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return do_route(*dims, *di, L, x, W_r, b, topk_idx, topk_gate, gap, ws,
                  static_cast<cudaStream_t>(stream));
}

int moe_dispatch(const moe_dims *dims, const moe_bf16 *x, const int32_t *topk_idx,
                 const float *topk_gate, int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                 float *perm_gate, int32_t *slot_pos, moe_bf16 *x_perm, void *ws,
                 size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(x, dims->T);
  MOE_CHECK_TOKEN_PTR(topk_idx, dims->T);
  MOE_CHECK_TOKEN_PTR(topk_gate, dims->T);
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(offsets);
  MOE_CHECK_TOKEN_PTR(perm_tok, dims->T);
  MOE_CHECK_TOKEN_PTR(perm_gate, dims->T);
  MOE_CHECK_TOKEN_PTR(slot_pos, dims->T);
  if (x_perm != nullptr) MOE_REQUIRE(aligned16(x_perm), MOE_ERR_ALIGN);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return do_dispatch(*dims, *di, L, x, topk_idx, topk_gate, counts, offsets, perm_tok,
                     perm_gate, slot_pos, x_perm, ws, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn(const moe_dims *dims, const moe_bf16 *x_perm, const int32_t *offsets,
                   const float *perm_gate, const moe_bf16 *W_g, const moe_bf16 *W_u,
                   const moe_bf16 *W_d, moe_bf16 *h, moe_bf16 *y_perm, void *ws,
                   size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_REQUIRE(!fp8_act(*dims), MOE_ERR_ARG);  // FP8 activations need FP8 weights
  MOE_REQUIRE(!fused_combine(*dims), MOE_ERR_ARG);  // moe_forward only
  MOE_CHECK_TOKEN_PTR(x_perm, dims->T);
  MOE_CHECK_PTR(offsets);
  MOE_CHECK_TOKEN_PTR(perm_gate, dims->T);
  MOE_CHECK_PTR(W_g);
  MOE_CHECK_PTR(W_u);
  MOE_CHECK_PTR(W_d);
  MOE_CHECK_TOKEN_PTR(h, dims->T);
  MOE_CHECK_TOKEN_PTR(y_perm, dims->T);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return do_expert_ffn(*dims, *di, L, x_perm, offsets, perm_gate, W_g, W_u, W_d, h, y_perm, ws,
                       static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_gather(const moe_dims *dims, const moe_bf16 *x, const int32_t *perm_tok,
                          const int32_t *offsets, const float *perm_gate, const moe_bf16 *W_g,
                          const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *h,
                          moe_bf16 *y_perm, void *ws, size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_REQUIRE(!fp8_act(*dims) && !fused_combine(*dims), MOE_ERR_ARG);
  MOE_CHECK_TOKEN_PTR(x, dims->T);
  MOE_CHECK_TOKEN_PTR(perm_tok, dims->T);
  MOE_CHECK_PTR(offsets);
  MOE_CHECK_TOKEN_PTR(perm_gate, dims->T);
  MOE_CHECK_PTR(W_g);
  MOE_CHECK_PTR(W_u);
  MOE_CHECK_PTR(W_d);
  MOE_CHECK_TOKEN_PTR(h, dims->T);
  MOE_CHECK_TOKEN_PTR(y_perm, dims->T);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return do_expert_ffn(*dims, *di, L, nullptr, offsets, perm_gate, W_g, W_u, W_d, h, y_perm, ws,
                       static_cast<cudaStream_t>(stream), nullptr, x, perm_tok);
}

int moe_dense_ffn(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_g,
                  const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *h, moe_bf16 *y, void *ws,
                  size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  const moe_dims &d = *dims;
  MOE_REQUIRE(d.T >= 0 && d.d > 0 && d.d % 64 == 0 && d.I > 0 && d.I % 64 == 0 &&
                  (long long)d.T * d.I < (1ll << 31) && (long long)d.T * d.d < (1ll << 31),
              MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(x, d.T);
  MOE_CHECK_PTR(W_g);
  MOE_CHECK_PTR(W_u);
  MOE_CHECK_PTR(W_d);
  MOE_CHECK_TOKEN_PTR(h, d.T);
  MOE_CHECK_TOKEN_PTR(y, d.T);
  int rc = check_ws(ws, ws_bytes, kAlign);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  if (d.T == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int *status = at<int>(ws, 0);
  // One group of all T rows through the same grouped GEMMs as the experts (gate 1).
  const int tile_tokens = gemm_tile_tokens(d.T, 1, d.d);
  const bool p256 = tile_tokens != 256;
  GemmArgs up{};
  if (!make_map(&up.map_a0, W_g, (uint64_t)d.I, (uint64_t)d.d, 128, p256) ||
      !make_map(&up.map_a1, W_u, (uint64_t)d.I, (uint64_t)d.d, 128, p256) ||
      !make_map(&up.map_a01, W_g, (uint64_t)d.I, (uint64_t)d.d, 256, p256) ||
      !make_act_maps(up, x, (uint64_t)d.T, (uint64_t)d.d, p256) ||
      !make_stream_maps(up, W_g, W_u, (uint64_t)d.I, (uint64_t)d.d, true)) {
    return MOE_ERR_CUDA;
  }
  up.group_offsets = nullptr;
  up.num_groups = 1;
  up.rows = d.T;
  up.M = d.I;
  up.K = d.d;
  up.k_splits = 1;
  up.out = h;
  up.out_ld = d.I;
  up.status = status;
  if (launch_grouped_gemm(kEpiSwiGLU, up, di->sms, tile_tokens, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  GemmArgs down{};
  if (!make_map(&down.map_a0, W_d, (uint64_t)d.d, (uint64_t)d.I, 128, p256) ||
      !make_map(&down.map_a1, W_d, (uint64_t)d.d, (uint64_t)d.I, 128, p256) ||
      !make_map(&down.map_a01, W_d, (uint64_t)d.d, (uint64_t)d.I, 256, p256) ||
      !make_act_maps(down, h, (uint64_t)d.T, (uint64_t)d.I, p256) ||
      !make_stream_maps(down, W_d, W_d, (uint64_t)d.d, (uint64_t)d.I, true)) {
    return MOE_ERR_CUDA;
  }
  down.group_offsets = nullptr;
  down.num_groups = 1;
  down.rows = d.T;
  down.M = d.d;
  down.K = d.I;
  down.k_splits = 1;
  down.out = y;
  down.out_ld = d.d;
  down.row_scale = nullptr;  // gate 1
  down.status = status;
  return to_status(launch_grouped_gemm(kEpiGated, down, di->sms, tile_tokens, s));
}

int moe_combine(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *y_perm,
                const int32_t *topk_idx, const float *topk_gate, const int32_t *slot_pos,
                moe_bf16 *y, void *ws, size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(x, dims->T);
  MOE_CHECK_TOKEN_PTR(y_perm, dims->T);
  MOE_CHECK_TOKEN_PTR(topk_idx, dims->T);
  MOE_CHECK_TOKEN_PTR(topk_gate, dims->T);
  MOE_CHECK_TOKEN_PTR(slot_pos, dims->T);
  MOE_CHECK_TOKEN_PTR(y, dims->T);
  int rc = check_ws(ws, ws_bytes, kAlign);  // the status word only
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return to_status(launch_combine(x, y_perm, topk_idx, topk_gate, slot_pos, dims->T, dims->d,
                                  dims->N, dims->K, dims->T * dims->K, y, at<int>(ws, 0),
                                  static_cast<cudaStream_t>(stream)));
}

int moe_router_logits(const moe_dims *dims, const void *ws, size_t ws_bytes, float *logits,
                      void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(logits, dims->T);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return to_status(launch_router_logits(at<float>(const_cast<void *>(ws), L.logits), L.splits,
                                        dims->T, dims->N + dims->Z, logits, di->sms,
                                        static_cast<cudaStream_t>(stream)));
}

int moe_debug_set_wait_limit(int64_t cycles) {
  MOE_REQUIRE(cycles >= 0, MOE_ERR_ARG);
  gemm_set_wait_limit((long long)cycles);
  return MOE_OK;
}

int moe_bias_update(const moe_dims *dims, const int32_t *counts, float *b, float *pid_state,
                    const moe_pid_params *params, void *stream) {
  MOE_REQUIRE(dims != nullptr && params != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(b);
  MOE_CHECK_PTR(pid_state);
  MOE_REQUIRE(std::isfinite(params->balance_gamma), MOE_ERR_ARG);
  const DeviceInfo *di = nullptr;
  const int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return to_status(launch_pid(counts, dims->N, dims->K, dims->T, b, pid_state, params->target,
                              params->kp, params->ki, params->kd, params->balance_gamma,
                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

int forward_impl(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r, const float *b,
                 const moe_bf16 *W_g, const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *y,
                 int32_t *counts, void *ws, size_t ws_bytes, void *const *ev, void *stream,
                 const Fp8Weights *fw = nullptr) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims), MOE_ERR_SHAPE);
  MOE_CHECK_TOKEN_PTR(x, dims->T);
  MOE_CHECK_PTR(W_r);
  MOE_CHECK_PTR(b);
  if (fw == nullptr) {
    MOE_REQUIRE(!fp8_act(*dims), MOE_ERR_ARG);  // FP8 activations need FP8 weights
    MOE_CHECK_PTR(W_g);
    MOE_CHECK_PTR(W_u);
    MOE_CHECK_PTR(W_d);
  } else {
    MOE_REQUIRE(fp8_dims_ok(*dims), MOE_ERR_SHAPE);
    MOE_REQUIRE(!fused_combine(*dims), MOE_ERR_ARG);  // bf16 weights only
    MOE_CHECK_PTR(fw->q_g);
    MOE_CHECK_PTR(fw->q_u);
    MOE_CHECK_PTR(fw->q_d);
    MOE_CHECK_PTR(fw->s_g);
    MOE_CHECK_PTR(fw->s_u);
    MOE_CHECK_PTR(fw->s_d);
  }
  MOE_CHECK_TOKEN_PTR(y, dims->T);
  if (counts != nullptr) MOE_REQUIRE(aligned16(counts), MOE_ERR_ALIGN);
  if (ev != nullptr)
    for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i) MOE_REQUIRE(ev[i] != nullptr, MOE_ERR_ARG);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.total);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const moe_dims &d = *dims;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t *cnt = counts != nullptr ? counts : at<int32_t>(ws, L.counts);
  int32_t *topk_idx = at<int32_t>(ws, L.topk_idx);
  float *topk_gate = at<float>(ws, L.topk_gate);
  int32_t *offsets = at<int32_t>(ws, L.offsets);
  int32_t *perm_tok = at<int32_t>(ws, L.perm_tok);
  float *perm_gate = at<float>(ws, L.perm_gate);
  int32_t *slot_pos = at<int32_t>(ws, L.slot_pos);
  moe_bf16 *x_perm = at<moe_bf16>(ws, L.x_perm);
  moe_bf16 *h = at<moe_bf16>(ws, L.h);
  moe_bf16 *y_perm = at<moe_bf16>(ws, L.y_perm);
  if ((rc = record(ev, 0, s)) != MOE_OK) return rc;
  rc = do_route(d, *di, L, x, W_r, b, topk_idx, topk_gate, at<float>(ws, L.gap), ws, s, ev);
  if (rc != MOE_OK) return rc;
  if ((rc = record(ev, 2, s)) != MOE_OK) return rc;
  // The gathered copy x_perm and tiled token loads: faster at large T than gathering rows
  // inside the up-projection (moe_expert_ffn_gather), whose row-by-row copies cost more.
  // With FP8 activations the up-projection's quantiser reads the token rows from x itself.
  const bool fp8_rows = fw != nullptr && fp8_act(d);
  rc = do_dispatch(d, *di, L, x, topk_idx, topk_gate, cnt, offsets, perm_tok, perm_gate,
                   slot_pos, fp8_rows ? nullptr : x_perm, ws, s);
  if (rc != MOE_OK) return rc;
  if ((rc = record(ev, 3, s)) != MOE_OK) return rc;
  GemmArgs cmb{};
  if (fused_combine(d)) {
    cmb.cmb_x = x;
    cmb.cmb_perm_tok = perm_tok;
    cmb.cmb_idx = topk_idx;
    cmb.cmb_gate = topk_gate;
    cmb.cmb_slot = slot_pos;
    cmb.cmb_count = at<int>(ws, L.cmb_count);
    cmb.cmb_y = y;
    cmb.cmb_K = d.K;
    cmb.cmb_N = d.N;
    cmb.cmb_blocks = combine_blocks(d);
  }
  rc = fp8_rows
           ? do_expert_ffn_e4m3(d, *di, L, nullptr, offsets, perm_gate, *fw, y_perm, ws, s, ev,
                                x, perm_tok)
           : do_expert_ffn(d, *di, L, x_perm, offsets, perm_gate, W_g, W_u, W_d, h, y_perm, ws,
                           s, ev, nullptr, nullptr, fw, fused_combine(d) ? &cmb : nullptr);
  if (rc != MOE_OK) return rc;
  if ((rc = record(ev, 5, s)) != MOE_OK) return rc;
  // With the fused combine only tokens without an FFN slot are left (the zero-only pass).
  rc = to_status(launch_combine(x, y_perm, topk_idx, topk_gate, slot_pos, d.T, d.d, d.N, d.K,
                                d.T * d.K, y, at<int>(ws, L.status), s, fused_combine(d)));
  if (rc != MOE_OK) return rc;
  return record(ev, 6, s);
}

}  // namespace

extern "C" {

int moe_forward(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r, const float *b,
                const moe_bf16 *W_g, const moe_bf16 *W_u, const moe_bf16 *W_d, moe_bf16 *y,
                int32_t *counts, void *ws, size_t ws_bytes, void *stream) {
  return forward_impl(dims, x, W_r, b, W_g, W_u, W_d, y, counts, ws, ws_bytes, nullptr, stream);
}

int moe_forward_timed(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r,
                      const float *b, const moe_bf16 *W_g, const moe_bf16 *W_u,
                      const moe_bf16 *W_d, moe_bf16 *y, int32_t *counts, void *ws,
                      size_t ws_bytes, void *const *stage_events, void *stream) {
  MOE_REQUIRE(stage_events != nullptr, MOE_ERR_ARG);
  return forward_impl(dims, x, W_r, b, W_g, W_u, W_d, y, counts, ws, ws_bytes, stage_events,
                      stream);
}

int moe_quantize_fp8(const moe_bf16 *w, int64_t G, int64_t R, int64_t C, uint8_t *q,
                     float *scale, void *stream) {
  MOE_REQUIRE(G >= 0 && R >= 0 && C >= 0 && R % 128 == 0 && C % 128 == 0, MOE_ERR_SHAPE);
  MOE_REQUIRE(G < (1ll << 31) && R < (1ll << 31) && C < (1ll << 31), MOE_ERR_SHAPE);
  // one CTA per 128 x 128 block: the block count must fit a grid dimension
  MOE_REQUIRE(G == 0 || R == 0 || C == 0 ||
                  (R / 128) * (C / 128) <= ((1ll << 31) - 1) / G,
              MOE_ERR_SHAPE);
  if (G == 0 || R == 0 || C == 0) return MOE_OK;
  MOE_CHECK_PTR(w);
  MOE_CHECK_PTR(q);
  MOE_CHECK_PTR(scale);
  const DeviceInfo *di = nullptr;
  const int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return to_status(launch_quantize_fp8(w, G, R, C, q, scale, static_cast<cudaStream_t>(stream)));
}

int moe_quantize_fp8_rows(const moe_bf16 *x, int64_t R, int64_t C, uint8_t *q, float *scale,
                          void *stream) {
  MOE_REQUIRE(R >= 0 && C >= 0 && C % 128 == 0 && C < (1ll << 31), MOE_ERR_SHAPE);
  MOE_REQUIRE(R <= ((1ll << 31) - 1) * 8 / std::max<int64_t>(1, (C / 128 + 1) / 2), MOE_ERR_SHAPE);
  if (R == 0 || C == 0) return MOE_OK;
  MOE_CHECK_PTR(x);
  MOE_CHECK_PTR(q);
  MOE_CHECK_PTR(scale);
  const DeviceInfo *di = nullptr;
  const int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  return to_status(launch_quantize_fp8_rows(x, R, (int)C, nullptr, q, scale,
                                            static_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn_fp8(const moe_dims *dims, const moe_bf16 *x_perm, const int32_t *offsets,
                       const float *perm_gate, const uint8_t *q_g, const float *s_g,
                       const uint8_t *q_u, const float *s_u, const uint8_t *q_d,
                       const float *s_d, moe_bf16 *h, moe_bf16 *y_perm, void *ws,
                       size_t ws_bytes, void *stream) {
  MOE_REQUIRE(dims != nullptr, MOE_ERR_ARG);
  MOE_REQUIRE(dims_ok(dims) && fp8_dims_ok(*dims), MOE_ERR_SHAPE);
  MOE_REQUIRE(!fused_combine(*dims), MOE_ERR_ARG);  // moe_forward only
  MOE_CHECK_TOKEN_PTR(x_perm, dims->T);
  MOE_CHECK_PTR(offsets);
  MOE_CHECK_TOKEN_PTR(perm_gate, dims->T);
  const Fp8Weights fw{q_g, q_u, q_d, s_g, s_u, s_d};
  MOE_CHECK_PTR(q_g);
  MOE_CHECK_PTR(q_u);
  MOE_CHECK_PTR(q_d);
  MOE_CHECK_PTR(s_g);
  MOE_CHECK_PTR(s_u);
  MOE_CHECK_PTR(s_d);
  if (!fp8_act(*dims)) MOE_CHECK_TOKEN_PTR(h, dims->T);  // unused with FP8 activations
  MOE_CHECK_TOKEN_PTR(y_perm, dims->T);
  const Layout L = layout_of(*dims);
  int rc = check_ws(ws, ws_bytes, L.scratch_end);
  if (rc != MOE_OK) return rc;
  const DeviceInfo *di = nullptr;
  rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  if (fp8_act(*dims))
    return do_expert_ffn_e4m3(*dims, *di, L, x_perm, offsets, perm_gate, fw, y_perm, ws,
                              static_cast<cudaStream_t>(stream));
  return do_expert_ffn(*dims, *di, L, x_perm, offsets, perm_gate, nullptr, nullptr, nullptr, h,
                       y_perm, ws, static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr,
                       &fw);
}

int moe_forward_fp8(const moe_dims *dims, const moe_bf16 *x, const moe_bf16 *W_r,
                    const float *b, const uint8_t *q_g, const float *s_g, const uint8_t *q_u,
                    const float *s_u, const uint8_t *q_d, const float *s_d, moe_bf16 *y,
                    int32_t *counts, void *ws, size_t ws_bytes, void *const *stage_events,
                    void *stream) {
  const Fp8Weights fw{q_g, q_u, q_d, s_g, s_u, s_d};
  return forward_impl(dims, x, W_r, b, nullptr, nullptr, nullptr, y, counts, ws, ws_bytes,
                      stage_events, stream, &fw);
}

int moe_last_device_error(void *ws, void *stream) {
  if (ws == nullptr) return MOE_ERR_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return -1;
  int code = 0;
  int *status = at<int>(ws, 0);
  if (cudaMemcpy(&code, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  if (code != 0 && cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return -1;
  return code;
}

}  // extern "C"
