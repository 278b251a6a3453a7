// noalloc.cu -- moe_dispatch_noalloc: the dispatch stage for callers that cannot give the
// library any device memory of its own.
//
// moe_dispatch needs a little scratch (one histogram row of N+Z counters per chunk of 256
// tokens), which every other entry point takes from a caller-provided workspace.  Some callers
// have no way to provide one: a plugin inside a host process that owns every byte of device
// memory through its own pool and gives plugins none, or a deployment with a fixed memory
// budget where no extra cudaMalloc may happen after start-up.  For them this variant keeps its
// scratch in a fixed array that is part of the library image itself: it exists on every GPU
// that loads the library and stays there until the process exits, whether used or not.
//
// Limits and behaviour:
//   - scratch capacity kNoAllocScratchInts int32 (1 MiB); a call needs ceil(T/256) * (N+Z) of
//     them (e.g. N+Z = 768 allows T <= 87,296) and larger requests return MOE_ERR_WORKSPACE;
//   - the array is shared by every call on a device and keeps the last call's contents; the
//     histogram kernel overwrites every entry a call reads before reading it, so nothing needs
//     clearing; two calls whose kernels overlap on the GPU (different streams) race on it;
//   - device-side checks (an expert id out of range) still skip the bad access but have no
//     status word to report to;
//   - the first call on each device looks up the array's device address (once, with that
//     device current) and checks the GPU is sm_100; make that first call before any stream
//     capture.  No call allocates or frees memory.
#include <mutex>

#include "kernels.cuh"
#include "../../include/moe.h"

constexpr size_t kNoAllocScratchInts = 262144;  // 1 MiB

// The scratch itself: one copy per device, part of the loaded library image.
static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchInts];

namespace moe {
namespace {

constexpr int kNoAllocMaxDevices = 64;

struct NoAllocDevice {
  bool ready = false;
  int status = MOE_OK;
  int sms = 0;
  int32_t *scratch = nullptr;  // device address of g_dispatch_scratch on this device
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

// Once per device, with that device current: architecture check, SM count, and the device
// address of the scratch array (the host-side name is only a stand-in for it).
int noalloc_device(const NoAllocDevice **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice &nd = g_noalloc_dev[dev];
  if (!nd.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      return MOE_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
      nd.status = MOE_ERR_ARCH;
    } else {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr)
        return MOE_ERR_CUDA;
      nd.scratch = static_cast<int32_t *>(p);
      nd.status = MOE_OK;
    }
    nd.sms = sms;
    nd.ready = true;
  }
  *out = &nd;
  return nd.status;
}

bool ok16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" int moe_dispatch_noalloc(const moe_dims *dims, const moe_bf16 *x,
                                    const int32_t *topk_idx, const float *topk_gate,
                                    int32_t *counts, int32_t *offsets, int32_t *perm_tok,
                                    float *perm_gate, int32_t *slot_pos, moe_bf16 *x_perm,
                                    void *stream) {
  using namespace moe;
  if (dims == nullptr) return MOE_ERR_ARG;
  if (moe_scratch_size(dims) == 0) return MOE_ERR_SHAPE;  // same limits as every entry point
  const int T = dims->T;
  const void *token_bufs[] = {x, topk_idx, topk_gate, perm_tok, perm_gate, slot_pos};
  for (const void *p : token_bufs) {
    if (T > 0 && p == nullptr) return MOE_ERR_ARG;
    if (p != nullptr && !ok16(p)) return MOE_ERR_ALIGN;
  }
  // As in moe_dispatch, a NULL x_perm skips the row copy (for moe_expert_ffn_gather).
  if (x_perm != nullptr && !ok16(x_perm)) return MOE_ERR_ALIGN;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_ARG;
  if (!ok16(counts) || !ok16(offsets)) return MOE_ERR_ALIGN;
  const int E = dims->N + dims->Z;
  if ((size_t)dispatch_chunks(T) * (size_t)E > kNoAllocScratchInts) return MOE_ERR_WORKSPACE;
  const NoAllocDevice *nd = nullptr;
  const int rc = noalloc_device(&nd);
  if (rc != MOE_OK) return rc;
  const cudaError_t e = launch_dispatch(x, topk_idx, topk_gate, T, dims->d, dims->N, E,
                                        dims->K, nd->scratch, counts, offsets, perm_tok,
                                        perm_gate, slot_pos, x_perm, nullptr, nd->sms,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
