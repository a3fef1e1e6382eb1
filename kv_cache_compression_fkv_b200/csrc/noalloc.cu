// fkv_score_segments_noalloc: segment scoring for callers that cannot
// allocate device memory.
//
// Some callers of this library never get to call cudaMalloc: a plugin run by
// a host inference runtime is handed only its input and output buffers (the
// runtime owns every byte of HBM and offers no workspace hook), and serving
// loops that reserve nearly all of HBM for their own KV pool up front must
// not allocate later, because an extra allocation can fail or stall the
// device.  fkv_score_segments needs a caller-provided workspace for its
// per-frame partial softmax statistics; this variant keeps that scratch in a
// fixed-size array that is part of the library's device image instead.
//
// The array is static: every GPU that loads the library holds its
// kNoAllocScratchBytes until the process exits, and all calls on a device
// share it.  Host code must not hand `g_noalloc_scratch` to a kernel -- on the
// host that name is only a stand-in, not a device address -- so the device
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) on the first call there, and cached.
#include <mutex>
#include <stdio.h>

#include "fkv_internal.cuh"

namespace fkv {

// Scratch bound: covers the 480P single-layer workload (about 6.6 MB of
// per-block partial statistics) and any token-mode call with up to 32768
// (layer, head) pairs; larger frame-mode calls (1080P, the 30-layer batch)
// need a workspace.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, or nullptr.
void* scratch_address(int32_t* st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fprintf(stderr, "fkv_score_segments_noalloc: no usable current device (%s)\n",
            cudaGetErrorString(e));
    *st = FKV_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      fprintf(stderr, "fkv_score_segments_noalloc: cudaGetSymbolAddress failed on device %d (%s)\n",
              dev, cudaGetErrorString(e));
      *st = FKV_ERR_CUDA;
      return nullptr;
    }
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}
}  // namespace

}  // namespace fkv

extern "C" int32_t fkv_score_segments_noalloc(const fkv_params_t* p, const void* q_cur,
                                              const void* q_score, const void* k_hist,
                                              const void* k_cur, const uint8_t* head_role,
                                              float* seg_score, void* stream) {
  int32_t st = fkv_check_params(p);
  if (st != FKV_OK) return st;
  size_t need = 0;
  st = fkv_workspace_size(p, &need);
  if (st != FKV_OK) return st;
  if (need > fkv::kNoAllocScratchBytes) {
    fprintf(stderr,
            "fkv_score_segments_noalloc: these sizes need %zu bytes of scratch, above the static "
            "maximum of %zu bytes; use fkv_score_segments with a workspace\n",
            need, fkv::kNoAllocScratchBytes);
    return FKV_ERR_WORKSPACE;
  }
  void* scratch = fkv::scratch_address(&st);
  if (!scratch) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The status block at the start of the scratch is cleared on every call, so
  // that a failure recorded by an earlier call does not mark this one; the
  // partial statistics after it are fully written before they are read.
  cudaError_t e = cudaMemsetAsync(scratch, 0, 256, s);
  if (e != cudaSuccess) {
    fprintf(stderr, "fkv_score_segments_noalloc: %s\n", cudaGetErrorString(e));
    return FKV_ERR_CUDA;
  }
  // Same validation and kernels as fkv_score_segments, with the static array
  // (256-byte aligned, large enough as checked above) as the workspace.  The
  // caller has no status word to read, so a device-side failure of the
  // scoring (a bounded wait that gave up) turns the dynamic heads' scores
  // into NaN instead of leaving stale values behind.
  return fkv::score_segments_checked(p, q_cur, q_score, k_hist, k_cur, head_role, seg_score,
                                     scratch, stream, true);
}
