// noalloc.cu -- mf_block_fwd_noalloc: the block forward for callers that cannot
// allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a plugin that runs inside
// a host application which owns all device memory and hands its plugins no
// allocator, or a caller on a latency-critical path that must not make a call
// which can synchronise the device. Such callers cannot supply the workspace
// mf_block_fwd needs for its fused RoPE (the (cos, sin) table and the rotated
// k). This entry point takes that workspace from a file-scope device array
// instead, so the caller passes only inputs and outputs.
//
// The array is part of the library's device image: every GPU that loads the
// library holds MF_NOALLOC_SCRATCH_BYTES for it until the process exits. Every
// call shares it and it keeps the last call's contents; nothing in it needs to
// start at zero (each call rewrites all of the table and rotated k it reads).
// Calls that overlap on the GPU (on different streams, or from different host
// threads) race on the array and must be serialised by the caller.
#include <cuda_runtime_api.h>

#include <mutex>

#include "mf.h"
#include "mf_internal.h"

namespace mf {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[MF_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of the array on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up once per
// device, with that device current, and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace mf

extern "C" mf_status mf_block_fwd_noalloc(
    const mf_bf16* x, const mf_bf16* q, const mf_bf16* k, const mf_bf16* v, const float* mod,
    const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h, const int32_t* pos_ids,
    const int32_t* tok_sample, const uint8_t* tok_mod, int32_t S, int32_t H, int32_t D,
    int32_t rope_axes, float base, float eps, mf_bf16* x_mod, mf_bf16* y, cudaStream_t stream) {
  if (cu_seqlens_h == nullptr || S < 1 || S > MF_MAX_SAMPLES || H < 1 || D < 1)
    return MF_ERR_INVALID;
  // a malformed pack is an argument error whatever its size
  int32_t T = 0;
  if (!mf::check_offsets(cu_seqlens_h, S, &T)) return MF_ERR_INVALID;
  const size_t need = mf_workspace_size(T, H, D, 1);
  if (need > MF_NOALLOC_SCRATCH_BYTES) return MF_ERR_UNSUPPORTED;  // pack too large
  void* scratch = nullptr;
  if (mf::scratch_address(&scratch) != cudaSuccess) return MF_ERR_CUDA;
  return mf_block_fwd(x, q, k, v, mod, cu_seqlens_d, cu_seqlens_h, pos_ids, tok_sample, tok_mod,
                      S, H, D, rope_axes, base, eps, x_mod, y, scratch, MF_NOALLOC_SCRATCH_BYTES,
                      stream);
}
