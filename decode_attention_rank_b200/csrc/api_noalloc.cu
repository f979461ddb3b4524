// Decode attention for callers that cannot allocate device memory: the same
// kernels as starkv_decode_attn, with their scratch in a fixed device array of
// this library instead of a caller workspace.
#include <limits.h>

#include <mutex>
#include <string>

#include "starkv_internal.cuh"

namespace starkv {

// One array per device that loads the library, alive until process exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[STARKV_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace starkv

using namespace starkv;

extern "C" starkv_status starkv_decode_attn_noalloc(const starkv_layer* L, const void* pool, int64_t n_pages,
                                                    const int32_t* page_table, int max_pages, int batch,
                                                    const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                                                    void* out, starkv_stream_t stream) {
  set_error("");
  if (L == nullptr) {
    set_error("layer is NULL");
    return STARKV_ERR_ARG;
  }
  if (batch < 0) {
    set_error("negative batch");
    return STARKV_ERR_ARG;
  }
  if (batch == 0) return STARKV_OK;
  if (!(pool && page_table && seq_lens && q && out) || n_pages <= 0 || max_pages <= 0) {
    set_error("NULL buffer or empty pool / page table");
    return STARKV_ERR_ARG;
  }
  if (max_pages > INT_MAX / kPage) {
    set_error("max_pages * 16 overflows int");
    return STARKV_ERR_ARG;
  }
  // the alignment rules of starkv_decode_attn, checked before the scratch lookup
  if ((((uintptr_t)pool | (uintptr_t)q | (uintptr_t)out) & 15) != 0 ||
      (((uintptr_t)page_table | (uintptr_t)seq_lens | (uintptr_t)q_pos) & 3) != 0) {
    set_error("pool, q and out must be 16-byte aligned, page_table, seq_lens and q_pos 4-byte aligned");
    return STARKV_ERR_ARG;
  }
  const size_t need = starkv_workspace_bytes(L, batch, max_pages * kPage, 1);
  if (need > STARKV_NOALLOC_SCRATCH_BYTES) {
    set_error("decode needs " + std::to_string(need) + " bytes of scratch; the built-in array holds " +
              std::to_string((size_t)STARKV_NOALLOC_SCRATCH_BYTES) + " (use starkv_decode_attn with a workspace)");
    return STARKV_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    set_error(std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    return STARKV_ERR_CUDA;
  }
  return starkv_decode_attn(L, pool, n_pages, page_table, max_pages, batch, seq_lens, q_pos, q, out, scratch,
                            STARKV_NOALLOC_SCRATCH_BYTES, stream);
}
