// Decode step for callers that cannot allocate device memory.
//
// palu_decode_attn needs a workspace for its per-split partial results and its
// device status word.  Some callers have no way to provide one: a plug-in whose
// host framework owns every byte of device memory and forbids further
// cudaMalloc calls, a process with a fixed device-memory budget, or a
// latency-critical path that must not pay for an allocation (cudaMalloc can
// synchronise the device).  For them this file keeps that scratch in a
// fixed-size array of device memory that the library owns: every GPU that loads
// the library holds it until the process exits.
#include <mutex>

#include "palu_common.cuh"
#include "palu_internal.h"

namespace {

// Status word (256 bytes) followed by the split partials.
constexpr size_t kNoAllocScratchBytes = PALU_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex[kMaxDevices];
void* g_scratch_ptr[kMaxDevices] = {};

// The array's name is only a host-side stand-in in host code: the device
// address comes from cudaGetSymbolAddress, with that device current.  Only a
// successful lookup is kept; after a failed one (for instance a first call
// made while the stream was being captured) the next call looks again.
palu_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PALU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex[dev]);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();   // do not leave the failed lookup as this thread's sticky error
      return PALU_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PALU_OK;
}

}  // namespace

extern "C" palu_status palu_decode_attn_noalloc(
    const palu_config* cfg, int batch, const void* q, const int32_t* q_pos, const void* zk_pool,
    const void* zv_pool, const void* zk_scales, const void* zv_scales, const int32_t* pos_pool,
    const int32_t* page_table, int max_pages, const int32_t* seq_lens, int num_pages, const void* B_k,
    const void* B_v, void* out, float* lse, int num_splits, palu_stream_t stream, int32_t* status_out) {
  size_t need = 0;
  palu_status s = palu_decode_workspace_size(cfg, batch, max_pages, num_splits, &need);
  if (s != PALU_OK) return s;
  if (need > kNoAllocScratchBytes) return PALU_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = scratch_address(&scratch);
  if (s != PALU_OK) return s;
  // The array keeps the previous call's contents: the status word must start
  // at zero; the partials are rewritten in full by every call.
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, sizeof(palu::DevStatus), st) != cudaSuccess) return PALU_ERR_CUDA;
  s = palu_decode_attn(cfg, batch, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales, pos_pool, page_table,
                       max_pages, seq_lens, num_pages, B_k, B_v, out, lse, scratch, kNoAllocScratchBytes,
                       num_splits, stream);
  if (s != PALU_OK || status_out == nullptr) return s;
  int32_t detail = 0;
  s = palu_get_device_status(scratch, stream, &detail);
  *status_out = detail;
  return s;
}
