// pa_decode_noalloc: paged decode for callers that cannot allocate device
// memory. Same kernels and arguments as pa_decode, but the scratch (work list,
// per-split partial results, status word) lives in one file-scope device array
// of fixed size instead of a caller-provided workspace.
//
// Who needs it: a process that hands nearly all of HBM to its KV-cache pool up
// front leaves no room for a second allocation, and code on a latency-critical
// path cannot afford cudaMalloc's implicit device synchronisation; neither can
// then obtain a workspace for pa_decode.
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
namespace {

// Fixed scratch, 32 MiB. It is part of this library's device image, so every
// GPU that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t{32} << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// In host code the array's name is only a host-side stand-in; its device
// address is looked up once per device with that device current.
std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

pa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && (dev < 0 || dev >= 64)) e = cudaErrorInvalidDevice;
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e == cudaSuccess) g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
  }
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_decode_noalloc(const pa_kv_cache* cache, float* out, const void* q,
                                       const int32_t* block_tables, int32_t bt_stride,
                                       const int32_t* context_lens, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t max_context_len,
                                       float scale, const pa_decode_options* opts,
                                       pa_stream_t stream) {
  // pa_decode's own checks first, so a bad argument is reported as such and
  // not as a scratch that is too small; the size of the scratch is the last
  pa::DecodeChoice ch;
  const pa_status chk = pa::check_decode_args(cache, out, q, block_tables, bt_stride,
                                              context_lens, num_seqs, num_q_heads,
                                              max_context_len, scale, opts, &ch);
  if (chk != PA_OK) return chk;
  if (ch.empty) return PA_OK;
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, cache->head_dim,
                                               max_context_len, cache->block_size, ch.split);
  if (need > pa::kNoAllocScratchBytes) return PA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const pa_status st = pa::scratch_address(&scratch);
  if (st != PA_OK) return st;
  return pa_decode(cache, out, q, block_tables, bt_stride, context_lens, num_seqs, num_q_heads,
                   max_context_len, scale, opts, scratch, pa::kNoAllocScratchBytes, stream);
}

extern "C" pa_status pa_decode_noalloc_status(pa_stream_t stream) {
  void* scratch = nullptr;
  const pa_status st = pa::scratch_address(&scratch);
  if (st != PA_OK) return st;
  // the status word sits at the start of the scratch, as in a workspace
  return pa_decode_status(scratch, stream);
}
