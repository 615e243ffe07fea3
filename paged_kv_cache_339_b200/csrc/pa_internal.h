// Host-side declarations shared by the C-ABI shim and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"
#include "pa_workspace.h"

namespace pa {

struct PlanParams {
  const int32_t* context_lens;
  float* out;
  uint8_t* ws;
  size_t pairs_off, nsplit_off, split_off, cnt_off;
  int32_t num_seqs, num_q_heads, num_kv_heads, head_dim;
  int32_t bt_stride, block_size, max_context_len;
  int32_t split_tokens;   // explicit split, or 0 = choose on the device
  int32_t min_split;      // lower bound of an automatic split
  int32_t max_splits;
  int32_t num_ctas;       // item streams of the decode kernel (CTAs x streams per CTA)
  // shared prefixes (share_prefixes = 1): groups of consecutive sequences
  // whose tables start with the same blocks; their common whole pieces go to
  // a list of their own (gpairs_off), taken by a launch of group_ctas item
  // streams that reads each shared tile once for up to share_members
  // sequences
  const int32_t* block_tables;
  int32_t share_prefixes, share_members, group_ctas;
  size_t gpairs_off;
  // 1: the decode kernel reads KV heads in pairs; items and merge counters
  // are per pair, pieces are cut to the same work as for one head
  int32_t pair_heads;
};

// Everything a decode main kernel needs; filled by the C-ABI shim.
struct DecodeParams {
  const void* k_cache;
  const void* v_cache;
  const void* q;
  float* out;
  const int32_t* block_tables;
  uint8_t* ws;
  size_t pairs_off, nsplit_off, split_off, cnt_off, ml_off, o_off;
  int32_t bt_stride, num_blocks, num_kv_heads, num_q_heads, head_dim,
      block_size, num_seqs, max_splits;
  float scale_log2;  // scale * log2(e): scores kept in log2 units
  int32_t dtype;     // pa_dtype
  // 1: this launch takes the group list (shared prefixes): an item is a run
  // of whole pieces common to `members` consecutive sequences, its query rows
  // those sequences' rows of the KV head
  int32_t group_mode;
  size_t gpairs_off;
  // 1: the tensor-core kernel reads KV heads in pairs (its items, and the
  // plan's, count num_kv_heads / 2 virtual heads of 2G query heads)
  int32_t pair_heads;
};

// Largest batch whose shared prefixes pa_decode looks for.
constexpr int32_t kShareMaxSeqs = 1024;

// Launched with programmatic stream serialisation (PDL): the plan may be
// scheduled while its predecessor in the stream (the KV write) finishes.
cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream);

// CUDA-core decode. Returns cudaErrorInvalidValue for an unsupported shape.
bool simt_supported(int dtype, int head_dim, int group);
cudaError_t simt_num_ctas(int dtype, int head_dim, int group, int* num_ctas);
cudaError_t launch_decode_simt(const DecodeParams& p, int num_ctas,
                               cudaStream_t stream);
// The CUDA-core kernel over the group list (16 query rows per item).
cudaError_t launch_decode_simt_groups(const DecodeParams& p, int num_ctas,
                                      cudaStream_t stream);

// Tensor-core (tcgen05) decode for 16-bit KV, head_dim 128, 4 <= G <= 16.
bool tc_supported(int dtype, int head_dim, int group);
cudaError_t tc_num_ctas(int dtype, int group, int* num_ctas);
cudaError_t launch_decode_tc(const DecodeParams& p, int num_ctas,
                             cudaStream_t stream);
// The tensor-core kernel over the group list: 16-row tiles of 16 / G
// sequences x G heads (16-bit KV, head_dim 128, G a divisor of 16 up to 8).
bool tc_group_supported(int dtype, int head_dim, int group);
// The tensor-core kernel can read KV heads in pairs (block size 8, an even
// number of KV heads, 4 or 8 query heads per KV head).
bool tc_pair_supported(int block_size, int num_kv_heads, int group);
cudaError_t launch_decode_tc_groups(const DecodeParams& p, int num_ctas,
                                    cudaStream_t stream);

// KV write and block copy.
cudaError_t launch_write_kv(void* k_cache, void* v_cache, const void* key,
                            const void* value, const int64_t* slots,
                            int32_t num_tokens, int32_t num_kv_heads,
                            int32_t block_size, int32_t row_bytes, int32_t elem_bytes,
                            int64_t num_slots, cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache,
                               const int64_t* pairs, int32_t num_pairs,
                               int64_t block_bytes, int32_t num_blocks,
                               cudaStream_t stream);
cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* pairs, int32_t num_pairs, int64_t block_bytes,
                               int32_t src_blocks, int32_t dst_blocks, cudaStream_t stream);

int num_sms();

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while its predecessor in the stream is still running; it must execute
// griddepcontrol.wait (pdl_wait) before touching anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// What check_decode_args decided for a valid pa_decode call.
struct DecodeChoice {
  int group;       // query heads per KV head
  int32_t split;   // explicit split (0 = automatic)
  bool use_tc;     // tensor-core kernel (else CUDA cores)
  bool share;      // look for shared prefixes (CUDA-core path, 2..1024 sequences)
  bool empty;      // no sequences: nothing to enqueue
};

// Every host-side check of pa_decode's arguments except those of the
// workspace (pointer, alignment, size), in pa_decode's order; PA_OK and the
// choice, or the status pa_decode would return.
pa_status check_decode_args(const pa_kv_cache* cache, const float* out, const void* q,
                            const int32_t* block_tables, int32_t bt_stride,
                            const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                            int32_t max_context_len, float scale, const pa_decode_options* opts,
                            DecodeChoice* ch);

// Store a CUDA error for pa_last_cuda_error() on this thread.
void record_cuda_error(cudaError_t e);

}  // namespace pa
