// C-ABI entry points (include/pa.h): host-side argument checks, dispatch,
// launch. No device memory is allocated or freed here.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "pa.h"
#include "pa_internal.h"

namespace pa {

namespace {

thread_local char g_cuda_error[256] = "";

pa_status cuda_fail(cudaError_t e) {
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s",
                cudaGetErrorName(e), cudaGetErrorString(e));
  return PA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status check_cache(const pa_kv_cache* c) {
  if (c == nullptr || c->k_cache == nullptr || c->v_cache == nullptr) return PA_ERR_INVALID_ARG;
  if (c->num_blocks <= 0 || c->num_kv_heads <= 0 || c->block_size <= 0 || c->head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  if (c->dtype != PA_F32 && c->dtype != PA_F16 && c->dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32) return PA_ERR_UNSUPPORTED;
  if (!aligned16(c->k_cache) || !aligned16(c->v_cache)) return PA_ERR_MISALIGNED;
  return PA_OK;
}

int elem_bytes(int dtype) { return dtype == PA_F32 ? 4 : 2; }

// Persistent-grid sizes, computed once per (device, kernel flavour).
struct CtaCache {
  std::mutex mu;
  int dev = -1;
  int simt[3][2][3] = {};   // [dtype][head_dim 64/128][gpw 1/2/4]
  int tc[3][17] = {};       // [dtype][group]
};
CtaCache g_ctas;

cudaError_t cached_ctas(bool tc, int dtype, int head_dim, int group, int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_ctas.mu);
  if (g_ctas.dev != dev) {
    std::memset(g_ctas.simt, 0, sizeof(g_ctas.simt));
    std::memset(g_ctas.tc, 0, sizeof(g_ctas.tc));
    g_ctas.dev = dev;
  }
  int* slot;
  if (tc) {
    slot = &g_ctas.tc[dtype][group];
  } else {
    const int gpw = group == 1 ? 0 : (group == 2 ? 1 : 2);
    slot = &g_ctas.simt[dtype][head_dim == 64 ? 0 : 1][gpw];
  }
  if (*slot == 0) {
    e = tc ? tc_num_ctas(dtype, group, slot) : simt_num_ctas(dtype, head_dim, group, slot);
    if (e != cudaSuccess) {
      *slot = 0;
      return e;
    }
  }
  *out = *slot;
  return cudaSuccess;
}

}  // namespace

void record_cuda_error(cudaError_t e) {
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Every host check of a pa_decode call that does not involve the workspace,
// and the kernel it will run. ch->empty: nothing to enqueue (no sequences).
pa_status check_decode_args(const pa_kv_cache* cache, const float* out, const void* q,
                            const int32_t* block_tables, int32_t bt_stride,
                            const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                            int32_t max_context_len, float scale, const pa_decode_options* opts,
                            DecodeChoice* ch) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0) return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int group = num_q_heads / cache->num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  const int32_t split = opts ? opts->split_tokens : 0;
  const int32_t path = opts ? opts->path : PA_PATH_AUTO;
  const int32_t share = opts ? opts->share_prefixes : 0;
  if (split < 0 || path < PA_PATH_AUTO || path > PA_PATH_TCGEN05) return PA_ERR_INVALID_ARG;
  if (share != 0 && share != 1) return PA_ERR_INVALID_ARG;
  if (split > 0) {
    if (split % cache->block_size != 0) return PA_ERR_INVALID_ARG;
    if (max_context_len > 0 && ceil_div(max_context_len, split) > kMaxSplits)
      return PA_ERR_INVALID_ARG;
  }
  ch->group = group;
  ch->split = split;
  ch->use_tc = false;
  ch->share = false;
  ch->empty = num_seqs == 0;
  if (ch->empty) return PA_OK;
  if (out == nullptr || q == nullptr || block_tables == nullptr || context_lens == nullptr)
    return PA_ERR_INVALID_ARG;
  if (bt_stride <= 0) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(bt_stride) * cache->block_size)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_MISALIGNED;
  // the planning kernel keeps the lengths in shared memory
  if (static_cast<int64_t>(num_seqs) * 4 > 220 * 1024) return PA_ERR_UNSUPPORTED;
  // query rows are 32-bit coordinates of the copies
  if (static_cast<int64_t>(num_seqs) * num_q_heads > INT32_MAX) return PA_ERR_UNSUPPORTED;

  // the tensor-core kernel loads query tiles of 16 rows: it needs >= 16 query rows
  const bool tc_ok = tc_supported(cache->dtype, cache->head_dim, group) &&
                     static_cast<int64_t>(num_seqs) * num_q_heads >= 16;
  bool use_tc = false;
  if (path == PA_PATH_TCGEN05) {
    if (!tc_ok) return PA_ERR_UNSUPPORTED;
    use_tc = true;
  } else if (path == PA_PATH_AUTO) {
    use_tc = tc_ok;
  }
  if (!use_tc && !simt_supported(cache->dtype, cache->head_dim, group)) return PA_ERR_UNSUPPORTED;
  ch->use_tc = use_tc;
  // shared prefixes are read once per group of at least two sequences (at
  // most 16 query rows: G <= 8), for batches of up to kShareMaxSeqs
  ch->share = share == 1 && group <= 8 && num_seqs >= 2 && num_seqs <= kShareMaxSeqs;
  return PA_OK;
}

// An NVTX range over one host call, named after the call, so a timeline
// profiler shows where each call's work was enqueued; without a tool
// attached, push and pop cost a call each.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace pa

using namespace pa;

extern "C" {

pa_status pa_write_kv(const pa_kv_cache* cache, const void* key, const void* value,
                      const int64_t* slot_mapping, int32_t num_tokens, pa_stream_t stream) {
  NvtxRange range("pa_write_kv");
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (key == nullptr || value == nullptr || slot_mapping == nullptr) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_MISALIGNED;
  const int32_t row_bytes = cache->head_dim * elem_bytes(cache->dtype);
  const int64_t num_slots = static_cast<int64_t>(cache->num_blocks) * cache->block_size;
  cudaError_t e = launch_write_kv(cache->k_cache, cache->v_cache, key, value, slot_mapping,
                                  num_tokens, cache->num_kv_heads, cache->block_size, row_bytes,
                                  elem_bytes(cache->dtype), num_slots,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

pa_status pa_copy_blocks(const pa_kv_cache* cache, const int64_t* block_pairs, int32_t num_pairs,
                         pa_stream_t stream) {
  NvtxRange range("pa_copy_blocks");
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (block_pairs == nullptr) return PA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(block_pairs) & 7u) return PA_ERR_MISALIGNED;
  const int64_t block_bytes = static_cast<int64_t>(cache->num_kv_heads) * cache->block_size *
                              cache->head_dim * elem_bytes(cache->dtype);
  cudaError_t e = launch_copy_blocks(cache->k_cache, cache->v_cache, block_pairs, num_pairs,
                                     block_bytes, cache->num_blocks,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

// Device address of page-locked host memory the device can reach; nullptr if
// it cannot (pageable memory, or not mapped).
static void* device_view_of_host(void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost) return nullptr;
  return a.devicePointer;
}

pa_status pa_swap_blocks(const pa_kv_cache* cache, void* host_k, void* host_v,
                         int32_t host_num_blocks, const int64_t* block_pairs, int32_t num_pairs,
                         int32_t direction, pa_stream_t stream) {
  NvtxRange range("pa_swap_blocks");
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || host_num_blocks < 0) return PA_ERR_INVALID_ARG;
  if (direction != PA_SWAP_OUT && direction != PA_SWAP_IN) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (block_pairs == nullptr || host_k == nullptr || host_v == nullptr) return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_pairs) & 7u) || !aligned16(host_k) || !aligned16(host_v))
    return PA_ERR_MISALIGNED;
  void* hk = device_view_of_host(host_k);
  void* hv = device_view_of_host(host_v);
  if (hk == nullptr || hv == nullptr) return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = static_cast<int64_t>(cache->num_kv_heads) * cache->block_size *
                              cache->head_dim * elem_bytes(cache->dtype);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      direction == PA_SWAP_OUT
          ? launch_swap_blocks(hk, hv, cache->k_cache, cache->v_cache, block_pairs, num_pairs,
                               block_bytes, cache->num_blocks, host_num_blocks, s)
          : launch_swap_blocks(cache->k_cache, cache->v_cache, hk, hv, block_pairs, num_pairs,
                               block_bytes, host_num_blocks, cache->num_blocks, s);
  return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t block_size,
                                int32_t split_tokens) {
  (void)block_size;
  if (num_seqs < 0 || num_q_heads < 0 || head_dim < 0 || max_context_len < 0) return 0;
  return ws_layout(num_seqs, num_q_heads, head_dim, max_context_len, split_tokens).total;
}

pa_status pa_decode(const pa_kv_cache* cache, float* out, const void* q,
                    const int32_t* block_tables, int32_t bt_stride, const int32_t* context_lens,
                    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
                    const pa_decode_options* opts, void* workspace, size_t workspace_bytes,
                    pa_stream_t stream) {
  NvtxRange range("pa_decode");
  DecodeChoice ch;
  pa_status st = check_decode_args(cache, out, q, block_tables, bt_stride, context_lens, num_seqs,
                                   num_q_heads, max_context_len, scale, opts, &ch);
  if (st != PA_OK) return st;
  if (ch.empty) return PA_OK;
  if (workspace == nullptr) return PA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return PA_ERR_MISALIGNED;
  const int group = ch.group;
  const int32_t split = ch.split;
  const bool use_tc = ch.use_tc;
  // the workspace size is the last check
  const WsLayout lay = ws_layout(num_seqs, num_q_heads, cache->head_dim, max_context_len, split);
  if (workspace_bytes < lay.total) return PA_ERR_WORKSPACE_TOO_SMALL;

  int ctas = 0;
  cudaError_t e = cached_ctas(use_tc, cache->dtype, cache->head_dim, group, &ctas);
  if (e != cudaSuccess) return cuda_fail(e);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // At block size 8 the tensor-core kernel reads two KV heads' pages with one
  // copy (its items, and the plan's, are then pairs of heads: one head of 2G
  // query heads); not with shared prefixes, whose launches count real heads.
  // Pairs halve the (sequence, head) units the plan deals out and the pieces
  // it cuts, so they are used where enough items remain: with at least two
  // pairs per item stream (many sequences), or with fewer pairs than streams
  // (few sequences, cut into pieces) when even the longest possible context
  // leaves the halved pieces above the workspace's smallest split (its bound
  // on pieces per sequence); in between, and for few short sequences, the
  // coarser items cost more at the end of the call than the saved copies gain.
  const int64_t pair_units = static_cast<int64_t>(num_seqs) * (cache->num_kv_heads / 2);
  const int64_t streams = 2 * static_cast<int64_t>(ctas);
  bool pair = use_tc && !ch.share &&
              tc_pair_supported(cache->block_size, cache->num_kv_heads, group);
  if (pair && pair_units < 2 * streams) {
    // an upper bound of the halved piece (the plan's half share, halved)
    const int64_t piece = static_cast<int64_t>(num_seqs) * max_context_len *
                          cache->num_kv_heads / streams / 4;
    pair = pair_units < streams && piece >= auto_min_split(max_context_len);
  }

  PlanParams pp;
  pp.context_lens = context_lens;
  pp.out = out;
  pp.ws = ws;
  pp.pairs_off = lay.pairs_off;
  pp.nsplit_off = lay.nsplit_off;
  pp.split_off = lay.split_off;
  pp.cnt_off = lay.cnt_off;
  pp.num_seqs = num_seqs;
  pp.num_q_heads = num_q_heads;
  pp.num_kv_heads = cache->num_kv_heads;
  pp.pair_heads = pair ? 1 : 0;
  pp.head_dim = cache->head_dim;
  pp.bt_stride = bt_stride;
  pp.block_size = cache->block_size;
  pp.max_context_len = max_context_len;
  pp.split_tokens = split;
  pp.min_split = split > 0 ? split : auto_min_split(max_context_len);
  pp.max_splits = lay.max_splits;
  // the tensor-core kernel runs two independent item streams per CTA
  pp.num_ctas = use_tc ? 2 * ctas : ctas;
  pp.block_tables = block_tables;
  pp.share_prefixes = ch.share ? 1 : 0;
  pp.share_members = 16 / group;
  pp.gpairs_off = lay.gpairs_off;
  // the group list runs on the tensor cores where its 16-row tiles fit
  // (16-bit KV, head_dim 128, G dividing 16), else on the CUDA cores
  const bool tc_groups = ch.share && tc_group_supported(cache->dtype, cache->head_dim, group);
  int gctas = 0;
  if (ch.share) {
    e = cached_ctas(tc_groups, cache->dtype, cache->head_dim, 16, &gctas);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  pp.group_ctas = tc_groups ? 2 * gctas : gctas;   // item streams of that launch
  e = launch_plan(pp, s);
  if (e != cudaSuccess) return cuda_fail(e);

  DecodeParams dp;
  dp.k_cache = cache->k_cache;
  dp.v_cache = cache->v_cache;
  dp.q = q;
  dp.out = out;
  dp.block_tables = block_tables;
  dp.ws = ws;
  dp.pairs_off = lay.pairs_off;
  dp.nsplit_off = lay.nsplit_off;
  dp.split_off = lay.split_off;
  dp.cnt_off = lay.cnt_off;
  dp.ml_off = lay.ml_off;
  dp.o_off = lay.o_off;
  dp.bt_stride = bt_stride;
  dp.num_blocks = cache->num_blocks;
  dp.num_kv_heads = cache->num_kv_heads;
  dp.num_q_heads = num_q_heads;
  dp.head_dim = cache->head_dim;
  dp.block_size = cache->block_size;
  dp.num_seqs = num_seqs;
  dp.max_splits = lay.max_splits;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.dtype = cache->dtype;
  dp.gpairs_off = lay.gpairs_off;
  dp.pair_heads = 0;
  if (ch.share) {
    // the groups' common pieces first (each member's piece is counted there),
    // then every sequence's own pieces
    dp.group_mode = 1;
    e = tc_groups ? launch_decode_tc_groups(dp, gctas, s) : launch_decode_simt_groups(dp, gctas, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  dp.group_mode = 0;
  dp.pair_heads = pair ? 1 : 0;
  e = use_tc ? launch_decode_tc(dp, ctas, s) : launch_decode_simt(dp, ctas, s);
  if (e != cudaSuccess) return cuda_fail(e);


  return PA_OK;
}

pa_status pa_decode_status(const void* workspace, pa_stream_t stream) {
  if (workspace == nullptr) return PA_ERR_INVALID_ARG;
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost,
                                  static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return static_cast<pa_status>(word);
}

const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape or dtype not supported";
    case PA_ERR_MISALIGNED: return "PA_ERR_MISALIGNED: pointer not 16-byte aligned";
    case PA_ERR_WORKSPACE_TOO_SMALL: return "PA_ERR_WORKSPACE_TOO_SMALL: workspace too small";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA call failed";
    case PA_ERR_DEVICE_TIMEOUT: return "PA_ERR_DEVICE_TIMEOUT: a kernel gave up waiting";
  }
  return "unknown pa_status";
}

const char* pa_last_cuda_error(void) { return g_cuda_error; }

const char* pa_version(void) { return "pagedattn 0.1.0 (sm_100a)"; }

}  // extern "C"
