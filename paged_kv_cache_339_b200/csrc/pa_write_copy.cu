// pa_write_kv, pa_copy_blocks and pa_swap_blocks kernels: bit-exact 16-byte
// vector copies.
//
// write: each new token's K/V row of one KV head (head_dim elements) goes to
//   pool[slot / BS][head][slot % BS][:]   (slot < 0: padding, skipped)
// at the positions the in-block storage order gives (pa_common.cuh).
// "Paged Attention: Virtual Memory for the KV Cache", "The fix borrowed from
// operating systems": a request fills its current block, then asks for more.
//
// copy: block dst of both pools becomes a copy of block src, all heads: the
// copy a diverging sequence gets of a shared block ("Sharing comes almost for
// free").
//
// swap: the same block copy between the device pools and a host pool the
// device can address (preemption by swapping, "What it does not fix"); the
// kernel reads or writes host memory directly over the host link.
//
// Consecutive threads touch consecutive 16-byte vectors of a row (coalesced
// on both sides). Indices outside the pool are skipped, never dereferenced.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kCopyThreads = 256;

// A CTA takes whole tokens (one slot load per token) and its threads walk the
// token's (head, 16-byte vector) pairs; every size that appears in the index
// arithmetic (vectors per row, 64-column halves, the 16-token group) is a
// power of two, so it is all shifts and masks.
__global__ void __launch_bounds__(kCopyThreads)
    write_kv_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                    const uint4* __restrict__ key,
                    const uint4* __restrict__ value,
                    const int64_t* __restrict__ slots, int32_t num_tokens,
                    int32_t num_kv_heads, int32_t block_size,
                    int32_t row_vecs, int32_t head_dim, int64_t num_slots) {
  pdl_launch_dependents();   // the decode plan may start; it waits for us before it ends
  const int per_token = num_kv_heads * row_vecs;
  const int rv_shift = __ffs(row_vecs) - 1;
  const int vec_elems = head_dim >> rv_shift;           // elements per 16-byte vector
  const int vh_shift = __ffs(64 / vec_elems) - 1;       // vectors per 64-column half
  const int sh = tile_sub_height(block_size);
  const int sh_shift = __ffs(sh) - 1;
  const int nh = head_dim >> 6;
  for (int t = blockIdx.x; t < num_tokens; t += gridDim.x) {
    const int64_t slot = slots[t];
    if (slot < 0 || slot >= num_slots) continue;
    const int64_t blk = slot / block_size;
    const int off = static_cast<int>(slot - blk * block_size);
    // vector offset of (token off, half 0, column 0) inside a tile, and of
    // the tile of head 0
    const int row_base = (((off >> sh_shift) * nh) << sh_shift) * (64 / vec_elems) +
                         (off & (sh - 1)) * (64 / vec_elems);
    const int64_t tile0 = blk * num_kv_heads * (static_cast<int64_t>(block_size) << rv_shift);
    const size_t src0 = static_cast<size_t>(t) * per_token;
    for (int r = threadIdx.x; r < per_token; r += blockDim.x) {
      const int h = r >> rv_shift, v = r & (row_vecs - 1);
      const int half = v >> vh_shift, vin = v & ((1 << vh_shift) - 1);
      const int64_t dst = tile0 + (static_cast<int64_t>(h) * block_size << rv_shift) + row_base +
                          ((half << sh_shift) << vh_shift) + vin;
      kc[dst] = key[src0 + r];
      vc[dst] = value[src0 + r];
    }
  }
}

// Block copies (copy-on-write within the pools, or swap between the pools
// and a host pool): a CTA takes one (pair, 16 KB part) at a time, four
// 16-byte vectors per thread in flight; pairs with an index outside its pool
// are skipped.
constexpr int kPartVecs = 4 * kCopyThreads;

__global__ void __launch_bounds__(kCopyThreads)
    block_copy_kernel(uint4* __restrict__ dk, uint4* __restrict__ dv,
                      const uint4* __restrict__ sk, const uint4* __restrict__ sv,
                      const int64_t* __restrict__ pairs, int32_t num_pairs, int64_t block_vecs,
                      int32_t src_blocks, int32_t dst_blocks) {
  pdl_launch_dependents();   // the decode plan may start; it waits for us before it ends
  const int parts = static_cast<int>((block_vecs + kPartVecs - 1) / kPartVecs);
  const int64_t work = static_cast<int64_t>(num_pairs) * parts;
  for (int64_t c = blockIdx.x; c < work; c += gridDim.x) {
    const int p = static_cast<int>(c / parts);
    const int part = static_cast<int>(c - static_cast<int64_t>(p) * parts);
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) continue;
    const int64_t v0 = static_cast<int64_t>(part) * kPartVecs + threadIdx.x;
    uint4 a[4], b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t v = v0 + k * kCopyThreads;
      if (v < block_vecs) {
        a[k] = sk[src * block_vecs + v];
        b[k] = sv[src * block_vecs + v];
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t v = v0 + k * kCopyThreads;
      if (v < block_vecs) {
        dk[dst * block_vecs + v] = a[k];
        dv[dst * block_vecs + v] = b[k];
      }
    }
  }
}

}  // namespace

cudaError_t launch_write_kv(void* k_cache, void* v_cache, const void* key,
                            const void* value, const int64_t* slots,
                            int32_t num_tokens, int32_t num_kv_heads,
                            int32_t block_size, int32_t row_bytes, int32_t elem_bytes,
                            int64_t num_slots, cudaStream_t stream) {
  const int32_t row_vecs = row_bytes / 16;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  const int grid = static_cast<int>(num_tokens < cap ? (num_tokens > 0 ? num_tokens : 1) : cap);
  write_kv_kernel<<<grid, kCopyThreads, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), slots,
      num_tokens, num_kv_heads, block_size, row_vecs, row_vecs * 16 / elem_bytes, num_slots);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                               int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               cudaStream_t stream) {
  return launch_swap_blocks(k_cache, v_cache, k_cache, v_cache, pairs, num_pairs, block_bytes,
                            num_blocks, num_blocks, stream);
}

cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* pairs, int32_t num_pairs, int64_t block_bytes,
                               int32_t src_blocks, int32_t dst_blocks, cudaStream_t stream) {
  const int64_t block_vecs = block_bytes / 16;
  const int64_t work = static_cast<int64_t>(num_pairs) * ((block_vecs + kPartVecs - 1) / kPartVecs);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  const int grid = static_cast<int>(work < cap ? (work > 0 ? work : 1) : cap);
  block_copy_kernel<<<grid, kCopyThreads, 0, stream>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), pairs, num_pairs, block_vecs, src_blocks, dst_blocks);
  return cudaGetLastError();
}

}  // namespace pa
