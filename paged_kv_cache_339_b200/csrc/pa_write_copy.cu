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

// A thread per 16-byte vector of the new K (and V) rows, four vectors apart by
// the grid's width in flight at once: the four slot loads and eight row loads
// are all issued before the first store, so neither the slot lookup nor the
// load of one token waits for another's. Vector i of the input is row
// i / row_vecs ((token, head) = divmod(row, num_kv_heads)), vector
// i % row_vecs of it; consecutive threads read consecutive vectors, and each
// run of 64 columns lands as one contiguous half-row of the tile. Sizes in the
// index arithmetic other than the head count are powers of two (shifts).
constexpr int kWriteUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads)
    write_kv_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                    const uint4* __restrict__ key,
                    const uint4* __restrict__ value,
                    const int64_t* __restrict__ slots, int64_t total_vecs,
                    int32_t num_kv_heads, int32_t bs_shift, int32_t rv_shift,
                    int32_t head_dim, int64_t num_slots) {
  pdl_launch_dependents();   // the decode plan may start; it waits for us before it ends
  const int row_vecs = 1 << rv_shift;
  const int vec_elems = head_dim >> rv_shift;           // elements per 16-byte vector
  const int vh_shift = __ffs(64 / vec_elems) - 1;       // vectors per 64-column half
  const int block_size = 1 << bs_shift;
  const int sh = tile_sub_height(block_size);
  const int sh_shift = __ffs(sh) - 1;
  const int nh = head_dim >> 6;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       base < total_vecs; base += kWriteUnroll * stride) {
    uint4 a[kWriteUnroll], b[kWriteUnroll];
    int64_t dst[kWriteUnroll];
#pragma unroll
    for (int k = 0; k < kWriteUnroll; ++k) {
      const int64_t i = base + k * stride;
      dst[k] = -1;
      if (i < total_vecs) {
        a[k] = key[i];
        b[k] = value[i];
        const int64_t row = i >> rv_shift;
        // 32-bit division where the row index allows it (all realistic sizes)
        const int64_t t = row <= 0x7fffffff
                              ? static_cast<int64_t>(static_cast<uint32_t>(row) /
                                                     static_cast<uint32_t>(num_kv_heads))
                              : row / num_kv_heads;
        const int h = static_cast<int>(row - t * num_kv_heads);
        const int64_t slot = slots[t];
        if (slot >= 0 && slot < num_slots) {
          const int64_t blk = slot >> bs_shift;
          const int off = static_cast<int>(slot & (block_size - 1));
          const int v = static_cast<int>(i & (row_vecs - 1));
          const int half = v >> vh_shift, vin = v & ((1 << vh_shift) - 1);
          // tile (blk, h), then (token off, half, vector vin) inside it
          dst[k] = ((blk * num_kv_heads + h) << (bs_shift + rv_shift)) +
                   ((((off >> sh_shift) * nh + half) << sh_shift) << vh_shift) +
                   ((off & (sh - 1)) << vh_shift) + vin;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kWriteUnroll; ++k) {
      if (dst[k] >= 0) {
        kc[dst[k]] = a[k];
        vc[dst[k]] = b[k];
      }
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
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * row_vecs;
  const int64_t per_cta = static_cast<int64_t>(kCopyThreads) * kWriteUnroll;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  int64_t grid = (total + per_cta - 1) / per_cta;
  grid = grid < 1 ? 1 : (grid > cap ? cap : grid);
  write_kv_kernel<<<static_cast<int>(grid), kCopyThreads, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), slots, total,
      num_kv_heads, __builtin_ctz(static_cast<unsigned>(block_size)),
      __builtin_ctz(static_cast<unsigned>(row_vecs)), row_vecs * 16 / elem_bytes, num_slots);
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
