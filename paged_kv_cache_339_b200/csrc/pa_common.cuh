// Device helpers shared by the paged-KV kernels (sm_100a only).
//
// Everything asynchronous here is a plain CTA-local form: bulk copies and TMA
// tensor loads write this CTA's shared memory, completion is tracked by
// mbarrier transaction counts, and no copy uses cluster multicast.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_workspace.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is built for sm_100a only"
#endif

namespace pa {

// Time limit of every barrier wait in the kernels (nanoseconds). A correct
// launch never comes near it; if a wait does run out, the kernel records
// PA_ERR_DEVICE_TIMEOUT in the workspace status word and returns early.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed, for at
// most kWaitLimitNs. On time-out (or when another role of the CTA already
// gave up, `abrt` != 0) it records the status, raises `abrt` and returns
// false; callers then leave their loops.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abrt,
                                          int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abrt) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abrt = 1;
        atomicExch(status, 6 /* PA_ERR_DEVICE_TIMEOUT */);
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Bulk copies global -> this CTA's shared memory (no multicast)
// ---------------------------------------------------------------------------
// Contiguous bytes; dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src,
                                         uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled TMA load of the box at (x, y) of `tmap` (x innermost, in
// elements; x * element size must be a multiple of 16 bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tmap,
                                            int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::"
      "complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y),
      "r"(smem_u32(bar))
      : "memory");
}

// L2 cache policy for data read once per call (the KV tiles): its lines are
// the first to be evicted, so the streamed pool does not push out of L2 what
// the next call reads again (block tables, lengths, the workspace, the
// kernels' code). Used as the cache-hint operand of the copies below.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 3-D tiled TMA load of the box at (x, y, z) of `tmap` (x innermost, in
// elements; x * element size a multiple of 16 bytes).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tmap, int32_t x,
                                            int32_t y, int32_t z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::"
      "complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// tma_load_2d with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* tmap, int32_t x,
                                                 int32_t y, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::"
      "complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap))
               : "memory");
}

// Generic-proxy writes to shared memory made visible to the async proxy
// (tensor core / TMA) before they read or overwrite it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier among `nthreads` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Element conversions (exact widening to fp32)
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  __device__ static __forceinline__ void unpack4(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ static __forceinline__ float load1(const void* p) {
    return *reinterpret_cast<const float*>(p);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  // bf16 -> fp32 is a 16-bit left shift of the bit pattern.
  __device__ static __forceinline__ void unpack2(uint32_t w, float* f) {
    f[0] = __uint_as_float(w << 16);
    f[1] = __uint_as_float(w & 0xffff0000u);
  }
  __device__ static __forceinline__ float load1(const void* p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  }
};

template <>
struct Elem<__half> {
  static constexpr int kBytes = 2;
  __device__ static __forceinline__ void unpack2(uint32_t w, float* f) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    float2 x = __half22float2(h);
    f[0] = x.x;
    f[1] = x.y;
  }
  __device__ static __forceinline__ float load1(const void* p) {
    return __half2float(*reinterpret_cast<const __half*>(p));
  }
};

// Unpack a 16-byte vector into fp32 values: 4 (fp32) or 8 (16-bit types).
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& v, float* f) {
  if constexpr (sizeof(T) == 4) {
    Elem<float>::unpack4(v, f);
  } else {
    Elem<T>::unpack2(v.x, f + 0);
    Elem<T>::unpack2(v.y, f + 2);
    Elem<T>::unpack2(v.z, f + 4);
    Elem<T>::unpack2(v.w, f + 6);
  }
}

// In-block storage order of one (block, KV head) tile of block_size x
// head_dim elements: rows cut into 64-element halves and grouped 16 tokens at
// a time, so element (t, d) sits at
//   ((t / SH) * NH + d / 64) * SH * 64 + (t % SH) * 64 + d % 64,
// SH = min(block_size, 16), NH = head_dim / 64 (row-major when head_dim = 64).
// A whole tile is one contiguous range, and each 16-token group of one half
// is a run of 128-byte (16-bit) rows that a single 2-D TMA box and the tensor
// cores consume directly.
__host__ __device__ __forceinline__ int tile_sub_height(int block_size) {
  return block_size < 16 ? block_size : 16;
}
__host__ __device__ __forceinline__ int tile_offset(int t, int d, int block_size, int head_dim) {
  const int sh = tile_sub_height(block_size), nh = head_dim >> 6;
  return ((t / sh) * nh + (d >> 6)) * sh * 64 + (t % sh) * 64 + (d & 63);
}

// Work-item record written by the planning kernel: one per (sequence, split);
// the KV-head index is folded into the claimed item number.
struct __align__(16) WorkPair {
  int32_t seq;
  int32_t split_n;  // split index (low 16 bits) | number of splits of the sequence << 16
  int32_t t_begin;  // first token of the range
  int32_t t_end;    // one past the last token
};
__device__ __forceinline__ int item_split(int32_t split_n) { return split_n & 0xffff; }
__device__ __forceinline__ int item_nsplit(int32_t split_n) { return (split_n >> 16) & 0x3fff; }
// Set on a sequence's only piece of its own when all its other pieces are
// shared-prefix group pieces, complete before the launch that takes it: that
// piece folds their partial results into its own and writes the output rows.
constexpr int32_t kFoldGroupPieces = 1 << 30;
__device__ __forceinline__ bool item_folds(int32_t split_n) {
  return (split_n & kFoldGroupPieces) != 0;
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until the previous kernel has completed and its writes
// are visible. Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Split-context merge, done by the last piece of a (sequence, KV head) to
// finish. With per-piece running max m_p (log2 units), sum l_p and
// unnormalised accumulator a_p:
//   M = max_p m_p,  L = sum_p l_p 2^(m_p - M),  o = sum_p a_p 2^(m_p - M) / L.
// This regrouping is exact algebra on the softmax sums; the pages do not
// discuss splitting a context. The pieces were written by other CTAs of the
// same grid, so they are read through L2 (ld.global.cg).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void merge_split_rows(float* out, const float2* ml, const float* po,
                                                 size_t row0, int nrows, int D, int nsp,
                                                 int max_splits, int tid, int nthreads) {
  // a thread per (row, 4 columns); one pass over the pieces with a running
  // maximum, 8 pieces' loads in flight at a time
  const int vpr = D / 4;
  for (int idx = tid; idx < nrows * vpr; idx += nthreads) {
    const int h = idx / vpr, c4 = idx - h * vpr;
    const size_t row = row0 + h;
    const float2* mr = ml + row * max_splits;
    const float4* pr = reinterpret_cast<const float4*>(po + row * max_splits * D) + c4;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nsp; s0 += 8) {
      float2 e[8];
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool in = s0 + j < nsp;
        e[j] = in ? __ldcg(mr + s0 + j) : make_float2(-INFINITY, 0.f);
        v[j] = in ? __ldcg(pr + static_cast<size_t>(s0 + j) * vpr) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mb = M;
#pragma unroll
      for (int j = 0; j < 8; ++j) mb = fmaxf(mb, e[j].x);
      const float sc = exp2f(M - mb);   // M = -inf on the first batch: 0
      L *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float w = exp2f(e[j].x - mb);   // 0 for the padding entries
        L = fmaf(e[j].y, w, L);
        acc.x = fmaf(w, v[j].x, acc.x);
        acc.y = fmaf(w, v[j].y, acc.y);
        acc.z = fmaf(w, v[j].z, acc.z);
        acc.w = fmaf(w, v[j].w, acc.w);
      }
      M = mb;
    }
    const float inv = 1.0f / L;
    reinterpret_cast<float4*>(out + row * D)[c4] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

}  // namespace pa
