// Work planning and split-context merge for pa_decode.
//
// plan_kernel (one CTA) reads the context lengths, checks them, picks the
// split size, and writes the list of (sequence, split) work pairs in
// split-major order (every sequence's first split, then every second split,
// ...), so the persistent decode kernels claim the longest ranges first.
//
// merge_kernel combines the partial softmax results of sequences that were
// split: with per-split running max m_p (log2 units), sum l_p and
// unnormalised accumulator a_p,
//   M = max_p m_p,  L = sum_p l_p 2^(m_p - M),  o = sum_p a_p 2^(m_p - M) / L.
// This regrouping is exact algebra on the softmax sums; the pages do not
// discuss splitting a context.
//
// Launched with programmatic stream serialisation: it may start while the KV
// write before it is still running (it reads only the lengths), and waits for
// that kernel before it exits, so the decode kernel that waits on the plan
// also sees the new tokens.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kPlanMaxThreads = 1024;

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

__global__ void __launch_bounds__(kPlanMaxThreads, 1) plan_kernel(PlanParams p) {
  pdl_launch_dependents();
  __shared__ long long s_sum[32];
  __shared__ int s_max[32];
  __shared__ int s_bad[32];
  __shared__ int s_split;
  __shared__ int s_maxn;
  __shared__ int s_total;
  extern __shared__ int cell_cnt[];   // [levels][32-sequence groups]

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  WorkPair* pairs = reinterpret_cast<WorkPair*>(p.ws + p.pairs_off);
  int32_t* nsplit = reinterpret_cast<int32_t*>(p.ws + p.nsplit_off);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int64_t cap = static_cast<int64_t>(p.bt_stride) * p.block_size;

  // 1. validate lengths, total and maximum
  long long tot = 0;
  int mx = 0, bad = 0;
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = p.context_lens[i];
    if (L < 0 || L > p.max_context_len || L > cap) {
      bad = 1;
    } else {
      tot += L;
      mx = max(mx, L);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (lane == 0) {
    s_sum[warp] = tot;
    s_max[warp] = mx;
    s_bad[warp] = bad;
  }
  __syncthreads();
  if (tid == 0) {
    long long t = 0;
    int m = 0, b = 0;
    for (int w = 0; w < nwarps; ++w) {
      t += s_sum[w];
      m = max(m, s_max[w]);
      b |= s_bad[w];
    }
    int S = p.split_tokens;
    if (S <= 0) {
      // Aim for ~items_per_cta work items per persistent CTA.
      long long per_cta = (t * p.num_kv_heads + p.num_ctas - 1) / p.num_ctas;
      long long want = (per_cta + p.items_per_cta - 1) / p.items_per_cta;
      want = (want + kAutoSplitQuantum - 1) / kAutoSplitQuantum * kAutoSplitQuantum;
      if (want < p.min_split) want = p.min_split;
      if (want > (1 << 30)) want = 1 << 30;
      S = static_cast<int>(want);
    }
    s_split = S;
    s_maxn = m > 0 ? (m + S - 1) / S : 0;
    hdr->status = b ? 1 /* PA_ERR_INVALID_ARG */ : 0;
    hdr->split_tokens = S;
    hdr->max_splits = p.max_splits;
  }
  __syncthreads();
  const int S = s_split;
  const int maxn = min(s_maxn, p.max_splits);

  // 2. splits per sequence; sequences with nothing to attend to get zero rows
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = p.context_lens[i];
    const bool ok = !(L < 0 || L > p.max_context_len || L > cap);
    const int n = (ok && L > 0) ? (L + S - 1) / S : 0;
    nsplit[i] = n;
    if (n == 0) {
      float4* row = reinterpret_cast<float4*>(
          p.out + static_cast<size_t>(i) * p.num_q_heads * p.head_dim);
      const int n4 = p.num_q_heads * p.head_dim / 4;
      for (int e = 0; e < n4; ++e) row[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();

  // 3. split-major pair list: position of (i, s) = base_s + rank_s(i), with
  // base_s = number of pairs at levels < s and rank_s(i) = number of
  // sequences j < i with more than s splits. Per 32-sequence group and level,
  // a ballot gives the group's count and each lane's rank inside the group;
  // one scan over the (level, group) counts gives every group's base.
  const int ngroups = (p.num_seqs + 31) / 32;
  const int ncells = maxn * ngroups;   // (level, group) cells, level-major
  for (int cell = warp; cell < ncells; cell += nwarps) {
    const int s = cell / ngroups, g = cell - s * ngroups;
    const int i = g * 32 + lane;
    const int n = i < p.num_seqs ? nsplit[i] : 0;
    const unsigned m = __ballot_sync(0xffffffffu, n > s);
    if (lane == 0) cell_cnt[cell] = __popc(m);
  }
  __syncthreads();
  // exclusive scan of cell_cnt (level-major) by warp 0
  if (warp == 0) {
    int carry = 0;
    for (int c0 = 0; c0 < ncells; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < ncells ? cell_cnt[c] : 0;
      const int inc = warp_incl_scan(v, lane);
      if (c < ncells) cell_cnt[c] = carry + inc - v;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) s_total = carry;
  }
  __syncthreads();
  for (int cell = warp; cell < ncells; cell += nwarps) {
    const int s = cell / ngroups, g = cell - s * ngroups;
    const int i = g * 32 + lane;
    int n = 0, L = 0;
    if (i < p.num_seqs) {
      n = nsplit[i];
      L = p.context_lens[i];
    }
    const unsigned m = __ballot_sync(0xffffffffu, n > s);
    if (n > s) {
      WorkPair w;
      w.seq = i;
      w.split_n = s | (n << 16);
      w.t_begin = s * S;
      w.t_end = min(L, (s + 1) * S);
      pairs[cell_cnt[cell] + __popc(m & ((1u << lane) - 1u))] = w;
    }
  }
  const int base = s_total;
  if (tid == 0) {
    hdr->num_pairs = base;
    hdr->num_items = base * p.num_kv_heads;
    hdr->work_counter = 0;
  }
  // complete only after the kernel before this one (the KV write) has
  pdl_wait();
}

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(MergeParams p) {
  pdl_wait();   // every partial of the decode kernel is written and visible
  extern __shared__ float s_w[];  // [G][max_splits] normalised weights
  const int seq = blockIdx.x / p.num_kv_heads;
  const int kvh = blockIdx.x % p.num_kv_heads;
  const int32_t* nsplit = reinterpret_cast<const int32_t*>(p.ws + p.nsplit_off);
  const int n = nsplit[seq];
  if (n <= 1) return;
  const int G = p.num_q_heads / p.num_kv_heads;
  const float2* ml = reinterpret_cast<const float2*>(p.ws + p.ml_off);
  const float* po = reinterpret_cast<const float*>(p.ws + p.o_off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  for (int g = warp; g < G; g += kMergeThreads / 32) {
    const size_t row = static_cast<size_t>(seq) * p.num_q_heads + kvh * G + g;
    const float2* r = ml + row * p.max_splits;
    float M = -INFINITY;
    for (int s = lane; s < n; s += 32) M = fmaxf(M, r[s].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < n; s += 32) L += r[s].y * exp2f(r[s].x - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float inv = 1.0f / L;
    for (int s = lane; s < n; s += 32) s_w[g * p.max_splits + s] = exp2f(r[s].x - M) * inv;
  }
  __syncthreads();
  const int D = p.head_dim;
  for (int idx = threadIdx.x; idx < G * D; idx += kMergeThreads) {
    const int g = idx / D, d = idx % D;
    const size_t row = static_cast<size_t>(seq) * p.num_q_heads + kvh * G + g;
    const float* src = po + row * p.max_splits * D + d;
    const float* w = s_w + g * p.max_splits;
    float acc = 0.f;
#pragma unroll 4
    for (int s = 0; s < n; ++s) acc = fmaf(w[s], src[static_cast<size_t>(s) * D], acc);
    p.out[row * D + d] = acc;
  }
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  if (p.max_splits <= 1 || p.num_seqs == 0) return cudaSuccess;
  const int G = p.num_q_heads / p.num_kv_heads;
  const size_t smem = static_cast<size_t>(G) * p.max_splits * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(merge_kernel, dim3(p.num_seqs * p.num_kv_heads), dim3(kMergeThreads), smem,
                    stream, p);
}

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream) {
  int threads = (p.num_seqs + 31) / 32 * 32;
  threads = threads < 64 ? 64 : (threads > kPlanMaxThreads ? kPlanMaxThreads : threads);
  const size_t cells = static_cast<size_t>(p.max_splits) * ((p.num_seqs + 31) / 32);
  const size_t smem = cells * sizeof(int);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, plan_kernel, p);
}

}  // namespace pa
