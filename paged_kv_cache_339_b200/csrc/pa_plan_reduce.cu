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
  // dynamic: lengths [num_seqs], splits [num_seqs], cell counts [levels][32-sequence groups]
  extern __shared__ int s_dyn[];
  int* s_len = s_dyn;
  int* s_n = s_dyn + p.num_seqs;
  int* cell_cnt = s_dyn + 2 * p.num_seqs;

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
    s_len[i] = L;
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
    const int L = s_len[i];
    const bool ok = !(L < 0 || L > p.max_context_len || L > cap);
    const int n = (ok && L > 0) ? (L + S - 1) / S : 0;
    nsplit[i] = n;
    s_n[i] = n;
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
    const int n = i < p.num_seqs ? s_n[i] : 0;
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
      n = s_n[i];
      L = s_len[i];
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

// One warp per output row (sequence, query head) for head_dim 128, one
// half-warp per row for head_dim 64: each lane owns 4 consecutive columns.
// The row's splits are read in batches of 8 independent 16-byte loads, and
// the per-split weights 2^(m_p - M) / L travel between lanes by shuffle.
template <int D>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(MergeParams p) {
  constexpr int VPR = D / 4;        // float4 columns per row = lanes per row
  constexpr int RPW = 32 / VPR;     // rows per warp
  pdl_wait();   // every partial of the decode kernel is written and visible
  const int lane = threadIdx.x & 31;
  const int cv = lane % VPR, base = lane - cv;
  const int total_rows = p.num_seqs * p.num_q_heads;
  const int row = (blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5)) * RPW + lane / VPR;
  const int32_t* nsplit = reinterpret_cast<const int32_t*>(p.ws + p.nsplit_off);
  const int n = row < total_rows ? nsplit[row / p.num_q_heads] : 0;
  int nw = n;   // loop bound shared by the rows of the warp
#pragma unroll
  for (int o = VPR; o < 32; o <<= 1) nw = max(nw, __shfl_xor_sync(0xffffffffu, nw, o));
  if (nw <= 1) return;   // no split row here: the decode kernel wrote the output

  const size_t r = row < total_rows ? static_cast<size_t>(row) : 0;
  const float2* ml = reinterpret_cast<const float2*>(p.ws + p.ml_off) + r * p.max_splits;
  const float4* src = reinterpret_cast<const float4*>(p.ws + p.o_off) + r * p.max_splits * VPR + cv;

  float M = -INFINITY;
  for (int s = cv; s < nw; s += VPR)
    if (s < n) M = fmaxf(M, ml[s].x);
#pragma unroll
  for (int o = VPR / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  for (int s = cv; s < nw; s += VPR)
    if (s < n) {
      const float2 e = ml[s];
      L += e.y * exp2f(e.x - M);
    }
#pragma unroll
  for (int o = VPR / 2; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const float inv = n > 1 ? 1.0f / L : 0.f;

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < nw; s0 += VPR) {
    const int sl = s0 + cv;
    const float wl = sl < n ? exp2f(ml[sl].x - M) * inv : 0.f;
    const int jn = min(VPR, nw - s0);
    for (int j0 = 0; j0 < jn; j0 += 8) {
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int sj = s0 + j0 + j;
        v[j] = sj < n ? __ldg(src + static_cast<size_t>(sj) * VPR) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float w = __shfl_sync(0xffffffffu, wl, base + j0 + j);
        acc.x = fmaf(w, v[j].x, acc.x);
        acc.y = fmaf(w, v[j].y, acc.y);
        acc.z = fmaf(w, v[j].z, acc.z);
        acc.w = fmaf(w, v[j].w, acc.w);
      }
    }
  }
  if (n > 1) reinterpret_cast<float4*>(p.out)[r * VPR + cv] = acc;
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  if (p.max_splits <= 1 || p.num_seqs == 0) return cudaSuccess;
  const int rows_per_cta = (kMergeThreads / 32) * (p.head_dim == 64 ? 2 : 1);
  const int rows = p.num_seqs * p.num_q_heads;
  const dim3 grid((rows + rows_per_cta - 1) / rows_per_cta);
  if (p.head_dim == 64) return launch_pdl(merge_kernel<64>, grid, dim3(kMergeThreads), 0, stream, p);
  if (p.head_dim == 128) return launch_pdl(merge_kernel<128>, grid, dim3(kMergeThreads), 0, stream, p);
  return cudaErrorInvalidValue;
}

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream) {
  // many warps even for small batches: the (level, group) cells are spread over them
  const int threads = kPlanMaxThreads;
  const size_t cells = static_cast<size_t>(p.max_splits) * ((p.num_seqs + 31) / 32);
  const size_t smem = (cells + 2 * static_cast<size_t>(p.num_seqs)) * sizeof(int);
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
