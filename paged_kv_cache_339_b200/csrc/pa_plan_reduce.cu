// Work planning for pa_decode.
//
// plan_kernel (one CTA) reads the context lengths, checks them, picks the
// split size S and cuts every sequence into pieces (work pairs). It lists
// the pairs longest first (bucketed by 128-token chunk count), so the
// persistent decode kernels, which claim pairs in list order, end on short
// pieces and finish together. Pieces: as many whole S-token pieces as fit,
// then the rest of the sequence. The automatic S is one stream's fair share
// of the work (splits cost partial results and a merge, so only sequences
// longer than that are cut), or half a share when there are fewer
// (sequence, KV head) units than streams; when the rests hold too little
// work to even out the streams' finishing times (a few long sequences), each
// sequence's last S-token pieces are cut into tail pieces of about an eighth
// of a share.
//
// The partial results of a split sequence are merged inside the decode
// kernels by the last piece to finish (pa_common.cuh, merge_split_rows); the
// plan zeroes the merge counters they count on.
//
// Launched with programmatic stream serialisation: it may start while the KV
// write before it is still running (it reads only the lengths and rewrites
// the workspace), and waits for that kernel before it writes the zero rows of
// empty sequences into `out` and exits, so the decode kernel that waits on
// the plan also sees the new tokens.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kPlanMaxThreads = 1024;
constexpr int kKeys = 64;   // length buckets: 1..63 chunks of 128 tokens, and >= 64 chunks

__device__ __forceinline__ int piece_key(int tokens) {
  const int k = (tokens + 127) >> 7;
  return k < kKeys ? k : kKeys;
}

struct PieceRule {
  int S;      // whole-piece size
  int cut;    // 1: the last `e` whole pieces (and the rest) are cut into ~sB-token pieces
  int e, sB, ms;
};

// Pieces of one sequence of L tokens: nA whole pieces of S tokens, then the
// remaining L - nA*S tokens as k pieces of sb tokens (the last one shorter).
// n = nA + k <= ms always: S >= max_context_len / ms by the workspace sizing.
__device__ __forceinline__ void seq_pieces(int L, const PieceRule& r, int& nA, int& sb, int& k) {
  const int nf = L / r.S;
  if (!r.cut) {
    nA = nf;
    sb = L - nf * r.S;
    k = sb > 0 ? 1 : 0;
    return;
  }
  nA = nf - min(r.e, nf);
  const int rest = L - nA * r.S;
  if (rest == 0) {
    sb = 0;
    k = 0;
    return;
  }
  const int room = r.ms - nA;   // >= 1: nA * S < L <= ms * S
  const int need = (rest + room - 1) / room;
  sb = need > r.sB ? (need + 127) / 128 * 128 : r.sB;
  k = (rest + sb - 1) / sb;
}

__global__ void __launch_bounds__(kPlanMaxThreads, 1) plan_kernel(PlanParams p) {
  pdl_launch_dependents();
  __shared__ long long s_sum[32];
  __shared__ int s_bad[32];
  __shared__ int s_hist[kKeys + 1];
  __shared__ int s_fill[kKeys + 1];
  __shared__ PieceRule s_rule;
  __shared__ int s_nsplit_seqs;
  extern __shared__ int s_len[];   // [num_seqs]

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  WorkPair* pairs = reinterpret_cast<WorkPair*>(p.ws + p.pairs_off);
  int32_t* nsplit = reinterpret_cast<int32_t*>(p.ws + p.nsplit_off);
  int32_t* cnt = reinterpret_cast<int32_t*>(p.ws + p.cnt_off);
  int32_t* split_list = reinterpret_cast<int32_t*>(p.ws + p.split_off);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_nsplit_seqs = 0;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int64_t cap = static_cast<int64_t>(p.bt_stride) * p.block_size;
  auto valid_len = [&](int L) { return !(L < 0 || L > p.max_context_len || L > cap); };

  // 1. validate lengths; total
  long long tot = 0;
  int bad = 0;
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = p.context_lens[i];
    s_len[i] = L;
    if (!valid_len(L)) {
      bad = 1;
    } else {
      tot += L;
    }
  }
  for (int k = tid; k <= kKeys; k += nthreads) s_hist[k] = 0;

#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (lane == 0) {
    s_sum[warp] = tot;
    s_bad[warp] = bad;
  }
  __syncthreads();
  if (warp == 0) {
    long long t = lane < nwarps ? s_sum[lane] : 0;
    int b = lane < nwarps ? s_bad[lane] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t += __shfl_xor_sync(0xffffffffu, t, o);
      b |= __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
      // one stream's fair share of the work, in tokens of one KV head
      const long long share = (t * p.num_kv_heads + p.num_ctas - 1) / p.num_ctas;
      int S = p.split_tokens;
      if (S <= 0) {
        // Whole pieces of up to one share: every split costs partial results
        // and a merge, so only sequences longer than a share are cut; the
        // longest-first order evens the CTAs out with the short sequences.
        // With fewer (sequence, KV head) units than streams there are no
        // short sequences to do that: every stream works on pieces of the
        // few long ones, and a stream whose CTA partner has run dry slows
        // down. Pieces of half a share then give each stream two or more,
        // so the claiming order can even them out.
        long long base = share;
        if (static_cast<long long>(p.num_seqs) * p.num_kv_heads < p.num_ctas)
          base = (share + 1) / 2;
        long long want = (base + kAutoSplitQuantum - 1) / kAutoSplitQuantum * kAutoSplitQuantum;
        if (want < p.min_split) want = p.min_split;
        if (want > (1 << 30)) want = 1 << 30;
        S = static_cast<int>(want);
      }
      s_rule.S = S;
      s_rule.cut = 0;
      s_rule.e = 0;
      // tail pieces, if the list needs them: about an eighth of a share
      long long sb = share / 8 / kAutoSplitQuantum * kAutoSplitQuantum;
      if (sb < kAutoSplitQuantum) sb = kAutoSplitQuantum;
      if (sb > S) sb = S;
      s_rule.sB = static_cast<int>(sb);
      s_rule.ms = p.max_splits;
      hdr->status = b ? 1 /* PA_ERR_INVALID_ARG */ : 0;
      hdr->split_tokens = S;
      hdr->max_splits = p.max_splits;
    }
  }
  __syncthreads();
  const int S = s_rule.S;

  // 2. short work: the rests (pieces shorter than S) of at most two tail
  // pieces, in tokens of one KV head
  if (p.split_tokens <= 0) {
    const int short_max = 2 * s_rule.sB;
    long long rem = 0;
    for (int i = tid; i < p.num_seqs; i += nthreads) {
      const int L = s_len[i];
      const int rest = valid_len(L) ? L % S : 0;
      if (rest <= short_max) rem += rest;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rem += __shfl_xor_sync(0xffffffffu, rem, o);
    if (lane == 0) s_sum[warp] = rem;
    __syncthreads();
    if (warp == 0) {
      long long r = lane < nwarps ? s_sum[lane] : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
      // The list should end on enough short work to even the streams out:
      // about two tail pieces per stream. Few or equally long sequences
      // leave too little in short rests; then the last whole pieces (and
      // rest) of every sequence are cut into tail pieces.
      const long long target =
          2LL * p.num_ctas * s_rule.sB / p.num_kv_heads;   // tokens of one KV head
      if (lane == 0 && r < target && p.num_seqs > 0) {
        const long long per_seq = static_cast<long long>(p.num_seqs) * S;
        s_rule.cut = 1;
        s_rule.e = static_cast<int>(min((target - r + per_seq - 1) / per_seq, 1LL << 20));
      }
    }
    __syncthreads();
  }
  const PieceRule rule = s_rule;

  // 3. pieces per sequence (a thread per sequence): split counts, zeroed merge
  // counters and the list of split sequences, and the length histogram (a
  // sequence's pieces form at most three runs of equal length)
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = s_len[i];
    int nA = 0, sb = 0, k = 0;
    if (valid_len(L) && L > 0) seq_pieces(L, rule, nA, sb, k);
    const int n = nA + k;
    nsplit[i] = n;
    if (n > 1) {
      for (int h = 0; h < p.num_kv_heads; ++h) cnt[static_cast<size_t>(i) * p.num_kv_heads + h] = 0;
      split_list[atomicAdd(&s_nsplit_seqs, 1)] = i;
    }
    if (nA > 0) atomicAdd(&s_hist[piece_key(S)], nA);
    if (k > 1) atomicAdd(&s_hist[piece_key(sb)], k - 1);
    if (k > 0) atomicAdd(&s_hist[piece_key(L - nA * S - (k - 1) * sb)], 1);
  }
  __syncthreads();
  // 4. longest first: bucket bases in descending length order (warp 0 scans
  // the kKeys buckets, two per lane)
  if (warp == 0) {
    const int k0 = kKeys - 2 * lane, k1 = k0 - 1;   // descending keys
    const int h0 = s_hist[k0], h1 = k1 >= 1 ? s_hist[k1] : 0;
    int inc = h0 + h1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    const int excl = inc - h0 - h1;
    s_fill[k0] = excl;
    if (k1 >= 1) s_fill[k1] = excl + h0;
    if (lane == 31) {
      hdr->num_pairs = inc;
      hdr->num_items = inc * p.num_kv_heads;
      // every item stream takes item (its index) first without claiming it
      // (no atomic on the start-up path); claims continue from here
      hdr->work_counter = p.num_ctas;
      hdr->num_split_seqs = s_nsplit_seqs;
      hdr->merge_counter = 0;
    }
  }
  __syncthreads();
  // 5. place every piece: a thread per sequence reserves each run's slots
  // with one atomic. The order inside a bucket is whatever the atomics give;
  // results do not depend on it (every piece's split index and token range
  // are fixed by the sequence).
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = s_len[i];
    if (!valid_len(L) || L == 0) continue;
    int nA, sb, k;
    seq_pieces(L, rule, nA, sb, k);
    const int n = nA + k;
    WorkPair w;
    w.seq = i;
    if (nA > 0) {
      const int pos = atomicAdd(&s_fill[piece_key(S)], nA);
      for (int j = 0; j < nA; ++j) {
        w.split_n = j | (n << 16);
        w.t_begin = j * S;
        w.t_end = w.t_begin + S;
        pairs[pos + j] = w;
      }
    }
    if (k > 1) {
      const int pos = atomicAdd(&s_fill[piece_key(sb)], k - 1);
      for (int q = 0; q < k - 1; ++q) {
        w.split_n = (nA + q) | (n << 16);
        w.t_begin = nA * S + q * sb;
        w.t_end = w.t_begin + sb;
        pairs[pos + q] = w;
      }
    }
    if (k > 0) {
      w.split_n = (n - 1) | (n << 16);
      w.t_begin = nA * S + (k - 1) * sb;
      w.t_end = L;
      pairs[atomicAdd(&s_fill[piece_key(L - w.t_begin)], 1)] = w;
    }
  }
  // complete only after the kernel before this one (the KV write) has
  pdl_wait();
  // Sequences with nothing to attend to get zero rows. These stores come
  // after the wait: the kernel before this one may still read or write `out`
  // until it has completed.
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = s_len[i];
    if (valid_len(L) && L > 0) continue;
    float4* row = reinterpret_cast<float4*>(
        p.out + static_cast<size_t>(i) * p.num_q_heads * p.head_dim);
    const int n4 = p.num_q_heads * p.head_dim / 4;
    for (int e = 0; e < n4; ++e) row[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

}  // namespace

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream) {
  // a thread per sequence
  int threads = (p.num_seqs + 31) / 32 * 32;
  threads = threads < 128 ? 128 : (threads > kPlanMaxThreads ? kPlanMaxThreads : threads);
  const size_t smem = static_cast<size_t>(p.num_seqs) * sizeof(int);
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
  // the largest shared-memory carveout, as the decode kernels use: an SM that
  // ran this kernel need not be reconfigured before it takes a decode CTA
  cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, plan_kernel, p);
}

}  // namespace pa
