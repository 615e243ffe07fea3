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
#include <climits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kPlanMaxThreads = 1024;
constexpr int kKeys = 64;   // length buckets: 1..63 chunks of 128 tokens, and >= 64 chunks
// Shared prefixes: a group needs at least this many common tokens, and its
// common whole pieces are at most this long (automatic split).
constexpr int kShareMinTokens = 256;
constexpr int kShareSplit = 512;

__device__ __forceinline__ int piece_key(int tokens) {
  const int k = (tokens + 127) >> 7;
  return k < kKeys ? k : kKeys;
}

struct PieceRule {
  int S;      // whole-piece size
  int cut;    // 1: the last `e` whole pieces (and the rest) are cut into ~sB-token pieces
  int e, sB, ms;
  int q;      // tail pieces are multiples of q tokens (one ring position)
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
  sb = need > r.sB ? (need + r.q - 1) / r.q * r.q : r.sB;
  k = (rest + sb - 1) / sb;
}

// Inclusive scans over the CTA's threads in thread order (every thread
// calls them; tmp: 32 shared ints).
__device__ __forceinline__ int block_scan_max(int v, int* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = max(v, n);
  }
  if (lane == 31) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? tmp[lane] : INT_MIN;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t = max(t, n);
    }
    if (lane < nw) tmp[lane] = t;
  }
  __syncthreads();
  if (warp > 0) v = max(v, tmp[warp - 1]);
  __syncthreads();
  return v;
}
__device__ __forceinline__ int block_scan_sum(int v, int* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    if (lane < nw) tmp[lane] = t;
  }
  __syncthreads();
  if (warp > 0) v += tmp[warp - 1];
  __syncthreads();
  return v;
}

// SHARE: also group sequences that share leading blocks (one thread per
// sequence: launched with kPlanMaxThreads threads, num_seqs <= kShareMaxSeqs).
template <bool SHARE>
__global__ void __launch_bounds__(kPlanMaxThreads, 1) plan_kernel(PlanParams p) {
  pdl_launch_dependents();
  __shared__ long long s_sum[32];
  __shared__ int s_bad[32];
  __shared__ int s_hist[kKeys + 1];
  __shared__ int s_fill[kKeys + 1];
  __shared__ PieceRule s_rule;
  __shared__ int s_nsplit_seqs;
  __shared__ int s_ngroups, s_ngpairs;
  __shared__ int s_scan[32];
  extern __shared__ int s_len[];   // [num_seqs]; with shared prefixes 4 more arrays follow
  // shared prefixes: per sequence, the leading full blocks it shares with the
  // one before it, then (at a group's first member) the group's common whole
  // pieces; the group's first member (or -1); at the first member, the common
  // prefix in tokens, then the member count; at the first member, the group's
  // first slot in the group list
  int* s_aux = s_len + p.num_seqs;
  int* s_lead = s_aux + p.num_seqs;
  int* s_pre = s_lead + p.num_seqs;
  int* s_goff = s_pre + p.num_seqs;

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  WorkPair* pairs = reinterpret_cast<WorkPair*>(p.ws + p.pairs_off);
  int32_t* nsplit = reinterpret_cast<int32_t*>(p.ws + p.nsplit_off);
  int32_t* cnt = reinterpret_cast<int32_t*>(p.ws + p.cnt_off);
  int32_t* split_list = reinterpret_cast<int32_t*>(p.ws + p.split_off);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    s_nsplit_seqs = 0;
    s_ngroups = 0;
    s_ngpairs = 0;
  }
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
  if constexpr (SHARE) {
    // 1b. Shared prefixes ("Paged Attention: Virtual Memory for the KV
    // Cache", "Sharing comes almost for free": sequences forked from one
    // another point at the same physical blocks). Each sequence counts the
    // leading full blocks its table has in common with the previous
    // sequence's: a thread per sequence checks the first entry, then a warp
    // per sequence whose first entries match compares the rest, 256 entries
    // per round (8 loads in flight per lane).
    const int i = tid;   // num_seqs <= threads
    int La = 0, nb = 0;
    if (i < p.num_seqs) {
      La = s_len[i];
      const int Lb = i > 0 ? s_len[i - 1] : 0;
      nb = i > 0 && valid_len(La) && valid_len(Lb) ? min(La, Lb) / p.block_size : 0;
      if (nb > 0) {
        const int32_t* ra = p.block_tables + static_cast<size_t>(i) * p.bt_stride;
        if (ra[0] != ra[-p.bt_stride]) nb = 0;
      }
      s_aux[i] = nb;   // an upper bound, exact below
      s_lead[i] = -1;
    }
    __syncthreads();
    for (int w = warp; w < p.num_seqs; w += nwarps) {
      const int n = s_aux[w];
      if (n <= 1) continue;
      const int32_t* ra = p.block_tables + static_cast<size_t>(w) * p.bt_stride;
      const int32_t* rb = ra - p.bt_stride;
      int common = n;
      for (int j0 = 0; j0 < n; j0 += 256) {
        bool diff[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + 32 * q + lane;
          diff[q] = j < n && ra[j] != rb[j];
        }
        unsigned first = 0xffffffffu;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const unsigned m = __ballot_sync(0xffffffffu, diff[q]);
          if (m != 0u && first == 0xffffffffu) first = 32 * q + __ffs(m) - 1;
        }
        if (first != 0xffffffffu) {
          common = j0 + static_cast<int>(first);
          break;
        }
      }
      if (lane == 0) s_aux[w] = common;
    }
    __syncthreads();
    // Groups: runs of consecutive sequences each sharing >= kShareMinTokens
    // with the one before, cut into groups of at most share_members members
    // (their query rows fill one 16-row tile). A run starts at the last
    // sequence that does not share with its predecessor (a max scan); a
    // member whose offset in its run is a multiple of share_members leads a
    // group if the next sequence is in the run too. The group's common
    // prefix is the smallest count among its members after the first.
    auto shares = [&](int j) { return s_aux[j] * p.block_size >= kShareMinTokens; };
    const bool in = i < p.num_seqs;
    const int run_start = block_scan_max(in && !(i > 0 && shares(i)) ? i : -1, s_scan);
    const bool leader = in && (i - run_start) % p.share_members == 0 && i + 1 < p.num_seqs &&
                        shares(i + 1);
    if (leader) {
      int m = i + 1, P = 1 << 30;
      for (; m < p.num_seqs && m - i < p.share_members && shares(m); ++m) P = min(P, s_aux[m]);
      s_pre[i] = P * p.block_size;
      s_goff[i] = m - i;   // members, until the offsets are known
    }
    const int any = __syncthreads_or(leader);
    if (leader) {
      for (int m = i; m < i + s_goff[i]; ++m) s_lead[m] = i;
    }
    if (tid == 0) s_ngroups = any;
    __syncthreads();
  }
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
        // groups share whole pieces: keep them short enough that a prefix
        // holds several
        if (s_ngroups > 0) {
          const long long cap_s = p.min_split > kShareSplit ? p.min_split : kShareSplit;
          if (want > cap_s) want = cap_s;
        }
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
      s_rule.q = kAutoSplitQuantum;
      hdr->status = b ? 1 /* PA_ERR_INVALID_ARG */ : 0;
      hdr->max_splits = p.max_splits;
    }
  }
  __syncthreads();

  // 2. short work: the rests (pieces shorter than S) of at most two tail
  // pieces, in tokens of one KV head
  if (p.split_tokens <= 0) {
    const int S1 = s_rule.S, short_max = 2 * s_rule.sB;
    long long rem = 0;
    for (int i = tid; i < p.num_seqs; i += nthreads) {
      const int L = s_len[i];
      const int rest = valid_len(L) ? L % S1 : 0;
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
        const long long per_seq = static_cast<long long>(p.num_seqs) * S1;
        s_rule.cut = 1;
        s_rule.e = static_cast<int>(min((target - r + per_seq - 1) / per_seq, 1LL << 20));
      }
      // Paired KV heads: an item token is a token of two heads, so the same
      // work takes half the tokens: whole and tail pieces of half the size
      // (whole pieces no shorter than the workspace's bound on pieces per
      // sequence allows), twice as many cut, in multiples of one 64-token
      // ring position.
      if (lane == 0 && p.pair_heads) {
        s_rule.S = max(s_rule.S / 2, p.min_split);
        s_rule.sB = min(max(s_rule.sB / 2, kAutoSplitQuantum / 2), s_rule.S);
        s_rule.e = min(2 * s_rule.e, 1 << 20);
        s_rule.q = kAutoSplitQuantum / 2;
      }
    }
    __syncthreads();
  }
  const PieceRule rule = s_rule;
  const int S = rule.S;
  if (tid == 0) hdr->split_tokens = S;
  // KV heads per sequence as the items count them (pairs when paired)
  const int Hi = p.pair_heads ? p.num_kv_heads / 2 : p.num_kv_heads;

  if constexpr (SHARE) {
    // 2b. A group's common whole pieces: the S-token pieces inside its
    // common prefix, short of every member's last token (so each member
    // keeps a piece of its own, which completes and merges its result). The
    // group list gets them once, with the members' query rows; each member's
    // own part (the rest of its sequence) is cut by the usual rule, with that
    // many pieces fewer of room. Group list offsets: a sum scan.
    const int i = tid;
    const bool leader = i < p.num_seqs && s_lead[i] == i;
    int kg = 0, members = 0;
    if (leader) {
      members = s_goff[i];
      kg = s_pre[i] / S;
      for (int m = i; m < i + members; ++m) kg = min(kg, (s_len[m] - 1) / S);
    }
    const int incl = block_scan_sum(kg, s_scan);
    if (leader) {
      s_aux[i] = kg;
      s_pre[i] = members;
      s_goff[i] = incl - kg;
    }
    if (tid == nthreads - 1) {
      s_ngpairs = incl;
      hdr->num_group_items = incl * p.num_kv_heads;
      hdr->group_work_counter = p.group_ctas;
    }
    __syncthreads();
  }
  // whole pieces of sequence i that a group lists for it
  auto shared_pieces = [&](int i) { return SHARE && s_lead[i] >= 0 ? s_aux[s_lead[i]] : 0; };
  auto s_lead_is = [&](int i) { return SHARE && s_lead[i] == i; };
  WorkPair* gpairs = reinterpret_cast<WorkPair*>(p.ws + p.gpairs_off);
  // pieces of sequence i (valid, L > 0): the kg whole pieces its group lists,
  // then its own part [kg*S, L) as nA whole pieces of S tokens and k pieces
  // of sb tokens (the last one shorter); n = kg + nA + k <= ms
  auto pieces_of = [&](int i, int L, int& kg, int& nA, int& sb, int& k) {
    kg = shared_pieces(i);
    PieceRule r = rule;
    r.ms -= kg;
    seq_pieces(L - kg * S, r, nA, sb, k);
  };

  // 3. pieces per sequence (a thread per sequence): split counts, zeroed merge
  // counters and the list of split sequences, and the length histogram (a
  // sequence's pieces form at most three runs of equal length)
  for (int i = tid; i < p.num_seqs; i += nthreads) {
    const int L = s_len[i];
    int kg = 0, nA = 0, sb = 0, k = 0;
    if (valid_len(L) && L > 0) pieces_of(i, L, kg, nA, sb, k);
    const int n = kg + nA + k;
    nsplit[i] = n;
    if (n > 1) {
      for (int h = 0; h < Hi; ++h) cnt[static_cast<size_t>(i) * Hi + h] = 0;
      split_list[atomicAdd(&s_nsplit_seqs, 1)] = i;
    }
    if (nA > 0) atomicAdd(&s_hist[piece_key(S)], nA);
    if (k > 1) atomicAdd(&s_hist[piece_key(sb)], k - 1);
    if (k > 0) atomicAdd(&s_hist[piece_key(L - kg * S - nA * S - (k - 1) * sb)], 1);
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
      hdr->num_items = inc * Hi;
      if (!SHARE) hdr->num_group_items = 0;
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
    int kg, nA, sb, k;
    pieces_of(i, L, kg, nA, sb, k);
    const int n = kg + nA + k, base = kg * S;
    // a member's only own piece folds the group pieces in itself
    const int32_t fold = kg > 0 && nA + k == 1 ? kFoldGroupPieces : 0;
    WorkPair w;
    w.seq = i;
    if (nA > 0) {
      const int pos = atomicAdd(&s_fill[piece_key(S)], nA);
      for (int j = 0; j < nA; ++j) {
        w.split_n = (kg + j) | (n << 16) | fold;
        w.t_begin = base + j * S;
        w.t_end = w.t_begin + S;
        pairs[pos + j] = w;
      }
    }
    if (k > 1) {
      const int pos = atomicAdd(&s_fill[piece_key(sb)], k - 1);
      for (int q = 0; q < k - 1; ++q) {
        w.split_n = (kg + nA + q) | (n << 16);
        w.t_begin = base + nA * S + q * sb;
        w.t_end = w.t_begin + sb;
        pairs[pos + q] = w;
      }
    }
    if (k > 0) {
      w.split_n = (n - 1) | (n << 16) | fold;
      w.t_begin = base + nA * S + (k - 1) * sb;
      w.t_end = L;
      pairs[atomicAdd(&s_fill[piece_key(L - w.t_begin)], 1)] = w;
    }
    if (s_lead_is(i)) {
      // the group list: the group's common whole pieces, each with the
      // members' count in place of the split count
      WorkPair g;
      g.seq = i;
      for (int j = 0; j < kg; ++j) {
        g.split_n = j | (s_pre[i] << 16);
        g.t_begin = j * S;
        g.t_end = g.t_begin + S;
        gpairs[s_goff[i] + j] = g;
      }
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
  // a thread per sequence (all threads for the table comparison of shared
  // prefixes)
  int threads = (p.num_seqs + 31) / 32 * 32;
  threads = threads < 128 ? 128 : (threads > kPlanMaxThreads ? kPlanMaxThreads : threads);
  if (p.share_prefixes) threads = kPlanMaxThreads;
  auto kern = p.share_prefixes ? plan_kernel<true> : plan_kernel<false>;
  // the lengths, and with shared prefixes four more arrays per sequence
  const size_t smem = static_cast<size_t>(p.num_seqs) * sizeof(int) * (p.share_prefixes ? 5 : 1);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace pa
