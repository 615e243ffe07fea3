// Paged decode on CUDA cores (any dtype, head_dim 64/128, up to 16 query
// heads per KV head). Used for MHA, fp32 caches and small GQA groups, where
// the work is about one FMA per byte read and tensor cores would only add
// padding.
//
// Persistent, warp-specialised CTA:
//   warp 0      producer: claims work items (sequence, split, KV head) from the
//               planned list, reads the block table, and streams each chunk of
//               64 logical tokens into a shared-memory ring with cp.async.bulk:
//               one bulk copy per (block, KV head) tile for K and one for V
//               (the tile is contiguous in the pool layout), completion tracked
//               by an mbarrier transaction count.
//   warps 1..4  consumers: scores with 8 lanes per token (16-byte shared loads,
//               3 shuffle steps), an online softmax in log2 units per
//               16-token sub-block, P.V with each lane owning head_dim/32
//               output columns; at the end of an item the warps' partial
//               (max, sum, acc) are merged and written as the final row or as a
//               split partial.
// Tiles are kept in the in-block storage order (pa_common.cuh) in shared
// memory too; rows are addressed through it.
// The block table is followed page by page, so the sequence is read in its
// logical order although its blocks sit anywhere in the pool ("Paged
// Attention: Virtual Memory for the KV Cache", "The fix borrowed from
// operating systems"; glossary "Paged attention", "What is Paged Attention?").
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

struct __align__(16) ChunkMeta {
  int32_t seq, kvh, split_raw, t0, valid, flags, pad0, pad1;
};

template <typename T, int D, int GPW>
struct SimtTraits {
  static constexpr int E = sizeof(T);
  static constexpr int ROW = D * E;            // bytes of one token's K (or V) row
  static constexpr int CHUNK = 64;             // tokens per pipeline stage
  static constexpr int NCW = 4;                // consumer warps
  static constexpr int NTHREADS = (NCW + 1) * 32;
  static constexpr int STAGE = 2 * CHUNK * ROW;  // K rows, then V rows
  static constexpr int NST_RAW = (96 * 1024) / STAGE;
  static constexpr int NST = NST_RAW < 3 ? 3 : (NST_RAW > 8 ? 8 : NST_RAW);
  static constexpr int NV = ROW / 128;         // 16-B vectors per lane per score row
  static constexpr int EPV = 16 / E;           // elements per 16-B vector
  static constexpr int QPL = NV * EPV;         // q elements per lane per head (= D/8)
  static constexpr int EPL = D / 32;           // output columns per lane
  static constexpr int PVB = ROW / 32;         // bytes per lane per V row
  static constexpr int SUB = 16;               // tokens per softmax sub-block
  static constexpr int NH = D / 64;            // 64-element halves per row
  static constexpr int HALF = 64 * E;          // bytes of one half-row
  static constexpr int CMB = GPW * D + 2 * GPW;  // floats per warp in the merge area
  static constexpr size_t OFF_BAR = static_cast<size_t>(NST) * STAGE;
  static constexpr size_t OFF_META = OFF_BAR + (2 * NST + 2) * 8;
  static constexpr size_t OFF_PSCR = (OFF_META + NST * sizeof(ChunkMeta) + 15) / 16 * 16;
  static constexpr size_t OFF_CMB = OFF_PSCR + NCW * SUB * 4 * 4;
  static constexpr size_t OFF_ABORT = OFF_CMB + NCW * CMB * 4;
  static constexpr size_t SMEM = OFF_ABORT + 16;
  static_assert(NV >= 1, "row must be at least 128 bytes");
  static_assert(OFF_BAR % 16 == 0 && OFF_META % 16 == 0 && OFF_PSCR % 16 == 0 &&
                    OFF_CMB % 16 == 0 && OFF_ABORT % 16 == 0,
                "16-byte aligned shared regions");
  static_assert(EPL == 2 || EPL == 4, "head_dim 64 or 128");
};

template <typename T, int N>
__device__ __forceinline__ void load_row_slice(const uint8_t* src, float* f) {
  // N bytes (4, 8 or 16) of a row, widened to fp32
  if constexpr (N == 16) {
    unpack16<T>(*reinterpret_cast<const uint4*>(src), f);
  } else if constexpr (N == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    if constexpr (sizeof(T) == 4) {
      f[0] = __uint_as_float(w.x);
      f[1] = __uint_as_float(w.y);
    } else {
      Elem<T>::unpack2(w.x, f);
      Elem<T>::unpack2(w.y, f + 2);
    }
  } else {
    static_assert(N == 4 && sizeof(T) == 2, "4-byte slices are 16-bit pairs");
    Elem<T>::unpack2(*reinterpret_cast<const uint32_t*>(src), f);
  }
}

// Bounded arrive-and-wait among the consumer threads (an mbarrier, so a
// stalled peer cannot hang the others).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase,
                                           volatile int* abrt, int* status) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, abrt, status);
  phase ^= 1u;
  return ok;
}

// Wait used only on the way out after an abort: bounded, ignores the flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
}

// GRP: the launch over the group list of shared prefixes (group items only).
template <typename T, int D, int GPW, bool GRP>
__global__ void __launch_bounds__(SimtTraits<T, D, GPW>::NTHREADS, 2)
    simt_decode_kernel(const DecodeParams p) {
  __shared__ volatile int s_last;   // this piece completed its sequence
  __shared__ volatile int s_lastm[16];   // group items: this piece completed member m
  using Tr = SimtTraits<T, D, GPW>;
  constexpr int CHUNK = Tr::CHUNK, ROW = Tr::ROW, NST = Tr::NST;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* gbar = empty + NST;
  ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(smem + Tr::OFF_META);
  float* pscr = reinterpret_cast<float*>(smem + Tr::OFF_PSCR);
  float* cmb = reinterpret_cast<float*>(smem + Tr::OFF_CMB);
  volatile int* abrt = reinterpret_cast<volatile int*>(smem + Tr::OFF_ABORT);

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  int* status = &hdr->status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Tr::NCW);
    }
    mbar_init(&gbar[0], Tr::NCW * 32);
    *abrt = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();   // the plan (and the KV write before it) are complete from here on
  // (no early launch of dependents: the next call's plan rewrites the workspace)

  // the group list (shared prefixes) or the work list
  const int num_items = GRP ? hdr->num_group_items : hdr->num_items;
  int* const work_counter = GRP ? &hdr->group_work_counter : &hdr->work_counter;
  const int Hkv = p.num_kv_heads, BS = p.block_size;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const WorkPair* pairs =
        reinterpret_cast<const WorkPair*>(p.ws + (GRP ? p.gpairs_off : p.pairs_off));
    const uint64_t pol = l2_evict_first_policy();   // K and V tiles: read once per call
    uint32_t c = 0;
    bool ok = true;
    // the first item is this CTA's own (the plan starts the claim counter
    // after one item per CTA)
    int kraw = blockIdx.x;
    int k = static_cast<int>(blockIdx.x);
    while (k < num_items) {
      const int pi = k / Hkv, kvh = k - pi * Hkv;
      const WorkPair wp = pairs[pi];
      const int32_t* bt_row = p.block_tables + static_cast<size_t>(wp.seq) * p.bt_stride;
      bool claimed = false;
      for (int cs = wp.t_begin; cs < wp.t_end; cs += CHUNK) {
        // next claim in flight two chunks before this item ends (a claim held
        // for a whole item would lengthen the tail)
        if (!claimed && wp.t_end - cs <= 2 * CHUNK) {
          if (lane == 0) kraw = atomicAdd(work_counter, 1);
          claimed = true;
        }
        const int valid = min(CHUNK, wp.t_end - cs);
        const int npg = (valid + BS - 1) / BS;
        int blk = 0;
        if (lane < npg) {
          blk = bt_row[cs / BS + lane];
          if (blk < 0 || blk >= p.num_blocks) {
            atomicCAS(status, 0, 1 /* PA_ERR_INVALID_ARG */);
            blk = 0;
          }
        }
        const int stage = c % NST;
        if (!mbar_wait(&empty[stage], ((c / NST) & 1u) ^ 1u, abrt, status)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          ChunkMeta m;
          m.seq = wp.seq;
          m.kvh = kvh;
          m.split_raw = wp.split_n;
          m.t0 = cs;
          m.valid = valid;
          m.flags = (cs == wp.t_begin ? kFirst : 0) | (cs + CHUNK >= wp.t_end ? kLast : 0);
          m.pad0 = m.pad1 = 0;
          meta[stage] = m;
          mbar_arrive_expect_tx(&full[stage], 2u * valid * ROW);
        }
        __syncwarp();
        if (lane < npg) {
          // one copy per tile; a partly used last tile copies only its valid
          // rows, one 16-token half-row segment at a time
          const int rows = min(BS, valid - lane * BS);
          const size_t src = (static_cast<size_t>(blk) * Hkv + kvh) * BS * ROW;
          const uint8_t* gk = static_cast<const uint8_t*>(p.k_cache) + src;
          const uint8_t* gv = static_cast<const uint8_t*>(p.v_cache) + src;
          uint8_t* dk = stages + static_cast<size_t>(stage) * Tr::STAGE + lane * BS * ROW;
          if (rows == BS || Tr::NH == 1) {
            bulk_g2s_hint(dk, gk, rows * ROW, &full[stage], pol);
            bulk_g2s_hint(dk + CHUNK * ROW, gv, rows * ROW, &full[stage], pol);
          } else {
            const int sh = tile_sub_height(BS);
            for (int sp = 0; sp * sh < rows; ++sp) {
              const uint32_t nb = static_cast<uint32_t>(min(sh, rows - sp * sh)) * Tr::HALF;
#pragma unroll
              for (int h = 0; h < Tr::NH; ++h) {
                const int seg = (sp * Tr::NH + h) * sh * Tr::HALF;
                bulk_g2s_hint(dk + seg, gk + seg, nb, &full[stage], pol);
                bulk_g2s_hint(dk + CHUNK * ROW + seg, gv + seg, nb, &full[stage], pol);
              }
            }
          }
        }
        ++c;
      }
      if (!ok) break;
      if (!claimed && lane == 0) kraw = atomicAdd(work_counter, 1);
      k = __shfl_sync(kFull, kraw, 0);
    }
    if (ok) {
      const int stage = c % NST;
      if (mbar_wait(&empty[stage], ((c / NST) & 1u) ^ 1u, abrt, status)) {
        if (lane == 0) {
          meta[stage].flags = kEnd;
          mbar_arrive(&full[stage]);
        }
      } else {
        ok = false;
      }
    }
    if (!ok && lane == 0) {
      // copies may still be landing in the last NST stages: let them finish
      for (uint32_t cc = c > NST ? c - NST : 0; cc < c; ++cc)
        drain_wait(&full[cc % NST], (cc / NST) & 1u);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1;
    const int G = p.num_q_heads / Hkv;
    // query rows an item has at most: G, or 16 for group items (members x G)
    const int GL = GRP ? 16 : G;
    const int HG = (GL + GPW - 1) / GPW;
    const int HGp = HG <= 1 ? 1 : (HG <= 2 ? 2 : 4);
    const int WPG = Tr::NCW / HGp;
    const int hg = cw / WPG, wg = cw % WPG;
    const bool active = hg < HG;
    const int TPW = CHUNK / WPG;
    const int gi = lane >> 3, j = lane & 7;
    float* ps_w = pscr + cw * Tr::SUB * 4;
    // in-block storage order: byte offset of token t's first half-row inside
    // a stage region (pages packed in table order); half h adds h * seg
    const int bs_shift = __ffs(BS) - 1;
    const int sh = tile_sub_height(BS), sh_shift = __ffs(sh) - 1;
    const int seg = sh * Tr::HALF;
    auto row_off = [&](int t) -> int {
      const int r = t & (BS - 1);
      return (t >> bs_shift) * BS * ROW + (r >> sh_shift) * Tr::NH * seg + (r & (sh - 1)) * Tr::HALF;
    };
    // Rows of consecutive groups of sh tokens are sh * ROW bytes apart (pages
    // are packed), so inside a 16-token sub-block (which starts on a multiple of
    // 16) token tb + i is at row_off(tb) + (i / sh) * sh * ROW + (i % sh) * HALF.
    const int grp_stride = sh * ROW;
    // score loads: vector j + 8v of a row lies in half v * EPV / 8
    int kofs[Tr::NV];
#pragma unroll
    for (int v = 0; v < Tr::NV; ++v)
      kofs[v] = ((v * Tr::EPV) >> 3) * seg + ((j + 8 * v) * 16) % Tr::HALF;
    // PV: this lane's columns d = lane * EPL .. lie in half (lane * EPL) / 64
    const int pv_off = ((lane * Tr::EPL) >> 6) * seg + (lane * Tr::PVB) % Tr::HALF;
    float q[GPW][Tr::QPL];
    float m[GPW], l[GPW], o[GPW][Tr::EPL];
    uint32_t c = 0, gphase = 0;

    while (true) {
      const int stage = c % NST;
      if (!mbar_wait(&full[stage], (c / NST) & 1u, abrt, status)) break;
      const ChunkMeta mt = meta[stage];
      if (mt.flags & kEnd) break;
      if (mt.flags & kFirst) {
#pragma unroll
        for (int g = 0; g < GPW; ++g) {
          m[g] = -INFINITY;
          l[g] = 0.f;
#pragma unroll
          for (int e = 0; e < Tr::EPL; ++e) o[g][e] = 0.f;
          // query row of row slot hl (spare slots repeat the first row): head
          // hl of the sequence, or for a group item head hl % G of member hl / G
          const int hl = hg * GPW + g;
          size_t qr;
          if constexpr (GRP) {
            const int hr = hl < item_nsplit(mt.split_raw) * G ? hl : 0;
            const int mb = hr / G;
            qr = static_cast<size_t>(mt.seq + mb) * p.num_q_heads + mt.kvh * G + (hr - mb * G);
          } else {
            qr = static_cast<size_t>(mt.seq) * p.num_q_heads + mt.kvh * G + (hl < G ? hl : 0);
          }
          const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + qr * ROW;
#pragma unroll
          for (int v = 0; v < Tr::NV; ++v) {
            float f[Tr::EPV];
            unpack16<T>(*reinterpret_cast<const uint4*>(qrow + (j + 8 * v) * 16), f);
#pragma unroll
            for (int e = 0; e < Tr::EPV; ++e) q[g][v * Tr::EPV + e] = f[e] * p.scale_log2;
          }
        }
      }
      if (active) {
        const uint8_t* Kst = stages + static_cast<size_t>(stage) * Tr::STAGE;
        const uint8_t* Vst = Kst + CHUNK * ROW;
        const int tw0 = wg * TPW;
        const int tend = min(tw0 + TPW, mt.valid);
        for (int tb = tw0; tb < tend; tb += Tr::SUB) {
          const int sb_off = row_off(tb);
          auto tok_off = [&](int i) {   // token tb + i, 0 <= i < 16
            return sb_off + (i >> sh_shift) * grp_stride + (i & (sh - 1)) * Tr::HALF;
          };
          // scores of tokens tb .. tb+15 (lane group gi takes every 4th)
          float s[4][GPW];
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            const int t = tb + pp * 4 + gi;
            const uint8_t* krow = Kst + tok_off(pp * 4 + gi);
            float acc[GPW];
#pragma unroll
            for (int g = 0; g < GPW; ++g) acc[g] = 0.f;
#pragma unroll
            for (int v = 0; v < Tr::NV; ++v) {
              float f[Tr::EPV];
              unpack16<T>(*reinterpret_cast<const uint4*>(krow + kofs[v]), f);
#pragma unroll
              for (int g = 0; g < GPW; ++g)
#pragma unroll
                for (int e = 0; e < Tr::EPV; ++e)
                  acc[g] = fmaf(q[g][v * Tr::EPV + e], f[e], acc[g]);
            }
#pragma unroll
            for (int g = 0; g < GPW; ++g) {
              acc[g] += __shfl_xor_sync(kFull, acc[g], 1);
              acc[g] += __shfl_xor_sync(kFull, acc[g], 2);
              acc[g] += __shfl_xor_sync(kFull, acc[g], 4);
              s[pp][g] = (t < tend) ? acc[g] : -INFINITY;
            }
          }
          // online softmax over the sub-block
          float pr[4][GPW];
#pragma unroll
          for (int g = 0; g < GPW; ++g) {
            float mb = fmaxf(fmaxf(s[0][g], s[1][g]), fmaxf(s[2][g], s[3][g]));
            mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, 8));
            mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, 16));
            const float mn = fmaxf(m[g], mb);
            const float alpha = exp2f(m[g] - mn);
            m[g] = mn;
            l[g] *= alpha;
#pragma unroll
            for (int e = 0; e < Tr::EPL; ++e) o[g][e] *= alpha;
            float psum = 0.f;
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              pr[pp][g] = exp2f(s[pp][g] - mn);
              psum += pr[pp][g];
            }
            l[g] += psum;
          }
          if (j == 0) {
#pragma unroll
            for (int pp = 0; pp < 4; ++pp)
#pragma unroll
              for (int g = 0; g < GPW; ++g) ps_w[(pp * 4 + gi) * 4 + g] = pr[pp][g];
          }
          __syncwarp();
          const int nt = min(Tr::SUB, tend - tb);
#pragma unroll 4
          for (int tt = 0; tt < nt; ++tt) {
            const float4 pw = *reinterpret_cast<const float4*>(ps_w + tt * 4);
            const float pv[4] = {pw.x, pw.y, pw.z, pw.w};
            float vf[Tr::EPL];
            load_row_slice<T, Tr::PVB>(Vst + tok_off(tt) + pv_off, vf);
#pragma unroll
            for (int g = 0; g < GPW; ++g)
#pragma unroll
              for (int e = 0; e < Tr::EPL; ++e) o[g][e] = fmaf(pv[g], vf[e], o[g][e]);
          }
          __syncwarp();
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);

      if (mt.flags & kLast) {
        // merge the warps that share a head group; write final row or partial
        float* mine = cmb + cw * Tr::CMB;
#pragma unroll
        for (int g = 0; g < GPW; ++g) {
          float lg = l[g];
          lg += __shfl_xor_sync(kFull, lg, 8);
          lg += __shfl_xor_sync(kFull, lg, 16);
#pragma unroll
          for (int e = 0; e < Tr::EPL; ++e) mine[g * D + lane * Tr::EPL + e] = active ? o[g][e] : 0.f;
          if (lane == 0) {
            mine[GPW * D + g] = active ? m[g] : -INFINITY;
            mine[GPW * D + GPW + g] = active ? lg : 0.f;
          }
        }
        if (!group_sync(&gbar[0], gphase, abrt, status)) break;
        const int tid = threadIdx.x - 32;
        float2* ml = reinterpret_cast<float2*>(p.ws + p.ml_off);
        float* po = reinterpret_cast<float*>(p.ws + p.o_off);
        int* cnt = reinterpret_cast<int*>(p.ws + p.cnt_off);
        // row h of the item, merged over the warps of its head group
        auto combine = [&](int h, int d, float& M, float& L, float& O) {
          const int hgi = h / GPW, g = h - hgi * GPW;
          M = -INFINITY;
          for (int w = 0; w < WPG; ++w) M = fmaxf(M, cmb[(hgi * WPG + w) * Tr::CMB + GPW * D + g]);
          L = 0.f;
          O = 0.f;
          for (int w = 0; w < WPG; ++w) {
            const float* src = cmb + (hgi * WPG + w) * Tr::CMB;
            const float sc = exp2f(src[GPW * D + g] - M);
            L = fmaf(src[GPW * D + GPW + g], sc, L);
            O = fmaf(src[g * D + d], sc, O);
          }
        };
        const int split = item_split(mt.split_raw);
        if (GRP) {
          // A group item: whole pieces common to `members` consecutive
          // sequences (the same physical blocks), rows h = member x G + head.
          // Each member counts the piece on its own (sequence, KV head)
          // counter; a member whose pieces are then all counted is merged
          // here, as by the last piece of any split sequence.
          const int members = item_nsplit(mt.split_raw);
          const int32_t* nsplit_of = reinterpret_cast<const int32_t*>(p.ws + p.nsplit_off);
          for (int idx = tid; idx < members * G * D; idx += Tr::NCW * 32) {
            const int h = idx / D, d = idx - (idx / D) * D;
            float M, L, O;
            combine(h, d, M, L, O);
            const int mb = h / G;
            const size_t row = static_cast<size_t>(mt.seq + mb) * p.num_q_heads + mt.kvh * G + (h - mb * G);
            if (nsplit_of[mt.seq + mb] == 1) {
              p.out[row * D + d] = O / L;
            } else {
              const size_t pr_ = row * p.max_splits + split;
              po[pr_ * D + d] = O;
              if (d == 0) ml[pr_] = make_float2(M, L);
            }
          }
          __threadfence();   // the partial results, before they are counted
          if (!group_sync(&gbar[0], gphase, abrt, status)) break;
          if (tid < members) {
            const int sq = mt.seq + tid;
            const int nspm = nsplit_of[sq];
            s_lastm[tid] = nspm > 1 &&
                           atomicAdd(cnt + static_cast<size_t>(sq) * Hkv + mt.kvh, 1) == nspm - 1;
          }
          if (!group_sync(&gbar[0], gphase, abrt, status)) break;
          for (int mb = 0; mb < members; ++mb) {
            if (!s_lastm[mb]) continue;
            __threadfence();   // every other piece counted before us is visible
            const int sq = mt.seq + mb;
            merge_split_rows(p.out, ml, po, static_cast<size_t>(sq) * p.num_q_heads + mt.kvh * G, G,
                             D, nsplit_of[sq], p.max_splits, tid, Tr::NCW * 32);
          }
        } else {
          const int nsp = item_nsplit(mt.split_raw);
          // the sequence's only own piece after its shared-prefix group
          // pieces (complete before this launch) folds them in itself
          const bool fold = item_folds(mt.split_raw);
          const bool single = nsp == 1 || fold;   // this item writes the output rows
          const size_t row0 = static_cast<size_t>(mt.seq) * p.num_q_heads + mt.kvh * G;
          for (int idx = tid; idx < G * D; idx += Tr::NCW * 32) {
            const int h = idx / D, d = idx - (idx / D) * D;
            float M, L, O;
            combine(h, d, M, L, O);
            const size_t row = row0 + h;
            if (fold) {
              // (m, l, o) of pieces 0 .. split-1, 8 pieces' loads in flight
              const size_t pr0 = row * p.max_splits;
              for (int s0 = 0; s0 < split; s0 += 8) {
                float2 e[8];
                float v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  const bool in = s0 + jj < split;
                  e[jj] = in ? __ldcg(ml + pr0 + s0 + jj) : make_float2(-INFINITY, 0.f);
                  v[jj] = in ? __ldcg(po + (pr0 + s0 + jj) * D + d) : 0.f;
                }
                float mb = M;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) mb = fmaxf(mb, e[jj].x);
                const float sc = exp2f(M - mb);
                L *= sc;
                O *= sc;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  const float w = exp2f(e[jj].x - mb);   // 0 for the padding entries
                  L = fmaf(e[jj].y, w, L);
                  O = fmaf(w, v[jj], O);
                }
                M = mb;
              }
            }
            if (single) {
              p.out[row * D + d] = O / L;
            } else {
              const size_t pr_ = row * p.max_splits + split;
              po[pr_ * D + d] = O;
              if (d == 0) ml[pr_] = make_float2(M, L);
            }
          }
          if (!single) __threadfence();   // this piece's partial result, before it is counted
          if (!group_sync(&gbar[0], gphase, abrt, status)) break;
          if (!single) {
            // the last piece of the (sequence, KV head) to finish merges them all
            if (tid == 0)
              s_last = atomicAdd(cnt + static_cast<size_t>(mt.seq) * Hkv + mt.kvh, 1) == nsp - 1;
            if (!group_sync(&gbar[0], gphase, abrt, status)) break;
            if (s_last) {
              __threadfence();   // every other piece counted before us is visible
              merge_split_rows(p.out, ml, po, row0, G, D, nsp, p.max_splits, tid, Tr::NCW * 32);
            }
          }
        }
      }
      ++c;
    }
  }
  __syncthreads();
}

template <typename T, int D, int GPW, bool GRP = false>
cudaError_t launch_t(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  using Tr = SimtTraits<T, D, GPW>;
  auto kern = simt_decode_kernel<T, D, GPW, GRP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Tr::SMEM));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(num_ctas), dim3(Tr::NTHREADS), Tr::SMEM, stream, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T, int D, int GPW>
cudaError_t launch_groups_t(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  return launch_t<T, D, GPW, true>(p, num_ctas, stream);
}

template <typename T, int D, int GPW>
cudaError_t ctas_t(int* n) {
  using Tr = SimtTraits<T, D, GPW>;
  auto kern = simt_decode_kernel<T, D, GPW, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Tr::SMEM));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Tr::NTHREADS, Tr::SMEM);
  if (e != cudaSuccess) return e;
  *n = num_sms() * (per_sm > 0 ? per_sm : 1);
  return cudaSuccess;
}

int gpw_for(int group) { return group == 1 ? 1 : (group == 2 ? 2 : 4); }

}  // namespace

bool simt_supported(int dtype, int head_dim, int group) {
  return (dtype >= 0 && dtype <= 2) && (head_dim == 64 || head_dim == 128) &&
         group >= 1 && group <= 16;
}

#define PA_SIMT_DISPATCH(FN, ...)                                                  \
  do {                                                                             \
    const int gpw = gpw_for(group);                                                \
    if (dtype == 0) {                                                              \
      if (head_dim == 64) {                                                        \
        if (gpw == 1) return FN<float, 64, 1>(__VA_ARGS__);                        \
        if (gpw == 2) return FN<float, 64, 2>(__VA_ARGS__);                        \
        return FN<float, 64, 4>(__VA_ARGS__);                                      \
      }                                                                            \
      if (gpw == 1) return FN<float, 128, 1>(__VA_ARGS__);                         \
      if (gpw == 2) return FN<float, 128, 2>(__VA_ARGS__);                         \
      return FN<float, 128, 4>(__VA_ARGS__);                                       \
    } else if (dtype == 1) {                                                       \
      if (head_dim == 64) {                                                        \
        if (gpw == 1) return FN<__half, 64, 1>(__VA_ARGS__);                       \
        if (gpw == 2) return FN<__half, 64, 2>(__VA_ARGS__);                       \
        return FN<__half, 64, 4>(__VA_ARGS__);                                     \
      }                                                                            \
      if (gpw == 1) return FN<__half, 128, 1>(__VA_ARGS__);                        \
      if (gpw == 2) return FN<__half, 128, 2>(__VA_ARGS__);                        \
      return FN<__half, 128, 4>(__VA_ARGS__);                                      \
    } else {                                                                       \
      if (head_dim == 64) {                                                        \
        if (gpw == 1) return FN<__nv_bfloat16, 64, 1>(__VA_ARGS__);                \
        if (gpw == 2) return FN<__nv_bfloat16, 64, 2>(__VA_ARGS__);                \
        return FN<__nv_bfloat16, 64, 4>(__VA_ARGS__);                              \
      }                                                                            \
      if (gpw == 1) return FN<__nv_bfloat16, 128, 1>(__VA_ARGS__);                 \
      if (gpw == 2) return FN<__nv_bfloat16, 128, 2>(__VA_ARGS__);                 \
      return FN<__nv_bfloat16, 128, 4>(__VA_ARGS__);                               \
    }                                                                              \
  } while (0)

cudaError_t simt_num_ctas(int dtype, int head_dim, int group, int* num_ctas) {
  if (!simt_supported(dtype, head_dim, group)) return cudaErrorInvalidValue;
  PA_SIMT_DISPATCH(ctas_t, num_ctas);
}

cudaError_t launch_decode_simt(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  const int dtype = p.dtype, head_dim = p.head_dim, group = p.num_q_heads / p.num_kv_heads;
  if (!simt_supported(dtype, head_dim, group)) return cudaErrorInvalidValue;
  PA_SIMT_DISPATCH(launch_t, p, num_ctas, stream);
}

cudaError_t launch_decode_simt_groups(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  // 16 query rows per item: the 4-rows-per-warp flavour
  const int dtype = p.dtype, head_dim = p.head_dim, group = 16;
  if (!p.group_mode || !simt_supported(dtype, head_dim, group)) return cudaErrorInvalidValue;
  PA_SIMT_DISPATCH(launch_groups_t, p, num_ctas, stream);
}

}  // namespace pa
