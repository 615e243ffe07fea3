// Paged decode on the 5th-generation tensor cores (tcgen05), for 16-bit KV,
// head_dim 128 and 4..16 query heads per KV head. With grouped-query
// attention ("Paged Attention: Virtual Memory for the KV Cache", "What it does
// not fix") the G query heads that share a KV head form a real dense tile, so
// the two contractions of a 128-token chunk run as MMAs:
//
//   S'[256 half-rows, NS] = K'[256 half-rows, 64] . Q'^T[64, NS]  (two M = 128 MMAs, A = K', K-major)
//   O^T[128 d, NPV]       = V^T[128 d, 128 tok] . P^T[128 tok, NPV] (A = V^T, MN-major)
//
// K' views the chunk's K as 128-byte half-rows (token, half h of d), Q' holds
// the query rows' first halves then their second halves, and a token's score
// is the sum of its two half-row terms K_h[t] . Q_h[g]. Query heads sit on
// the N side (padded to 16; spare columns are ignored).
// The probabilities are rounded to 16 bits for the second MMA as a sum of two
// terms, p = hi + lo (columns [0, NPV/2) and [NPV/2, NPV) of P^T), so the
// product keeps ~16 significant bits of p at no extra tensor-core passes.
//
// Persistent, warp-specialised CTA (one per SM, ~220 KB shared memory) that
// runs two independent item streams, so one stream's serial steps (the MMA
// round trips, the end-of-item reduction and stores) overlap the other's:
//   warp 11     scheduler: claims (sequence, split, KV head) items for the two
//               streams and describes their 128-token chunks alternately (ring
//               position c belongs to stream c & 1): metadata, query row and
//               the physical blocks read from the block table. It runs up to
//               8 positions ahead through a shared-memory descriptor queue.
//               When a stream runs out of items its position carries END and
//               the other stream takes every later position (its first chunk
//               after that is marked SOLO), so a stream left alone at the end
//               has the whole ring; two STOPs end the producer.
//   warp 0      producer: for each descriptor loads each page's K and V tile
//               (two 64-column halves each) plus the Q tile with 2-D TMA
//               (128-byte swizzle) into a 3-stage ring; completion by mbarrier
//               transaction count. K and Q' of a stage are refilled as soon as
//               the score MMA has read them, V once the P.V MMA has: the score
//               MMA and the softmax of a chunk run while its V is still in
//               flight, and V's slot is held only for the P.V MMA.
//   warps 1, 2  MMA issuers (one elected lane each), one per stream: S^T into
//               the stream's TMEM columns, then O^T once its softmax group has
//               published P; warp 1 also allocates and frees TMEM.
//   warps 3-6,  softmax and correction groups, one per stream: thread r reads
//   7-10        half-row r of both score tiles (tcgen05.ld), owns one of the
//               two tokens in them and takes its partner lane's half of that
//               token's score; the column maxima and sums over the group use
//               transposed warp reductions. Thread r also owns output column
//               d = r for the correction O = alpha O + O_c. A split item
//               writes its partial result to the workspace; after its last
//               item the group merges split rows (merge tasks).
// Paired KV heads (block size 8, 4 or 8 query heads per KV head): the pool
// stores a block's KV heads one after the other, so the pages of KV heads 2j
// and 2j + 1 of a block are one contiguous 4 KiB run. The kernel then treats
// the pair as one virtual KV head of 2G query heads whose pages hold 2 x 8
// virtual tokens (head 2j's 8 tokens, then head 2j + 1's), loaded with one
// box per block instead of one per (block, head): a 128-token ring position
// holds 64 tokens of both heads. A softmax thread's token belongs to one of
// the two heads, so it keeps the scores, probabilities and sums of that
// head's G query heads only (the others' probabilities are zero). Halving
// the copies matters at block size 8, where the copy engine's request rate,
// not HBM, bounds 2 KiB boxes.
// No load uses cluster multicast; every wait is bounded (see pa_common.cuh).
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kFirst = 1, kLast = 2, kEnd = 4, kSolo = 8, kStop = 16;
constexpr int kChunk = 128;   // tokens per stage (= MMA M)
constexpr int kD = 128;       // head_dim
constexpr int kNst = 3;       // pipeline stages
constexpr int kTile = kChunk * 256;           // K (or V) of 128 tokens: 256 half-rows x 128 B
constexpr int kQReg = 32 * 128;               // Q' region: up to 32 half-rows x 128 B
constexpr int kStage = 2 * kTile + kQReg;     // K, V, Q' of one chunk
constexpr int kQd = 8;        // chunk descriptors the scheduler may run ahead
constexpr int kMaxPages = kChunk / 8;          // pages per chunk at the smallest block size
constexpr int kSchedWarp = 11;
constexpr int kThreads = 384;  // producer, 2 MMA issuers, 2 softmax groups of 4 warps, scheduler

struct __align__(16) ChunkMeta {
  int32_t seq, kvh, split_raw, t0, valid, flags, pad0, pad1;
};

// One ring position as the scheduler hands it to the producer: what the
// consumers will read (meta), the query row and the chunk's physical blocks.
struct __align__(16) ChunkDesc {
  ChunkMeta meta;
  int32_t q_row, npg, pad0, pad1;
  int32_t blk[kMaxPages];
};

template <int GT>
struct TcLayout {
  static constexpr int NPV = GT * 2 < 16 ? 16 : GT * 2;  // P^T columns: hi, lo (M=128 needs N%16==0)
  static constexpr int PBUF = (NPV / 8) * 2048;      // P^T buffer bytes (one per group)
  static constexpr size_t OFF_P = static_cast<size_t>(kNst) * kStage;
  static constexpr size_t OFF_BAR = OFF_P + 2 * PBUF;
  // barriers: kfull[3][2], vfull[3][2], kempty[3], vempty[3]; per group:
  // s_full, s_free, p_full, o_full, o_free, group barrier, MMA drain;
  // descriptor queue full/empty
  static constexpr int NBAR = 6 * kNst + 14 + 2 * kQd;
  static constexpr size_t OFF_META = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;  // 16-B vector stores
  static constexpr size_t OFF_DESC = (OFF_META + 2 * kNst * sizeof(ChunkMeta) + 15) / 16 * 16;
  static constexpr size_t OFF_RED = OFF_DESC + kQd * sizeof(ChunkDesc);
  static constexpr size_t OFF_LRED = OFF_RED + 2 * 2 * 4 * 16 * 4;
  static constexpr size_t OFF_MISC = OFF_LRED + 2 * 2 * 4 * 16 * 4;
  static constexpr size_t SMEM_USED = OFF_MISC + 16;
  static constexpr size_t SMEM = SMEM_USED + 1024;   // slack to align the base to 1 KB
  static constexpr int NS = GT <= 8 ? 16 : 32;       // score MMA N: two halves x heads
  // per stream: two score accumulators (NS columns each) and the O^T accumulator
  static constexpr int COLS_PER_STREAM = 2 * NS + NPV;
  // End-of-item work deferred into the next chunk (needs 2 GT + 4 spare
  // registers per softmax thread; the 16-head tile has none)
  static constexpr bool DEFER_END = GT <= 8;
  static constexpr uint32_t TMEM_COLS = 2 * COLS_PER_STREAM <= 128 ? 128 : 256;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(kStage % 1024 == 0 && OFF_P % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(OFF_BAR % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(OFF_META % 16 == 0 && OFF_DESC % 16 == 0 && OFF_RED % 16 == 0 &&
                    OFF_LRED % 16 == 0 && OFF_MISC % 16 == 0,
                "16-byte aligned shared regions");
};

// ---------------------------------------------------------------------------
// tcgen05 wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (16-byte units), version 1, layout type in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(layout) << 61);
}
constexpr uint32_t kSw128 = 2, kSwNone = 0;

// Instruction descriptor, kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t fmt, bool a_mn, bool b_mn, int M, int N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* f) {
  uint32_t v[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
}

// 16 columns of this warp's 32 TMEM lanes, without waiting for them; the
// values are valid only after tmem_wait16 on the same array.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
// Wait for every outstanding tcgen05.ld of the thread; v is tied to the wait
// so no use of it can be scheduled before it.
__device__ __forceinline__ void tmem_wait16(uint32_t* v) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}
// Orders later uses of v after an earlier tmem_wait16 (no instruction).
__device__ __forceinline__ void tmem_after_wait16(uint32_t* v) {
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

// 2^x with the hardware approximation (ex2.approx.ftz: relative error below
// 2^-22; -inf gives +0), for the probabilities of 16-bit caches.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Round p to 16 bits (hi) and the remainder p - hi to 16 bits (lo), for two
// values at once: p0 in the low half of each word, p1 in the high half (one
// 2-wide conversion per word).
template <typename T>
__device__ __forceinline__ void split16x2(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  } else {
    const __half2 h = __floats2half2_rn(p0, p1);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(p0 - hf.x, p1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  }
}

// Barrier among the 4 warps of a softmax group: one arrival per warp. The
// result is made warp-uniform so a time-out never splits a warp.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, volatile int* abrt,
                                           int* status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = __all_sync(kFull, mbar_wait(bar, phase, abrt, status));
  phase ^= 1u;
  return ok;
}

// Max (MAX) or sum of NC values per lane over SPAN lanes (the warp, or a half
// warp), all NC columns at once: each step hands half of the lane's columns
// to its partner at the step's distance and keeps the other half, so the
// first log2(NC) shuffles cover every column; the remaining steps reduce the
// one column left. On return, lane l holds the result for column
// (l % SPAN) / (SPAN / NC).
template <int NC, int SPAN, bool MAX>
__device__ __forceinline__ float xreduce(float (&v)[NC], int lane) {
  static_assert(NC >= 1 && NC <= SPAN && (NC & (NC - 1)) == 0, "power-of-two columns");
  int o = SPAN / 2;
#pragma unroll
  for (int w = NC; w > 1; w >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < w / 2; ++j) {
      const float send = up ? v[j] : v[j + w / 2];
      const float keep = up ? v[j + w / 2] : v[j];
      const float got = __shfl_xor_sync(kFull, send, o);
      v[j] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
#pragma unroll
  for (; o > 0; o >>= 1) {
    const float got = __shfl_xor_sync(kFull, v[0], o);
    v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
  }
  return v[0];
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
}

// GRP: the launch over the group list of shared prefixes (group items only).
// PAIR: paired KV heads (items, query rows and counts per virtual KV head).
template <typename T, int GT, bool GRP, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    tc_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_q) {
  using Ly = TcLayout<GT>;
  constexpr int NPV = Ly::NPV;
  __shared__ volatile int s_last[2];   // per group: this piece completed its sequence
  extern __shared__ uint8_t smem_raw[];
  // 1 KB alignment for the 128-byte-swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pbuf = smem + Ly::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::OFF_BAR);
  // A stage holds K and Q' (released once the score MMA has read them) and V
  // (released after the P.V MMA), each with its own full / empty barriers.
  // kfull / vfull[2 * stage + (c & 1)]: one barrier per (stage, position
  // parity), so the consumers of ring position c see every phase of the
  // barrier they wait on: it serves every 2 x kNst-th position, and its phase
  // parity at c is (c / (2 kNst)) & 1, whichever stream c belongs to.
  uint64_t* kfull = bars;                // [kNst][2]
  uint64_t* vfull = bars + 2 * kNst;     // [kNst][2]
  uint64_t* kempty = bars + 4 * kNst;    // [kNst]
  uint64_t* vempty = bars + 5 * kNst;    // [kNst]
  uint64_t* s_full = bars + 6 * kNst;    // [2] per group
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_free = o_full + 2;
  uint64_t* grp = o_free + 2;            // [2] group barriers
  uint64_t* drain = grp + 2;             // [2] MMA drain
  uint64_t* desc_full = drain + 2;       // [kQd]
  uint64_t* desc_empty = desc_full + kQd;  // [kQd]
  ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(smem + Ly::OFF_META);   // [kNst][2]
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + Ly::OFF_DESC);
  float* red = reinterpret_cast<float*>(smem + Ly::OFF_RED);    // [2 grp][2][4][16]
  float* lred = reinterpret_cast<float*>(smem + Ly::OFF_LRED);  // [2 grp][2 item parity][4][16]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Ly::OFF_MISC);
  volatile int* abrt = reinterpret_cast<volatile int*>(smem + Ly::OFF_MISC + 4);

  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  int* status = &hdr->status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNst; ++s) {
      for (int g = 0; g < 2; ++g) {
        mbar_init(&kfull[2 * s + g], 1);
        mbar_init(&vfull[2 * s + g], 1);
      }
      mbar_init(&kempty[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      // the softmax groups arrive once per warp (lane 0, after __syncwarp)
      mbar_init(&s_free[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], 4);
      mbar_init(&grp[b], 4);
      mbar_init(&drain[b], 1);
    }
    for (int q = 0; q < kQd; ++q) {
      mbar_init(&desc_full[q], 1);                           // scheduler, lane 0
      mbar_init(&desc_empty[q], 1);                          // producer, lane 0
    }
    *abrt = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(Ly::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();   // the plan (and the KV write before it) are complete from here on
  // (no early launch of dependents: the next call's plan rewrites the workspace)

  // the group list (shared prefixes) or the work list
  const int num_items = GRP ? hdr->num_group_items : hdr->num_items;
  // KV heads as the items see them (virtual ones when paired), query heads
  // per item head, tokens a page box holds and tokens per ring position
  const int Hkv = PAIR ? p.num_kv_heads / 2 : p.num_kv_heads, BS = p.block_size;
  const int G = p.num_q_heads / Hkv;
  const int PB = PAIR ? 2 * BS : BS;
  constexpr int CH = PAIR ? kChunk / 2 : kChunk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Takes ring position c's descriptor from the scheduler, waits for the
    // stage halves, and issues the chunk's copies: Q' (two boxes) and one K
    // box per page, then one V box per page; or forwards an END / STOP
    // marker.
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_v);
    }
    const uint64_t pol = l2_evict_first_policy();   // K and V tiles: read once per call
    int stops = 0;
    uint32_t ck = 0, cv = 0;   // positions whose K / V copies (or markers) were issued
    bool ok = true;
    for (uint32_t c = 0;; ++c) {
      const int qd = c % kQd;
      if (!mbar_wait(&desc_full[qd], (c / kQd) & 1u, abrt, status)) {
        ok = false;
        break;
      }
      const ChunkDesc& d = desc[qd];
      const int flags = d.meta.flags;
      const int kvh = d.meta.kvh;
      const int npg = d.npg;
      const int blk = d.blk[lane & (kMaxPages - 1)];
      uint4 m0 = make_uint4(0, 0, 0, 0), m1 = m0;
      int q_row = 0, q_y = 0;
      if (lane == 0) {
        m0 = reinterpret_cast<const uint4*>(&d.meta)[0];
        m1 = reinterpret_cast<const uint4*>(&d.meta)[1];
        q_row = d.q_row;
        q_y = d.pad0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_empty[qd]);   // every lane has its copy of the descriptor
      const int stage = c % kNst;
      const uint32_t epar = ((c / kNst) & 1u) ^ 1u;
      const int bi = 2 * stage + (c & 1);
      const bool data = !(flags & (kEnd | kStop));
      uint8_t* st = smem + static_cast<size_t>(stage) * kStage;
      {
        // K and Q' (and the chunk's metadata) once the score MMA of the
        // stage's previous chunk is done
        if (!mbar_wait(&kempty[stage], epar, abrt, status)) {
          ok = false;
          break;
        }
        if (data) {
          if (lane == 0) {
            reinterpret_cast<uint4*>(&meta[bi])[0] = m0;
            reinterpret_cast<uint4*>(&meta[bi])[1] = m1;
            // K: one box of 2*PB half-rows per page; Q': the group's query
            // rows, first halves then second halves (NS/2 rows each)
            mbar_arrive_expect_tx(&kfull[bi],
                                  static_cast<uint32_t>(npg * PB * 256 + Ly::NS * 128));
            if (GRP) {
              tma_load_3d(st + 2 * kTile, &tm_q, 0, q_y, q_row, &kfull[bi]);
              tma_load_3d(st + 2 * kTile + (Ly::NS / 2) * 128, &tm_q, 64, q_y, q_row, &kfull[bi]);
            } else {
              tma_load_2d(st + 2 * kTile, &tm_q, 0, q_row, &kfull[bi]);
              tma_load_2d(st + 2 * kTile + (Ly::NS / 2) * 128, &tm_q, 64, q_row, &kfull[bi]);
            }
          }
          __syncwarp();
          if (lane < npg)
            tma_load_2d_hint(st + lane * PB * 256, &tm_k, 0, (blk * Hkv + kvh) * PB * 2,
                             &kfull[bi], pol);
        } else {
          if (lane == 0) {
            meta[bi].flags = flags;
            mbar_arrive(&kfull[bi]);
          }
          __syncwarp();
        }
        ++ck;
      }
      {
        // V once the P.V MMA of the stage's previous chunk is done
        if (!mbar_wait(&vempty[stage], epar, abrt, status)) {
          ok = false;
          break;
        }
        if (data) {
          if (lane == 0) mbar_arrive_expect_tx(&vfull[bi], static_cast<uint32_t>(npg * PB * 256));
          __syncwarp();
          if (lane < npg)
            tma_load_2d_hint(st + kTile + lane * PB * 256, &tm_v, 0, (blk * Hkv + kvh) * PB * 2,
                             &vfull[bi], pol);
        } else {
          if (lane == 0) mbar_arrive(&vfull[bi]);
          __syncwarp();
        }
        ++cv;
      }
      if ((flags & kStop) && ++stops == 2) break;
    }
    if (!ok && lane == 0) {
      // copies may still be landing in the last kNst positions: let them finish
      for (uint32_t cc = ck > kNst ? ck - kNst : 0; cc < ck; ++cc)
        drain_wait(&kfull[2 * (cc % kNst) + (cc & 1)], (cc / (2 * kNst)) & 1u);
      for (uint32_t cc = cv > kNst ? cv - kNst : 0; cc < cv; ++cc)
        drain_wait(&vfull[2 * (cc % kNst) + (cc & 1)], (cc / (2 * kNst)) & 1u);
    }
  } else if (warp == kSchedWarp) {
    // ------------------------------------------------------------ scheduler
    // Two item streams; ring position c belongs to stream (group) c & 1. The
    // scheduler claims (sequence, split, KV head) items, follows the block
    // table and writes one descriptor per position, up to kQd positions ahead
    // of the producer, so none of this global-memory latency sits on the copy
    // issue path.
    const WorkPair* pairs =
        reinterpret_cast<const WorkPair*>(p.ws + (GRP ? p.gpairs_off : p.pairs_off));
    int* const work_counter = GRP ? &hdr->group_work_counter : &hdr->work_counter;
    // Per-stream state (warp-uniform), plus a window of block-table entries:
    // lane j holds entries wbase + j and wbase + 32 + j of the current item.
    // The next item of each stream is prefetched one step per emission
    // (claim -> work pair -> first table window), starting with the current
    // item's last chunk. The loop below is unrolled over the two
    // streams so each stream's state sits in its own registers.
    struct Stream {
      int seq, kvh, split_n, tb, te, cs;   // current item, next chunk start
      int wbase, w0, w1;                   // table window of the current item
      int nst;                             // next item: 0 none, 1 claimed, 2 pair, 3 window, 4 no more
      int nkraw;                           // claim result (lane 0)
      int nseq, nkvh, nsplit_n, ntb, nte;  // next item's work pair
      int nw0, nw1;                        // next item's first window
      bool ended;
    };
    auto load_window = [&](int sq, int first_page, int& a, int& b) {
      const int32_t* row = p.block_tables + static_cast<size_t>(sq) * p.bt_stride;
      const int i0 = first_page + lane, i1 = first_page + 32 + lane;
      a = i0 < p.bt_stride ? row[i0] : 0;
      b = i1 < p.bt_stride ? row[i1] : 0;
    };
    auto claim = [&]() {
      int kr = 0;
      if (lane == 0) kr = atomicAdd(work_counter, 1);
      return kr;
    };
    // one prefetch step for the next item of stream `cur`
    auto prefetch_step = [&](Stream& cur) {
      if (cur.nst == 0) {
        cur.nkraw = claim();
        cur.nst = 1;
      } else if (cur.nst == 1) {
        const int k = __shfl_sync(kFull, cur.nkraw, 0);
        if (k < num_items) {
          const int pi = k / Hkv;
          const WorkPair wp = pairs[pi];
          cur.nseq = wp.seq;
          cur.nkvh = k - pi * Hkv;
          cur.nsplit_n = wp.split_n;
          cur.ntb = wp.t_begin;
          cur.nte = wp.t_end;
          cur.nst = 2;
        } else {
          cur.nst = 4;
        }
      } else if (cur.nst == 2) {
        load_window(cur.nseq, cur.ntb / BS, cur.nw0, cur.nw1);
        cur.nst = 3;
      }
    };
    // Each stream's first item is its own, unclaimed: stream 2b + t of CTA b
    // takes item 2b + t (the plan starts the claim counter after one item per
    // stream), so the start-up path has no atomic.
    Stream st0 = {};
    st0.nkraw = 2 * static_cast<int>(blockIdx.x);
    st0.nst = 1;
    Stream st1 = {};
    st1.nkraw = 2 * static_cast<int>(blockIdx.x) + 1;
    st1.nst = 1;
    // the two first items' work pairs, then their first table windows: each
    // pair of loads is in flight together, two round trips in all
    prefetch_step(st0);
    prefetch_step(st1);
    prefetch_step(st0);
    prefetch_step(st1);
    int stops = 0;
    uint32_t c = 0;
    int solo = -1;            // once one stream has ended: the stream (0 / 1) that takes every position
    bool solo_mark = false;   // its next chunk carries kSolo
    // describe position c for stream t = `cur` (a chunk, or an END / STOP
    // marker); returns false when the scheduler should stop
    auto emit = [&](Stream& cur, const Stream& other, int t) -> bool {
      int kind = 0;   // 0 data, 1 end, 3 stop
      if (!cur.ended && cur.cs >= cur.te) {
        // current item done: finish the prefetch of the next one, then switch
        while (cur.nst < 3) prefetch_step(cur);
        if (cur.nst == 4) {
          cur.ended = true;
          kind = 1;
          if (!other.ended) {
            solo = t ^ 1;
            solo_mark = true;
          }
        } else {
          cur.seq = cur.nseq;
          cur.kvh = cur.nkvh;
          cur.split_n = cur.nsplit_n;
          cur.tb = cur.ntb;
          cur.te = cur.nte;
          cur.cs = cur.ntb;
          cur.wbase = cur.ntb / BS;
          cur.w0 = cur.nw0;
          cur.w1 = cur.nw1;
          cur.nst = 0;
        }
      } else if (cur.ended) {
        kind = 3;   // a stream is only described again once both have ended
      }
      int valid = 0, npg = 0, blk = 0;
      if (kind == 0) {
        valid = min(CH, cur.te - cur.cs);
        npg = (valid + BS - 1) / BS;
        const int p0 = cur.cs / BS;
        if (p0 + npg > cur.wbase + 64) {   // chunk runs past the window: next window
          cur.wbase = p0;
          load_window(cur.seq, p0, cur.w0, cur.w1);
        }
        const int j = p0 - cur.wbase + lane;   // window index of this lane's page
        const int e0 = __shfl_sync(kFull, cur.w0, j & 31);
        const int e1 = __shfl_sync(kFull, cur.w1, j & 31);
        blk = j < 32 ? e0 : e1;
        if (lane < npg && (blk < 0 || blk >= p.num_blocks)) {
          atomicCAS(status, 0, 1 /* PA_ERR_INVALID_ARG */);
          blk = 0;
        }
        // advance the next item's prefetch by one step; the claim itself waits
        // until the current item has its last chunk left, so a stream never
        // holds an unstarted item for long (it would lengthen the tail); the
        // scheduler runs far enough ahead of the copies to cover the claim,
        // work pair and table window loads
        if (cur.nst != 0 || cur.te - cur.cs <= CH) prefetch_step(cur);
      }
      const int qd = c % kQd;
      if (!mbar_wait(&desc_empty[qd], ((c / kQd) & 1u) ^ 1u, abrt, status)) return false;
      ChunkDesc& d = desc[qd];
      if (kind == 0) {
        if (lane == 0) {
          ChunkMeta m;
          m.seq = cur.seq;
          m.kvh = cur.kvh;
          m.split_raw = cur.split_n;
          m.t0 = cur.cs;
          m.valid = valid;
          m.flags = (cur.cs == cur.tb ? kFirst : 0) | (cur.cs + CH >= cur.te ? kLast : 0) |
                    (solo_mark ? kSolo : 0);
          m.pad0 = m.pad1 = 0;
          d.meta = m;
          // the query rows: G heads of the sequence (a row of the [B * Hq,
          // 128] map), or for a group item, from its first member on, G heads
          // of each member (the [B, Hq, 128] map at (kvh * G, seq))
          d.q_row = GRP ? cur.seq : cur.seq * p.num_q_heads + cur.kvh * G;
          d.pad0 = cur.kvh * G;
          d.npg = npg;
        }
        if (lane < kMaxPages) d.blk[lane] = lane < npg ? blk : 0;
        cur.cs += CH;
        solo_mark = false;
      } else if (lane == 0) {
        d.meta.flags = kind == 1 ? kEnd : kStop;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_full[qd]);
      ++c;
      return !(kind == 3 && ++stops == 2);
    };
    // alternate until a stream ends (the position after its END belongs to
    // the other stream), then the other stream alone
    bool run = true;
    while (run && solo < 0) {
      run = emit(st0, st1, 0);
      if (run && solo < 0) run = emit(st1, st0, 1);
    }
    if (solo == 0)
      while (run) run = emit(st0, st1, 0);
    if (solo == 1)
      while (run) run = emit(st1, st0, 1);
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    const int t = warp - 1;   // group served
    if (lane == 0) {
      const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      const uint32_t idesc_s = instr_desc(fmt, false, false, 128, Ly::NS);
      const uint32_t sh = static_cast<uint32_t>(tile_sub_height(BS));
      const uint32_t v_sbo = sh == 16 ? 1024u : 2048u;   // 8-token groups
      const uint32_t idesc_pv = instr_desc(fmt, true, true, 128, NPV);
      const uint32_t sbase = smem_u32(smem);
      const uint32_t pb = smem_u32(pbuf) + t * Ly::PBUF;
      const uint32_t s_tm = tmem + t * Ly::COLS_PER_STREAM;   // two NS-column score tiles
      const uint32_t o_tm = s_tm + 2 * Ly::NS;
      uint32_t n = 0;      // data chunks of this group so far
      uint32_t step = 2;   // 1 once this stream takes every position
      for (uint32_t c = t;; c += step) {
        const int stage = c % kNst;
        const uint32_t fpar = (c / (2 * kNst)) & 1u;
        const int bi = 2 * stage + static_cast<int>(c & 1u);
        if (!mbar_wait(&kfull[bi], fpar, abrt, status)) break;
        const ChunkMeta mt = meta[bi];
        if (mt.flags & kStop) break;
        if (mt.flags & kSolo) step = 1;
        const uint32_t par = n & 1u;
        if (mt.flags & kEnd) {
          // release only after the softmax group has seen END (it acknowledges
          // on p_full); a slot refilled earlier could complete the next phase of
          // kfull[] before the group observed this one
          if (!mbar_wait(&p_full[t], par, abrt, status)) break;
          mbar_arrive(&kempty[stage]);
          // V's slot only after the producer has passed this position's V half
          // (its vfull arrival): an earlier release would complete two phases
          // of vempty[] before the producer waits on the first
          if (!mbar_wait(&vfull[bi], fpar, abrt, status)) break;
          mbar_arrive(&vempty[stage]);
          break;   // the stream's last position (later ones go to the other stream)
        }
        // Half-row scores: the K region holds 256 half-rows (token, half) of
        // 128 B; Q' holds the query rows' first halves then their second
        // halves. S'[(t, h), (h', g)] = K_h[t] . Q_h'[g]; the softmax group
        // adds the two h == h' terms of each token.
        if (!mbar_wait(&s_free[t], par ^ 1u, abrt, status)) break;
        tc_fence_after();
        const uint32_t stg = sbase + stage * kStage;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = smem_desc(stg + m * 16384 + kk * 32, 16, 1024, kSw128);
            const uint64_t b = smem_desc(stg + 2 * kTile + kk * 32, 16, 1024, kSw128);
            mma_f16(s_tm + m * Ly::NS, a, b, idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&s_full[t]);
        mma_commit(&kempty[stage]);   // K and Q' are free once these MMAs completed
        // O^T = V^T . P^T once the softmax group has written P and V has landed
        if (!mbar_wait(&p_full[t], par, abrt, status)) break;
        if (!mbar_wait(&o_free[t], par ^ 1u, abrt, status)) break;
        if (!mbar_wait(&vfull[bi], fpar, abrt, status)) break;
        tc_fence_after();
        // 16-token steps; paired, the loaded blocks' 2 x BS virtual tokens each
        const int nks = PAIR ? (mt.valid + BS - 1) / BS * (2 * BS) / 16 : (mt.valid + 15) >> 4;
        for (int ks = 0; ks < nks; ++ks) {
          // V^T for tokens 16ks..16ks+15: 4 KB of half-rows; M atoms (column
          // halves) sh * 128 B apart, 8-token groups v_sbo apart
          const uint64_t a = smem_desc(stg + kTile + ks * 4096, sh * 128, v_sbo, kSw128);
          const uint64_t b = smem_desc(pb + ks * 256, 128, 2048, kSwNone);
          mma_f16(o_tm, a, b, idesc_pv, ks > 0 ? 1u : 0u);
        }
        mma_commit(&o_full[t]);
        mma_commit(&vempty[stage]);
        ++n;
      }
      // all MMAs this thread issued have completed before TMEM is released
      mma_commit(&drain[t]);
      drain_wait(&drain[t], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / correction
    const int t = (warp - 3) >> 2;          // group 0: warps 3-6, group 1: warps 7-10
    const int wq = (warp - 3) & 3;           // 0..3 within the group
    const int r = 32 * (warp & 3) + lane;    // TMEM lane: score half-row / output column d
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const uint32_t s_col = t * Ly::COLS_PER_STREAM, o_col = s_col + 2 * Ly::NS;
    const float sl2 = p.scale_log2;
    // Half-row r of score tile m is (token tk0 + 64 m, half hh); its partner
    // half-row (same token, other half) is lane r ^ sh of the same warp.
    const int sh = tile_sub_height(BS);
    const int hh = (r / sh) & 1;
    const int tk0 = (r / (2 * sh)) * sh + r % sh;
    const int own_t = hh ? tk0 + 64 : tk0;   // the token whose P row / V row this thread writes
    // Paired heads (block size 8, 2 G = GT): virtual token v is token
    // (v / 16) 8 + v % 8 of the chunk, of the pair's KV head hd = (v / 8) & 1,
    // whose query heads are the item's columns [hd GT/2, hd GT/2 + GT/2).
    // tk0 and tk0 + 64 are of the same head and 32 tokens apart; the lanes of
    // one head are one half of the warp, and a lane and lane ^ 8 hold the two
    // halves of the same tokens.
    const int rt0 = PAIR ? (tk0 / (2 * BS)) * BS + tk0 % BS : tk0;
    const int rt1 = PAIR ? rt0 + 32 : tk0 + 64;
    const int own_rt = hh ? rt1 : rt0;
    const int hd = PAIR ? (tk0 / BS) & 1 : 0;
    constexpr int GH = GT / 2;   // query heads of one KV head of a pair
    uint8_t* pdst_base = pbuf + t * Ly::PBUF + own_t * 16;
    // own token's V half-rows in the stage: (t / sh) * sh * 256 + (t % sh) * 128, + sh * 128
    const int vrow_off = kTile + (own_t / sh) * sh * 256 + (own_t % sh) * 128;
    float* red_t = red + t * 128;
    float* lred_t = lred + t * 128;
    uint64_t* gbar = &grp[t];
    float2* ml = reinterpret_cast<float2*>(p.ws + p.ml_off);
    float* po = reinterpret_cast<float*>(p.ws + p.o_off);
    int* cnt = reinterpret_cast<int*>(p.ws + p.cnt_off);
    float m_run[GT], l_thr[GT], o[GT];
    uint32_t gphase = 0, n = 0;
    // an item's end: per-warp sums of l are written at its last chunk into
    // lred_t[item parity]; the cross-warp sum, normalisation and stores
    // (finish) run after the next chunk's max barrier, once that chunk's P is
    // published, or at END after one barrier
    float o_pend[Ly::DEFER_END ? GT : 1], m_pend[Ly::DEFER_END ? GT : 1];
    int pend_seq = 0, pend_kvh = 0, pend_split = 0;
    bool pend = false;
    uint32_t lpar = 0;   // parity of the next item to end
    // an item's result: the output rows, or the piece's partial result and,
    // for the last piece of the (sequence, KV head) to finish, the merge of
    // all of them; false when a barrier gave up
    auto finish = [&](const float* lr, int seq, int kvh, int split_raw, const float* ov_,
                      const float* mv_) -> bool {
      // a group item (shared prefix) is a piece of each of its members,
      // never their only one (each keeps a piece of its own); its rows are
      // member x G + head
      const int members = GRP ? item_nsplit(split_raw) : 1;
      const int nsp = GRP ? 0 : item_nsplit(split_raw);
      const int rows = members * G;
      const int split = item_split(split_raw);
      const size_t row0 = static_cast<size_t>(seq) * p.num_q_heads + kvh * G;
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        if (g >= rows) break;
        const float L = lr[g] + lr[16 + g] + lr[32 + g] + lr[48 + g];
        size_t row = row0 + g;
        if constexpr (GRP) {
          const int mb = g / G;
          row = row0 + static_cast<size_t>(mb) * p.num_q_heads + (g - mb * G);
        }
        if (nsp == 1) {
          p.out[row * kD + r] = ov_[g] / L;
        } else {
          const size_t pr_ = row * p.max_splits + split;
          po[pr_ * kD + r] = ov_[g];
          if (r == 0) ml[pr_] = make_float2(mv_[g], L);
        }
      }
      if (nsp == 1) return true;
      __threadfence();   // this piece's partial result, before it is counted
      if (!group_sync(gbar, gphase, abrt, status)) return false;
      // counted (for each member); the merge runs after the main loop (merge
      // tasks below), in the launch of the members' own pieces for group items
      if (wq == 0 && lane < members) atomicAdd(cnt + static_cast<size_t>(seq + lane) * Hkv + kvh, 1);
      return true;
    };

    uint32_t step = 2;   // 1 once this stream takes every position
    for (uint32_t c = t;; c += step) {
      const int stage = c % kNst;
      const uint32_t fpar = (c / (2 * kNst)) & 1u;
      const int bi = 2 * stage + static_cast<int>(c & 1u);
      if (!__all_sync(kFull, mbar_wait(&kfull[bi], fpar, abrt, status))) break;
      const ChunkMeta mt = meta[bi];
      if (mt.flags & kSolo) step = 1;
      // query rows of the chunk's item: G, or members x G for a group item
      const int rows = GRP ? item_nsplit(mt.split_raw) * G : G;
      if (mt.flags & kEnd) {
        if (Ly::DEFER_END && pend) {
          if (!group_sync(gbar, gphase, abrt, status)) break;
          if (!finish(lred_t + (lpar ^ 1u) * 64, pend_seq, pend_kvh, pend_split, o_pend, m_pend))
            break;
          pend = false;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);   // acknowledge END so the slot can be released
        break;
      }
      if (mt.flags & kFirst) {
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          m_run[g] = -INFINITY;
          l_thr[g] = 0.f;
          o[g] = 0.f;
        }
      }
      const uint32_t par = n & 1u;
      // ---- the half-row scores of tokens tk0 (tile 0) and tk0 + 64 (tile 1)
      if (!__all_sync(kFull, mbar_wait(&s_full[t], par, abrt, status))) break;
      tc_fence_after();
      // The thread's own token's scores (hh = 0: token tk0 of tile 0, hh = 1:
      // token tk0 + 64 of tile 1) for its query columns: all GT, or paired,
      // the GH of its own KV head. A half-row term is K_h[t] . Q_h[g]; the
      // thread holds half hh of both tiles' tokens, so it keeps its own
      // token's term (own) and trades the other tile's term (snd) with its
      // partner (lane ^ sh), which holds the other half. Score columns: the
      // query rows' first halves [0, NS/2), then their second halves.
      constexpr int NC = PAIR ? GH : GT;
      constexpr int SPAN = PAIR ? 16 : 32;   // lanes of one KV head
      float own[NC], snd[NC];
      // column g of the thread's (paired: own head's) query columns in a run
      // of first or second halves
      auto pick = [&](const float* x, int g) { return PAIR ? (hd ? x[GH + g] : x[g]) : x[g]; };
      if constexpr (Ly::NS == 16) {
        // both score tiles requested at once, one wait
        uint32_t su0[16], su1[16];
        tmem_ld16_async(lane_addr + s_col, su0);
        tmem_ld16_async(lane_addr + s_col + Ly::NS, su1);
        tmem_wait16(su0);
        tmem_after_wait16(su1);
        float sv0[16], sv1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          sv0[i] = __uint_as_float(su0[i]);
          sv1[i] = __uint_as_float(su1[i]);
        }
#pragma unroll
        for (int g = 0; g < NC; ++g) {
          own[g] = hh ? pick(sv1 + 8, g) : pick(sv0, g);
          snd[g] = hh ? pick(sv0 + 8, g) : pick(sv1, g);
        }
      } else {
        // 64 columns, 16 at a time, each kept only where the thread uses it
        float x[16];
        tmem_ld16(lane_addr + s_col, x);   // tile 0, first halves
#pragma unroll
        for (int g = 0; g < NC; ++g) own[g] = pick(x, g);
        tmem_ld16(lane_addr + s_col + Ly::NS, x);   // tile 1, first halves
#pragma unroll
        for (int g = 0; g < NC; ++g) snd[g] = pick(x, g);
        tmem_ld16(lane_addr + s_col + 16, x);   // tile 0, second halves
#pragma unroll
        for (int g = 0; g < NC; ++g) snd[g] = hh ? pick(x, g) : snd[g];
        tmem_ld16(lane_addr + s_col + Ly::NS + 16, x);   // tile 1, second halves
#pragma unroll
        for (int g = 0; g < NC; ++g) own[g] = hh ? pick(x, g) : own[g];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[t]);
      // hardware 2^x (ex2.approx)
      auto ex2 = [](float x) { return exp2_approx(x); };
      const bool own_ok = own_rt < mt.valid;
      float so[NC];
#pragma unroll
      for (int g = 0; g < NC; ++g) {
        const float full = own[g] + __shfl_xor_sync(kFull, snd[g], sh);
        so[g] = (own_ok && (PAIR || g < rows)) ? full * sl2 : -INFINITY;
      }
      // ---- chunk max per head across the group's 128 threads (paired: per
      // half warp)
      float* rb = red_t + par * 64;
      {
        float v[NC];
#pragma unroll
        for (int g = 0; g < NC; ++g) v[g] = so[g];
        const float mx = xreduce<NC, SPAN, true>(v, lane);
        const int cg = (lane & (SPAN - 1)) / (SPAN / NC);
        if ((lane & (SPAN / NC - 1)) == 0) rb[wq * 16 + hd * GH + cg] = mx;
      }
      if (!group_sync(gbar, gphase, abrt, status)) break;
      float alpha[GT];
      float cmx[GT];   // the chunk's max per column over the group's four warps
#pragma unroll
      for (int g4 = 0; g4 < GT; g4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(rb + g4);
        const float4 b = *reinterpret_cast<const float4*>(rb + 16 + g4);
        const float4 c = *reinterpret_cast<const float4*>(rb + 32 + g4);
        const float4 d = *reinterpret_cast<const float4*>(rb + 48 + g4);
        cmx[g4] = fmaxf(fmaxf(a.x, b.x), fmaxf(c.x, d.x));
        cmx[g4 + 1] = fmaxf(fmaxf(a.y, b.y), fmaxf(c.y, d.y));
        cmx[g4 + 2] = fmaxf(fmaxf(a.z, b.z), fmaxf(c.z, d.z));
        cmx[g4 + 3] = fmaxf(fmaxf(a.w, b.w), fmaxf(c.w, d.w));
      }
      float pv[NC];   // the thread's token's probabilities for its query columns
      if constexpr (PAIR) {
        // every column's running max and rescale (the correction below takes
        // all of them), then the own head's probabilities
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float cm = cmx[g];
          const float mn = fmaxf(m_run[g], cm);
          alpha[g] = (mn == -INFINITY) ? 0.f : ex2(m_run[g] - mn);
          m_run[g] = mn;
        }
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          const float mn = hd ? m_run[GH + g] : m_run[g];
          const float al = hd ? alpha[GH + g] : alpha[g];
          const float pr = (mn == -INFINITY) ? 0.f : ex2(so[g] - mn);
          l_thr[g] = fmaf(l_thr[g], al, pr);
          pv[g] = pr;
        }
      } else {
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float cm = cmx[g];
          const float mn = fmaxf(m_run[g], cm);
          // rows g >= rows never see a finite score; keep them inert (alpha 0, p 0)
          alpha[g] = (mn == -INFINITY) ? 0.f : ex2(m_run[g] - mn);
          const float pr = (mn == -INFINITY) ? 0.f : ex2(so[g] - mn);
          m_run[g] = mn;
          l_thr[g] = fmaf(l_thr[g], alpha[g], pr);
          pv[g] = pr;
        }
      }
      // P^T row own_t: columns [0, GT) hold the hi parts, [GT, 2 GT) the lo
      // parts (paired: the own head's columns; the other head's are zero),
      // two columns to a word
      uint32_t wd[NPV / 2];
#pragma unroll
      for (int i = 0; i < NPV / 2; ++i) wd[i] = 0u;
#pragma unroll
      for (int k = 0; k < NC / 2; ++k) {
        uint32_t hi, lo;
        split16x2<T>(pv[2 * k], pv[2 * k + 1], hi, lo);
        if constexpr (PAIR) {
          wd[k] = hd ? 0u : hi;
          wd[GH / 2 + k] = hd ? hi : 0u;
          wd[GT / 2 + k] = hd ? 0u : lo;
          wd[GT / 2 + GH / 2 + k] = hd ? lo : 0u;
        } else {
          wd[k] = hi;
          wd[GT / 2 + k] = lo;
        }
      }
#pragma unroll
      for (int ng = 0; ng < NPV / 8; ++ng)
        *reinterpret_cast<uint4*>(pdst_base + ng * 2048) =
            make_uint4(wd[4 * ng], wd[4 * ng + 1], wd[4 * ng + 2], wd[4 * ng + 3]);
      bool vok = true;
      // past the chunk's valid tokens but inside the last 16-token step of
      // the P.V MMA (paired: inside the last loaded block): make V finite
      // (zero) once the stage's V has landed
      const int v_end = PAIR ? (mt.valid + BS - 1) / BS * BS : (mt.valid + 15) & ~15;
      if (own_rt >= mt.valid && own_rt < v_end) {
        vok = mbar_wait(&vfull[bi], fpar, abrt, status);
        if (vok) {
          uint8_t* vrow = smem + static_cast<size_t>(stage) * kStage + vrow_off;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            reinterpret_cast<uint4*>(vrow)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(vrow + sh * 128)[i] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      if (!__all_sync(kFull, vok)) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
      if (Ly::DEFER_END && pend) {
        // the previous item's end, while the P.V MMA runs (the max barrier
        // above made every warp's l sums visible)
        if (!finish(lred_t + (lpar ^ 1u) * 64, pend_seq, pend_kvh, pend_split, o_pend, m_pend))
          break;
        pend = false;
      }
      // ---- correction: O = alpha * O + O_chunk (thread r owns column d = r)
      if (!__all_sync(kFull, mbar_wait(&o_full[t], par, abrt, status))) break;
      tc_fence_after();
      float ov[NPV];
      tmem_ld16(lane_addr + o_col, ov);
      if constexpr (NPV == 32) tmem_ld16(lane_addr + o_col + 16, ov + 16);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[t]);
#pragma unroll
      for (int g = 0; g < GT; ++g) o[g] = fmaf(o[g], alpha[g], ov[g] + ov[GT + g]);
      ++n;

      if (mt.flags & kLast) {
        // per-warp sum of l over the group's 128 tokens
        float* lr = lred_t + (Ly::DEFER_END ? lpar : 0u) * 64;
        {
          float v[NC];   // paired: the own head's sums
#pragma unroll
          for (int g = 0; g < NC; ++g) v[g] = l_thr[g];
          const float lg = xreduce<NC, SPAN, false>(v, lane);
          const int cg = (lane & (SPAN - 1)) / (SPAN / NC);
          if ((lane & (SPAN / NC - 1)) == 0) lr[wq * 16 + hd * GH + cg] = lg;
        }
        if constexpr (Ly::DEFER_END) {
#pragma unroll
          for (int g = 0; g < GT; ++g) {
            o_pend[g] = o[g];
            m_pend[g] = m_run[g];
          }
          pend_seq = mt.seq;
          pend_kvh = mt.kvh;
          pend_split = mt.split_raw;
          pend = true;
          lpar ^= 1u;
        } else {
          if (!group_sync(gbar, gphase, abrt, status)) break;
          if (!finish(lr, mt.seq, mt.kvh, mt.split_raw, o, m_run)) break;
        }
      }
    }
    // ---- merges of the split sequences, one output row per task. After its
    // last item the group claims tasks, waits until every piece of the row's
    // (sequence, KV head) has been counted, and merges the row: warp w of the
    // group folds pieces w, w + 4, ... (lane l: columns 4l .. 4l + 3, 8
    // pieces' loads in flight), then thread r combines the four warps'
    // results for column r. Outside the main loop, so the merge neither
    // stalls the ring nor adds to the loop's registers; the groups that
    // finish first share the merges out. A group waits only on pieces that
    // streams of running CTAs have claimed (every item was claimed before any
    // stream saw END), so every wait ends.
    // (None in the launch over the group list: its pieces are merged by the
    // launch of the members' own pieces, which runs after it.)
    if (!GRP && !*abrt) {
      const int32_t* split_list = reinterpret_cast<const int32_t*>(p.ws + p.split_off);
      const int32_t* nsplit_of = reinterpret_cast<const int32_t*>(p.ws + p.nsplit_off);
      const int Hq = p.num_q_heads;
      const int ntasks = hdr->num_split_seqs * Hq;
      // the group's P buffer (free once its stream has ended): per warp its
      // running max and sum, then its 128 column sums
      float* wml = reinterpret_cast<float*>(pbuf + t * Ly::PBUF);
      float* wacc = wml + 8;
      static_assert(Ly::PBUF >= (8 + 4 * kD) * 4, "merge scratch fits the P buffer");
      for (;;) {
        if (wq == 0 && lane == 0) {
          int k = atomicAdd(&hdr->merge_counter, 1);
          if (k < ntasks) {
            const int j = k / Hq;
            const int sq = split_list[j];
            const int kv = (k - j * Hq) / G;
            const int nsp = nsplit_of[sq];
            volatile int* c = cnt + static_cast<size_t>(sq) * Hkv + kv;
            const unsigned long long t0 = global_timer_ns();
            while (*c < nsp) {
              if (*abrt || global_timer_ns() - t0 > kWaitLimitNs) {
                if (!*abrt) atomicExch(status, 6 /* PA_ERR_DEVICE_TIMEOUT */);
                *abrt = 1;
                k = ntasks;
                break;
              }
            }
          }
          s_last[t] = k;
        }
        if (!group_sync(gbar, gphase, abrt, status)) break;
        const int k = s_last[t];
        if (k >= ntasks) break;
        __threadfence();   // the counted pieces' partial results are visible
        const int j = k / Hq;
        const int sq = split_list[j];
        const int nsp = nsplit_of[sq];
        const size_t row = static_cast<size_t>(sq) * Hq + (k - j * Hq);
        const float2* mr = ml + row * p.max_splits;
        const float4* pr4 = reinterpret_cast<const float4*>(po + row * p.max_splits * kD) + lane;
        float M = -INFINITY, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = wq; s0 < nsp; s0 += 32) {
          float2 e[8];
          float4 v[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int sp = s0 + 4 * jj;
            const bool in = sp < nsp;
            e[jj] = in ? __ldcg(mr + sp) : make_float2(-INFINITY, 0.f);
            v[jj] = in ? __ldcg(pr4 + static_cast<size_t>(sp) * (kD / 4))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float mb = M;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) mb = fmaxf(mb, e[jj].x);
          const float sc = exp2f(M - mb);   // M = -inf on the first batch: 0
          L *= sc;
          acc.x *= sc;
          acc.y *= sc;
          acc.z *= sc;
          acc.w *= sc;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float w = exp2f(e[jj].x - mb);   // 0 for the padding entries
            L = fmaf(e[jj].y, w, L);
            acc.x = fmaf(w, v[jj].x, acc.x);
            acc.y = fmaf(w, v[jj].y, acc.y);
            acc.z = fmaf(w, v[jj].z, acc.z);
            acc.w = fmaf(w, v[jj].w, acc.w);
          }
          M = mb;
        }
        // a warp without pieces (nsp < 4) leaves M = -inf, L = 0: weight 0
        if (lane == 0) {
          wml[2 * wq] = M;
          wml[2 * wq + 1] = L;
        }
        reinterpret_cast<float4*>(wacc + wq * kD)[lane] = acc;
        if (!group_sync(gbar, gphase, abrt, status)) break;
        float Mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) Mt = fmaxf(Mt, wml[2 * w]);
        float Lt = 0.f, at = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float sw = exp2f(wml[2 * w] - Mt);
          Lt = fmaf(wml[2 * w + 1], sw, Lt);
          at = fmaf(wacc[w * kD + r], sw, at);
        }
        p.out[row * kD + r] = at / Lt;
        // the task slot and the scratch are rewritten only after every
        // thread has read them
        if (!group_sync(gbar, gphase, abrt, status)) break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Ly::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps and launch
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D map over a [rows, cols] 16-bit matrix with the given row pitch, box =
// 64 columns x box_rows rows, 128-byte swizzle; out-of-range rows read as zero.
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                     uint64_t row_bytes, uint32_t box_rows, bool bf16) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D map over q as [num_seqs, num_q_heads, 128] 16-bit elements, box = 64
// columns x G heads x 16 / G sequences (16 rows in the 2-D box's order),
// 128-byte swizzle; sequences past the end read as zero.
cudaError_t make_q_group_map(CUtensorMap* m, const void* q, int num_seqs, int num_q_heads, int G,
                             bool bf16) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (G < 1 || 16 % G != 0) return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(num_seqs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2,
                           static_cast<cuuint64_t>(num_q_heads) * kD * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(16 / G)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T, int GT, bool GRP = false, bool PAIR = false>
cudaError_t launch_t(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  using Ly = TcLayout<GT>;
  const bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap mk, mv, mq;
  // pools as [half-rows, 64]: a (block, head) tile is 2 * block_size
  // consecutive 128-byte half-rows in its storage order, loaded as one box
  // (two heads' tiles when paired)
  const uint64_t half_rows =
      static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * p.block_size * 2;
  const uint32_t box_rows = (PAIR ? 4 : 2) * p.block_size;
  cudaError_t e = make_map(&mk, p.k_cache, 64, half_rows, 128, box_rows, bf16);
  if (e == cudaSuccess) e = make_map(&mv, p.v_cache, 64, half_rows, 128, box_rows, bf16);
  // q as [rows, 128]: one box per column half, NS/2 query rows; for the
  // group list, the rows of G heads of 16 / G consecutive sequences
  if (e == cudaSuccess) {
    if constexpr (GRP) {
      static_assert(Ly::NS / 2 == 16, "group items fill a 16-row tile");
      e = make_q_group_map(&mq, p.q, p.num_seqs, p.num_q_heads, p.num_q_heads / p.num_kv_heads,
                           bf16);
    } else {
      e = make_map(&mq, p.q, kD, static_cast<uint64_t>(p.num_seqs) * p.num_q_heads, kD * 2,
                   Ly::NS / 2, bf16);
    }
  }
  if (e != cudaSuccess) return e;
  auto kern = tc_decode_kernel<T, GT, GRP, PAIR>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(Ly::SMEM));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(num_ctas), dim3(kThreads), Ly::SMEM, stream, p, mk, mv, mq);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

bool tc_supported(int dtype, int head_dim, int group) {
  return (dtype == 1 || dtype == 2) && head_dim == kD && group >= 4 && group <= 16 &&
         encode_fn() != nullptr;
}

cudaError_t tc_num_ctas(int dtype, int group, int* num_ctas) {
  (void)dtype;
  (void)group;
  *num_ctas = num_sms();   // one CTA per SM (shared memory and TMEM sized for it)
  return cudaSuccess;
}

bool tc_group_supported(int dtype, int head_dim, int group) {
  return (dtype == 1 || dtype == 2) && head_dim == kD && group >= 1 && group <= 8 &&
         16 % group == 0 && encode_fn() != nullptr;
}

cudaError_t launch_decode_tc_groups(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  const int group = p.num_q_heads / p.num_kv_heads;
  if (!p.group_mode || !tc_group_supported(p.dtype, p.head_dim, group)) return cudaErrorInvalidValue;
  if (p.dtype == 2) return launch_t<__nv_bfloat16, 16, true>(p, num_ctas, stream);
  return launch_t<__half, 16, true>(p, num_ctas, stream);
}

bool tc_pair_supported(int block_size, int num_kv_heads, int group) {
  // a pair of KV heads of 4 (8) query heads each fills the 8-row (16-row)
  // tile exactly
  return block_size == 8 && num_kv_heads % 2 == 0 && (group == 4 || group == 8);
}

cudaError_t launch_decode_tc(const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  const int group = p.num_q_heads / p.num_kv_heads;
  if (!tc_supported(p.dtype, p.head_dim, group)) return cudaErrorInvalidValue;
  if (p.pair_heads) {
    // a pair is one KV head of 2G query heads
    if (!tc_pair_supported(p.block_size, p.num_kv_heads, group)) return cudaErrorInvalidValue;
    if (p.dtype == 2) {
      if (group == 4) return launch_t<__nv_bfloat16, 8, false, true>(p, num_ctas, stream);
      return launch_t<__nv_bfloat16, 16, false, true>(p, num_ctas, stream);
    }
    if (group == 4) return launch_t<__half, 8, false, true>(p, num_ctas, stream);
    return launch_t<__half, 16, false, true>(p, num_ctas, stream);
  }
  if (p.dtype == 2) {
    if (group <= 4) return launch_t<__nv_bfloat16, 4>(p, num_ctas, stream);
    if (group <= 8) return launch_t<__nv_bfloat16, 8>(p, num_ctas, stream);
    return launch_t<__nv_bfloat16, 16>(p, num_ctas, stream);
  }
  if (group <= 4) return launch_t<__half, 4>(p, num_ctas, stream);
  if (group <= 8) return launch_t<__half, 8>(p, num_ctas, stream);
  return launch_t<__half, 16>(p, num_ctas, stream);
}

}  // namespace pa
