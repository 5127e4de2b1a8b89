// Paged MLA split-KV decode kernel for sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes: for each (sequence, KV head, row group of up to 128 query
// rows) and each scheduler part, the softmax attention of the rows over the
// part's pages of the sequence (FlashMLA overview, section 2.2 attention
// equation, absorbed form: 576-wide keys, values = first 512 columns of the
// same cached row; pages through block_table, section 4.2(1)).  A piece that
// covers a whole sequence writes o (bf16) and lse directly; a piece of a split
// sequence writes a normalised fp32 partial and its lse, merged later by the
// combine kernel (the "merge of split results" kernel the article names).
//
// Design (B200-specific; the Hopper design on the pages is prior art only).
// A 128-row tile needs the query (128x576 bf16), S = Q K^T (fp32) and the
// output accumulator O (128x512 fp32 = all 512 TMEM columns of an SM).  That
// does not fit one SM, so every work unit is a 2-CTA cluster with split roles:
//
//   CTA 0 ("S-CTA"): the latent part of Q (512 columns) lives in TMEM as an MMA
//     A operand (256 columns of bf16 pairs), its RoPE part (64 columns) in
//     shared memory; S is double-buffered in the other 2 x 128 TMEM columns.
//     Two TMA producer threads stream 16 KB chunk stages through an 8-stage
//     ring: chunk c of two consecutive pages (rows 0-63 page A, rows 64-127
//     page B, 64 columns, 128B swizzle; one producer per page), so one MMA
//     covers 128 tokens (N = 128 runs the tensor core at full rate, N = 64
//     does not).  The query arrives through the same ring; the MMA thread
//     copies its latent chunks into TMEM (tcgen05.cp) and issues per page pair
//     32 TS MMAs (latent, A from TMEM) + 4 SS MMAs (RoPE).  Two softmax
//     warpgroups (one row per thread, one page of the pair each) read S, apply
//     the mask, exchange row maxima, keep the running max/sum in fp32 with a
//     lazy rescale (the reference max only moves when a pair's max exceeds it
//     by 2^8), stage P (bf16, swizzled K-major MMA layout) plus per-row
//     factors in shared memory, and one thread bulk-copies them into a P slot
//     of CTA 1, completing bytes on CTA 1's slot barrier.
//   CTA 1 ("O-CTA"): a TMA warp streams the value part of the same pages in
//     32 KB half-page stages (mostly L2 hits: CTA 0 just read the page); one
//     thread issues O += P V as 8 MMAs per page (M=128, N=256, K=16, V
//     MN-major) into the 512-column accumulator; a relay warp re-arms each
//     consumed P slot's barrier and returns the slot to CTA 0; two correction
//     warpgroups (256 accumulator columns each) sum the bf16 weights they see
//     into the row sums, rescale O rows when CTA 0 moved a row's reference
//     max, and run the epilogue (O / l -> bf16 o, or fp32 partials) at the end
//     of each piece.
//
// Pair variant (two or more row groups per KV head, e.g. two query tokens x 128
// heads): the two 128-row groups of a (sequence, part) read the same pages, so
// they share one 4-CTA cluster built from two CTA pairs (cta_group::2) instead
// of two independent clusters:
//   ranks 0, 1 (S pair): each CTA holds the query of its own row group in TMEM
//     and streams only its own page of each page pair from HBM (rank 0 page A,
//     rank 1 page B, chunk stages of 16 KB = two 64-column chunks); one thread
//     of rank 0 issues M = 256 score MMAs whose B operand (the 128 tokens of the
//     pair) is split between the two CTAs' shared memory, so every page byte
//     enters one SM once and feeds both tensor cores.  Each CTA's softmax
//     warpgroups then work on their own 128 rows exactly as above and send P
//     to the O-CTA of their row group (rank + 2).
//   ranks 2, 3 (O pair): each loads only its half of the value columns of each
//     page ({0,1,4,5} or {2,3,6,7} of the eight 64-column chunks); one thread
//     of rank 2 issues M = 256 (both row groups) by N = 256 MMAs whose B operand
//     (the value tile) is split the same way; each CTA keeps its row group's
//     128 x 512 accumulator.  Rescale and epilogue commands go to both CTAs.
// Compared with two independent clusters this halves the bytes each page puts
// through shared memory and the B-operand shared-memory reads per MMA.
//
// Launch: a programmatic dependent of the counter-clear kernel (setup overlaps
// the kernels before it; the schedule is read after griddepcontrol.wait); its
// own dependent, the merge kernel, may start as soon as every CTA is resident.
// Every wait is bounded (see ptx.cuh); a timeout records an error code and
// makes all roles leave their loops, drain their in-flight copies and MMAs,
// free TMEM and exit.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kThreads = 384;  // 4 role warps + two 4-warp groups
constexpr int kRing = 8;                           // S-CTA chunk stages
constexpr int kStageBufs = 4;                      // S-CTA P staging buffers
constexpr uint32_t kChunkBytes = 128 * 64 * 2;     // 128 rows x 64 columns bf16
constexpr uint32_t kPageChunkBytes = 64 * 64 * 2;  // one page's 64 tokens x 64 columns
constexpr int kVStages = 4;                        // O-CTA half-page stages
constexpr uint32_t kVStageBytes = 4 * kPageChunkBytes;  // 64 tokens x 256 columns
constexpr int kPSlots = 5;
constexpr uint32_t kPBytes = kRows * kPage * 2;    // 128 x 64 bf16

struct SideSlot {        // per-P-slot row data sent with every P tile
  uint32_t wflag[4];     // per softmax warp: some row of the warp moved its reference max
  float alpha[kRows];    // O row rescale factors (1 = unchanged)
};
constexpr uint32_t kSideBytes = sizeof(SideSlot);
constexpr uint32_t kPFullTx = kPBytes + kSideBytes;  // bytes every P message carries

struct Mailbox {         // MMA thread -> correction warps (O-CTA)
  int cmd;               // kCmdRescale or kCmdEpilogue
  int slot;              // P slot whose alpha to apply (rescale)
  int b;
  int part_slot;         // partial slot index, or -1 for a direct write
  float lr_x[2][2][kRows];  // [piece parity][correction group] row-sum halves
};
enum : int { kCmdRescale = 1, kCmdEpilogue = 2 };

// mbarriers: one index space for both CTAs, each CTA initialises its own
enum : int {
  kBarRingFull = 0,                      // S [kRing] chunk stage loaded (TMA tx)
  kBarRingEmpty = kBarRingFull + kRing,  // S [kRing] chunk stage consumed
  kBarSFull = kBarRingEmpty + kRing,     // S [2] S tile ready (commit)
  kBarSFree = kBarSFull + 2,             // S [2] S tile read by softmax warps (256)
  kBarQrFull = kBarSFree + 2,            // S Q RoPE chunk loaded (TMA tx)
  kBarQrEmpty = kBarQrFull + 1,          // S Q RoPE chunk no longer read (commit)
  kBarPFree = kBarQrEmpty + 1,           // S [kPSlots] P slot free again (remote arrival)
  kBarStageFree = kBarPFree + kPSlots,   // S [kStageBufs] staging buffer copied out (remote arrival)
  kBarVFull = kBarStageFree + kStageBufs,  // O [4] V half-stage loaded (TMA tx)
  kBarVEmpty = kBarVFull + kVStages,     // O [4] V half-stage consumed (commit)
  kBarPFull = kBarVEmpty + kVStages,     // O [kPSlots] P slot written (armed + bulk-copy tx)
  kBarPCons = kBarPFull + kPSlots,       // O [kPSlots] P slot consumed (commit + 8 warps; pair: + 8 of the mate)
  kBarPeerP = kBarPCons + kPSlots,       // O [kPSlots] pair: the mate O-CTA's P slot landed (remote arrival)
  kBarFlagsRead = kBarPeerP + kPSlots,   // O [kPSlots] pair: this CTA's 8 correction warps read the mate's flags
  kBarSFreeFwd = kBarFlagsRead + kPSlots,  // S [2] pair, odd CTA: its softmax read S (relayed to the leader)
  kBarCmdFull = kBarSFreeFwd + 2,        // O mailbox command posted (1)
  kBarCmdDone = kBarCmdFull + 1,         // O command done (256; pair: 1 per O-CTA, on rank 2)
  kBarDrain = kBarCmdDone + 1,           // both: all issued MMAs complete
  kNumBars = kBarDrain + 1
};

struct Ctrl {
  uint64_t bar[kNumBars];
  uint32_t tmem_base;
  int abort_flag;
};

// shared-memory layouts (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_QROPE = 0;                                 // S-CTA: Q RoPE chunk
constexpr uint32_t OFF_RING = kChunkBytes;                        // S-CTA: chunk ring
constexpr uint32_t OFF_STAGE = OFF_RING + kRing * kChunkBytes;    // S-CTA: P staging
constexpr uint32_t OFF_V = 0;                                     // O-CTA: V ring
constexpr uint32_t OFF_P = OFF_V + kVStages * kVStageBytes;       // O-CTA: P slots
constexpr uint32_t OFF_SIDE = OFF_P + kPSlots * kPBytes;          // O-CTA: side slots
constexpr uint32_t OFF_MAIL = OFF_SIDE + kPSlots * kSideBytes;    // O-CTA: mailbox
constexpr uint32_t OFF_STAGE_SIDE = OFF_STAGE + kStageBufs * kPBytes;  // S-CTA: staged side data
constexpr uint32_t OFF_XCH = OFF_STAGE_SIDE + kStageBufs * kSideBytes;  // S-CTA: row exchange
constexpr uint32_t kXchBytes = (2 * 2 * kRows + 2 * kRows) * 4;  // max x2 pairs, l
constexpr uint32_t cmax(uint32_t a, uint32_t b) { return a > b ? a : b; }
constexpr uint32_t OFF_CTRL =  // both: after the larger of the two CTA layouts
    (cmax(OFF_XCH + kXchBytes, OFF_MAIL + (uint32_t)sizeof(Mailbox)) + 15u) & ~15u;
constexpr uint32_t SMEM_BYTES = OFF_CTRL + sizeof(Ctrl);
static_assert(OFF_MAIL + sizeof(Mailbox) <= OFF_CTRL, "O-CTA regions overlap the control block");
static_assert(SMEM_BYTES <= 232448, "shared memory budget exceeded");
static_assert(OFF_P % 1024 == 0 && OFF_RING % 1024 == 0 && OFF_STAGE % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(OFF_SIDE % 16 == 0 && kSideBytes % 16 == 0, "side slots need 16-byte alignment");

// TMEM column map
constexpr uint32_t kTmemQ = 0;      // S-CTA: latent Q, 256 columns of bf16 pairs
constexpr uint32_t kTmemS = 256;    // S-CTA: two 128-column S tiles
constexpr uint32_t kTmemO = 0;      // O-CTA: 512 columns

constexpr float kLn2 = 0.69314718055994531f;
constexpr float kTau = 8.0f;        // lazy rescale threshold (log2 units)

struct Ring {
  uint32_t idx = 0, phase = 0;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++idx == n) { idx = 0; phase ^= 1u; }
  }
};

// Iterates the pieces of a scheduler part: calls f(b, p0, p1, ordinal).
// Pieces of a part run in sequence order on odd parts and in reverse on even
// parts.  A sequence cut between parts c and c + 1 then has both of its pieces
// processed first when c is even (its merge can run while the decode is still
// going); when c is odd both come last.  In plain order every cut sequence would
// wait for the end of a part.
struct PartIter {
  int b0, pg0, b1, pg1, ord0;
  bool rev;
  __device__ PartIter(const DecodeParams& P, int part) {
    const int32_t* m = P.meta + (size_t)part * kMetaInts;
    b0 = max(m[0], 0);
    pg0 = max(m[1], 0);
    b1 = min(m[2], P.batch);
    pg1 = m[3];
    ord0 = max(m[4], 0);
    rev = (part & 1) == 0;
  }
};

__device__ __forceinline__ int seq_pages(const DecodeParams& P, int b) {
  int L = P.seqlens[b];
  L = L < 0 ? 0 : L;
  int n = (L + kPage - 1) / kPage;
  return n < P.max_pages ? n : P.max_pages;
}

// A sequence longer than its block table (cache_seqlens[b] > 64 * max_pages)
// is skipped by every role alike -- nothing of it is read -- and recorded in
// the device error word; the merge kernel writes its rows as empty.
__device__ __forceinline__ bool seq_too_long(const DecodeParams& P, int b) {
  return (long long)P.seqlens[b] > (long long)P.max_pages * kPage;
}

template <class F>
__device__ __forceinline__ void for_each_piece(const DecodeParams& P, const PartIter& it, F&& f) {
  const int last = min(it.b1, P.batch - 1);
  for (int k = 0; k <= last - it.b0; ++k) {
    const int b = it.rev ? last - k : it.b0 + k;
    if (seq_too_long(P, b)) {
      if (threadIdx.x == 0) atomicCAS(P.err, 0, kErrBadSeqlen);
      continue;
    }
    const int n = seq_pages(P, b);
    const int p0 = (b == it.b0) ? min(it.pg0, n) : 0;
    const int p1 = (b == it.b1) ? min(max(it.pg1, 0), n) : n;
    if (p0 >= p1) continue;
    if (!f(b, p0, p1, b == it.b0 ? it.ord0 : 0)) return;
  }
}

__device__ __forceinline__ int piece_slot(const DecodeParams& P, int b, int ordinal) {
  const int s0 = P.num_splits[b], s1 = P.num_splits[b + 1];
  return (s1 - s0 >= 2) ? s0 + ordinal : -1;
}

__device__ __forceinline__ int load_page(const DecodeParams& P, int b, int p) {
  int page = P.block_table[(size_t)b * P.max_pages + p];
  if (page < 0 || page >= P.num_pages) {
    atomicCAS(P.err, 0, kErrBadPage);
    page = P.num_pages;  // outside the tensor map: TMA fills zeros
  }
  return page;
}

// TMA the 64-column chunk c of this tile's 128 query rows into `dst`
// (boxes of min(hpk,128) rows; rows past R are left untouched).  Returns bytes.
// kPairLoad: the bytes complete on `bar`, a barrier of either CTA of the pair.
template <bool kPairLoad = false>
__device__ __forceinline__ uint32_t load_q_chunk(const DecodeParams& P, const CUtensorMap* tmap_q,
                                                 uint32_t dst, uint32_t bar, int b, int g, int rg,
                                                 int c, uint64_t pol, bool issue) {
  const int qbox = P.hpk < kRows ? P.hpk : kRows;
  uint32_t bytes = 0;
  for (int j = 0; j < kRows / qbox; ++j) {
    const int rr0 = rg * kRows + j * qbox;
    if (rr0 >= P.R) break;
    if (issue) {
      const int qi = rr0 / P.hpk;
      const int row = (b * P.s_q + qi) * P.h_q + g * P.hpk + rr0 % P.hpk;
      if constexpr (kPairLoad)
        tma_load_2d_pair(dst + (uint32_t)(j * qbox * 128), tmap_q, bar, c * 64, row, pol);
      else
        tma_load_2d(dst + (uint32_t)(j * qbox * 128), tmap_q, bar, c * 64, row, pol);
    }
    bytes += (uint32_t)qbox * 128u;
  }
  return bytes;
}

// Error path of the pair variant: copies a CTA issued complete on the leader's
// barriers, which it cannot wait on, so it lets them land for a fixed time
// (far above any copy's latency) before its shared memory may be released.
__device__ __forceinline__ void settle_inflight_copies() {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
}

// kPair = false: 2-CTA clusters (S-CTA, O-CTA), one per 128-row group.
// kPair = true: 4-CTA clusters (S pair, O pair), one per two row groups; every
// tcgen05 instruction of this variant is a cta_group::2 one.
// The cluster shape is set at launch (2 or 4 CTAs along x).
template <bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_q,
              const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_kv2,
              const DecodeParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (sbase & 1023u) {  // layout assumption broken: report and leave (uniform branch)
    if (tid == 0) atomicCAS(P.err, 0, kErrBadSmemAlign);
    if (P.follows_decode && blockIdx.x == 0 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  constexpr int kClusterCtas = kPair ? 4 : 2;
  const uint32_t crank = cluster_ctarank();
  // role: 0 = S-CTA, 1 = O-CTA; half: which CTA of the pair (pair variant)
  const uint32_t rank = kPair ? (crank >> 1) : crank;
  const uint32_t half = kPair ? (crank & 1u) : 0u;
  const bool leader = half == 0;
  const uint32_t lead_rank = crank & ~1u;             // the pair's MMA-issuing CTA
  const uint32_t mate = crank ^ 1u;                   // the other CTA of the pair
  const uint16_t pair_mask = (uint16_t)(3u << lead_rank);
  const int cluster_id = blockIdx.x / kClusterCtas;
  const int units = kPair ? (P.n_rg + 1) / 2 : P.n_rg;  // clusters per KV head and part
  const int groups = P.h_kv * units;
  const int part = P.part0 + cluster_id / groups;
  const int g = (cluster_id % groups) / units;
  const int rg = kPair ? 2 * ((cluster_id % groups) % units) + (int)half : (cluster_id % groups) % units;

  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + OFF_CTRL);
  SideSlot* side = reinterpret_cast<SideSlot*>(smem + OFF_SIDE);
  Mailbox* mail = reinterpret_cast<Mailbox*>(smem + OFF_MAIL);
  volatile int* abortf = &ctrl->abort_flag;
  auto bar = [&](int i) { return smem_u32(&ctrl->bar[i]); };

  if (tid == 0) {
    if (rank == 0) {
      for (int s = 0; s < kRing; ++s) {
        // one arrival per TMA producer; pair: the leader's producer arms both CTAs' bytes
        mbar_init(bar(kBarRingFull + s), kPair ? 1 : 2);
        mbar_init(bar(kBarRingEmpty + s), 1);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(kBarSFull + s), 1);
        mbar_init(bar(kBarSFree + s), kPair ? 2 : 256);  // pair: one arrival per S-CTA
      }
      mbar_init(bar(kBarQrFull), 1);
      mbar_init(bar(kBarQrEmpty), 1);
      for (int s = 0; s < 2; ++s) mbar_init(bar(kBarSFreeFwd + s), 1);
      for (int s = 0; s < kPSlots; ++s) mbar_init(bar(kBarPFree + s), 1);
      for (int s = 0; s < kStageBufs; ++s) mbar_init(bar(kBarStageFree + s), 1);
    } else {
      for (int s = 0; s < kVStages; ++s) {
        mbar_init(bar(kBarVFull + s), 1);
        mbar_init(bar(kBarVEmpty + s), 1);
      }
      for (int s = 0; s < kPSlots; ++s) {
        mbar_init(bar(kBarPFull + s), 1);
        // commit + this CTA's 8 correction warps (+ pair: the mate's, relayed once)
        mbar_init(bar(kBarPCons + s), kPair ? 1 + 8 + 1 : 1 + 8);
        mbar_init(bar(kBarPeerP + s), 1);
        mbar_init(bar(kBarFlagsRead + s), 8);
      }
      mbar_init(bar(kBarCmdFull), 1);
      mbar_init(bar(kBarCmdDone), kPair ? 2 : 256);
    }
    mbar_init(bar(kBarDrain), 1);
    ctrl->abort_flag = 0;
    fence_mbar_init();
    if (rank == 1) {
      // arm every P slot for its first message (the relay re-arms after each use)
      for (int s = 0; s < kPSlots; ++s) mbar_arrive_expect_tx(bar(kBarPFull + s), kPFullTx);
    }
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(&ctrl->tmem_base), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_kv);
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_v);
    if (kPair) tma_prefetch_desc(&tmap_kv2);
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  // launched as a programmatic dependent of the counter clear: the setup above
  // overlaps the kernels before it; the schedule and the cleared counters are
  // read only after this wait (the clear's grid completes after the schedule's).
  // A decode launch that follows the call's first decode kernel (the 2-CTA
  // clusters on the SMs the 4-CTA clusters leave free) skips it: it is launched
  // only once every CTA of that kernel has passed this wait and triggered, so
  // the schedule and the clear have completed, and waiting here would wait for
  // that whole kernel.
  if (!P.follows_decode) asm volatile("griddepcontrol.wait;" ::: "memory");
  // every CTA of this grid is resident now: the next kernel (the merge, or the
  // second decode launch), launched as a programmatic dependent, may start on
  // SMs as they free up (the merge waits for the completion signals of the
  // pieces it merges)
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const PartIter it(P, part);
  // the CTA on the other side of the P hand-off (S-CTA <-> O-CTA of a row group)
  const uint32_t peer = kPair ? (crank ^ 2u) : (crank ^ 1u);

  if (rank == 0) {
    // =========================================================== S-CTA
    if ((warp == 0 || warp == 2) && lane == 0) {
      if constexpr (!kPair) {
      // ---- two TMA producers walk the same chunk-stage sequence; every stage's
      // full barrier takes one arrival from each.  Producer 0 loads the query
      // chunks and page A of each pair, producer 1 page B: one thread alone
      // cannot issue 8 KB tiles fast enough to keep the SM's fill rate up.
      const int prod = warp >> 1;
      Ring st;
      uint32_t qr_phase = 0;
      bool ok = true, qr_issued = false;
      uint32_t qr_issued_phase = 0;
      uint32_t issued_phase[kRing];
      bool issued[kRing];
      for (int s = 0; s < kRing; ++s) issued[s] = false;
      const uint64_t pol_q = policy_evict_last();
      const uint64_t pol_kv = policy_evict_normal();
      for_each_piece(P, it, [&](int b, int p0, int p1, int) {
        // latent query chunks 0..7 through the ring
        for (int c = 0; c < 8; ++c) {
          ok = mbar_wait(bar(kBarRingEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 1);
          if (!ok) return false;
          const uint32_t fb = bar(kBarRingFull + st.idx);
          if (prod == 0) {
            const uint32_t dst = sbase + OFF_RING + st.idx * kChunkBytes;
            mbar_arrive_expect_tx(fb, load_q_chunk(P, &tmap_q, dst, fb, b, g, rg, c, pol_q, false));
            load_q_chunk(P, &tmap_q, dst, fb, b, g, rg, c, pol_q, true);
            issued[st.idx] = true;
            issued_phase[st.idx] = st.phase;
          } else {
            mbar_arrive(fb);
          }
          st.next(kRing);
        }
        // RoPE chunk 8 into its own buffer (freed when the piece's MMAs are done)
        if (prod == 0) {
          ok = mbar_wait(bar(kBarQrEmpty), qr_phase ^ 1u, abortf, P.err, kErrWaitBase + 2);
          if (!ok) return false;
          const uint32_t fb = bar(kBarQrFull);
          mbar_arrive_expect_tx(fb, load_q_chunk(P, &tmap_q, sbase + OFF_QROPE, fb, b, g, rg, 8, pol_q, false));
          load_q_chunk(P, &tmap_q, sbase + OFF_QROPE, fb, b, g, rg, 8, pol_q, true);
          qr_issued = true;
          qr_issued_phase = qr_phase;
          qr_phase ^= 1u;
        }
        // page pairs: chunk c of page A at +0, of page B at +8 KB
        for (int pa = p0; pa < p1; pa += 2) {
          const bool has = prod == 0 || pa + 1 < p1;
          const int page = has ? load_page(P, b, pa + prod) : 0;
          const uint32_t off = (uint32_t)prod * kPageChunkBytes;
          for (int c = 0; c < 9; ++c) {
            ok = mbar_wait(bar(kBarRingEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 3);
            if (!ok) return false;
            const uint32_t fb = bar(kBarRingFull + st.idx);
            if (has) {
              mbar_arrive_expect_tx(fb, kPageChunkBytes);
              tma_load_3d(sbase + OFF_RING + st.idx * kChunkBytes + off, &tmap_kv, fb, c * 64, g,
                          page * kPage, pol_kv);
              issued[st.idx] = true;
              issued_phase[st.idx] = st.phase;
            } else {
              mbar_arrive(fb);
            }
            st.next(kRing);
          }
        }
        return true;
      });
      if (!ok) {  // drain copies still in flight before the CTA may exit
        for (int s = 0; s < kRing; ++s)
          if (issued[s]) mbar_wait_drain(bar(kBarRingFull + s), issued_phase[s]);
        if (qr_issued) mbar_wait_drain(bar(kBarQrFull), qr_issued_phase);
      }
      } else {
        // ---- pair: the two producers of each S-CTA take turns over the stages.
        // Each CTA loads its own row group's query and its own page of every
        // pair (rank 0 page A, rank 1 page B; a missing page B reads as zeros,
        // from outside the tensor map), the page in stages of two 64-column
        // chunks; all bytes complete on the leader's barriers, which the
        // leader's producer arms for both CTAs.
        const int prod = warp >> 1;
        Ring st;
        uint32_t turn = 0;  // running stage count: stage k belongs to producer k % 2
        uint32_t qr_phase = 0;
        bool ok = true;
        const uint64_t pol_q = policy_evict_last();
        const uint64_t pol_kv = policy_evict_normal();
        const uint32_t lead_full0 = map_to_rank(bar(kBarRingFull), lead_rank);
        const uint32_t lead_qr = map_to_rank(bar(kBarQrFull), lead_rank);
        const uint32_t q_bytes = load_q_chunk(P, &tmap_q, 0, 0, 0, g, rg, 0, 0, false) +
                                 load_q_chunk(P, &tmap_q, 0, 0, 0, g, rg ^ 1, 0, 0, false);
        for_each_piece(P, it, [&](int b, int p0, int p1, int) {
          for (int c = 0; c < 8; ++c, ++turn) {
            if ((turn & 1u) == (uint32_t)prod) {
              ok = mbar_wait<true>(bar(kBarRingEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 1);
              if (!ok) return false;
              if (leader) mbar_arrive_expect_tx(bar(kBarRingFull + st.idx), q_bytes);
              load_q_chunk<true>(P, &tmap_q, sbase + OFF_RING + st.idx * kChunkBytes, lead_full0 + 8u * st.idx,
                                 b, g, rg, c, pol_q, true);
            }
            st.next(kRing);
          }
          if (prod == 0) {
            ok = mbar_wait<true>(bar(kBarQrEmpty), qr_phase ^ 1u, abortf, P.err, kErrWaitBase + 2);
            if (!ok) return false;
            if (leader) mbar_arrive_expect_tx(bar(kBarQrFull), q_bytes);
            load_q_chunk<true>(P, &tmap_q, sbase + OFF_QROPE, lead_qr, b, g, rg, 8, pol_q, true);
            qr_phase ^= 1u;
          }
          for (int pa = p0; pa < p1; pa += 2) {
            const int page = half == 0 ? load_page(P, b, pa) : (pa + 1 < p1 ? load_page(P, b, pa + 1) : P.num_pages);
            for (int s = 0; s < 5; ++s, ++turn) {
              if ((turn & 1u) == (uint32_t)prod) {
                ok = mbar_wait<true>(bar(kBarRingEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 3);
                if (!ok) return false;
                const uint32_t dst = sbase + OFF_RING + st.idx * kChunkBytes;
                const uint32_t fb = lead_full0 + 8u * st.idx;
                if (leader) mbar_arrive_expect_tx(bar(kBarRingFull + st.idx), (s < 4 ? 4u : 2u) * kPageChunkBytes);
                if (s < 4)  // chunks 2s and 2s+1 of the page, chunk-major
                  tma_load_4d_pair(dst, &tmap_kv2, fb, 0, page * kPage, 2 * s, g, pol_kv);
                else        // the RoPE chunk
                  tma_load_3d_pair(dst, &tmap_kv, fb, 8 * 64, g, page * kPage, pol_kv);
              }
              st.next(kRing);
            }
          }
          return true;
        });
        if (!ok) settle_inflight_copies();
      }
    } else if (warp == 1 && lane == 0) {
      if constexpr (!kPair) {
      // ---- MMA issuer: S = Q K^T for page pairs (N = 128) or a single page (N = 64)
      Ring st, sb;
      uint32_t qr_phase = 0;
      bool ok = true;
      const uint32_t idesc128 = make_idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc64 = make_idesc_bf16(128, 64, 0, 0);
      const uint64_t ring_desc0 = make_smem_desc(sbase + OFF_RING, 16, 1024, 2);
      const uint64_t qr_desc = make_smem_desc(sbase + OFF_QROPE, 16, 1024, 2);
      const uint32_t ring_empty0 = bar(kBarRingEmpty);
      const uint32_t ring_full0 = bar(kBarRingFull);
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        // latent query chunks 0..7 -> TMEM columns [32c, 32c + 32) by tcgen05.cp;
        // the copies execute in order with the MMAs below (and after the previous
        // piece's MMAs, which still read the old query)
        for (int c = 0; c < 8; ++c) {
          if (!mbar_wait(ring_full0 + 8u * st.idx, st.phase, abortf, P.err, kErrWaitBase + 9))
            return false;
          tc_fence_after();
          const uint64_t qd = ring_desc0 + (uint64_t)(st.idx * (kChunkBytes >> 4));
#pragma unroll
          for (int k = 0; k < 4; ++k) tmem_cp_128x256b(tmem + kTmemQ + 32u * c + 8u * k, qd + 2 * k);
          tc_commit(ring_empty0 + 8u * st.idx);
          st.next(kRing);
        }
        bool first = true;
        for (int pa = p0; pa < p1; pa += 2) {
          const int npg = (pa + 1 < p1) ? 2 : 1;
          const uint32_t idesc = npg == 2 ? idesc128 : idesc64;
          const bool last_pair = pa + 2 >= p1;
          ok = mbar_wait(bar(kBarSFree + sb.idx), sb.phase ^ 1u, abortf, P.err, kErrWaitBase + 4);
          if (!ok) return false;
          const uint32_t dS = tmem + kTmemS + 128u * sb.idx;
          // the pair's 9 chunk stages, issued fully unrolled with precomputed
          // stage indices: per-chunk waits stay (TMA streams chunk by chunk) but
          // no descriptor or ring arithmetic sits between the MMAs
          tc_fence_after();
          uint32_t sidx[9], sph[9];
#pragma unroll
          for (int c = 0; c < 9; ++c) {
            sidx[c] = st.idx;
            sph[c] = st.phase;
            st.next(kRing);
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (!mbar_wait(ring_full0 + 8u * sidx[c], sph[c], abortf, P.err, kErrWaitBase + 6))
              return false;
            const uint64_t bd = ring_desc0 + (uint64_t)(sidx[c] * (kChunkBytes >> 4));
            const uint32_t a = tmem + kTmemQ + 32u * c;
            mma_ts(dS, a, bd, idesc, c > 0);
            mma_ts(dS, a + 8, bd + 2, idesc, 1);
            mma_ts(dS, a + 16, bd + 4, idesc, 1);
            mma_ts(dS, a + 24, bd + 6, idesc, 1);
            tc_commit(ring_empty0 + 8u * sidx[c]);
          }
          if (!mbar_wait(ring_full0 + 8u * sidx[8], sph[8], abortf, P.err, kErrWaitBase + 7))
            return false;
          if (first) {
            if (!mbar_wait(bar(kBarQrFull), qr_phase, abortf, P.err, kErrWaitBase + 8)) return false;
            qr_phase ^= 1u;
          }
          {
            const uint64_t bd = ring_desc0 + (uint64_t)(sidx[8] * (kChunkBytes >> 4));
            mma_ss(dS, qr_desc, bd, idesc, 1);
            mma_ss(dS, qr_desc + 2, bd + 2, idesc, 1);
            mma_ss(dS, qr_desc + 4, bd + 4, idesc, 1);
            mma_ss(dS, qr_desc + 6, bd + 6, idesc, 1);
            tc_commit(ring_empty0 + 8u * sidx[8]);
          }
          tc_commit(bar(kBarSFull + sb.idx));
          if (last_pair) tc_commit(bar(kBarQrEmpty));
          sb.next(2);
          first = false;
        }
        return true;
      });
      tc_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
      } else if (leader) {
        // ---- pair MMA issuer (rank 0): S = Q K^T of both row groups, M = 256
        // (rows of rank 0 then rank 1), N = 128 (page A from rank 0's shared
        // memory, page B from rank 1's), K in stages of two chunks
        Ring st, sb;
        uint32_t qr_phase = 0;
        const uint32_t idesc = make_idesc_bf16(256, 128, 0, 0);
        const uint64_t ring_desc0 = make_smem_desc(sbase + OFF_RING, 16, 1024, 2);
        const uint64_t qr_desc = make_smem_desc(sbase + OFF_QROPE, 16, 1024, 2);
        const uint32_t ring_empty0 = bar(kBarRingEmpty);
        const uint32_t ring_full0 = bar(kBarRingFull);
        for_each_piece(P, it, [&](int, int p0, int p1, int) {
          // each CTA's latent query chunks into its own TMEM columns [32c, 32c + 32)
          for (int c = 0; c < 8; ++c) {
            if (!mbar_wait<true>(ring_full0 + 8u * st.idx, st.phase, abortf, P.err, kErrWaitBase + 9))
              return false;
            tc_fence_after();
            const uint64_t qd = ring_desc0 + (uint64_t)(st.idx * (kChunkBytes >> 4));
#pragma unroll
            for (int k = 0; k < 4; ++k) tmem_cp_128x256b_pair(tmem + kTmemQ + 32u * c + 8u * k, qd + 2 * k);
            tc_commit_pair_mc(ring_empty0 + 8u * st.idx, pair_mask);
            st.next(kRing);
          }
          bool first = true;
          for (int pa = p0; pa < p1; pa += 2) {
            const bool last_pair = pa + 2 >= p1;
            if (!mbar_wait<true>(bar(kBarSFree + sb.idx), sb.phase ^ 1u, abortf, P.err, kErrWaitBase + 4))
              return false;
            const uint32_t dS = tmem + kTmemS + 128u * sb.idx;
            // the pair's five stages (four of two chunks, then the RoPE chunk), issued
            // unrolled with precomputed stage indices: the per-stage waits stay (TMA
            // streams stage by stage) but no ring arithmetic or fence sits between MMAs
            tc_fence_after();
            uint32_t sidx[5], sph[5];
#pragma unroll
            for (int s = 0; s < 5; ++s) {
              sidx[s] = st.idx;
              sph[s] = st.phase;
              st.next(kRing);
            }
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              if (!mbar_wait(ring_full0 + 8u * sidx[s], sph[s], abortf, P.err, kErrWaitBase + 6)) return false;
              const uint64_t bd = ring_desc0 + (uint64_t)(sidx[s] * (kChunkBytes >> 4));
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const int c = 2 * s + j;
                const uint32_t a = tmem + kTmemQ + 32u * c;
                const uint64_t bj = bd + (uint64_t)(j * (kPageChunkBytes >> 4));
                mma_ts_pair(dS, a, bj, idesc, c > 0);
                mma_ts_pair(dS, a + 8, bj + 2, idesc, 1);
                mma_ts_pair(dS, a + 16, bj + 4, idesc, 1);
                mma_ts_pair(dS, a + 24, bj + 6, idesc, 1);
              }
              tc_commit_pair_mc(ring_empty0 + 8u * sidx[s], pair_mask);
            }
            if (!mbar_wait(ring_full0 + 8u * sidx[4], sph[4], abortf, P.err, kErrWaitBase + 7)) return false;
            if (first) {
              if (!mbar_wait<true>(bar(kBarQrFull), qr_phase, abortf, P.err, kErrWaitBase + 8)) return false;
              qr_phase ^= 1u;
            }
            {
              const uint64_t bd = ring_desc0 + (uint64_t)(sidx[4] * (kChunkBytes >> 4));
              mma_ss_pair(dS, qr_desc, bd, idesc, 1);
              mma_ss_pair(dS, qr_desc + 2, bd + 2, idesc, 1);
              mma_ss_pair(dS, qr_desc + 4, bd + 4, idesc, 1);
              mma_ss_pair(dS, qr_desc + 6, bd + 6, idesc, 1);
              tc_commit_pair_mc(ring_empty0 + 8u * sidx[4], pair_mask);
            }
            tc_commit_pair_mc(bar(kBarSFull + sb.idx), pair_mask);
            if (last_pair) tc_commit_pair_mc(bar(kBarQrEmpty), pair_mask);
            sb.next(2);
            first = false;
          }
          return true;
        });
        tc_commit_pair(bar(kBarDrain));
        mbar_wait_drain(bar(kBarDrain), 0);
      }
    } else if (kPair && warp == 3 && lane == 0 && !leader) {
      // ---- pair, odd S-CTA: forward "this CTA's S tile was read" to the leader
      Ring sb;
      const uint32_t lead_sfree = map_to_rank(bar(kBarSFree), lead_rank);
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        for (int pa = p0; pa < p1; pa += 2) {
          if (!mbar_wait(bar(kBarSFreeFwd + sb.idx), sb.phase, abortf, P.err, kErrWaitBase + 26)) return false;
          mbar_arrive_remote(lead_sfree + 8u * sb.idx);
          sb.next(2);
        }
        return true;
      });
    } else if (warp >= 4) {
      // ---- two softmax warpgroups: thread (wg, r) owns query row r; of each page
      // pair, warpgroup 0 handles the first page and warpgroup 1 the second
      const int wg = (tid - 128) >> 7;
      const int r = (tid - 128) & 127;
      const uint32_t bar_wg = 1u + (uint32_t)wg;  // named barrier of this warpgroup (128)
      const uint32_t bar_all = 3u;                // named barrier of both groups (256)
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const int rr = rg * kRows + r;
      const bool valid = rr < P.R;
      const int qi = valid ? rr / P.hpk : 0;
      const int head = valid ? g * P.hpk + rr % P.hpk : 0;
      const float c = P.scale_log2;
      float* xmax = reinterpret_cast<float*>(smem + OFF_XCH);  // [2 pair parities][2 groups][128]
      float* xl = xmax + 4 * kRows;                            // [2][128] exact row sums
      Ring sb;
      uint32_t kp = 0;    // running page index of this cluster (P slot = kp % 4)
      uint32_t npair = 0; // running pair index (exchange-buffer parity)
      bool ok = true;
      const uint32_t p_remote = map_to_rank(sbase + OFF_P, peer);
      const uint32_t side_remote = map_to_rank(smem_u32(side), peer);
      const uint32_t pfull_remote = map_to_rank(bar(kBarPFull), peer);
      const uint32_t prow_off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
      // Every bounded wait is followed by an AND over all 256 threads, so both
      // groups always leave together (named barriers have no timeout).
      for_each_piece(P, it, [&](int b, int p0, int p1, int ordinal) {
        const int L = max(P.seqlens[b], 0);
        const int limit = valid ? (P.causal ? L - P.s_q + qi : L - 1) : -1;
        // this group's share of the exact row sum l (for lse; the O-CTA sums the
        // bf16-rounded weights that normalise O itself)
        float m_ref = -INFINITY, l = 0.f;
        for (int pa = p0; pa < p1; pa += 2, ++npair) {
          const int npg = (pa + 1 < p1) ? 2 : 1;
          const bool last_pair = pa + 2 >= p1;
          const bool mine = wg < npg;  // uniform per group
          ok = named_bar_and(bar_all, 256, mbar_wait<kPair>(bar(kBarSFull + sb.idx), sb.phase, abortf, P.err,
                                                            kErrWaitBase + 10));
          if (!ok) return false;
          tc_fence_after();
          const int jw = (pa + wg) * kPage;  // first token of this group's page
          uint32_t s0[32], s1[32];
          if (mine) {
            tmem_ld64_sync(tmem + lane_off + kTmemS + 128u * sb.idx + 64u * (uint32_t)wg, s0, s1);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) { s0[j] = 0xff800000u; s1[j] = 0xff800000u; }  // -inf
          }
          tc_fence_before();
          const uint32_t s_used = sb.idx;
          if constexpr (!kPair) mbar_arrive(bar(kBarSFree + s_used));
          sb.next(2);
          const bool tail = mine && (jw + kPage - 1 > limit);
          if (tail) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (jw + j > limit) s0[j] = 0xff800000u;
              if (jw + 32 + j > limit) s1[j] = 0xff800000u;
            }
          }
          float mloc;
          {
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = fmaxf(__uint_as_float(s0[u]), __uint_as_float(s1[u]));
#pragma unroll
            for (int j = 8; j < 32; ++j)
              m8[j & 7] = fmaxf(m8[j & 7], fmaxf(__uint_as_float(s0[j]), __uint_as_float(s1[j])));
            mloc = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                         fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          }
          // exchange the row max with the other group (buffer alternates by pair)
          float* xm = xmax + (npair & 1u) * (2 * kRows);
          xm[wg * kRows + r] = mloc;
          named_bar_sync(bar_all, 256);
          if constexpr (kPair) {
            // all 256 threads have read this CTA's S tile: one arrival per CTA on
            // the leader's barrier releases it for the next pair's MMAs
            if (tid == 128) {
              // the odd CTA's arrival is relayed by warp 3: an arrival on another
              // CTA's barrier takes ~1 us from a thread with stores in flight
              if (leader)
                mbar_arrive(bar(kBarSFree + s_used));
              else
                mbar_arrive(bar(kBarSFreeFwd + s_used));
            }
          }
          const float mx = fmaxf(mloc, xm[(wg ^ 1) * kRows + r]);
          // identical lazy-rescale update in both groups
          const float mxs = (mx == -INFINITY) ? -INFINITY : mx * c;
          float alpha = 1.f;
          bool resc = false;
          if (mxs > m_ref + kTau) {
            if (m_ref != -INFINITY) {
              alpha = ex2(m_ref - mxs);
              resc = true;
              l *= alpha;
            }
            m_ref = mxs;
          }
          const float base = (m_ref == -INFINITY) ? 0.f : m_ref;
          const uint32_t wany = __any_sync(0xffffffffu, resc) ? 1u : 0u;
          const uint32_t kk = kp + (uint32_t)wg;
          const uint32_t slot = kk % kPSlots, buf = kk % kStageBufs;
          // the destination slot must be consumed and the staging buffer copied out
          bool got = true;
          if (mine)
            got = mbar_wait<true>(bar(kBarPFree + slot), ((kk / kPSlots) & 1u) ^ 1u, abortf, P.err,
                                  kErrWaitBase + 11) &&
                  mbar_wait<true>(bar(kBarStageFree + buf), ((kk / kStageBufs) & 1u) ^ 1u, abortf,
                                  P.err, kErrWaitBase + 21);
          ok = named_bar_and(bar_all, 256, got);
          if (!ok) return false;
          uint32_t pk[32];
          if (mine) {
            // P = exp2(S*c - base) -> bf16; masked entries are -inf and weigh exactly 0
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float e0 = ex2(fmaf(__uint_as_float(s0[2 * j]), c, -base));
              float e1 = ex2(fmaf(__uint_as_float(s0[2 * j + 1]), c, -base));
              float e2 = ex2(fmaf(__uint_as_float(s1[2 * j]), c, -base));
              float e3 = ex2(fmaf(__uint_as_float(s1[2 * j + 1]), c, -base));
              if (tail) {  // also exact when c == 0
                e0 = s0[2 * j] == 0xff800000u ? 0.f : e0;
                e1 = s0[2 * j + 1] == 0xff800000u ? 0.f : e1;
                e2 = s1[2 * j] == 0xff800000u ? 0.f : e2;
                e3 = s1[2 * j + 1] == 0xff800000u ? 0.f : e3;
              }
              pk[j] = pack_bf16x2(e0, e1);
              pk[16 + j] = pack_bf16x2(e2, e3);
              ls[j & 3] += (e0 + e1) + (e2 + e3);
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          }
          if (mine) {
            // P row and the row's factors into the local staging buffers, then
            // one bulk copy each into the O-CTA's slot
            uint8_t* srow = smem + OFF_STAGE + buf * kPBytes + prow_off;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(srow + ((q ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            SideSlot* ss = reinterpret_cast<SideSlot*>(smem + OFF_STAGE_SIDE + buf * kSideBytes);
            ss->alpha[r] = wg == 0 ? alpha : 1.f;
            if (lane == 0) ss->wflag[warp & 3] = wg == 0 ? wany : 0u;
            fence_proxy_async_cta();  // staged data is read by the bulk copies (async proxy)
            named_bar_sync(bar_wg, 128);
            if (r == 0) {
              const uint32_t rbar = pfull_remote + slot * 8u;
              bulk_copy_to_peer(p_remote + slot * kPBytes, sbase + OFF_STAGE + buf * kPBytes, kPBytes, rbar);
              bulk_copy_to_peer(side_remote + slot * kSideBytes, sbase + OFF_STAGE_SIDE + buf * kSideBytes,
                                kSideBytes, rbar);
            }
          }
          kp += (uint32_t)npg;
          if (last_pair) {  // the piece's row sum: both groups' shares
            xl[wg * kRows + r] = l;
            named_bar_sync(bar_all, 256);
          }
          if (last_pair && wg == 0) {
            const int pslot = piece_slot(P, b, ordinal);
            if (valid) {
              const float ltot = l + xl[kRows + r];
              const float lse_v = ltot > 0.f ? (m_ref + __log2f(ltot)) * kLn2 : -INFINITY;
              if (pslot < 0)
                P.lse[((size_t)b * P.h_q + head) * P.s_q + qi] = lse_v;
              else
                P.part_lse[((size_t)pslot * P.h_kv + g) * P.R + rr] = lse_v;
            }
            if (pslot >= 0) {  // split piece: signal the merge kernel (lse half)
              __threadfence();
              named_bar_sync(bar_wg, 128);
              if (r == 0 && rg < P.n_rg) atomicAdd(&P.seq_done[((size_t)b * P.h_kv + g) * P.n_rg + rg], 1);
            }
          }
        }
        return true;
      });
    }
  } else {
    // =========================================================== O-CTA
    if (warp == 0 && lane == 0) {
      if constexpr (!kPair) {
      // ---- TMA producer: value part of each page as two half-page stages
      Ring st;
      bool ok = true;
      uint32_t issued_phase[kVStages];
      bool issued[kVStages] = {false, false, false, false};
      const uint64_t pol = policy_evict_first();
      for_each_piece(P, it, [&](int b, int p0, int p1, int) {
        for (int p = p0; p < p1 && ok; ++p) {
          const int page = load_page(P, b, p);
          for (int hh = 0; hh < 2 && ok; ++hh) {
            ok = mbar_wait(bar(kBarVEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 12);
            if (!ok) break;
            const uint32_t fb = bar(kBarVFull + st.idx);
            mbar_arrive_expect_tx(fb, kVStageBytes);
            const uint32_t dst = sbase + OFF_V + st.idx * kVStageBytes;
            // one box: 4 column chunks x 64 tokens, chunk-major in shared memory
            tma_load_4d(dst, &tmap_v, fb, 0, page * kPage, 4 * hh, g, pol);
            issued[st.idx] = true;
            issued_phase[st.idx] = st.phase;
            st.next(kVStages);
          }
        }
        return ok;
      });
      if (!ok) {
        for (int s = 0; s < kVStages; ++s)
          if (issued[s]) mbar_wait_drain(bar(kBarVFull + s), issued_phase[s]);
      }
      } else {
        // ---- pair: this CTA's half of each page's value columns, chunks
        // {2h, 2h+1} for the first N = 256 MMA and {4+2h, 5+2h} for the second
        // (h = this CTA's half), one 32 KB stage per page, completing on the
        // leader's barrier (armed there for both CTAs)
        Ring st;
        bool ok = true;
        const uint64_t pol = policy_evict_first();
        const uint32_t lead_vfull0 = map_to_rank(bar(kBarVFull), lead_rank);
        for_each_piece(P, it, [&](int b, int p0, int p1, int) {
          for (int p = p0; p < p1; ++p) {
            const int page = load_page(P, b, p);
            ok = mbar_wait<true>(bar(kBarVEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 12);
            if (!ok) return false;
            if (leader) mbar_arrive_expect_tx(bar(kBarVFull + st.idx), 2 * kVStageBytes);
            const uint32_t dst = sbase + OFF_V + st.idx * kVStageBytes;
            const uint32_t fb = lead_vfull0 + 8u * st.idx;
            tma_load_4d_pair(dst, &tmap_kv2, fb, 0, page * kPage, 2 * (int)half, g, pol);
            tma_load_4d_pair(dst + 2 * kPageChunkBytes, &tmap_kv2, fb, 0, page * kPage, 4 + 2 * (int)half, g, pol);
            st.next(kVStages);
          }
          return true;
        });
        if (!ok) settle_inflight_copies();
      }
    } else if (warp == 1 && lane == 0) {
      if constexpr (!kPair) {
      // ---- MMA issuer: O += P V, plus the command stream to the correction warps
      Ring st;
      uint32_t kp = 0, done_phase = 0, drain_phase = 0;
      bool pending_epilogue = false, ok = true;
      const uint32_t idesc = make_idesc_bf16(128, 256, 0, 1);
      const uint64_t v_desc0 = make_smem_desc(sbase + OFF_V, 8192, 1024, 2);
      const uint64_t p_desc0 = make_smem_desc(sbase + OFF_P, 16, 1024, 2);
      for_each_piece(P, it, [&](int b, int p0, int p1, int ordinal) {
        for (int p = p0; p < p1; ++p, ++kp) {
          const uint32_t ps = kp % kPSlots, pph = (kp / kPSlots) & 1u;
          if (!mbar_wait<true>(bar(kBarPFull + ps), pph, abortf, P.err, kErrWaitBase + 13)) return false;
          const volatile uint32_t* wf = side[ps].wflag;
          const bool resc = (wf[0] | wf[1] | wf[2] | wf[3]) != 0u;
          const bool first = (p == p0), last = (p == p1 - 1);
          if (first && pending_epilogue) {  // accumulator still being drained by the epilogue
            ok = mbar_wait(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 14);
            done_phase ^= 1u;
            pending_epilogue = false;
            if (!ok) return false;
          }
          if (resc && !first) {
            // a row's reference max moved: finish all issued MMAs, rescale O rows
            tc_commit(bar(kBarDrain));
            ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 15);
            drain_phase ^= 1u;
            if (!ok) return false;
            mail->cmd = kCmdRescale;
            mail->slot = (int)ps;
            tc_fence_before();
            mbar_arrive(bar(kBarCmdFull));
            ok = mbar_wait(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 16);
            done_phase ^= 1u;
            if (!ok) return false;
          }
          const uint64_t pd = p_desc0 + (uint64_t)(ps * (kPBytes >> 4));
          uint32_t vidx[2];
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            vidx[n] = st.idx;
            if (!mbar_wait(bar(kBarVFull + st.idx), st.phase, abortf, P.err, kErrWaitBase + 17))
              return false;
            st.next(kVStages);
          }
          tc_fence_after();
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            const uint64_t vd = v_desc0 + (uint64_t)(vidx[n] * (kVStageBytes >> 4));
            const uint32_t d = tmem + kTmemO + 256u * n;
            mma_ss(d, pd, vd, idesc, !first);
            mma_ss(d, pd + 2, vd + 128, idesc, 1);
            mma_ss(d, pd + 4, vd + 256, idesc, 1);
            mma_ss(d, pd + 6, vd + 384, idesc, 1);
            tc_commit(bar(kBarVEmpty + vidx[n]));
          }
          tc_commit(bar(kBarPCons + ps));  // P slot consumed -> relay warp
          if (last) {
            // last page of the piece: wait for the accumulator, hand it to the epilogue
            tc_commit(bar(kBarDrain));
            ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 18);
            drain_phase ^= 1u;
            if (!ok) return false;
            mail->cmd = kCmdEpilogue;
            mail->b = b;
            mail->part_slot = piece_slot(P, b, ordinal);
            tc_fence_before();
            mbar_arrive(bar(kBarCmdFull));
            pending_epilogue = true;
          }
        }
        return true;
      });
      if (pending_epilogue) mbar_wait(bar(kBarCmdDone), done_phase, abortf, nullptr, 0);
      tc_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), drain_phase);
      } else if (leader) {
        // ---- pair MMA issuer (rank 2): O += P V for both row groups, M = 256
        // (P rows of rank 2 then rank 3), N = 256 twice (value columns split
        // between the two CTAs), plus the command stream to both CTAs'
        // correction warps
        Ring st;
        uint32_t kp = 0, done_phase = 0, drain_phase = 0;
        bool pending_epilogue = false, ok = true;
        const uint32_t idesc = make_idesc_bf16(256, 256, 0, 1);
        const uint64_t v_desc0 = make_smem_desc(sbase + OFF_V, 8192, 1024, 2);
        const uint64_t p_desc0 = make_smem_desc(sbase + OFF_P, 16, 1024, 2);
        const uint32_t mate_side = map_to_rank(smem_u32(side), mate);
        const uint32_t mate_mail = map_to_rank(smem_u32(mail), mate);
        const uint32_t mate_cmdfull = map_to_rank(bar(kBarCmdFull), mate);
        auto post = [&](int cmd, int slot, int b, int pslot) {
          mail->cmd = cmd;
          mail->slot = slot;
          mail->b = b;
          mail->part_slot = pslot;
          st_cluster_u32(mate_mail + (uint32_t)offsetof(Mailbox, cmd), (uint32_t)cmd);
          st_cluster_u32(mate_mail + (uint32_t)offsetof(Mailbox, slot), (uint32_t)slot);
          st_cluster_u32(mate_mail + (uint32_t)offsetof(Mailbox, b), (uint32_t)b);
          st_cluster_u32(mate_mail + (uint32_t)offsetof(Mailbox, part_slot), (uint32_t)pslot);
          tc_fence_before();
          mbar_arrive(bar(kBarCmdFull));
          mbar_arrive_remote(mate_cmdfull);
        };
        for_each_piece(P, it, [&](int b, int p0, int p1, int ordinal) {
          for (int p = p0; p < p1; ++p, ++kp) {
            const uint32_t ps = kp % kPSlots, pph = (kp / kPSlots) & 1u;
            if (!mbar_wait<true>(bar(kBarPFull + ps), pph, abortf, P.err, kErrWaitBase + 13)) return false;
            if (!mbar_wait<true>(bar(kBarPeerP + ps), pph, abortf, P.err, kErrWaitBase + 24)) return false;
            const volatile uint32_t* wf = side[ps].wflag;
            const uint32_t ms = mate_side + ps * kSideBytes;  // wflag[0..3] lead the side slot
            const bool resc = ((wf[0] | wf[1] | wf[2] | wf[3]) | (ld_cluster_u32(ms) | ld_cluster_u32(ms + 4) |
                                                                 ld_cluster_u32(ms + 8) | ld_cluster_u32(ms + 12))) != 0u;
            const bool first = (p == p0), last = (p == p1 - 1);
            if (first && pending_epilogue) {  // accumulators still being drained by the epilogue
              ok = mbar_wait<true>(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 14);
              done_phase ^= 1u;
              pending_epilogue = false;
              if (!ok) return false;
            }
            if (resc && !first) {
              // a row's reference max moved in either row group: finish all issued
              // MMAs, then both CTAs rescale their O rows
              tc_commit_pair(bar(kBarDrain));
              ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 15);
              drain_phase ^= 1u;
              if (!ok) return false;
              post(kCmdRescale, (int)ps, 0, 0);
              ok = mbar_wait<true>(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 16);
              done_phase ^= 1u;
              if (!ok) return false;
            }
            if (!mbar_wait(bar(kBarVFull + st.idx), st.phase, abortf, P.err, kErrWaitBase + 17))
              return false;
            tc_fence_after();
            const uint64_t pd = p_desc0 + (uint64_t)(ps * (kPBytes >> 4));
            const uint64_t vd = v_desc0 + (uint64_t)(st.idx * (kVStageBytes >> 4));
#pragma unroll
            for (int n = 0; n < 2; ++n) {
              const uint64_t vn = vd + (uint64_t)(n * (2 * kPageChunkBytes >> 4));
              const uint32_t d = tmem + kTmemO + 256u * n;
              mma_ss_pair(d, pd, vn, idesc, !first);
              mma_ss_pair(d, pd + 2, vn + 128, idesc, 1);
              mma_ss_pair(d, pd + 4, vn + 256, idesc, 1);
              mma_ss_pair(d, pd + 6, vn + 384, idesc, 1);
            }
            tc_commit_pair_mc(bar(kBarVEmpty + st.idx), pair_mask);
            st.next(kVStages);
            tc_commit_pair_mc(bar(kBarPCons + ps), pair_mask);  // P slots consumed -> relay warps
            if (last) {
              tc_commit_pair(bar(kBarDrain));
              ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 18);
              drain_phase ^= 1u;
              if (!ok) return false;
              post(kCmdEpilogue, 0, b, piece_slot(P, b, ordinal));
              pending_epilogue = true;
            }
          }
          return true;
        });
        if (pending_epilogue) mbar_wait<true>(bar(kBarCmdDone), done_phase, abortf, nullptr, 0);
        tc_commit_pair(bar(kBarDrain));
        mbar_wait_drain(bar(kBarDrain), drain_phase);
      }
    } else if (warp == 2 && lane == 0) {
      // ---- relay: re-arm a consumed P slot and hand it back to the S-CTA
      uint32_t kp = 0;
      const uint32_t pfree_remote = map_to_rank(bar(kBarPFree), peer);
      const uint32_t mate_pcons = kPair ? map_to_rank(bar(kBarPCons), mate) : 0u;
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        for (int p = p0; p < p1; ++p, ++kp) {
          const uint32_t ps = kp % kPSlots, pph = (kp / kPSlots) & 1u;
          if constexpr (kPair) {
            // this CTA's correction warps have read the mate's flags of this
            // page: the mate may refill its slot once its own consumers are done
            if (!mbar_wait(bar(kBarFlagsRead + ps), pph, abortf, P.err, kErrWaitBase + 27)) return false;
            mbar_arrive_remote_relaxed(mate_pcons + ps * 8u);
          }
          if (!mbar_wait<kPair>(bar(kBarPCons + ps), pph, abortf, P.err, kErrWaitBase + 19)) return false;
          mbar_arrive_expect_tx(bar(kBarPFull + ps), kPFullTx);
          mbar_arrive_remote_relaxed(pfree_remote + ps * 8u);
        }
        return true;
      });
    } else if (warp == 3 && lane == 0) {
      // ---- land relay: once a P message has landed, its staging buffer in the
      // S-CTA may be reused
      uint32_t kp = 0;
      const uint32_t sfree_remote = map_to_rank(bar(kBarStageFree), peer);
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        for (int p = p0; p < p1; ++p, ++kp) {
          if (!mbar_wait<true>(bar(kBarPFull + kp % kPSlots), (kp / kPSlots) & 1u, abortf, P.err,
                               kErrWaitBase + 22))
            return false;
          mbar_arrive_remote_relaxed(sfree_remote + (kp % kStageBufs) * 8u);
          if constexpr (kPair) mbar_arrive_remote_relaxed(map_to_rank(bar(kBarPeerP + kp % kPSlots), mate));
        }
        return true;
      });
    } else if (warp >= 4) {
      // ---- two correction / epilogue warpgroups: thread (wg, r) owns TMEM lane
      // r (= row r) and accumulator columns [256 wg, 256 wg + 256)
      const int wg = (tid - 128) >> 7;
      const int r = (tid - 128) & 127;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t tcol = tmem + lane_off + kTmemO + 256u * (uint32_t)wg;
      const int rr = rg * kRows + r;
      const bool valid = rr < P.R;
      const int qi = valid ? rr / P.hpk : 0;
      const int head = valid ? g * P.hpk + rr % P.hpk : 0;
      uint32_t cmd_phase = 0, kp = 0, npiece = 0;
      // P row r of each page, the 32 tokens of this group: 4 swizzled 16-byte chunks
      const uint32_t prow_off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
      // Both groups meet at named barrier 4 (256 threads), so every bounded wait
      // is followed by an AND over all of them: all leave together or none.
      auto agree = [&](bool ok) { return named_bar_and(4, 256, ok); };
      // one command from the MMA thread
      auto wait_cmd = [&]() {
        if (!agree(mbar_wait<kPair>(bar(kBarCmdFull), cmd_phase, abortf, P.err, kErrWaitBase + 20)))
          return false;
        cmd_phase ^= 1u;
        tc_fence_after();
        return true;
      };
      // a command is done: every thread arrives (single CTA), or, in the pair
      // variant, one arrival per CTA on the leader's barrier once all 256 are done
      auto cmd_done = [&]() {
        tc_fence_before();
        if constexpr (kPair) {
          named_bar_sync(4, 256);
          if (tid == 128) {
            if (leader)
              mbar_arrive(bar(kBarCmdDone));
            else
              mbar_arrive_remote(map_to_rank(bar(kBarCmdDone), lead_rank));
          }
        } else {
          mbar_arrive(bar(kBarCmdDone));
        }
      };
      const uint32_t mate_side = kPair ? map_to_rank(smem_u32(side), mate) : 0u;
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        // lr: this group's half of the row's sum of the bf16 weights the MMA
        // multiplies, rescaled with O
        float lr = 0.f;
        for (int p = p0; p < p1; ++p, ++kp) {
          const uint32_t ps = kp % kPSlots, pph = (kp / kPSlots) & 1u;
          if (!agree(mbar_wait<true>(bar(kBarPFull + ps), pph, abortf, P.err, kErrWaitBase + 23)))
            return false;
          const volatile uint32_t* wf = side[ps].wflag;
          uint32_t any = wf[0] | wf[1] | wf[2] | wf[3];
          if constexpr (kPair) {
            // the MMA thread rescales when either row group moved a reference max:
            // read the mate's flags once its P slot has landed
            if (!agree(mbar_wait<true>(bar(kBarPeerP + ps), pph, abortf, P.err, kErrWaitBase + 25)))
              return false;
            const uint32_t ms = mate_side + ps * kSideBytes;
            any |= ld_cluster_u32(ms) | ld_cluster_u32(ms + 4) | ld_cluster_u32(ms + 8) | ld_cluster_u32(ms + 12);
          }
          const bool resc = p != p0 && any != 0u;
          const float a = side[ps].alpha[r];
          const uint8_t* prow = smem + OFF_P + ps * kPBytes + prow_off;
          float s4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 x = *reinterpret_cast<const uint4*>(prow + (((4 * wg + q) ^ (r & 7)) << 4));
            s4[q] = ((__uint_as_float(x.x << 16) + __uint_as_float(x.x & 0xffff0000u)) +
                     (__uint_as_float(x.y << 16) + __uint_as_float(x.y & 0xffff0000u))) +
                    ((__uint_as_float(x.z << 16) + __uint_as_float(x.z & 0xffff0000u)) +
                     (__uint_as_float(x.w << 16) + __uint_as_float(x.w & 0xffff0000u)));
          }
          lr = fmaf(lr, a, (s4[0] + s4[1]) + (s4[2] + s4[3]));
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(kBarPCons + ps));  // this warp is done with the slot
            // pair: and with the mate's flags (relay warp 2 tells the mate)
            if constexpr (kPair) mbar_arrive(bar(kBarFlagsRead + ps));
          }
          if (resc) {
            // the MMA thread drains and posts a rescale before this page's MMAs
            if (!wait_cmd()) return false;
            if (__any_sync(0xffffffffu, a != 1.f)) {  // tcgen05.ld/st are warp-collective
#pragma unroll 1
              for (int j = 0; j < 8; ++j) {
                uint32_t v[32];
                tmem_ld32_sync(tcol + 32 * j, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = __float_as_uint(__uint_as_float(v[u]) * a);
                tmem_st32(tcol + 32 * j, v);
              }
              tmem_wait_st();
            }
            cmd_done();
          }
        }
        {
          const bool okc = mbar_wait<kPair>(bar(kBarCmdFull), cmd_phase, abortf, P.err, kErrWaitBase + 20);
          float* xr = mail->lr_x[npiece & 1u][0];
          xr[wg * kRows + r] = lr;  // exchanged with the other group at the barrier
          if (!agree(okc)) return false;  // the piece's epilogue command
          cmd_phase ^= 1u;
          tc_fence_after();
          const float lrt = lr + xr[(wg ^ 1) * kRows + r];
          ++npiece;
          // epilogue: tcgen05.ld is warp-collective, so every thread loads and
          // only valid rows store
          const float linv = lrt > 0.f ? 1.f / lrt : 0.f;
          const int b = mail->b;
          const int pslot = mail->part_slot;
          // 64 accumulator columns per TMEM round trip
          if (pslot < 0) {
            uint16_t* dst = P.o + ((size_t)(b * P.s_q + qi) * P.h_q + head) * kDV + 256 * wg;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
              uint32_t v0[32], v1[32];
              tmem_ld64_sync(tcol + 64 * j, v0, v1);
              uint32_t pk[32];
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                pk[u] = pack_bf16x2(__uint_as_float(v0[2 * u]) * linv, __uint_as_float(v0[2 * u + 1]) * linv);
                pk[16 + u] =
                    pack_bf16x2(__uint_as_float(v1[2 * u]) * linv, __uint_as_float(v1[2 * u + 1]) * linv);
              }
              if (valid) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  st_global_v8(dst + 64 * j + 16 * u, pk[8 * u], pk[8 * u + 1], pk[8 * u + 2], pk[8 * u + 3],
                               pk[8 * u + 4], pk[8 * u + 5], pk[8 * u + 6], pk[8 * u + 7]);
              }
            }
          } else {
            // partials are chunk-major, [slot][h_kv][64 chunks of 8 columns][R][8], so
            // the 32 rows of a warp store 1 KB contiguous per chunk
            float* dst = P.part_o + (((size_t)pslot * P.h_kv + g) * (kDV / 8) + 32 * wg) * P.R * 8 +
                         (size_t)rr * 8;
            const size_t cstride = (size_t)P.R * 8;  // floats between consecutive chunks
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
              uint32_t v[2][32];
              tmem_ld64_sync(tcol + 64 * j, v[0], v[1]);
              if (valid) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                  for (int u = 0; u < 4; ++u)
                    st_global_v8(dst + (8 * j + 4 * h + u) * cstride,
                                 __float_as_uint(__uint_as_float(v[h][8 * u]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 1]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 2]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 3]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 4]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 5]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 6]) * linv),
                                 __float_as_uint(__uint_as_float(v[h][8 * u + 7]) * linv));
              }
            }
            // signal the merge kernel (partial o half) once all 256 threads stored
            __threadfence();
            named_bar_sync(4, 256);
            if (tid == 128 && rg < P.n_rg) atomicAdd(&P.seq_done[((size_t)b * P.h_kv + g) * P.n_rg + rg], 1);
          }
          cmd_done();
          return true;
        }
      });
    }
  }

  // ---- teardown: no peer access may be in flight when either CTA exits
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
  // a second decode launch completes only after the first (one CTA waits for
  // it), so that the merge grid's completion, which waits for this grid's, also
  // implies the first's: work queued after the call sees every output row
  if (P.follows_decode && blockIdx.x == 0 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

size_t decode_smem_bytes() { return SMEM_BYTES; }

cudaError_t decode_prepare(int device) {
  static bool done[64] = {};
  if (device >= 0 && device < 64 && done[device]) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess && device >= 0 && device < 64) done[device] = true;
  return e;
}

int decode_max_active_clusters(int device, bool pair, int* out) {
  cudaError_t e = decode_prepare(device);
  if (e != cudaSuccess) return (int)e;
  const int ctas = pair ? 4 : 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas * 512, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ctas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = pair ? cudaOccupancyMaxActiveClusters(&n, decode_kernel<true>, &cfg)
           : cudaOccupancyMaxActiveClusters(&n, decode_kernel<false>, &cfg);
  if (e != cudaSuccess) return (int)e;
  *out = n;
  return 0;
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_kv, const CUtensorMap& tmap_q,
                          const CUtensorMap& tmap_v, const CUtensorMap& tmap_kv2, bool pair, int parts,
                          cudaStream_t stream) {
  const int ctas = pair ? 4 : 2;
  const int units = pair ? (p.n_rg + 1) / 2 : p.n_rg;
  const int clusters = parts * p.h_kv * units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = ctas;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return pair ? cudaLaunchKernelEx(&cfg, decode_kernel<true>, tmap_kv, tmap_q, tmap_v, tmap_kv2, p)
              : cudaLaunchKernelEx(&cfg, decode_kernel<false>, tmap_kv, tmap_q, tmap_v, tmap_kv2, p);
}

}  // namespace pmla
