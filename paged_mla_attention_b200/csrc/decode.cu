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
// One 128-row tile needs Q (128x576 bf16 = 288 TMEM columns as an MMA A
// operand), S = QK^T (128x64 fp32, 64 columns, double-buffered) and the output
// accumulator O (128x512 fp32 = all 512 TMEM columns).  That does not fit one
// SM's TMEM, so each work unit runs on a 2-CTA cluster with split roles:
//
//   CTA 0 ("S-CTA"): Q lives in TMEM; a TMA warp streams whole 64-token pages
//     (9 chunks of 64 columns, 128B-swizzled) into a 3-stage ring; one thread
//     issues S = Q K^T as 36 tcgen05 MMAs (M=128, N=64, K=16, A from TMEM)
//     into a double-buffered TMEM tile; four softmax warps (one row per
//     thread) read S, keep the running max/sum in fp32 with a lazy rescale
//     (the reference max only moves when the page max exceeds it by 2^8), and
//     write P = exp2(S*c - m) as bf16 straight into CTA 1's shared memory
//     (distributed shared memory, in the swizzled K-major MMA layout).
//   CTA 1 ("O-CTA"): a TMA warp streams the value part of the same pages
//     (8 chunks); one thread issues O += P V as 8 MMAs (M=128, N=256, K=16,
//     V MN-major) into the 512-column TMEM accumulator; four correction warps
//     rescale O rows when the S-CTA moved a row's reference max, and run the
//     epilogue (O / l -> bf16 o, or fp32 partials) at the end of each piece.
//
// Every wait is bounded (see ptx.cuh); a timeout records an error code and
// makes all roles leave their loops, drain their in-flight copies and MMAs,
// free TMEM and exit.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kPSlots = 2;
constexpr uint32_t kChunkBytes = 64 * 64 * 2;             // 64 tokens x 64 columns bf16
constexpr uint32_t kKStageBytes = 9 * kChunkBytes;         // whole page row (576)
constexpr uint32_t kVStageBytes = 8 * kChunkBytes;         // value part (512)
constexpr uint32_t kPBytes = kRows * kPage * 2;            // 128 x 64 bf16

struct SideSlot {        // per-P-slot row data sent by the S-CTA
  uint32_t flags;        // bit0: some row moved its reference max; bit1: last page of piece
  uint32_t pad[3];
  float alpha[kRows];    // O row rescale factors (1 = unchanged)
  float linv[kRows];     // 1 / row sum, valid on the last page of a piece
};

struct Mailbox {         // MMA thread -> correction warps (O-CTA)
  int cmd;               // 1: rescale rows by side slot `slot`; 2: epilogue
  int slot;
  int b;
  int part_slot;         // partial slot index, or -1 for a direct write
  float linv[kRows];
};

enum : int { kCmdRescale = 1, kCmdEpilogue = 2 };

// mbarrier indices (same offsets in both CTAs; meaning depends on the role)
enum : int {
  kBarFull = 0,       // [3] page stage loaded (TMA tx)
  kBarEmpty = 3,      // [3] page stage consumed (MMA commit)
  kBarSFull = 6,      // S-CTA [2]: S tile ready (commit) | O-CTA [2]: P slot consumed (commit)
  kBarSFree = 8,      // S-CTA [2]: S tile read by softmax warps (128 arrivals)
  kBarQFull = 10,     // S-CTA: Q tile in TMEM (128) | O-CTA: mailbox command posted (1)
  kBarCmdDone = 11,   // O-CTA: command done (128)
  kBarPFree = 12,     // S-CTA [2]: P slot free again (remote arrival from the O-CTA)
  kBarPFull = 14,     // O-CTA [2]: P slot written (remote arrival from the S-CTA)
  kBarDrain = 16,     // both: all issued MMAs complete
  kNumBars = 17
};

struct Ctrl {
  uint64_t bar[kNumBars];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr uint32_t OFF_P = kStages * kVStageBytes;                          // O-CTA P slots
constexpr uint32_t OFF_SIDE = OFF_P + kPSlots * kPBytes;
constexpr uint32_t OFF_MAIL = OFF_SIDE + kPSlots * sizeof(SideSlot);
constexpr uint32_t OFF_CTRL = (OFF_MAIL + sizeof(Mailbox) + 15u) & ~15u;
constexpr uint32_t SMEM_BYTES = OFF_CTRL + sizeof(Ctrl);
static_assert(kStages * kKStageBytes <= OFF_CTRL, "S-CTA ring overlaps the control block");
static_assert(SMEM_BYTES <= 232448, "shared memory budget exceeded");
static_assert(OFF_P % 1024 == 0, "P slots must be 1024-byte aligned for the 128B swizzle");

// TMEM column map
constexpr uint32_t kTmemQ = 0;      // S-CTA: Q, 288 columns (bf16 pairs)
constexpr uint32_t kTmemS = 288;    // S-CTA: two 64-column S tiles
constexpr uint32_t kTmemO = 0;      // O-CTA: 512 columns

struct Ring {
  uint32_t idx = 0, phase = 0;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++idx == n) { idx = 0; phase ^= 1u; }
  }
};

// Iterates the pieces of a scheduler part: calls f(b, p0, p1, ordinal).
struct PartIter {
  int b0, pg0, b1, pg1, ord0;
  __device__ PartIter(const DecodeParams& P, int part) {
    const int32_t* m = P.meta + (size_t)part * kMetaInts;
    b0 = max(m[0], 0);
    pg0 = max(m[1], 0);
    b1 = min(m[2], P.batch);
    pg1 = m[3];
    ord0 = max(m[4], 0);
  }
};

__device__ __forceinline__ int seq_pages(const DecodeParams& P, int b) {
  int L = P.seqlens[b];
  L = L < 0 ? 0 : L;
  int n = (L + kPage - 1) / kPage;
  return n < P.max_pages ? n : P.max_pages;
}

template <class F>
__device__ __forceinline__ void for_each_piece(const DecodeParams& P, const PartIter& it, F&& f) {
  for (int b = it.b0; b <= it.b1 && b < P.batch; ++b) {
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_kv, const DecodeParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (sbase & 1023u) {  // layout assumption broken: report and leave (uniform branch)
    if (tid == 0) atomicCAS(P.err, 0, kErrBadSmemAlign);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const int cluster_id = blockIdx.x >> 1;
  const int groups = P.h_kv * P.n_rg;
  const int part = cluster_id / groups;
  const int g = (cluster_id % groups) / P.n_rg;
  const int rg = (cluster_id % groups) % P.n_rg;

  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + OFF_CTRL);
  SideSlot* side = reinterpret_cast<SideSlot*>(smem + OFF_SIDE);
  Mailbox* mail = reinterpret_cast<Mailbox*>(smem + OFF_MAIL);
  volatile int* abortf = &ctrl->abort_flag;
  auto bar = [&](int i) { return smem_u32(&ctrl->bar[i]); };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSFree + s), 128);
      mbar_init(bar(kBarPFree + s), 1);
      mbar_init(bar(kBarPFull + s), 1);
    }
    mbar_init(bar(kBarQFull), rank == 0 ? 128 : 1);
    mbar_init(bar(kBarCmdDone), 128);
    mbar_init(bar(kBarDrain), 1);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_kv);
  tc_fence_before();
  __syncthreads();
  cluster_arrive();
  cluster_wait();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  const PartIter it(P, part);
  const uint32_t peer = rank ^ 1u;

  if (rank == 0) {
    // =========================================================== S-CTA
    if (warp == 0 && lane == 0) {
      // ---- TMA producer: whole pages (9 chunks)
      Ring st;
      bool ok = true;
      uint32_t issued_phase[kStages];
      bool issued[kStages] = {false, false, false};
      const uint64_t pol = policy_evict_normal();
      for_each_piece(P, it, [&](int b, int p0, int p1, int) {
        for (int p = p0; p < p1 && ok; ++p) {
          ok = mbar_wait(bar(kBarEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 1);
          if (!ok) break;
          int page = P.block_table[(size_t)b * P.max_pages + p];
          if (page < 0 || page >= P.num_pages) {
            atomicCAS(P.err, 0, kErrBadPage);
            page = P.num_pages;  // out of the tensor map: TMA fills zeros
          }
          const uint32_t fb = bar(kBarFull + st.idx);
          mbar_arrive_expect_tx(fb, kKStageBytes);
          const uint32_t dst = sbase + st.idx * kKStageBytes;
#pragma unroll
          for (int c = 0; c < 9; ++c)
            tma_load_3d(dst + c * kChunkBytes, &tmap_kv, fb, c * 64, g, page * kPage, pol);
          issued[st.idx] = true;
          issued_phase[st.idx] = st.phase;
          st.next(kStages);
        }
        return ok;
      });
      if (!ok) {  // drain copies still in flight before the CTA may exit
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) mbar_wait_drain(bar(kBarFull + s), issued_phase[s]);
      }
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer: S = Q K^T
      Ring st, sb;
      uint32_t qphase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc_bf16(128, 64, 0, 0);
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        for (int p = p0; p < p1; ++p) {
          ok = mbar_wait(bar(kBarFull + st.idx), st.phase, abortf, P.err, kErrWaitBase + 2) &&
               mbar_wait(bar(kBarSFree + sb.idx), sb.phase ^ 1u, abortf, P.err, kErrWaitBase + 3);
          if (ok && p == p0) {
            ok = mbar_wait(bar(kBarQFull), qphase, abortf, P.err, kErrWaitBase + 4);
            qphase ^= 1u;
          }
          if (!ok) return false;
          tc_fence_after();
          const uint32_t kst = sbase + st.idx * kKStageBytes;
          const uint32_t dS = tmem + kTmemS + 64u * sb.idx;
#pragma unroll 4
          for (int s = 0; s < 36; ++s) {
            const uint64_t bdesc =
                make_smem_desc(kst + (s >> 2) * kChunkBytes + (s & 3) * 32, 16, 1024, 2);
            mma_ts(dS, tmem + kTmemQ + 8u * s, bdesc, idesc, s > 0);
          }
          tc_commit(bar(kBarEmpty + st.idx));
          tc_commit(bar(kBarSFull + sb.idx));
          st.next(kStages);
          sb.next(2);
        }
        return true;
      });
      tc_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
    } else if (warp >= 4) {
      // ---- softmax warpgroup: thread r owns query row r of the tile
      const int r = tid - 128;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const int rr = rg * kRows + r;
      const bool valid = rr < P.R;
      const int qi = valid ? rr / P.hpk : 0;
      const int head = valid ? g * P.hpk + rr % P.hpk : 0;
      const float c = P.scale_log2;
      const float kTau = 8.0f;
      Ring sb, ps;
      bool ok = true;
      for_each_piece(P, it, [&](int b, int p0, int p1, int ordinal) {
        const int L = max(P.seqlens[b], 0);
        const int limit = valid ? (P.causal ? L - P.s_q + qi : L - 1) : -1;
        // Q row -> TMEM columns [0, 288) as packed bf16 pairs
        {
          const uint4* src = reinterpret_cast<const uint4*>(
              P.q + ((size_t)(b * P.s_q + qi) * P.h_q + head) * kD);
#pragma unroll 1
          for (int j = 0; j < 9; ++j) {
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint4 x = valid ? __ldg(src + 8 * j + u) : make_uint4(0, 0, 0, 0);
              v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
            }
            tmem_st32(tmem + lane_off + kTmemQ + 32 * j, v);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(kBarQFull));
        }
        // l: exact row sum (for lse); lr: sum of the bf16-rounded weights the
        // MMA multiplies (normalises O so the applied weights sum to one)
        float m_ref = -INFINITY, l = 0.f, lr = 0.f;
        for (int p = p0; p < p1; ++p) {
          // every bounded wait is followed by a group-wide AND so that all 128
          // threads leave together (a named barrier has no timeout)
          ok = named_bar_and(1, 128,
                             mbar_wait(bar(kBarSFull + sb.idx), sb.phase, abortf, P.err, kErrWaitBase + 5));
          if (!ok) return false;
          tc_fence_after();
          uint32_t sa[32], sbv[32];
          tmem_ld64_sync(tmem + lane_off + kTmemS + 64u * sb.idx, sa, sbv);
          tc_fence_before();
          mbar_arrive(bar(kBarSFree + sb.idx));
          sb.next(2);
          float s[64];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            s[j] = __uint_as_float(sa[j]);
            s[32 + j] = __uint_as_float(sbv[j]);
          }
          // tokens past the row's last visible index get weight 0; only the
          // tail page(s) of a sequence carry such tokens
          const int j0 = p * kPage;
          const bool tail = j0 + kPage - 1 > limit;
          if (tail) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j0 + j > limit) s[j] = -INFINITY;
          }
          float mx = s[0];
#pragma unroll
          for (int j = 1; j < 64; ++j) mx = fmaxf(mx, s[j]);
          const float mxs = (mx == -INFINITY) ? -INFINITY : mx * c;
          float alpha = 1.f;
          bool resc = false;
          if (mxs > m_ref + kTau) {
            if (m_ref != -INFINITY) {
              alpha = ex2(m_ref - mxs);
              resc = true;
              l *= alpha;
              lr *= alpha;
            }
            m_ref = mxs;
          }
          const float base = (m_ref == -INFINITY) ? 0.f : m_ref;
          uint32_t pk[32];
          float lsum = 0.f, lrsum = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float e0 = ex2(fmaf(s[2 * j], c, -base));
            float e1 = ex2(fmaf(s[2 * j + 1], c, -base));
            if (tail) {
              e0 = (j0 + 2 * j > limit) ? 0.f : e0;
              e1 = (j0 + 2 * j + 1 > limit) ? 0.f : e1;
            }
            pk[j] = pack_bf16x2(e0, e1);
            lsum += e0 + e1;
            lrsum += __uint_as_float(pk[j] << 16) + __uint_as_float(pk[j] & 0xffff0000u);
          }
          l += lsum;
          lr += lrsum;
          const bool last = (p == p1 - 1);
          // wait until the O-CTA's MMAs have finished reading this P slot
          ok = named_bar_and(1, 128, mbar_wait<true>(bar(kBarPFree + ps.idx), ps.phase ^ 1u, abortf,
                                                      P.err, kErrWaitBase + 6));
          if (!ok) return false;
          const uint32_t prow = sbase + OFF_P + ps.idx * kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_cluster_v4(map_to_rank(prow + ((cc ^ (r & 7)) << 4), peer), pk[4 * cc],
                          pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          const uint32_t side_local = smem_u32(&side[ps.idx]);
          st_cluster_f32(map_to_rank(side_local + offsetof(SideSlot, alpha) + 4 * r, peer), alpha);
          if (last)
            st_cluster_f32(map_to_rank(side_local + offsetof(SideSlot, linv) + 4 * r, peer),
                           lr > 0.f ? 1.f / lr : 0.f);
          fence_proxy_async_cluster();
          const bool any = named_bar_or(1, 128, resc);
          if (r == 0) {
            st_cluster_u32(map_to_rank(side_local, peer), (any ? 1u : 0u) | (last ? 2u : 0u));
            mbar_arrive_remote(map_to_rank(bar(kBarPFull + ps.idx), peer));
          }
          ps.next(2);
        }
        if (valid) {
          const float lse_v = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          const int slot = piece_slot(P, b, ordinal);
          if (slot < 0)
            P.lse[((size_t)b * P.h_q + head) * P.s_q + qi] = lse_v;
          else
            P.part_lse[((size_t)slot * P.h_kv + g) * P.R + rr] = lse_v;
        }
        return true;
      });
    }
  } else {
    // =========================================================== O-CTA
    if (warp == 0 && lane == 0) {
      // ---- TMA producer: value part of each page (8 chunks)
      Ring st;
      bool ok = true;
      uint32_t issued_phase[kStages];
      bool issued[kStages] = {false, false, false};
      const uint64_t pol = policy_evict_first();
      for_each_piece(P, it, [&](int b, int p0, int p1, int) {
        for (int p = p0; p < p1 && ok; ++p) {
          ok = mbar_wait(bar(kBarEmpty + st.idx), st.phase ^ 1u, abortf, P.err, kErrWaitBase + 11);
          if (!ok) break;
          int page = P.block_table[(size_t)b * P.max_pages + p];
          if (page < 0 || page >= P.num_pages) page = P.num_pages;
          const uint32_t fb = bar(kBarFull + st.idx);
          mbar_arrive_expect_tx(fb, kVStageBytes);
          const uint32_t dst = sbase + st.idx * kVStageBytes;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            tma_load_3d(dst + cc * kChunkBytes, &tmap_kv, fb, cc * 64, g, page * kPage, pol);
          issued[st.idx] = true;
          issued_phase[st.idx] = st.phase;
          st.next(kStages);
        }
        return ok;
      });
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) mbar_wait_drain(bar(kBarFull + s), issued_phase[s]);
      }
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer: O += P V, plus the command stream to the correction warps
      Ring st, ps;
      uint32_t done_phase = 0, drain_phase = 0;
      bool pending_epilogue = false, ok = true;
      const uint32_t idesc = make_idesc_bf16(128, 256, 0, 1);
      for_each_piece(P, it, [&](int b, int p0, int p1, int ordinal) {
        for (int p = p0; p < p1; ++p) {
          ok = mbar_wait(bar(kBarFull + st.idx), st.phase, abortf, P.err, kErrWaitBase + 12) &&
               mbar_wait<true>(bar(kBarPFull + ps.idx), ps.phase, abortf, P.err,
                               kErrWaitBase + 13);
          if (!ok) return false;
          const uint32_t flags = *reinterpret_cast<volatile uint32_t*>(&side[ps.idx].flags);
          const bool first = (p == p0);
          if (first && pending_epilogue) {  // accumulator still being drained by the epilogue
            ok = mbar_wait(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 14);
            done_phase ^= 1u;
            pending_epilogue = false;
            if (!ok) return false;
          }
          if ((flags & 1u) && !first) {
            // a row's reference max moved: finish all issued MMAs, rescale O rows
            tc_commit(bar(kBarDrain));
            ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 15);
            drain_phase ^= 1u;
            if (!ok) return false;
            mail->cmd = kCmdRescale;
            mail->slot = ps.idx;
            tc_fence_before();
            mbar_arrive(bar(kBarQFull));
            ok = mbar_wait(bar(kBarCmdDone), done_phase, abortf, P.err, kErrWaitBase + 16);
            done_phase ^= 1u;
            if (!ok) return false;
          }
          tc_fence_after();
          const uint32_t vst = sbase + st.idx * kVStageBytes;
          const uint32_t pslot = sbase + OFF_P + ps.idx * kPBytes;
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t adesc = make_smem_desc(pslot + k * 32, 16, 1024, 2);
              const uint64_t bdesc =
                  make_smem_desc(vst + (4 * n) * kChunkBytes + k * 2048, 8192, 1024, 2);
              mma_ss(tmem + kTmemO + 256u * n, adesc, bdesc, idesc, !(first && k == 0));
            }
          tc_commit(bar(kBarEmpty + st.idx));
          tc_commit(bar(kBarSFull + ps.idx));  // P slot consumed -> relay warp
          if (flags & 2u) {
            // last page of the piece: wait for the accumulator, hand it to the epilogue
            tc_commit(bar(kBarDrain));
            ok = mbar_wait(bar(kBarDrain), drain_phase, abortf, P.err, kErrWaitBase + 17);
            drain_phase ^= 1u;
            if (!ok) return false;
            const float4* srcl = reinterpret_cast<const float4*>(side[ps.idx].linv);
            float4* dstl = reinterpret_cast<float4*>(mail->linv);
#pragma unroll 4
            for (int u = 0; u < kRows / 4; ++u) dstl[u] = srcl[u];
            mail->cmd = kCmdEpilogue;
            mail->b = b;
            mail->part_slot = piece_slot(P, b, ordinal);
            tc_fence_before();
            mbar_arrive(bar(kBarQFull));
            pending_epilogue = true;
          }
          st.next(kStages);
          ps.next(2);
        }
        return true;
      });
      if (pending_epilogue)
        mbar_wait(bar(kBarCmdDone), done_phase, abortf, nullptr, 0);
      tc_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), drain_phase);
    } else if (warp == 2 && lane == 0) {
      // ---- relay: tell the S-CTA a P slot may be overwritten once its MMAs completed
      Ring ps;
      for_each_piece(P, it, [&](int, int p0, int p1, int) {
        for (int p = p0; p < p1; ++p) {
          if (!mbar_wait(bar(kBarSFull + ps.idx), ps.phase, abortf, P.err, kErrWaitBase + 18))
            return false;
          mbar_arrive_remote(map_to_rank(bar(kBarPFree + ps.idx), peer));
          ps.next(2);
        }
        return true;
      });
    } else if (warp >= 4) {
      // ---- correction / epilogue warpgroup: thread r owns TMEM lane r (= row r)
      const int r = tid - 128;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const int rr = rg * kRows + r;
      const bool valid = rr < P.R;
      const int qi = valid ? rr / P.hpk : 0;
      const int head = valid ? g * P.hpk + rr % P.hpk : 0;
      uint32_t cmd_phase = 0;
      for_each_piece(P, it, [&](int, int, int, int) {
        for (;;) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait(bar(kBarQFull), cmd_phase, abortf, P.err, kErrWaitBase + 19)))
            return false;
          cmd_phase ^= 1u;
          tc_fence_after();
          const int cmd = *reinterpret_cast<volatile int*>(&mail->cmd);
          if (cmd == kCmdRescale) {
            const float a = side[mail->slot].alpha[r];
            if (__any_sync(0xffffffffu, a != 1.f)) {  // tcgen05.ld/st are warp-collective
#pragma unroll 1
              for (int j = 0; j < 16; ++j) {
                uint32_t v[32];
                tmem_ld32_sync(tmem + lane_off + kTmemO + 32 * j, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = __float_as_uint(__uint_as_float(v[u]) * a);
                tmem_st32(tmem + lane_off + kTmemO + 32 * j, v);
              }
              tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar(kBarCmdDone));
            continue;
          }
          // epilogue
          const float linv = mail->linv[r];
          const int b = mail->b;
          const int pslot = mail->part_slot;
          // tcgen05.ld is warp-collective: every thread loads, valid rows store
          if (pslot < 0) {
            uint4* dst = reinterpret_cast<uint4*>(
                P.o + ((size_t)(b * P.s_q + qi) * P.h_q + head) * kDV);
#pragma unroll 1
            for (int j = 0; j < 16; ++j) {
              uint32_t v[32];
              tmem_ld32_sync(tmem + lane_off + kTmemO + 32 * j, v);
              uint32_t pk[16];
#pragma unroll
              for (int u = 0; u < 16; ++u)
                pk[u] = pack_bf16x2(__uint_as_float(v[2 * u]) * linv,
                                    __uint_as_float(v[2 * u + 1]) * linv);
              if (valid) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  dst[4 * j + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
              }
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(
                P.part_o + (((size_t)pslot * P.h_kv + g) * P.R + rr) * kDV);
#pragma unroll 1
            for (int j = 0; j < 16; ++j) {
              uint32_t v[32];
              tmem_ld32_sync(tmem + lane_off + kTmemO + 32 * j, v);
              if (valid) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  dst[8 * j + u] = make_float4(__uint_as_float(v[4 * u]) * linv,
                                               __uint_as_float(v[4 * u + 1]) * linv,
                                               __uint_as_float(v[4 * u + 2]) * linv,
                                               __uint_as_float(v[4 * u + 3]) * linv);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(bar(kBarCmdDone));
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
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t decode_smem_bytes() { return SMEM_BYTES; }

cudaError_t decode_prepare(int device) {
  static bool done[64] = {};
  if (device >= 0 && device < 64 && done[device]) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess && device >= 0 && device < 64) done[device] = true;
  return e;
}

int decode_max_active_clusters(int device, int* out) {
  cudaError_t e = decode_prepare(device);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 512, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, decode_kernel, &cfg);
  if (e != cudaSuccess) return (int)e;
  *out = n;
  return 0;
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_kv, cudaStream_t stream) {
  const int clusters = p.num_parts * p.h_kv * p.n_rg;
  decode_kernel<<<2 * clusters, kThreads, SMEM_BYTES, stream>>>(tmap_kv, p);
  return cudaGetLastError();
}

}  // namespace pmla
