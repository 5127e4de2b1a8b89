// Length-balanced split-KV scheduler (get_mla_metadata).
//
// The FlashMLA pages name this step only by its interface (usage step 3:
// get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) returns
// tile_scheduler_metadata and num_splits) and describe it as tiling /
// load-balanced scheduling for variable-length sequences.  The algorithm here
// is our own plain reading, computed in parallel by one thread block:
//
//   cost of a piece    = its pages + F               (F = kPieceCostPages)
//   cost coordinate    = sequences laid end to end, each as F + its pages;
//                        position (b, page) sits at X = S_b + F + page, the
//                        start of sequence b at X = S_b
//   total              = S_batch
//   weights            = w_p = kPartWeightFull for parts p < num_main,
//                        kPartWeightAux after (parts run by slower clusters);
//                        C_p = w_0 + ... + w_{p-1}, W = C_P
//   boundary of part p = X_p = floor(C_p (total + (P-1) F) / W) - (p-1) F
//
// Every part is assumed to start inside a sequence and so pay one F of its
// own; the spacing of the X_p gives each part its weight's share of the total
// plus those P-1 overheads (with equal weights, p (total + (P-1) F) / P).  X_p is mapped back to (b, page) and snapped so that no
// piece is shorter than two pages: a start at page 1 moves to the sequence
// start, a start that would leave a one-page tail moves to the next sequence.
// Snapping is monotone, so parts stay ordered (some may be empty).  When the
// whole batch costs less than P (F + 1) the overhead assumption is dropped and
// X_p = floor(C_p total / W).
//
// A part's cost is at most ceil(w_p (total + (P-1) F) / W) + F + 2 in either
// regime; each thread finds its boundary by binary search, so the kernel
// takes a few microseconds for any batch.
#include "pagedmla_internal.cuh"

namespace pmla {

constexpr int kSchedThreads = 1024;
constexpr int kSchedWarps = kSchedThreads / 32;

namespace {

__device__ __forceinline__ int pages_of(const int32_t* seqlens, int b) {
  const int L = seqlens[b] > 0 ? seqlens[b] : 0;
  return (L + kPage - 1) / kPage;
}

// Exclusive block scan of one 64-bit value per thread (kSchedThreads threads).
__device__ long long block_exclusive_scan(long long v, long long* warp_tot, long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    long long t = warp_tot[lane];
    long long ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of the warp totals
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const long long r = warp_tot[warp] + inc - v;
  __syncthreads();  // warp_tot may be reused by the caller's next scan
  return r;
}

}  // namespace

__global__ void __launch_bounds__(kSchedThreads) metadata_kernel(const int32_t* __restrict__ seqlens,
                                                                 int batch, int num_parts, int num_main,
                                                                 int32_t* __restrict__ meta,
                                                                 int32_t* __restrict__ num_splits) {
  __shared__ long long chunk_base[kSchedThreads];  // cost coordinate of each chunk's first sequence
  __shared__ int chunk_ne[kSchedThreads];          // non-empty sequences before each chunk
  __shared__ long long warp_tot[kSchedWarps];
  __shared__ long long sh_total, sh_scratch;
  __shared__ int start_b[kMaxParts + 1], start_pg[kMaxParts + 1];
  __shared__ int cut_rank[kMaxParts + 1];  // cuts among parts <= p (inclusive)
  __shared__ int cut_seq[kMaxParts];       // sequence of each distinct cut, in order
  __shared__ int sh_ncuts;

  // the kernel queued next may start now (the counter clear, then the decode
  // kernel's setup); they wait for this grid before reading what it writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long F = kPieceCostPages;
  const int t = threadIdx.x;
  const int P = num_parts;

  // 1. every thread owns a contiguous chunk of sequences: chunk cost and
  //    non-empty count, then block scans give each chunk's base
  const int per = (batch + kSchedThreads - 1) / kSchedThreads;
  const int c0 = min(t * per, batch), c1 = min(c0 + per, batch);
  long long csum = 0;
  int cne = 0;
  for (int b = c0; b < c1; ++b) {
    const int n = pages_of(seqlens, b);
    if (n > 0) {
      csum += n + F;
      ++cne;
    }
  }
  chunk_base[t] = block_exclusive_scan(csum, warp_tot, &sh_total);
  chunk_ne[t] = (int)block_exclusive_scan(cne, warp_tot, &sh_scratch);
  const long long total = sh_total;  // the scans end with a barrier

  // 2. part boundaries (C_p <= 2^11 x 2^7 and A < 2^42: the products fit 64 bits)
  const long long A = total + (long long)(P - 1) * F;
  const bool overhead_model = A >= (long long)P * (F + 1);
  const int M = min(max(num_main, 0), P);
  const int W = M * kPartWeightFull + (P - M) * kPartWeightAux;
  const long long span = overhead_model ? A : total;
  for (int p = t; p <= P; p += kSchedThreads) {
    int sb = batch, spg = 0;
    if (p == 0) {
      sb = 0;
    } else if (p < P) {
      const int cw = p <= M ? p * kPartWeightFull : M * kPartWeightFull + (p - M) * kPartWeightAux;
      const long long X = (long long)cw * span / W - (overhead_model ? (long long)(p - 1) * F : 0);
      if (X < total) {
        // last chunk whose base is <= X (its cost is > 0 because X < total)
        int lo = 0, hi = kSchedThreads - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (chunk_base[mid] <= X) lo = mid; else hi = mid - 1;
        }
        long long S = chunk_base[lo];
        int b = min(lo * per, batch);
        // the sequence containing X (empty sequences cost nothing and are skipped)
        for (; b < batch; ++b) {
          const int n = pages_of(seqlens, b);
          const long long c = n > 0 ? n + F : 0;
          if (X < S + c) {
            long long pg = X - S - F;
            if (pg < 2) pg = 0;
            if (pg > 0 && n - pg < 2) {
              sb = b + 1;
              spg = 0;
            } else {
              sb = b;
              spg = (int)pg;
            }
            break;
          }
          S += c;
        }
      }
    }
    start_b[p] = sb;
    start_pg[p] = spg;
  }
  __syncthreads();

  // 3. distinct cut points (starts inside a sequence), ranked in order
  if (t == 0) sh_ncuts = 0;
  {
    // parts are few (<= kMaxParts): each thread ranks a contiguous run of them
    const int pp = (P + 1 + kSchedThreads - 1) / kSchedThreads;
    const int q0 = min(t * pp, P + 1), q1 = min(q0 + pp, P + 1);
    int mine = 0;
    for (int p = q0; p < q1; ++p)
      mine += (p > 0 && p < P && start_pg[p] > 0 &&
               (start_b[p] != start_b[p - 1] || start_pg[p] != start_pg[p - 1]));
    const long long before = block_exclusive_scan(mine, warp_tot, &sh_scratch);
    int r = (int)before;
    for (int p = q0; p < q1; ++p) {
      const bool cut = p > 0 && p < P && start_pg[p] > 0 &&
                       (start_b[p] != start_b[p - 1] || start_pg[p] != start_pg[p - 1]);
      if (cut) cut_seq[r++] = start_b[p];
      cut_rank[p] = r;
    }
    if (t == kSchedThreads - 1) sh_ncuts = r;
  }
  __syncthreads();
  const int ncuts = sh_ncuts;
  // number of cuts in sequences < b (lower bound) or <= b (upper bound)
  auto cuts_before = [&](int b, bool inclusive) {
    int lo = 0, hi = ncuts;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (inclusive ? cut_seq[mid] <= b : cut_seq[mid] < b) lo = mid + 1; else hi = mid;
    }
    return lo;
  };

  // 4. metadata rows
  for (int p = t; p < P; p += kSchedThreads) {
    int32_t* m = meta + (size_t)p * kMetaInts;
    const int b0 = start_b[p], pg0 = start_pg[p];
    m[0] = b0;
    m[1] = pg0;
    m[2] = start_b[p + 1];
    m[3] = start_pg[p + 1];
    m[4] = pg0 > 0 ? cut_rank[p] - cuts_before(b0, false) : 0;
    m[5] = p < M ? kPartWeightFull : kPartWeightAux;
    m[6] = 0;
    m[7] = 0;
  }

  // 5. num_splits = exclusive prefix of pieces: one per non-empty sequence plus
  //    one per cut inside it
  if (t == 0) num_splits[0] = 0;
  int ne = chunk_ne[t];
  int nc = c0 < c1 ? cuts_before(c0, false) : 0;
  for (int b = c0; b < c1; ++b) {
    ne += pages_of(seqlens, b) > 0;
    while (nc < ncuts && cut_seq[nc] <= b) ++nc;
    num_splits[b + 1] = ne + nc;
  }
}

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int num_main, int32_t* meta,
                            int32_t* num_splits, cudaStream_t stream) {
  metadata_kernel<<<1, kSchedThreads, 0, stream>>>(seqlens, batch, num_parts, num_main, meta, num_splits);
  return cudaGetLastError();
}

}  // namespace pmla
