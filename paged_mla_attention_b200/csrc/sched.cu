// Length-balanced split-KV scheduler (get_mla_metadata).
//
// The FlashMLA pages name this step only by its interface (usage step 3:
// get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) returns
// tile_scheduler_metadata and num_splits) and describe it as tiling /
// load-balanced scheduling for variable-length sequences.  The algorithm here
// is our own plain reading:
//
//   cost(piece) = pages in the piece + kPieceCostPages
//   target(p)   = ceil((remaining cost + expected split overhead) / parts
//                 left), recomputed as each part starts, so rounding slack is
//                 spread instead of piling up on the last part
//
// Walk the sequences in order and fill part after part up to its target; a
// sequence that does not fit in the rest of a part is cut, and the next part
// continues it (one more piece, one more fixed cost).  Pieces shorter than two
// pages are not cut off a sequence's tail.  The last part takes whatever is
// left.  One thread does the walk: it is O(batch + parts) and runs once per
// decode step, shared by all layers.
#include "pagedmla_internal.cuh"

namespace pmla {

constexpr int kSchedThreads = 256;
constexpr int kSchedSmemLens = 8192;  // lengths staged in shared memory (32 KB)

__global__ void __launch_bounds__(kSchedThreads) metadata_kernel(const int32_t* __restrict__ seqlens,
                                                                 int batch, int num_parts,
                                                                 int32_t* __restrict__ meta,
                                                                 int32_t* __restrict__ num_splits) {
  // All threads stage the page counts in shared memory (coalesced loads) and
  // reduce the total; thread 0 then walks them without global-memory latency.
  __shared__ int32_t pages_s[kSchedSmemLens];
  __shared__ long long partial[kSchedThreads / 32];
  const long long fixed = kPieceCostPages;
  const bool staged = batch <= kSchedSmemLens;
  long long mine = 0;
  for (int b = threadIdx.x; b < batch; b += kSchedThreads) {
    const int L = seqlens[b] > 0 ? seqlens[b] : 0;
    const int n = (L + kPage - 1) / kPage;
    if (staged) pages_s[b] = n;
    if (n > 0) mine += n + fixed;
  }
  for (int off = 16; off; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if ((threadIdx.x & 31) == 0) partial[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x != 0) return;
  auto pages_of = [&](int b) -> int {
    if (staged) return pages_s[b];
    const int L = seqlens[b] > 0 ? seqlens[b] : 0;
    return (L + kPage - 1) / kPage;
  };
  // remaining cost: unassigned pages plus one fixed cost per sequence (or
  // sequence remainder) that still has unassigned pages
  long long remaining = 0;
  for (int w = 0; w < kSchedThreads / 32; ++w) remaining += partial[w];
  auto target_for = [&](int part) {
    const long long left = num_parts - part;
    long long t = (remaining + fixed * (left - 1) + left - 1) / left;
    return t < fixed + 2 ? fixed + 2 : t;
  };

  int part = 0;
  long long load = 0;
  long long target = target_for(0);
  int32_t* m = meta;
  m[0] = 0; m[1] = 0; m[4] = 0; m[5] = 0; m[6] = 0; m[7] = 0;
  num_splits[0] = 0;
  int prefix = 0;  // running num_splits value (never re-read from global memory)
  for (int b = 0; b < batch; ++b) {
    const int n = pages_of(b);
    int pieces = 0;
    int p = 0;
    while (p < n) {
      const long long avail = target - load - fixed;
      if (avail < 1 && load > 0 && part < num_parts - 1) {
        // close this part at (b, p); the next one starts there
        m[2] = b; m[3] = p;
        remaining -= load;
        if (p > 0) remaining += fixed;  // the rest of b becomes a new piece
        ++part;
        m = meta + (size_t)part * kMetaInts;
        m[0] = b; m[1] = p; m[4] = pieces; m[5] = 0; m[6] = 0; m[7] = 0;
        load = 0;
        target = target_for(part);
        continue;
      }
      int take = n - p;
      if (part < num_parts - 1 && avail < take) {
        take = (int)(avail < 1 ? 1 : avail);
        if (n - p - take < 2) take = n - p;  // no tiny tail piece
      }
      p += take;
      load += take + fixed;
      ++pieces;
    }
    prefix += pieces;
    num_splits[b + 1] = prefix;
  }
  m[2] = batch; m[3] = 0;
  for (int q = part + 1; q < num_parts; ++q) {
    int32_t* e = meta + (size_t)q * kMetaInts;
    e[0] = batch; e[1] = 0; e[2] = batch; e[3] = 0;
    e[4] = 0; e[5] = 0; e[6] = 0; e[7] = 0;
  }
}

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int32_t* meta,
                            int32_t* num_splits, cudaStream_t stream) {
  metadata_kernel<<<1, kSchedThreads, 0, stream>>>(seqlens, batch, num_parts, meta, num_splits);
  return cudaGetLastError();
}

}  // namespace pmla
