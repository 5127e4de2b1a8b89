// Append of new tokens to the paged KV cache (the write side of the paged
// layout in the FlashMLA overview, section 4.2(1): logical 64-token blocks
// mapped to physical pages by block_table).
//
// Token t of the s_new new tokens of sequence b goes to position L_b + t:
// page block_table[b][(L_b + t) / 64], slot (L_b + t) % 64, and its 576-wide
// row [c^KV ; k^R] of KV head g is copied there unchanged (bf16 bits).
//
// One warp per (b, t, g) row: 72 16-byte vectors, lanes stride over them, so
// each warp reads and writes 1152 contiguous bytes.  A row whose position lies
// past the block table or whose page id is out of range is skipped and
// recorded in the device error word.  The kernel is HBM-bound: 2304 bytes per
// row (read + write).
#include "pagedmla_internal.cuh"

namespace pmla {

namespace {

constexpr int kAppendWarps = 8;
constexpr int kRowVecs = kD * 2 / 16;  // 72 16-byte vectors per row

__global__ void __launch_bounds__(32 * kAppendWarps) append_kernel(const AppendParams P) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kAppendWarps + warp;
  const long long rows = (long long)P.batch * P.s_new * P.h_kv;
  if (row >= rows) return;
  const int g = (int)(row % P.h_kv);
  const int t = (int)((row / P.h_kv) % P.s_new);
  const int b = (int)(row / ((long long)P.h_kv * P.s_new));
  const int L = P.seqlens[b] > 0 ? P.seqlens[b] : 0;
  const long long pos = (long long)L + t;
  if (pos >= (long long)P.max_pages * kPage) {
    if (lane == 0) atomicCAS(P.err, 0, kErrBadAppend);
    return;
  }
  const int page = P.block_table[(size_t)b * P.max_pages + (size_t)(pos / kPage)];
  if (page < 0 || page >= P.num_pages) {
    if (lane == 0) atomicCAS(P.err, 0, kErrBadPage);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(P.new_kv + (size_t)row * kD);
  uint4* dst = reinterpret_cast<uint4*>(
      P.kvcache + (((size_t)page * kPage + (size_t)(pos % kPage)) * P.h_kv + g) * kD);
#pragma unroll
  for (int i = lane; i < kRowVecs; i += 32) dst[i] = __ldg(src + i);
  if (P.new_seqlens && t == 0 && g == 0 && lane == 0) P.new_seqlens[b] = L + P.s_new;
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.batch * p.s_new * p.h_kv;
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + kAppendWarps - 1) / kAppendWarps;
  append_kernel<<<(unsigned)blocks, 32 * kAppendWarps, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pmla
