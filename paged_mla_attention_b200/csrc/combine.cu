// Merge of split-KV partial results (the "combine the split results" kernel
// the FlashMLA overview names in section 4.2(1)).
//
// For a query row of a sequence cut into n >= 2 pieces, each piece k left a
// normalised partial o_k (fp32) and its log-sum-exp lse_k.  The full result is
//   lse = log sum_k exp(lse_k),   o = sum_k exp(lse_k - lse) o_k,
// computed with the largest lse_k subtracted first.  Empty pieces
// (lse_k = -inf) weigh nothing; if every piece is empty, o = 0, lse = -inf.
// Sequences with no pages at all (n = 0) also get o = 0, lse = -inf here;
// unsplit sequences (n = 1) were written by the decode kernel directly.
//
// Layout: one warp per query row, each lane owns 16 of the 512 columns (four
// float4 per partial), so every partial row is read with fully coalesced
// 2 KB warp loads.  Grid: (row blocks of 8, h_kv, batch).
#include "pagedmla_internal.cuh"

#include <cuda_bf16.h>

namespace pmla {

namespace {

constexpr int kRowsPerBlock = 8;  // 8 warps, one row each

__global__ void __launch_bounds__(32 * kRowsPerBlock)
combine_kernel(const CombineParams P) {
  const int b = blockIdx.z;
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = blockIdx.x * kRowsPerBlock + warp;
  if (rr >= P.R) return;
  const int s0 = P.num_splits[b];
  const int n = P.num_splits[b + 1] - s0;
  if (n == 1) return;
  const int qi = rr / P.hpk;
  const int head = g * P.hpk + rr % P.hpk;
  uint4* orow = reinterpret_cast<uint4*>(P.o + ((size_t)(b * P.s_q + qi) * P.h_q + head) * kDV) +
                lane * 2;
  float* lse_out = P.lse + ((size_t)b * P.h_q + head) * P.s_q + qi;

  float m = -INFINITY;
  for (int k = lane; k < n; k += 32)
    m = fmaxf(m, P.part_lse[((size_t)(s0 + k) * P.h_kv + g) * P.R + rr]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (n == 0 || m == -INFINITY) {
    orow[0] = make_uint4(0, 0, 0, 0);
    orow[1] = make_uint4(0, 0, 0, 0);
    if (lane == 0) *lse_out = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = lane; k < n; k += 32)
    z += __expf(P.part_lse[((size_t)(s0 + k) * P.h_kv + g) * P.R + rr] - m);
#pragma unroll
  for (int off = 16; off; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float total = m + __logf(z);

  float acc[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) acc[u] = 0.f;
  for (int k = 0; k < n; ++k) {
    const size_t row = ((size_t)(s0 + k) * P.h_kv + g) * P.R + rr;
    const float w = __expf(P.part_lse[row] - total);
    const float4* src = reinterpret_cast<const float4*>(P.part_o + row * kDV) + lane * 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 v = __ldg(src + u);
      acc[4 * u] = fmaf(w, v.x, acc[4 * u]);
      acc[4 * u + 1] = fmaf(w, v.y, acc[4 * u + 1]);
      acc[4 * u + 2] = fmaf(w, v.z, acc[4 * u + 2]);
      acc[4 * u + 3] = fmaf(w, v.w, acc[4 * u + 3]);
    }
  }
  uint32_t pk[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
    pk[u] = *reinterpret_cast<uint32_t*>(&h2);
  }
  orow[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  orow[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0) *lse_out = total;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  dim3 grid((p.R + kRowsPerBlock - 1) / kRowsPerBlock, p.h_kv, p.batch);
  if (p.batch == 0) return cudaSuccess;
  combine_kernel<<<grid, 32 * kRowsPerBlock, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pmla
