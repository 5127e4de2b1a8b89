// Merge of split-KV partial results (the "combine the split results" kernel
// the FlashMLA overview names in section 4.2(1)).
//
// For a query row of a sequence cut into n >= 2 pieces, each piece k left a
// normalised partial o_k (fp32) and its log-sum-exp lse_k.  The full result is
//   lse = log sum_k exp(lse_k),   o = sum_k exp(lse_k - lse) o_k,
// computed with the largest lse_k subtracted first.  Empty pieces
// (lse_k = -inf) weigh nothing; if every piece is empty, o = 0, lse = -inf.
// Sequences with no pages at all (n = 0), and sequences longer than their
// block table (skipped by the decode kernel), also get o = 0, lse = -inf here;
// unsplit sequences (n = 1) were written by the decode kernel directly.
//
// Layout: the partials are chunk-major, [slot][h_kv][64 chunks of 8 columns]
// [R rows][8].  A block takes 32 consecutive rows and one column slice (all
// 512 columns, a quarter or an eighth) of one (sequence, KV head); warps take
// the chunks of that slice, lane = row, so every load is 1 KB contiguous, with
// the loads of several pieces in flight at once.  The merged rows go through
// shared memory and leave as contiguous 16-byte stores.  Grid: (row blocks of
// 32 x column slices, h_kv, batch).
//
// Overlap with the decode kernel: this kernel is launched as a programmatic
// dependent of the decode kernel, which lets it start once every decode CTA is
// resident.  Each finished split piece adds 2 to a counter per (sequence, KV
// head, row group) -- once after its lse, once after its o rows, each behind
// a device-scope fence -- and a block merges only after the counter reaches
// 2 x pieces (a bounded wait that records an error if it runs out).  The last
// block of the grid ends by waiting for the whole decode grid, so this grid
// cannot complete before the decode grid has, and work queued after it sees
// the decode kernel complete.  Every other block exits as soon as its rows are
// written: blocks parked on that wait would hold SM slots that blocks still to
// be dispatched need.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace pmla {

namespace {

constexpr int kMergeRows = 32;
constexpr int kMergeThreads = 256;
constexpr int kChunks = kDV / 8;  // 64 chunks of 8 columns

// kQuarters column slices per row block (one block each; a warp handles
// kCPW = 8 / kQuarters chunks of its slice) and kPieceBatch pieces whose loads
// are in flight together.  Few slices suit sequences cut into few pieces (less
// repeated lse work, fewer blocks waiting); many slices suit a long sequence
// cut into many pieces, whose merge would otherwise run on a handful of SMs.
// kGroups groups of 8 warps share a block and take the pieces in turns, each
// group keeping kPieceBatch pieces' loads in flight; their sums meet in shared
// memory (a sequence cut into ~70 pieces otherwise spends ~9 serial rounds of
// load latency in one block).
template <int kQuarters, int kPieceBatch, int kGroups = 1>
__global__ void __launch_bounds__(kMergeThreads * kGroups) combine_kernel(const CombineParams P) {
  constexpr int kQCols = kDV / kQuarters;
  constexpr int kQChunks = kChunks / kQuarters;
  constexpr int kCPW = kQChunks / 8;  // chunks per warp
  constexpr int kMaxPieces = kQuarters == 1 ? 64 : 128;  // lse values staged per round
  // merged rows, bf16; rows padded by 16 bytes so the lane-per-row stores hit distinct banks
  __shared__ __align__(16) uint16_t tile[kMergeRows][kQCols + 8];
  __shared__ float row_lse[kMergeRows];
  const int b = blockIdx.z;
  const int g = blockIdx.y;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warp = wid & 7, grp = wid >> 3;  // chunk warp within the group, piece group
  const int r0 = (blockIdx.x / kQuarters) * kMergeRows;
  const int quarter = blockIdx.x % kQuarters;
  const int s0 = P.num_splits[b];
  // a sequence longer than its block table was skipped by the decode kernel
  // (which recorded the error): its rows are written here as empty
  const int n = (long long)P.seqlens[b] > (long long)P.max_pages * kPage ? 0 : P.num_splits[b + 1] - s0;
  const bool last_block =
      blockIdx.x == gridDim.x - 1 && blockIdx.y == gridDim.y - 1 && blockIdx.z == gridDim.z - 1;
  if (n == 1) {  // written by the decode kernel directly
    if (last_block) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int rr = r0 + lane;
  const bool valid = rr < P.R;
  __shared__ int ready;
  if (n >= 2) {
    if (threadIdx.x == 0) {
      const int* ctr = P.seq_done + ((size_t)b * P.h_kv + g) * P.n_rg + r0 / kRows;
      const uint64_t t0 = global_timer_ns();
      int ok = 1;
      for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= 2 * n) break;
        if (global_timer_ns() - t0 > PMLA_WAIT_TIMEOUT_NS) {
          atomicCAS(P.err, 0, kErrWaitBase + 30);
          ok = 0;
          break;
        }
        __nanosleep(256);
      }
      ready = ok;
    }
    __syncthreads();
    if (!ready) {
      if (last_block) asm volatile("griddepcontrol.wait;" ::: "memory");
      return;
    }
  }

  // all lse_k of the block's rows in one round trip (warp w loads pieces w, w+8,
  // ...), then every thread derives its row's total and the merge weights from
  // shared memory; pieces beyond kMaxPieces go round again
  __shared__ float wsh[kMaxPieces][kMergeRows];
  float m = -INFINITY, z = 0.f;
  for (int k0 = 0; k0 < n; k0 += kMaxPieces) {
    const int nk = min(n - k0, kMaxPieces);
    __syncthreads();
    for (int k = wid; k < nk; k += 8 * kGroups)
      wsh[k][lane] = valid ? __ldcg(P.part_lse + ((size_t)(s0 + k0 + k) * P.h_kv + g) * P.R + rr)
                           : -INFINITY;
    __syncthreads();
    for (int k = 0; k < nk; ++k) {  // online max / sum of exp over this row's pieces
      const float x = wsh[k][lane];
      if (x > m) {
        z = z * __expf(m - x) + 1.f;
        m = x;
      } else if (x != -INFINITY) {
        z += __expf(x - m);
      }
    }
  }
  const float total = (m == -INFINITY) ? -INFINITY : m + __logf(z);
  if (wid == 0) row_lse[lane] = total;

  float acc[kCPW][8];
#pragma unroll
  for (int i = 0; i < kCPW; ++i)
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[i][u] = 0.f;
  if (valid && total != -INFINITY) {
    // pieces go kPieceBatch at a time so that 16 loads per thread are in flight
    const float4* base = reinterpret_cast<const float4*>(P.part_o) +
                         ((size_t)(quarter * kQChunks + warp) * P.R + rr) * 2;
    const size_t piece_stride = (size_t)P.h_kv * kChunks * P.R * 2;  // float4s between slots
    const size_t chunk8 = (size_t)8 * P.R * 2;                       // float4s between chunks c, c+8
    for (int k0 = grp * kPieceBatch; k0 < n; k0 += kPieceBatch * kGroups) {
      float w[kPieceBatch];
      float4 x[kPieceBatch][kCPW], y[kPieceBatch][kCPW];
#pragma unroll
      for (int j = 0; j < kPieceBatch; ++j) {
        const int k = k0 + j;
        w[j] = 0.f;
        if (k < n) {
          const size_t slot = (size_t)(s0 + k) * P.h_kv + g;
          const float lk = n <= kMaxPieces ? wsh[k][lane] : __ldcg(P.part_lse + slot * P.R + rr);
          w[j] = __expf(lk - total);
          const float4* src = base + (size_t)(s0 + k) * piece_stride + (size_t)g * kChunks * P.R * 2;
#pragma unroll
          for (int i = 0; i < kCPW; ++i) {  // written by a kernel still running: L2, not the L1 cache
            x[j][i] = __ldcg(src + i * chunk8);
            y[j][i] = __ldcg(src + i * chunk8 + 1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < kCPW; ++i) x[j][i] = y[j][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < kPieceBatch; ++j)
#pragma unroll
        for (int i = 0; i < kCPW; ++i) {
          acc[i][0] = fmaf(w[j], x[j][i].x, acc[i][0]);
          acc[i][1] = fmaf(w[j], x[j][i].y, acc[i][1]);
          acc[i][2] = fmaf(w[j], x[j][i].z, acc[i][2]);
          acc[i][3] = fmaf(w[j], x[j][i].w, acc[i][3]);
          acc[i][4] = fmaf(w[j], y[j][i].x, acc[i][4]);
          acc[i][5] = fmaf(w[j], y[j][i].y, acc[i][5]);
          acc[i][6] = fmaf(w[j], y[j][i].z, acc[i][6]);
          acc[i][7] = fmaf(w[j], y[j][i].w, acc[i][7]);
        }
    }
  }
  if constexpr (kGroups > 1) {
    // the other groups' sums join group 0's
    __shared__ float red[kGroups - 1][8][kCPW][8][kMergeRows];
    if (grp > 0)
#pragma unroll
      for (int i = 0; i < kCPW; ++i)
#pragma unroll
        for (int u = 0; u < 8; ++u) red[grp - 1][warp][i][u][lane] = acc[i][u];
    __syncthreads();
    if (grp == 0)
#pragma unroll
      for (int q = 0; q < kGroups - 1; ++q)
#pragma unroll
        for (int i = 0; i < kCPW; ++i)
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[i][u] += red[q][warp][i][u][lane];
  }
#pragma unroll
  for (int i = 0; i < kCPW; ++i) {
    if (grp > 0) break;
    uint32_t pk[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[i][2 * u], acc[i][2 * u + 1]);
      pk[u] = *reinterpret_cast<uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(&tile[lane][(warp + 8 * i) * 8]) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  __syncthreads();

  // rows r0.. of (b, g): row rr is query token rr / hpk, head g*hpk + rr % hpk
  constexpr int kVec = kQCols * 2 / 16;  // 16-byte pieces per row of the quarter
  for (int e = threadIdx.x; e < kMergeRows * kVec; e += kMergeThreads * kGroups) {
    const int row = e / kVec, c = e % kVec;
    const int r = r0 + row;
    if (r >= P.R) continue;
    const int qi = r / P.hpk, head = g * P.hpk + r % P.hpk;
    uint4* dst =
        reinterpret_cast<uint4*>(P.o + ((size_t)(b * P.s_q + qi) * P.h_q + head) * kDV + quarter * kQCols) + c;
    *dst = *reinterpret_cast<const uint4*>(&tile[row][c * 8]);
  }
  if (wid == 0 && valid && quarter == 0) {
    const int qi = rr / P.hpk, head = g * P.hpk + rr % P.hpk;
    P.lse[((size_t)b * P.h_q + head) * P.s_q + qi] = row_lse[lane];
  }
  if (last_block) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

namespace {

// Zeroes the merge's completion counters.  Launched as a programmatic dependent
// of whatever precedes it (normally the schedule), it lets its own dependent,
// the decode kernel, start its setup at once; it zeroes only after the
// preceding grid has completed (a decode kernel of an earlier call may still be
// counting), so when this grid completes, so has the one before it.
__global__ void __launch_bounds__(256) clear_counters_kernel(int* ctr, int n) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) ctr[i] = 0;
}

}  // namespace

cudaError_t launch_clear_counters(int* ctr, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n + 255) / 256 < 148 ? (n + 255) / 256 : 148), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, clear_counters_kernel, ctr, n);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  // a long sequence cut into many pieces shows as many scheduler parts per
  // sequence: spread each row block over 8 column slices then.  Otherwise a
  // sequence has a few pieces (mostly two, the halves of a cut): with one row
  // group per KV head, 4 column slices with both pieces' loads in flight at once
  // (the tail after the decode kernel: uniform 11.0 -> 6.5 us, varlen 17.3 ->
  // 7.8 us); with more row groups one block per row block (4 slices measured no
  // better on causal2).
  const bool many = p.num_parts >= 2 * p.batch;
  const bool sliced = !many && p.R <= kRows;
  const int slices = many ? 8 : sliced ? 4 : 1;
  cfg.gridDim = dim3(((p.R + kMergeRows - 1) / kMergeRows) * slices, p.h_kv, p.batch);
  cfg.blockDim = dim3(many ? 2 * kMergeThreads : kMergeThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (many) return cudaLaunchKernelEx(&cfg, combine_kernel<8, 8, 2>, p);
  return sliced ? cudaLaunchKernelEx(&cfg, combine_kernel<4, 2>, p) : cudaLaunchKernelEx(&cfg, combine_kernel<1, 1>, p);
}

}  // namespace pmla
