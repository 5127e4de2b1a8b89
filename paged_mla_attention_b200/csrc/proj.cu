// Absorbed MLA projections around the latent decode (FlashMLA overview,
// section 2.2): with k^C_{j,h} = W^UK_h c_j and v_{j,h} = W^UV_h c_j,
//   q~_h = W^UK_h^T q^C_h       (128 -> 512, before the decode: the 576-wide
//                                 query is [q~_h ; q^R_h])
//   o_h  = W^UV_h o^lat_h       (512 -> 128, after it)
// W^UK and W^UV are stored [h][128][512].  Per head these are small GEMMs over
// the tokens of the step, run on tcgen05 tensor cores: one CTA per (128
// tokens, head), operands staged into shared memory in the 128-byte-swizzled
// layouts the MMA reads, fp32 accumulation in TMEM, bf16 results.
//
//   absorb:   C[t][n] = sum_k q^C[t][k] W^UK[k][n]   M = tokens, N = 512, K = 128
//             (B = W^UK_h as stored: N contiguous, i.e. MN-major)
//   unabsorb: C[t][n] = sum_k o^lat[t][k] W^UV[n][k] M = tokens, N = 128, K = 512
//             (B = W^UV_h as stored: K contiguous, i.e. K-major; K in four
//              quarters so that the operands fit shared memory)
// Operands move by TMA (one thread issues every tile of the CTA, so a whole
// head's weight matrix is in flight at once): the kernels are bound by reading
// each head's 128 KB weight matrix.  Tokens past the end read as zeros.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kProjThreads = 128;
constexpr uint32_t kChunk = 16384;  // 128 rows x 128 bytes, one 64-column SW128 chunk

// Chunks are filled by TMA boxes of 64 columns x 128 rows (128-byte swizzle):
//   a map:  [T][H][K] as dims {K, H, T}, box {64, 1, 128}: 128 tokens of head h
//   w map:  [H*128][512] as dims {512, H*128}, box {64, 128}: 128 rows of head h
// absorb:  K = 128 in one phase; A (2 chunks) + B (8 N-chunks, MN-major) = 160 KB
//          behind two barriers (A and N 0..255, then N 256..511) so the first N
//          half's MMAs start while the second half lands.
// project: K = 512 in four phases of 128 (A 2 chunks + B 2 chunks = 64 KB each)
//          through three buffers; phase 3 reuses buffer 0 once phase 0's MMAs
//          have completed.
// Thread 0 issues the copies and the MMAs; all threads run the epilogue.
template <bool kAbsorb>
__global__ void __launch_bounds__(kProjThreads, 1)
proj_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
            const ProjParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full_bar[3];
  __shared__ uint64_t mma_bar[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  constexpr int N = kAbsorb ? 512 : 128;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * 128, h = blockIdx.y;
  const int t = t0 + tid;
  const bool valid = t < P.tokens;
  // the 128-byte swizzle needs 1024-byte aligned tiles: align the dynamic base
  // (one spare KB is part of the allocation)
  const uint32_t raw = smem_u32(smem);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const int wrow = h * 128;  // first row of this head's weight matrix

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&full_bar[i]), 1);
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&mma_bar[i]), 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid == 0) {
    const uint64_t pol_a = policy_evict_first();
    const uint64_t pol_w = policy_evict_last();  // re-read by the head's other token tiles
    bool ok = true;
    uint32_t issued = 0;  // bit i: full_bar[i] has a phase in flight
    uint32_t issued_par = 0;  // bit i: the parity of that phase
    if (kAbsorb) {
      const uint32_t f0 = smem_u32(&full_bar[0]), f1 = smem_u32(&full_bar[1]);
      mbar_arrive_expect_tx(f0, 6 * kChunk);
      for (int c = 0; c < 2; ++c) tma_load_3d(sbase + c * kChunk, &tmap_a, f0, c * 64, h, t0, pol_a);
      for (int c = 0; c < 4; ++c) tma_load_2d(sbase + (2 + c) * kChunk, &tmap_w, f0, c * 64, wrow, pol_w);
      mbar_arrive_expect_tx(f1, 4 * kChunk);
      for (int c = 4; c < 8; ++c) tma_load_2d(sbase + (2 + c) * kChunk, &tmap_w, f1, c * 64, wrow, pol_w);
      issued = 3u;
      const uint32_t idesc = make_idesc_bf16(128, 256, 0, 1);
      const uint64_t a0 = make_smem_desc(sbase, 16, 1024, 2);
      const uint64_t b0 = make_smem_desc(sbase + 2 * kChunk, kChunk, 1024, 2);
      for (int nh = 0; nh < 2 && ok; ++nh) {
        ok = mbar_wait(nh ? f1 : f0, 0u, &abort_flag, P.err, kErrWaitBase + 40);
        if (!ok) break;
        issued &= ~(1u << nh);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t ad = a0 + (uint64_t)(((ks >> 2) * kChunk + (ks & 3) * 32) >> 4);
          const uint64_t bd = b0 + (uint64_t)((nh * 4 * kChunk + ks * 2048) >> 4);
          mma_ss(tmem + 256u * nh, ad, bd, idesc, ks > 0);
        }
      }
      if (ok) tc_commit(smem_u32(&mma_bar[1]));
    } else {
      auto load_phase = [&](int ph, int buf) {
        const uint32_t f = smem_u32(&full_bar[buf]);
        const uint32_t dst = sbase + buf * 4 * kChunk;
        mbar_arrive_expect_tx(f, 4 * kChunk);
        issued_par = (issued_par & ~(1u << buf)) | ((uint32_t)(ph / 3) << buf);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(dst + c * kChunk, &tmap_a, f, ph * 128 + c * 64, h, t0, pol_a);
          tma_load_2d(dst + (2 + c) * kChunk, &tmap_w, f, ph * 128 + c * 64, wrow, pol_w);
        }
        issued |= 1u << buf;
      };
      for (int ph = 0; ph < 3; ++ph) load_phase(ph, ph);
      const uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
      for (int ph = 0; ph < 4 && ok; ++ph) {
        const int buf = ph % 3;
        ok = mbar_wait(smem_u32(&full_bar[buf]), (uint32_t)(ph / 3), &abort_flag, P.err, kErrWaitBase + 40);
        if (!ok) break;
        issued &= ~(1u << buf);
        tc_fence_after();
        const uint32_t base = sbase + buf * 4 * kChunk;
        const uint64_t a0 = make_smem_desc(base, 16, 1024, 2);
        const uint64_t b0 = make_smem_desc(base + 2 * kChunk, 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = ((ks >> 2) * kChunk + (ks & 3) * 32) >> 4;
          mma_ss(tmem, a0 + off, b0 + off, idesc, (ph > 0) || (ks > 0));
        }
        if (ph == 0) {
          tc_commit(smem_u32(&mma_bar[0]));
        } else if (ph == 1) {
          // buffer 0 is free once phase 0's MMAs have read it: load phase 3 there
          ok = mbar_wait(smem_u32(&mma_bar[0]), 0u, &abort_flag, P.err, kErrWaitBase + 40);
          if (ok) load_phase(3, 0);
        }
      }
      if (ok) tc_commit(smem_u32(&mma_bar[1]));
    }
    if (!ok) {  // no copy may still be writing this CTA's shared memory when it exits
      abort_flag = 1;
      for (int i = 0; i < 3; ++i)
        if (issued & (1u << i)) mbar_wait_drain(smem_u32(&full_bar[i]), (issued_par >> i) & 1u);
    }
  }
  // every thread waits for the accumulator
  const bool ok = __syncthreads_and(mbar_wait(smem_u32(&mma_bar[1]), 0u, &abort_flag, P.err, kErrWaitBase + 40));
  tc_fence_after();

  // ---- epilogue: row tid of the accumulator -> bf16 output row
  if (ok) {
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint16_t* out = P.out + ((size_t)t * P.heads + h) * (kAbsorb ? kD : 128);
#pragma unroll 1
    for (int j = 0; j < N / 64; ++j) {
      uint32_t v0[32], v1[32];
      tmem_ld64_sync(tmem + lane_off + 64u * j, v0, v1);
      uint32_t pk[32];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        pk[u] = pack_bf16x2(__uint_as_float(v0[2 * u]), __uint_as_float(v0[2 * u + 1]));
        pk[16 + u] = pack_bf16x2(__uint_as_float(v1[2 * u]), __uint_as_float(v1[2 * u + 1]));
      }
      if (valid) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_global_v8(out + 64 * j + 16 * u, pk[8 * u], pk[8 * u + 1], pk[8 * u + 2], pk[8 * u + 3],
                       pk[8 * u + 4], pk[8 * u + 5], pk[8 * u + 6], pk[8 * u + 7]);
      }
    }
    if (kAbsorb && valid) {  // the RoPE part of the query passes through
      const uint4* src = reinterpret_cast<const uint4*>(P.rope + ((size_t)t * P.heads + h) * 64);
      uint4* dst = reinterpret_cast<uint4*>(out + 512);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[u] = __ldg(src + u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, N);
  }
}

}  // namespace

size_t proj_smem_bytes(bool absorb) {
  return absorb ? (2 + 8) * (size_t)kChunk + 1024 : 3 * 4 * (size_t)kChunk + 1024;
}

cudaError_t launch_proj(const ProjParams& p, bool absorb, const CUtensorMap& tmap_a, const CUtensorMap& tmap_w,
                        cudaStream_t stream) {
  if (p.tokens == 0) return cudaSuccess;
  const size_t smem = proj_smem_bytes(absorb);
  cudaError_t e = absorb ? cudaFuncSetAttribute(proj_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                         : cudaFuncSetAttribute(proj_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.tokens + 127) / 128, p.heads);
  if (absorb)
    proj_kernel<true><<<grid, kProjThreads, smem, stream>>>(tmap_a, tmap_w, p);
  else
    proj_kernel<false><<<grid, kProjThreads, smem, stream>>>(tmap_a, tmap_w, p);
  return cudaGetLastError();
}

}  // namespace pmla
