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
// Operands move with cp.async (16-byte asynchronous copies, many in flight per
// thread): the kernels are bound by reading each head's 128 KB weight matrix.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kProjThreads = 128;
constexpr uint32_t kChunk = 16384;  // 128 rows x 128 bytes, one 64-column SW128 chunk

// 16-byte asynchronous global -> shared copy (L2 only); `src_bytes` 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Copies 128 rows x `kChunks` 64-column chunks into chunk-major SW128 tiles at
// `dst` (1024-byte aligned): row r's 16-byte unit u of chunk c lands at
// c * kChunk + r * 128 + ((u ^ (r & 7)) << 4).  Row r starts at `src` + r * `row_stride`
// elements (plus `col0`); rows with r >= `rows_valid` are zero-filled.  Eight
// consecutive threads cover one 128-byte chunk row, so each warp reads whole rows.
template <int kChunks>
__device__ __forceinline__ void stage_tile(uint32_t dst, const uint16_t* src, size_t row_stride, int col0,
                                           int rows_valid, int tid) {
#pragma unroll 4
  for (int i = tid; i < 128 * kChunks * 8; i += kProjThreads) {
    const int u = i & 7, c = (i >> 3) % kChunks, r = (i >> 3) / kChunks;
    const bool ok = r < rows_valid;
    const uint16_t* g = ok ? src + (size_t)r * row_stride + col0 + c * 64 + u * 8 : src;
    cp_async16(dst + c * kChunk + r * 128 + ((u ^ (r & 7)) << 4), g, ok ? 16u : 0u);
  }
}

// absorb:  K = 128 in one phase; A (2 chunks) + B (8 N-chunks, MN-major) = 160 KB,
//          copied as two groups (A and N 0..255, then N 256..511) so the first
//          N half's MMAs start while the second half lands.
// project: K = 512 in four phases of 128 (A 2 chunks + B 2 chunks = 64 KB each)
//          through three buffers; phase 3 reuses buffer 0 once phase 0's MMAs
//          have completed.
template <bool kAbsorb>
__global__ void __launch_bounds__(kProjThreads, 1) proj_kernel(const ProjParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  constexpr int N = kAbsorb ? 512 : 128;
  constexpr int K = kAbsorb ? 128 : 512;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * 128, h = blockIdx.y;
  const int t = t0 + tid;
  const bool valid = t < P.tokens;
  const int rows_valid = min(128, P.tokens - t0);
  // the 128-byte swizzle needs 1024-byte aligned tiles: align the dynamic base
  // (one spare KB is part of the allocation)
  const uint32_t raw = smem_u32(smem);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint16_t* a = P.a + ((size_t)t0 * P.heads + h) * K;   // token rows of this head
  const size_t a_stride = (size_t)P.heads * K;
  const uint16_t* w = P.w + (size_t)h * 128 * 512;             // [128][512]

  if (kAbsorb) {
    stage_tile<2>(sbase, a, a_stride, 0, rows_valid, tid);                  // A: q^C, K 0..127
    stage_tile<4>(sbase + 2 * kChunk, w, 512, 0, 128, tid);                 // B: N 0..255
    cp_async_commit();
    stage_tile<4>(sbase + 6 * kChunk, w, 512, 256, 128, tid);               // B: N 256..511
    cp_async_commit();
  } else {
#pragma unroll
    for (int ph = 0; ph < 3; ++ph) {
      stage_tile<2>(sbase + ph * 4 * kChunk, a, a_stride, ph * 128, rows_valid, tid);
      stage_tile<2>(sbase + (ph * 4 + 2) * kChunk, w, 512, ph * 128, 128, tid);
      cp_async_commit();
    }
  }
  if (tid == 0) {
    mbar_init(smem_u32(&mma_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;

  if (kAbsorb) {
    const uint32_t idesc = make_idesc_bf16(128, 256, 0, 1);
    const uint64_t a0 = make_smem_desc(sbase, 16, 1024, 2);
    const uint64_t b0 = make_smem_desc(sbase + 2 * kChunk, kChunk, 1024, 2);
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      if (nh == 0) cp_async_wait<1>(); else cp_async_wait<0>();
      fence_proxy_async_cta();  // cp.async writes (generic proxy) -> read by the MMA
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < K / 16; ++ks) {
          const uint64_t ad = a0 + (uint64_t)(((ks >> 2) * kChunk + (ks & 3) * 32) >> 4);
          const uint64_t bd = b0 + (uint64_t)((nh * 4 * kChunk + ks * 2048) >> 4);
          mma_ss(tmem + 256u * nh, ad, bd, idesc, ks > 0);
        }
        if (nh == 1) tc_commit(smem_u32(&mma_bar));
      }
    }
    ok = mbar_wait(smem_u32(&mma_bar), 0u, &abort_flag, P.err, kErrWaitBase + 40);
  } else {
    const uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int ph = 0; ph < 4; ++ph) {
      if (ph == 0) cp_async_wait<2>();
      else if (ph == 3) cp_async_wait<0>();
      else cp_async_wait<1>();
      fence_proxy_async_cta();
      __syncthreads();
      const uint32_t buf = sbase + (ph % 3) * 4 * kChunk;
      if (tid == 0) {
        tc_fence_after();
        const uint64_t a0 = make_smem_desc(buf, 16, 1024, 2);
        const uint64_t b0 = make_smem_desc(buf + 2 * kChunk, 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = ((ks >> 2) * kChunk + (ks & 3) * 32) >> 4;
          mma_ss(tmem, a0 + off, b0 + off, idesc, (ph > 0) || (ks > 0));
        }
        if (ph == 0 || ph == 3) tc_commit(smem_u32(&mma_bar));
      }
      if (ph == 1) {
        // buffer 0 is free once phase 0's MMAs have read it: load phase 3 there
        ok = __syncthreads_and(mbar_wait(smem_u32(&mma_bar), 0u, &abort_flag, P.err, kErrWaitBase + 40));
        if (!ok) {
          cp_async_commit();
          break;
        }
        stage_tile<2>(sbase, a, a_stride, 3 * 128, rows_valid, tid);
        stage_tile<2>(sbase + 2 * kChunk, w, 512, 3 * 128, 128, tid);
        cp_async_commit();
      }
    }
    if (ok) ok = mbar_wait(smem_u32(&mma_bar), 1u, &abort_flag, P.err, kErrWaitBase + 40);
  }
  cp_async_wait<0>();
  ok = __syncthreads_and(ok);
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

cudaError_t launch_proj(const ProjParams& p, bool absorb, cudaStream_t stream) {
  if (p.tokens == 0) return cudaSuccess;
  const size_t smem = proj_smem_bytes(absorb);
  cudaError_t e = absorb ? cudaFuncSetAttribute(proj_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                         : cudaFuncSetAttribute(proj_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.tokens + 127) / 128, p.heads);
  if (absorb)
    proj_kernel<true><<<grid, kProjThreads, smem, stream>>>(p);
  else
    proj_kernel<false><<<grid, kProjThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pmla
