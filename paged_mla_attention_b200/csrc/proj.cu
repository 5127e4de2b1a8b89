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
//             (B = W^UV_h as stored: K contiguous, i.e. K-major; K in two halves
//              so that the operands fit shared memory)
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kProjThreads = 128;
constexpr uint32_t kChunk = 16384;  // 128 rows x 128 bytes, one 64-column SW128 chunk

// Row `r` (bytes `src`, `kchunks` x 128 bytes) into chunk-major SW128 K-major layout.
__device__ __forceinline__ void stage_row(uint8_t* base, const uint8_t* src, int r, int kchunks) {
  for (int c = 0; c < kchunks; ++c) {
    const uint4* s = reinterpret_cast<const uint4*>(src + c * 128);
    uint8_t* d = base + c * kChunk + r * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(d + ((u ^ (r & 7)) << 4)) = __ldg(s + u);
  }
}

__device__ __forceinline__ void zero_row(uint8_t* base, int r, int kchunks) {
  for (int c = 0; c < kchunks; ++c)
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<uint4*>(base + c * kChunk + r * 128 + (u << 4)) = make_uint4(0, 0, 0, 0);
}

template <bool kAbsorb>
__global__ void __launch_bounds__(kProjThreads, 1) proj_kernel(const ProjParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  constexpr int N = kAbsorb ? 512 : 128;
  constexpr int K = kAbsorb ? 128 : 512;
  constexpr int kKHalf = kAbsorb ? K : K / 2;  // K staged per phase
  constexpr int kPhases = K / kKHalf;
  constexpr int kAChunks = kKHalf / 64;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * 128, h = blockIdx.y;
  const int t = t0 + tid;
  const bool valid = t < P.tokens;
  // the 128-byte swizzle needs 1024-byte aligned tiles: align the dynamic base
  // (one spare KB is part of the allocation)
  const uint32_t raw = smem_u32(smem);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sa = smem + (sbase - raw);                    // A: kAChunks chunks
  uint8_t* sb = sa + kAChunks * kChunk;                  // B
  if (tid == 0) {
    mbar_init(smem_u32(&done_bar), 1);
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
  const uint32_t idesc = make_idesc_bf16(128, kAbsorb ? 256 : 128, 0, kAbsorb ? 1 : 0);

  for (int ph = 0; ph < kPhases; ++ph) {
    // ---- stage A rows (token t) and B rows (row tid of the head's matrix)
    if (valid) {
      const uint8_t* arow =
          reinterpret_cast<const uint8_t*>(P.a + ((size_t)t * P.heads + h) * K + ph * kKHalf);
      stage_row(sa, arow, tid, kAChunks);
    } else {
      zero_row(sa, tid, kAChunks);
    }
    const uint16_t* w = P.w + (size_t)h * 128 * 512;
    if (kAbsorb) {
      // W^UK_h row k = tid: 512 N values -> MN-major chunks (64 N columns each)
      stage_row(sb, reinterpret_cast<const uint8_t*>(w + (size_t)tid * 512), tid, 8);
    } else {
      // W^UV_h row n = tid, K half ph: 256 K values -> K-major chunks
      stage_row(sb, reinterpret_cast<const uint8_t*>(w + (size_t)tid * 512 + ph * kKHalf), tid,
                kKHalf / 64);
    }
    fence_proxy_async_cta();  // generic shared-memory writes -> read by the MMA (async proxy)
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint64_t a0 = make_smem_desc(sbase, 16, 1024, 2);
      if (kAbsorb) {
        const uint64_t b0 = make_smem_desc(sbase + kAChunks * kChunk, kChunk, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < K / 16; ++ks) {
          const uint64_t ad = a0 + (uint64_t)(((ks >> 2) * kChunk + (ks & 3) * 32) >> 4);
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
            const uint64_t bd = b0 + (uint64_t)((nh * 4 * kChunk + ks * 2048) >> 4);
            mma_ss(tmem + 256u * nh, ad, bd, idesc, ks > 0);
          }
        }
      } else {
        const uint64_t b0 = make_smem_desc(sbase + kAChunks * kChunk, 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < kKHalf / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * kChunk + (ks & 3) * 32) >> 4;
          mma_ss(tmem, a0 + off, b0 + off, idesc, (ph > 0) || (ks > 0));
        }
      }
      tc_commit(smem_u32(&done_bar));
    }
    // every thread waits for the MMAs (they read this phase's shared memory)
    const bool ok = mbar_wait(smem_u32(&done_bar), (uint32_t)(ph & 1), &abort_flag, P.err,
                              kErrWaitBase + 40);
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
  }

  // ---- epilogue: row tid of the accumulator -> bf16 output row
  if (!abort_flag) {
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint16_t* out = kAbsorb ? P.out + ((size_t)t * P.heads + h) * kD : P.out + ((size_t)t * P.heads + h) * 128;
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
  return absorb ? (2 + 8) * (size_t)kChunk + 1024 : (4 + 4) * (size_t)kChunk + 1024;
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
