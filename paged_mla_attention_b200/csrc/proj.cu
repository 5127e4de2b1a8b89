// Absorbed MLA projections around the latent decode (FlashMLA overview,
// section 2.2): with k^C_{j,h} = W^UK_h c_j and v_{j,h} = W^UV_h c_j,
//   q~_h = W^UK_h^T q^C_h       (128 -> 512, before the decode: the 576-wide
//                                 query is [q~_h ; q^R_h])
//   o_h  = W^UV_h o^lat_h       (512 -> 128, after it)
// W^UK and W^UV are stored [h][128][512].  Per head these are small GEMMs over
// the tokens of the step, run on tcgen05 tensor cores with operands staged into
// shared memory by TMA in the 128-byte-swizzled layouts the MMA reads, fp32
// accumulation in TMEM and bf16 results.
//
//   absorb:   C[t][n] = sum_k q^C[t][k] W^UK[k][n]   M = tokens, N = 512, K = 128
//             (B = W^UK_h as stored: N contiguous, i.e. MN-major).  One CTA per
//             (128 tokens, head, half of N): A 32 KB + its W^UK half 64 KB.
//   unabsorb: C[t][n] = sum_k o^lat[t][k] W^UV[n][k] M = tokens, N = 128, K = 512
//             (B = W^UV_h as stored: K contiguous, i.e. K-major).  One CTA per
//             (128 tokens, head): K streams in eight 64-wide chunks (A 16 KB +
//             W 16 KB each) through a ring of slots.
// At decode sizes (a step's tokens are at most a few hundred) the kernels are
// bound by reading the weights (128 KB per head) and moving the activations.
// Absorb CTAs, and unabsorb CTAs when there are several token tiles, take 96 KB
// of shared memory and at most 256 TMEM columns, so two fit an SM and one's
// epilogue overlaps the other's loads; with one tile (at most 128 tokens) the
// unabsorb grid is one CTA per head, fewer than the SMs, and its ring has six
// slots (192 KB) so that six of the eight chunks are in flight at once.
// Results leave through shared memory by TMA stores (one 32-token x 64-column
// box per warp), which write whole 128-byte rows; tokens past the end read as
// zeros and are not stored.
//
// The kernels are launched as programmatic dependents of the preceding kernel
// on the stream: a CTA sets up, lets its own dependents launch, and prefetches
// its weights from HBM into L2, then waits (griddepcontrol.wait) for the
// preceding grid to complete before any load into shared memory or any store.
// The prefetch only warms L2, so the result is the same whatever kernel wrote
// the weights; back to back (one projection per layer) the weight fetch, launch
// and setup overlap the previous kernel's tail.
#include "pagedmla_internal.cuh"
#include "ptx.cuh"

namespace pmla {

namespace {

constexpr int kProjThreads = 128;
constexpr uint32_t kChunk = 16384;   // 128 rows x 128 bytes, one 64-column SW128 chunk
constexpr uint32_t kOutBox = 4096;   // 32 rows x 128 bytes: one warp's 64-column output box
constexpr uint32_t kOperandBytes = 6 * kChunk;
constexpr int kRingMax = 6;          // unabsorb ring slots (A chunk + W chunk each)

// Epilogue of both kernels: warp w owns accumulator lanes [32w, 32w+32) (tokens
// t0+32w...).  For each 64-column group j of the `ncols` accumulator columns
// from TMEM address `tmem` on, it converts to bf16, writes the warp's box at
// staging + (j*4 + w) * 4 KB in the 128-byte-swizzled layout of the output map
// (16-byte unit u of row r at unit u ^ (r & 7)), and one lane stores the box to
// output columns col0 + 64 j.  With `last`, that lane then waits until its
// stores have read their boxes (shared memory must outlive them).
__device__ __forceinline__ void drain_to_global(const CUtensorMap* tmap_out, uint32_t tmem, uint32_t staging,
                                                int ncols, int col0, int h, int t0, int tokens, bool last) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const bool any_row = t0 + 32 * warp < tokens;
#pragma unroll 1
  for (int j = 0; j < ncols / 64; ++j) {
    uint32_t v0[32], v1[32];
    __syncwarp();
    tmem_ld64_sync(tmem + lane_off + 64u * j, v0, v1);
    const uint32_t row = staging + (uint32_t)(j * 4 + warp) * kOutBox + (uint32_t)lane * 128u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t* src = u < 4 ? v0 + 8 * u : v1 + 8 * (u - 4);
      st_shared_v4(row + ((uint32_t)(u ^ (lane & 7)) << 4), pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
                   pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
                   pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
                   pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
    }
    fence_proxy_async_cta();  // the writes above, before the async proxy reads them
    __syncwarp();
    if (lane == 0 && any_row)
      tma_store_3d(tmap_out, staging + (uint32_t)(j * 4 + warp) * kOutBox, col0 + 64 * j, h, t0 + 32 * warp);
  }
  if (lane == 0 && any_row) {
    bulk_commit_group();
    if (last) bulk_wait_group_read0();
  }
}

// Absorb.  Maps: a = q^C [T][H][128] as dims {128, H, T}, box {64, 1, 128};
// w = W^UK as dims {512, H*128}, box {64, 128}; out = q [T][H][576] as dims
// {576, H, T}, box {64, 1, 32}.  Shared memory: A chunks 0-1 (K 0-63, 64-127),
// then the four W^UK chunks of this half (N 64 apart, each 128 K-rows).
// Barrier 0: A + W chunks 0-1 (N 0..127 of the half); barrier 1: W chunks 2-3.
__global__ void __launch_bounds__(kProjThreads, 2)
absorb_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
              const __grid_constant__ CUtensorMap tmap_out, const ProjParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full_bar[2];
  __shared__ uint64_t mma_bar[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * 128, h = blockIdx.y, nh = blockIdx.z;
  const int t = t0 + tid;
  const bool valid = t < P.tokens;
  const uint32_t sbase = (smem_u32(smem) + 1023u) & ~1023u;  // SW128 tiles need 1 KB alignment
  const int wrow = h * 128, ncol0 = 256 * nh;

  if (tid == 0) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&mma_bar[i]), 1);
    }
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_out);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid == 0) {
    // one tile of tokens: the weights are read once (let them go); several: the
    // other tiles' CTAs re-read them from L2
    const uint64_t pol_a = policy_evict_first();
    const uint64_t pol_w = P.tokens > 128 ? policy_evict_last() : policy_evict_first();
    if (blockIdx.x == 0)
      for (int c = 0; c < 4; ++c) tma_prefetch_l2_2d(&tmap_w, ncol0 + 64 * c, wrow, pol_w);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t f0 = smem_u32(&full_bar[0]), f1 = smem_u32(&full_bar[1]);
    mbar_arrive_expect_tx(f0, 4 * kChunk);
    for (int c = 0; c < 2; ++c) tma_load_3d(sbase + c * kChunk, &tmap_a, f0, c * 64, h, t0, pol_a);
    for (int c = 0; c < 2; ++c) tma_load_2d(sbase + (2 + c) * kChunk, &tmap_w, f0, ncol0 + 64 * c, wrow, pol_w);
    mbar_arrive_expect_tx(f1, 2 * kChunk);
    for (int c = 2; c < 4; ++c) tma_load_2d(sbase + (2 + c) * kChunk, &tmap_w, f1, ncol0 + 64 * c, wrow, pol_w);
    uint32_t pending = 3u;  // bit g: full_bar[g] not yet seen complete
    bool ok = true;
    const uint32_t idesc = make_idesc_bf16(128, 128, 0, 1);
    const uint64_t a0 = make_smem_desc(sbase, 16, 1024, 2);
    for (int g = 0; g < 2 && ok; ++g) {
      ok = mbar_wait(g ? f1 : f0, 0u, &abort_flag, P.err, kErrWaitBase + 40);
      if (!ok) break;
      pending &= ~(1u << g);
      tc_fence_after();
      // N 128g..128g+127 of the half: W chunks 2g, 2g+1 (LBO = one chunk along N)
      const uint64_t b0 = make_smem_desc(sbase + (2 + 2 * g) * kChunk, kChunk, 1024, 2);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = a0 + (uint64_t)(((ks >> 2) * kChunk + (ks & 3) * 32) >> 4);
        const uint64_t bd = b0 + (uint64_t)((ks * 2048) >> 4);
        mma_ss(tmem + 128u * g, ad, bd, idesc, ks > 0);
      }
      tc_commit(smem_u32(&mma_bar[g]));
    }
    if (!ok) {  // no copy may still be writing this CTA's shared memory when it exits
      abort_flag = 1;
      for (int g = 0; g < 2; ++g)
        if (pending & (1u << g)) mbar_wait_drain(smem_u32(&full_bar[g]), 0u);
    }
  }
  // every thread waits for the preceding grid: the RoPE columns are read from it
  // and no output may be written before it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (nh == 1 && valid) {  // the RoPE part of the query passes through
    const uint4* src = reinterpret_cast<const uint4*>(P.rope + ((size_t)t * P.heads + h) * 64);
    uint4* dst = reinterpret_cast<uint4*>(P.out + ((size_t)t * P.heads + h) * kD + 512);
    uint4 r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) r[u] = __ldg(src + u);
#pragma unroll
    for (int u = 0; u < 8; ++u) dst[u] = r[u];
  }
  // N 0..127 of the half leave while the MMAs of N 128..255 run: W chunks 0-1
  // are free once the first group's MMAs completed and stage its boxes, W chunks
  // 2-3 stage the second group's
  for (int g = 0; g < 2; ++g) {
    const bool ok = __syncthreads_and(mbar_wait(smem_u32(&mma_bar[g]), 0u, &abort_flag, P.err, kErrWaitBase + 40));
    if (!ok) break;
    tc_fence_after();
    drain_to_global(&tmap_out, tmem + 128u * g, sbase + (2 + 2 * g) * kChunk, 128, ncol0 + 128 * g, h, t0, P.tokens,
                    g == 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Unabsorb.  Maps: a = o^lat [T][H][512] as dims {512, H, T}, box {64, 1, 128};
// w = W^UV as dims {512, H*128}, box {64, 128}; out = o [T][H][128] as dims
// {128, H, T}, box {64, 1, 32}.  K chunk c (columns 64c..64c+63) goes to ring
// slot c % ring (ring = 3 or 6 slots): A chunk, then W chunk.  Thread 32 loads,
// thread 0 issues the MMAs and frees a slot with a commit once its four MMAs
// have read it.
__global__ void __launch_bounds__(kProjThreads, 2)
unabsorb_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                const __grid_constant__ CUtensorMap tmap_out, const ProjParams P, const int ring) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full_bar[kRingMax], empty_bar[kRingMax];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * 128, h = blockIdx.y;
  const uint32_t sbase = (smem_u32(smem) + 1023u) & ~1023u;
  const int wrow = h * 128;

  if (tid == 0) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = 0; i < ring; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    mbar_init(smem_u32(&mma_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_out);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid == 32) {  // producer
    const uint64_t pol_a = policy_evict_first();
    const uint64_t pol_w = P.tokens > 128 ? policy_evict_last() : policy_evict_first();
    if (blockIdx.x == 0)
      for (int c = 0; c < 8; ++c) tma_prefetch_l2_2d(&tmap_w, 64 * c, wrow, pol_w);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int issued = 0;  // chunks issued: slot s holds phases of chunks s, s + ring, ...
    for (int c = 0; c < 8; ++c) {
      const int s = c % ring;
      if (c >= ring && !mbar_wait(smem_u32(&empty_bar[s]), (uint32_t)((c / ring - 1) & 1), &abort_flag, P.err,
                                  kErrWaitBase + 41))
        break;
      const uint32_t f = smem_u32(&full_bar[s]);
      const uint32_t dst = sbase + (uint32_t)s * 2 * kChunk;
      mbar_arrive_expect_tx(f, 2 * kChunk);
      tma_load_3d(dst, &tmap_a, f, 64 * c, h, t0, pol_a);
      tma_load_2d(dst + kChunk, &tmap_w, f, 64 * c, wrow, pol_w);
      ++issued;
    }
    // no copy may still be writing this CTA's shared memory when it exits (on the
    // normal path every phase has completed already): the last chunk issued into
    // each slot
    for (int c = issued - 1; c >= 0 && c >= issued - ring; --c)
      mbar_wait_drain(smem_u32(&full_bar[c % ring]), (uint32_t)((c / ring) & 1));
  } else if (tid == 0) {  // MMA issuer
    const uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
    bool ok = true;
    for (int c = 0; c < 8 && ok; ++c) {
      const int s = c % ring;
      ok = mbar_wait(smem_u32(&full_bar[s]), (uint32_t)((c / ring) & 1), &abort_flag, P.err, kErrWaitBase + 40);
      if (!ok) break;
      tc_fence_after();
      const uint32_t base = sbase + (uint32_t)s * 2 * kChunk;
      const uint64_t a0 = make_smem_desc(base, 16, 1024, 2);
      const uint64_t b0 = make_smem_desc(base + kChunk, 16, 1024, 2);
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_ss(tmem, a0 + 2 * k, b0 + 2 * k, idesc, (c > 0) || (k > 0));
      tc_commit(smem_u32(&empty_bar[s]));
    }
    if (ok) tc_commit(smem_u32(&mma_bar));
    else abort_flag = 1;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // no output before the preceding grid completed
  const bool ok = __syncthreads_and(mbar_wait(smem_u32(&mma_bar), 0u, &abort_flag, P.err, kErrWaitBase + 40));
  tc_fence_after();
  // every chunk has been read by the MMAs: the first 32 KB of the ring stage the
  // output boxes
  if (ok) drain_to_global(&tmap_out, tmem, sbase, 128, 0, h, t0, P.tokens, true);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

cudaError_t launch_proj(const ProjParams& p, bool absorb, const CUtensorMap& tmap_a, const CUtensorMap& tmap_w,
                        const CUtensorMap& tmap_out, cudaStream_t stream) {
  // one token tile: one unabsorb CTA per head (fewer than the SMs) with a ring
  // of six K chunks; several tiles: two CTAs per SM with three
  const int ring = p.tokens <= 128 ? kRingMax : 3;
  // operands + alignment slack for the 1 KB aligned base
  const size_t smem = (absorb ? kOperandBytes : (size_t)ring * 2 * kChunk) + 1024;
  constexpr int kMaxSmem = kRingMax * 2 * kChunk + 1024;
  cudaError_t e = absorb ? cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                         : cudaFuncSetAttribute(unabsorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.tokens + 127) / 128, p.heads, absorb ? 2 : 1);
  cfg.blockDim = dim3(kProjThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return absorb ? cudaLaunchKernelEx(&cfg, absorb_kernel, tmap_a, tmap_w, tmap_out, p)
                : cudaLaunchKernelEx(&cfg, unabsorb_kernel, tmap_a, tmap_w, tmap_out, p, ring);
}

}  // namespace pmla
