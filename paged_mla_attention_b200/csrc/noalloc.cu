// Allocation-free variant of mla_decode_with_kvcache.
//
// Some callers cannot call cudaMalloc at all: code running inside a CUDA graph
// being captured, allocator-free serving runtimes that own all device memory up
// front, or plugins loaded into a host process whose memory manager forbids
// other allocations.  They can still pass their inputs and outputs, but not a
// workspace.  This entry point runs the same decode with the split-KV scratch
// (partial outputs and log-sum-exps of split sequences) taken from a
// fixed-size array that the library itself holds in device memory.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library's module is loaded holds it (kNoAllocScratchBytes) until the process
// exits.  In host code its name is only a stand-in, not a device address, so
// the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it; that first
// call should therefore come before any stream capture on that device.
//
// All calls share the one array, which keeps whatever the last call left in
// it.  The decode writes every scratch entry it later reads, so nothing needs
// clearing between calls, but calls whose work overlaps on the GPU (different
// streams, or different host threads without ordering) race on the array and
// must be serialised by the caller.
#include <cstdio>
#include <mutex>

#include "../../include/pagedmla.h"
#include "pagedmla_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

}  // namespace

extern "C" {

PMLA_API int mla_decode_with_kvcache_noalloc(
    const uint16_t* q, const uint16_t* kvcache, const int32_t* block_table,
    const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv, int d, int dv,
    int num_pages, int max_pages_per_seq, const int32_t* tile_scheduler_metadata, int num_parts,
    const int32_t* num_splits, int causal, float softmax_scale, uint16_t* o, float* lse,
    void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    pmla::set_last_error("mla_decode_with_kvcache_noalloc: no usable current CUDA device");
    return PMLA_ERR_CUDA;
  }
  if (h_kv >= 1 && h_q >= 1 && h_q % h_kv == 0 && batch >= 0 && num_parts >= 1 && s_q >= 1) {
    // the same upper bound mla_get_metadata_sizes reports for this shape
    const size_t R = (size_t)s_q * (size_t)(h_q / h_kv);
    const size_t need = R > (size_t(1) << 20) ? ~size_t(0)
                        : pmla::workspace_layout(batch, (int)R, h_kv, num_parts).bytes;
    if (need > kNoAllocScratchBytes) {
      char msg[256];
      snprintf(msg, sizeof msg,
               "shape needs %zu bytes of split scratch, above the built-in %zu-byte maximum of "
               "mla_decode_with_kvcache_noalloc; use mla_decode_with_kvcache with a workspace",
               need, kNoAllocScratchBytes);
      pmla::set_last_error(msg);
      return PMLA_ERR_WORKSPACE;
    }
  }
  void* scratch;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        pmla::set_last_error("mla_decode_with_kvcache_noalloc: cudaGetSymbolAddress of the scratch array failed");
        return PMLA_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return mla_decode_with_kvcache(q, kvcache, block_table, cache_seqlens, batch, s_q, h_q, h_kv, d,
                                 dv, num_pages, max_pages_per_seq, tile_scheduler_metadata,
                                 num_parts, num_splits, causal, softmax_scale, o, lse, scratch,
                                 kNoAllocScratchBytes, stream);
}

}  // extern "C"
