// extern "C" entry points of libpagedmla.so (declared in include/pagedmla.h).
//
// Argument checks happen here, on the host, before anything is launched; the
// kernels themselves only defend against device-side data they cannot check
// (page ids out of range, lost arrivals) and report through the device error
// word instead of faulting.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>

#include "../../include/pagedmla.h"
#include "pagedmla_internal.cuh"

namespace pmla {

WorkspaceLayout workspace_layout(int batch, int R, int h_kv, int num_parts) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  WorkspaceLayout w;
  const size_t slots = (size_t)batch + (size_t)num_parts;
  const size_t rows = slots * (size_t)h_kv * (size_t)R;
  w.lse_off = rows * kDV * sizeof(float);
  w.done_off = w.lse_off + up(rows * sizeof(float));
  w.done_count = (size_t)batch * (size_t)h_kv * (size_t)((R + kRows - 1) / kRows);
  w.bytes = w.done_off + up(w.done_count * sizeof(int));
  return w;
}

}  // namespace pmla

namespace {

thread_local std::string g_last_error;

__device__ int g_device_error;  // first error code any kernel reported

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int fail_cuda(cudaError_t e, const char* what) {
  return fail(PMLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

struct DeviceInfo {
  bool ready = false;
  int max_clusters = 0;       // 2-CTA decode clusters resident at once
  int max_clusters_pair = 0;  // 4-CTA decode clusters (two row groups each) resident at once
  int num_sms = 0;
  int* err_ptr = nullptr;
};
std::mutex g_mu;
DeviceInfo g_dev[64];

// Per-device one-time set-up: kernel attributes, cluster occupancy, the
// address of the device error word.  Returns 0 or a PMLA error.
int device_setup(int* device_out, DeviceInfo** info_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(PMLA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
      return fail(PMLA_ERR_UNSUPPORTED, "needs an sm_100 (B200-class) GPU, device %d is sm_%d%d",
                  dev, prop.major, prop.minor);
    if ((size_t)prop.sharedMemPerBlockOptin < pmla::decode_smem_bytes())
      return fail(PMLA_ERR_UNSUPPORTED, "device offers %zu B shared memory per block, need %zu",
                  (size_t)prop.sharedMemPerBlockOptin, pmla::decode_smem_bytes());
    int n = 0, n4 = 0;
    int rc = pmla::decode_max_active_clusters(dev, false, &n);
    if (rc == 0) rc = pmla::decode_max_active_clusters(dev, true, &n4);
    if (rc != 0) return fail_cuda((cudaError_t)rc, "cudaOccupancyMaxActiveClusters");
    if (n < 1 || n4 < 1) return fail(PMLA_ERR_UNSUPPORTED, "decode kernel cannot be resident on this device");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(device error word)");
    d.max_clusters = n;
    d.max_clusters_pair = n4;
    d.num_sms = prop.multiProcessorCount;
    d.err_ptr = static_cast<int*>(p);
    d.ready = true;
  }
  *device_out = dev;
  *info_out = &d;
  return PMLA_OK;
}

// Partial-result rows of the largest schedule for this shape, (batch + parts)
// x h_kv x R, must stay below 2^32 so that every workspace size and offset is
// far from overflowing (2^32 rows x 2 KB) and the counter count fits an int.
bool too_many_rows(int batch, long long R, int h_kv) {
  return ((long long)batch + pmla::kMaxParts) * (long long)h_kv * R > (1ll << 32);
}

int check_shape(int batch, int num_heads_per_head_k, int num_heads_k) {
  if (batch < 0 || batch > 65535) return fail(PMLA_ERR_INVALID_ARG, "batch %d not in [0, 65535]", batch);
  if (num_heads_per_head_k < 1 || num_heads_k < 1 || num_heads_k > 65535)
    return fail(PMLA_ERR_INVALID_ARG, "bad head counts (%d per KV head, %d KV heads)",
                num_heads_per_head_k, num_heads_k);
  if (num_heads_per_head_k > (1 << 20) || too_many_rows(batch, num_heads_per_head_k, num_heads_k))
    return fail(PMLA_ERR_UNSUPPORTED, "shape too large (batch %d, %d rows per KV head, %d KV heads)", batch,
                num_heads_per_head_k, num_heads_k);
  return PMLA_OK;
}

// Scheduler parts: as many (part, KV head, cluster) work units as decode clusters
// fit on the device at once.  A KV head with one 128-row group takes one 2-CTA
// cluster per part; with more, one 4-CTA cluster per two row groups, and the
// SMs those clusters leave free take further parts, each run by one 2-CTA
// cluster per row group and weighted kPartWeightAux in the schedule.
struct PartPlan {
  int main;  // parts of the call's first decode launch
  int aux;   // parts of the 2-CTA launch on the remaining SMs
};
PartPlan part_plan(const DeviceInfo& d, int num_heads_per_head_k, int num_heads_k) {
  const int n_rg = (num_heads_per_head_k + pmla::kRows - 1) / pmla::kRows;
  const bool pair = pmla::decode_uses_pairs(n_rg);
  const long long groups = (long long)(pair ? (n_rg + 1) / 2 : n_rg) * num_heads_k;
  long long parts = (pair ? d.max_clusters_pair : d.max_clusters) / groups;
  if (parts < 1) parts = 1;
  long long aux = 0;
  if (pair) {  // SMs left by the 4-CTA clusters, in 2-CTA clusters, one per row group
    const long long free_sms = (long long)d.num_sms - 4 * parts * groups;
    aux = free_sms > 0 ? (free_sms / 2) / ((long long)n_rg * num_heads_k) : 0;
  }
  return PartPlan{(int)parts, (int)aux};
}
int parts_for(const DeviceInfo& d, int num_heads_per_head_k, int num_heads_k) {
  const PartPlan pl = part_plan(d, num_heads_per_head_k, num_heads_k);
  return pl.main + pl.aux;
}
// Parts of the first decode launch for a call with num_parts parts: all of them
// unless num_parts is exactly what part_plan gives (the schedule then weighs
// the rest kPartWeightAux and they run as the 2-CTA launch).
int main_parts(const DeviceInfo& d, int num_heads_per_head_k, int num_heads_k, int num_parts) {
  const PartPlan pl = part_plan(d, num_heads_per_head_k, num_heads_k);
  return (pl.aux > 0 && num_parts == pl.main + pl.aux) ? pl.main : num_parts;
}

size_t workspace_for(int batch, int R, int h_kv, int num_parts, size_t* lse_offset) {
  const pmla::WorkspaceLayout w = pmla::workspace_layout(batch, R, h_kv, num_parts);
  *lse_offset = w.lse_off;
  return w.bytes;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

namespace pmla {
void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }
}  // namespace pmla

extern "C" {

const char* pmla_version(void) { return "pagedmla 0.1.0 (sm_100a)"; }

const char* pmla_last_error(void) { return g_last_error.c_str(); }

const char* mla_get_last_error(void) { return g_last_error.c_str(); }

int mla_get_metadata_sizes(int batch, int num_heads_per_head_k, int num_heads_k, int* num_parts,
                           size_t* workspace_bytes) {
  g_last_error.clear();
  if (!num_parts || !workspace_bytes) return fail(PMLA_ERR_INVALID_ARG, "null output pointer");
  int rc = check_shape(batch, num_heads_per_head_k, num_heads_k);
  if (rc) return rc;
  int dev;
  DeviceInfo* d;
  rc = device_setup(&dev, &d);
  if (rc) return rc;
  *num_parts = parts_for(*d, num_heads_per_head_k, num_heads_k);
  size_t lse_off;
  *workspace_bytes = workspace_for(batch, num_heads_per_head_k, num_heads_k, *num_parts, &lse_off);
  return PMLA_OK;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int num_heads_per_head_k,
                     int num_heads_k, int32_t* tile_scheduler_metadata, int num_parts,
                     int32_t* num_splits, void* stream) {
  g_last_error.clear();
  int rc = check_shape(batch, num_heads_per_head_k, num_heads_k);
  if (rc) return rc;
  if (!tile_scheduler_metadata || !num_splits || (batch > 0 && !cache_seqlens))
    return fail(PMLA_ERR_INVALID_ARG, "null pointer argument");
  if (num_parts < 1 || num_parts > pmla::kMaxParts)
    return fail(PMLA_ERR_INVALID_ARG, "num_parts %d outside [1, %d]", num_parts, pmla::kMaxParts);
  int dev;
  DeviceInfo* d;
  rc = device_setup(&dev, &d);
  if (rc) return rc;
  const int num_main = main_parts(*d, num_heads_per_head_k, num_heads_k, num_parts);
  cudaError_t e = pmla::launch_metadata(cache_seqlens, batch, num_parts, num_main, tile_scheduler_metadata,
                                        num_splits, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "metadata kernel launch");
  return PMLA_OK;
}

}  // extern "C"

namespace {

constexpr int kStageDecode = 1, kStageMerge = 2;

// Shared body of the three decode entry points: validates everything, then
// launches the split-KV decode kernel and/or the merge kernel.
int decode_impl(const uint16_t* q, const uint16_t* kvcache, const int32_t* block_table,
                const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv, int d, int dv,
                int num_pages, int max_pages_per_seq, const int32_t* tile_scheduler_metadata,
                int num_parts, const int32_t* num_splits, int causal, float softmax_scale, uint16_t* o,
                float* lse, void* workspace, size_t workspace_bytes, void* stream, int stages) {
  g_last_error.clear();
  if (d != PMLA_HEAD_DIM || dv != PMLA_HEAD_DIM_V)
    return fail(PMLA_ERR_UNSUPPORTED, "head dims must be d=576, dv=512 (got %d, %d)", d, dv);
  if (batch < 0 || batch > 65535 || s_q < 1 || h_q < 1 || h_kv < 1 || h_kv > 65535)
    return fail(PMLA_ERR_INVALID_ARG, "bad shape batch=%d s_q=%d h_q=%d h_kv=%d", batch, s_q, h_q,
                h_kv);
  if (h_q % h_kv != 0)
    return fail(PMLA_ERR_UNSUPPORTED, "h_q (%d) must be a multiple of h_kv (%d)", h_q, h_kv);
  {
    // the query tile is loaded by TMA in boxes of min(h_q/h_kv, 128) rows
    const int hpk = h_q / h_kv;
    const bool ok = hpk < pmla::kRows ? (pmla::kRows % hpk == 0 && hpk >= 8) : (hpk % pmla::kRows == 0);
    if (!ok)
      return fail(PMLA_ERR_UNSUPPORTED,
                  "h_q/h_kv = %d: must divide 128 (and be >= 8) or be a multiple of 128", hpk);
  }
  if (num_pages < 1 || max_pages_per_seq < 1 || num_parts < 1)
    return fail(PMLA_ERR_INVALID_ARG, "num_pages, max_pages_per_seq and num_parts must be >= 1");
  if ((long long)num_pages * pmla::kPage * h_kv > (1ll << 31))
    return fail(PMLA_ERR_UNSUPPORTED, "kv cache too large for 32-bit row coordinates");
  if (!std::isfinite(softmax_scale) || softmax_scale < 0.f)
    return fail(PMLA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (batch == 0) return PMLA_OK;  // nothing to read or write: buffers may be empty (null)
  if (!q || !kvcache || !block_table || !cache_seqlens || !tile_scheduler_metadata ||
      !num_splits || !o || !lse)
    return fail(PMLA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(kvcache) || !aligned32(o))
    return fail(PMLA_ERR_ALIGNMENT, "q and kvcache must be 16-byte aligned, o 32-byte aligned");
  const long long R = (long long)s_q * (h_q / h_kv);
  if (R > (1 << 20) || too_many_rows(batch, R, h_kv))
    return fail(PMLA_ERR_UNSUPPORTED, "s_q * h_q / h_kv too large for this batch");
  size_t lse_off;
  const size_t need = workspace_for(batch, (int)R, h_kv, num_parts, &lse_off);
  if (!workspace || workspace_bytes < need || !aligned32(workspace))
    return fail(PMLA_ERR_WORKSPACE, "workspace needs %zu bytes, 32-byte aligned (got %zu)", need,
                workspace_bytes);

  int dev;
  DeviceInfo* info;
  int rc = device_setup(&dev, &info);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (stages & kStageDecode) {
    auto encode = get_encode();
    if (!encode) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");

    // kvcache as a 3-D tensor: [576 columns] x [h_kv heads] x [num_pages*64 tokens];
    // each TMA box is 64 columns x 1 head x 64 tokens with the 128-byte swizzle.
    CUtensorMap tmap;
    cuuint64_t gdim[3] = {(cuuint64_t)pmla::kD, (cuuint64_t)h_kv,
                          (cuuint64_t)num_pages * pmla::kPage};
    cuuint64_t gstride[2] = {(cuuint64_t)pmla::kD * 2, (cuuint64_t)h_kv * pmla::kD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)pmla::kPage};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(kvcache),
                         gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)cr);

    // kvcache once more as a 4-D tensor [64 columns] x [tokens] x [9 column chunks]
    // x [h_kv heads] (the chunk stride, 128 bytes, is below the token stride): one
    // box of 64 columns x 64 tokens x 4 chunks lands as 4 chunk-major 8 KB tiles,
    // i.e. half of a page's value part in a single TMA instruction.
    CUtensorMap tmap_v;
    {
      cuuint64_t vdim[4] = {64, (cuuint64_t)num_pages * pmla::kPage, (cuuint64_t)pmla::kD / 64,
                            (cuuint64_t)h_kv};
      cuuint64_t vstride[3] = {(cuuint64_t)h_kv * pmla::kD * 2, 128, (cuuint64_t)pmla::kD * 2};
      cuuint32_t vbox[4] = {64, (cuuint32_t)pmla::kPage, 4, 1};
      cuuint32_t vestride[4] = {1, 1, 1, 1};
      cr = encode(&tmap_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(kvcache), vdim,
                  vstride, vbox, vestride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS)
        return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (value tiles) failed (%d)", (int)cr);
  }

    // the same 4-D view with boxes of 2 column chunks (16 KB): the pair variant's
    // page stages and value halves
    CUtensorMap tmap_kv2;
    {
      cuuint64_t vdim[4] = {64, (cuuint64_t)num_pages * pmla::kPage, (cuuint64_t)pmla::kD / 64,
                            (cuuint64_t)h_kv};
      cuuint64_t vstride[3] = {(cuuint64_t)h_kv * pmla::kD * 2, 128, (cuuint64_t)pmla::kD * 2};
      cuuint32_t vbox[4] = {64, (cuuint32_t)pmla::kPage, 2, 1};
      cuuint32_t vestride[4] = {1, 1, 1, 1};
      cr = encode(&tmap_kv2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(kvcache), vdim,
                  vstride, vbox, vestride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS)
        return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (two-chunk tiles) failed (%d)", (int)cr);
    }

    // q as a 2-D tensor: [576 columns] x [batch*s_q*h_q rows]; boxes of 64 columns
    // x min(h_q/h_kv, 128) rows with the 128-byte swizzle.
    CUtensorMap tmap_q;
    {
      const int hpk = h_q / h_kv;
      cuuint64_t qdim[2] = {(cuuint64_t)pmla::kD, (cuuint64_t)batch * s_q * h_q};
      cuuint64_t qstride[1] = {(cuuint64_t)pmla::kD * 2};
      cuuint32_t qbox[2] = {64, (cuuint32_t)(hpk < pmla::kRows ? hpk : pmla::kRows)};
      cuuint32_t qestride[2] = {1, 1};
      cr = encode(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(q), qdim,
                  qstride, qbox, qestride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS)
        return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)cr);
  }

    pmla::DecodeParams p;
    p.q = q;
    p.block_table = block_table;
    p.seqlens = cache_seqlens;
    p.meta = tile_scheduler_metadata;
    p.num_splits = num_splits;
    p.o = o;
    p.lse = lse;
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + lse_off);
    const pmla::WorkspaceLayout wl = pmla::workspace_layout(batch, (int)R, h_kv, num_parts);
    p.seq_done = reinterpret_cast<int*>(static_cast<char*>(workspace) + wl.done_off);
    p.err = info->err_ptr;
    p.batch = batch;
    p.s_q = s_q;
    p.h_q = h_q;
    p.h_kv = h_kv;
    p.hpk = h_q / h_kv;
    p.R = (int)R;
    p.n_rg = (int)((R + pmla::kRows - 1) / pmla::kRows);
    p.num_parts = num_parts;
    p.part0 = 0;
    p.follows_decode = 0;
    p.max_pages = max_pages_per_seq;
    p.num_pages = num_pages;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    const bool pair = pmla::decode_uses_pairs(p.n_rg);
    if ((long long)num_parts * h_kv * p.n_rg > (1ll << 28))
      return fail(PMLA_ERR_UNSUPPORTED, "grid too large");

    cudaError_t e = pmla::decode_prepare(dev);
    if (e != cudaSuccess) return fail_cuda(e, "decode kernel attributes");
    // the merge kernel counts completion signals from zero
    e = pmla::launch_clear_counters(p.seq_done, (int)wl.done_count, st);
    if (e != cudaSuccess) return fail_cuda(e, "clearing the completion counters");
    const int num_main = main_parts(*info, (int)R, h_kv, num_parts);
    e = pmla::launch_decode(p, tmap, tmap_q, tmap_v, tmap_kv2, pair, num_main, st);
    if (e != cudaSuccess) return fail_cuda(e, "decode kernel launch");
    if (num_main < num_parts) {
      // the remaining parts on the SMs the 4-CTA clusters leave free: 2-CTA
      // clusters, one per row group, launched as a programmatic dependent of
      // the first decode kernel (they start once all of its CTAs are resident)
      p.part0 = num_main;
      p.follows_decode = 1;
      e = pmla::launch_decode(p, tmap, tmap_q, tmap_v, tmap_kv2, false, num_parts - num_main, st);
      if (e != cudaSuccess) return fail_cuda(e, "decode kernel launch (remaining SMs)");
    }
  }
  if (!(stages & kStageMerge)) return PMLA_OK;

  const pmla::WorkspaceLayout wl2 = pmla::workspace_layout(batch, (int)R, h_kv, num_parts);
  pmla::CombineParams c;
  c.num_splits = num_splits;
  c.seqlens = cache_seqlens;
  c.max_pages = max_pages_per_seq;
  c.part_o = static_cast<float*>(workspace);
  c.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + wl2.lse_off);
  c.seq_done = reinterpret_cast<const int*>(static_cast<char*>(workspace) + wl2.done_off);
  c.err = info->err_ptr;
  c.o = o;
  c.lse = lse;
  c.batch = batch;
  c.s_q = s_q;
  c.h_q = h_q;
  c.h_kv = h_kv;
  c.hpk = h_q / h_kv;
  c.R = (int)R;
  c.n_rg = (int)((R + pmla::kRows - 1) / pmla::kRows);
  c.num_parts = num_parts;
  cudaError_t e = pmla::launch_combine(c, st);
  if (e != cudaSuccess) return fail_cuda(e, "combine kernel launch");
  return PMLA_OK;
}

}  // namespace

extern "C" {

#define PMLA_DECODE_ARGS                                                                       \
  q, kvcache, block_table, cache_seqlens, batch, s_q, h_q, h_kv, d, dv, num_pages,              \
      max_pages_per_seq, tile_scheduler_metadata, num_parts, num_splits, causal, softmax_scale, \
      o, lse, workspace, workspace_bytes, stream
#define PMLA_DECODE_PARAMS                                                                     \
  const uint16_t *q, const uint16_t *kvcache, const int32_t *block_table,                      \
      const int32_t *cache_seqlens, int batch, int s_q, int h_q, int h_kv, int d, int dv,      \
      int num_pages, int max_pages_per_seq, const int32_t *tile_scheduler_metadata,            \
      int num_parts, const int32_t *num_splits, int causal, float softmax_scale, uint16_t *o,  \
      float *lse, void *workspace, size_t workspace_bytes, void *stream

int mla_decode_with_kvcache(PMLA_DECODE_PARAMS) {
  return decode_impl(PMLA_DECODE_ARGS, kStageDecode | kStageMerge);
}
int mla_decode_splits(PMLA_DECODE_PARAMS) { return decode_impl(PMLA_DECODE_ARGS, kStageDecode); }
int mla_merge_splits(PMLA_DECODE_PARAMS) { return decode_impl(PMLA_DECODE_ARGS, kStageMerge); }

int mla_append_kvcache(const uint16_t* new_kv, const int32_t* block_table,
                       const int32_t* cache_seqlens, int batch, int s_new, int h_kv, int d,
                       uint16_t* kvcache, int num_pages, int max_pages_per_seq,
                       int32_t* new_seqlens, void* stream) {
  g_last_error.clear();
  if (d != PMLA_HEAD_DIM) return fail(PMLA_ERR_UNSUPPORTED, "head dim must be d=576 (got %d)", d);
  if (batch < 0 || batch > 65535 || s_new < 0 || h_kv < 1 || h_kv > 65535)
    return fail(PMLA_ERR_INVALID_ARG, "bad shape batch=%d s_new=%d h_kv=%d", batch, s_new, h_kv);
  if (num_pages < 1 || max_pages_per_seq < 1)
    return fail(PMLA_ERR_INVALID_ARG, "num_pages and max_pages_per_seq must be >= 1");
  if ((long long)batch * s_new * h_kv > (1ll << 40))
    return fail(PMLA_ERR_UNSUPPORTED, "too many rows");
  if ((long long)batch * s_new == 0) return PMLA_OK;
  if (!new_kv || !block_table || !cache_seqlens || !kvcache)
    return fail(PMLA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(new_kv) || !aligned16(kvcache))
    return fail(PMLA_ERR_ALIGNMENT, "new_kv and kvcache must be 16-byte aligned");
  int dev;
  DeviceInfo* info;
  int rc = device_setup(&dev, &info);
  if (rc) return rc;
  pmla::AppendParams a;
  a.new_kv = new_kv;
  a.block_table = block_table;
  a.seqlens = cache_seqlens;
  a.kvcache = kvcache;
  a.new_seqlens = new_seqlens;
  a.err = info->err_ptr;
  a.batch = batch;
  a.s_new = s_new;
  a.h_kv = h_kv;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  cudaError_t e = pmla::launch_append(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "append kernel launch");
  return PMLA_OK;
}

static int proj_call(const uint16_t* a, const uint16_t* rope, const uint16_t* w, int tokens, int heads,
                     uint16_t* out, void* stream, bool absorb) {
  g_last_error.clear();
  if (tokens < 0 || heads < 1 || heads > 65535 || (long long)tokens > (1ll << 31))
    return fail(PMLA_ERR_INVALID_ARG, "bad shape tokens=%d heads=%d", tokens, heads);
  if (tokens == 0) return PMLA_OK;
  if (!a || !w || !out || (absorb && !rope)) return fail(PMLA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(a) || !aligned16(w) || !aligned32(out) || (absorb && !aligned16(rope)))
    return fail(PMLA_ERR_ALIGNMENT, "inputs must be 16-byte aligned and the output 32-byte aligned");
  int dev;
  DeviceInfo* info;
  int rc = device_setup(&dev, &info);
  if (rc) return rc;
  pmla::ProjParams p;
  p.a = a;
  p.rope = rope;
  p.w = w;
  p.out = out;
  p.err = info->err_ptr;
  p.tokens = tokens;
  p.heads = heads;
  auto encode = get_encode();
  if (!encode) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  // activations [tokens][heads][K] as dims {K, heads, tokens}: a box of 64 columns x
  // 1 head x 128 tokens is one 128-row SW128 chunk of a head's token tile
  const cuuint64_t K = absorb ? 128 : 512;
  CUtensorMap tmap_a, tmap_w;
  {
    cuuint64_t dim[3] = {K, (cuuint64_t)heads, (cuuint64_t)tokens};
    cuuint64_t stride[2] = {K * 2, (cuuint64_t)heads * K * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult cr = encode(&tmap_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a), dim, stride,
                         box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (activations) failed (%d)", (int)cr);
  }
  // weights [heads][128][512] as dims {512, heads*128}: a box of 64 columns x 128 rows
  {
    cuuint64_t dim[2] = {512, (cuuint64_t)heads * 128};
    cuuint64_t stride[1] = {1024};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    CUresult cr = encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(w), dim, stride,
                         box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (weights) failed (%d)", (int)cr);
  }
  // output [tokens][heads][576 or 128] as dims {N, heads, tokens}: a box of 64
  // columns x 1 head x 32 tokens is one warp's share of a 64-column output group
  CUtensorMap tmap_out;
  {
    const cuuint64_t N = absorb ? 576 : 128;
    cuuint64_t dim[3] = {N, (cuuint64_t)heads, (cuuint64_t)tokens};
    cuuint64_t stride[2] = {N * 2, (cuuint64_t)heads * N * 2};
    cuuint32_t box[3] = {64, 1, 32};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult cr = encode(&tmap_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dim, stride, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(PMLA_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", (int)cr);
  }
  cudaError_t e = pmla::launch_proj(p, absorb, tmap_a, tmap_w, tmap_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "projection kernel launch");
  return PMLA_OK;
}

int mla_absorb_query(const uint16_t* q_nope, const uint16_t* q_rope, const uint16_t* w_uk, int tokens,
                     int heads, uint16_t* q_out, void* stream) {
  return proj_call(q_nope, q_rope, w_uk, tokens, heads, q_out, stream, true);
}

int mla_project_output(const uint16_t* o_latent, const uint16_t* w_uv, int tokens, int heads,
                       uint16_t* o_out, void* stream) {
  return proj_call(o_latent, nullptr, w_uv, tokens, heads, o_out, stream, false);
}

int pmla_device_error(void) {
  int dev;
  DeviceInfo* info;
  int rc = device_setup(&dev, &info);
  if (rc) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceSynchronize");
  int v = 0, zero = 0;
  e = cudaMemcpy(&v, info->err_ptr, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e, "reading the device error word");
  e = cudaMemcpy(info->err_ptr, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail_cuda(e, "clearing the device error word");
  return v;
}

}  // extern "C"
