// Internal definitions shared by the kernels and the C-ABI layer.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace pmla {

constexpr int kPage = 64;       // tokens per page
constexpr int kD = 576;         // q/k width
constexpr int kDV = 512;        // value width
constexpr int kRows = 128;      // query rows per tile (the MMA's M)
constexpr int kMetaInts = 8;    // int32 per scheduler part
constexpr int kMaxParts = 2048; // scheduler parts one metadata kernel handles

// Fixed cost, in pages, that the scheduler charges every piece of a sequence:
// loading the 128x576 query tile (144 KB, two pages' worth of bytes), the
// epilogue drain of the 128x512 accumulator, and for split pieces the partial
// write and its re-read by the merge kernel.
constexpr int kPieceCostPages = 3;

// Share weights of scheduler parts (tile_scheduler_metadata column 5).  With
// two or more row groups per KV head the parts run on 4-CTA clusters of the
// pair variant, which leave some SMs free (148 - 4 x 33 = 16 on B200); those
// take 2-CTA clusters of the one-row-group variant, one per row group of a
// part.  Running beside the 4-CTA clusters they cover a part at about 0.84 of
// their rate per SM, so their parts get that share of the work (on causal2,
// per-cluster end times: weight 91 left them idle for the last ~50 us of
// ~365 us, 107 ends both kinds of cluster within ~2 us of each other).
constexpr int kPartWeightFull = 128;
constexpr int kPartWeightAux = 107;

// Device error codes written by bounded waits that time out (first one wins).
enum DeviceError : int {
  kErrNone = 0,
  kErrBadSmemAlign = 1,
  kErrBadPage = 2,
  kErrBadAppend = 3,   // an appended token lies past the sequence's block table
  kErrBadSeqlen = 4,   // cache_seqlens[b] > 64 * max_pages: the sequence is treated as empty
  kErrWaitBase = 100,  // + the id of the wait that gave up
};

struct DecodeParams {
  const uint16_t* q;            // [b][s_q][h_q][576]
  const int32_t* block_table;   // [b][max_pages]
  const int32_t* seqlens;       // [b]
  const int32_t* meta;          // [num_parts][8]
  const int32_t* num_splits;    // [b+1]
  uint16_t* o;                  // [b][s_q][h_q][512]
  float* lse;                   // [b][h_q][s_q]
  float* part_o;                // [slots][h_kv][R][512]
  float* part_lse;              // [slots][h_kv][R]
  int* seq_done;                // [b][h_kv][n_rg] completion signals of split pieces
  int* err;                     // device error word
  int batch, s_q, h_q, h_kv;
  int hpk;                      // h_q / h_kv
  int R;                        // s_q * hpk rows per KV head
  int n_rg;                     // ceil(R / 128) row groups
  int num_parts, max_pages, num_pages, causal;
  int part0;                    // first scheduler part of this launch
  int follows_decode;           // 1: launched after the call's other decode kernel (see the kernel)
  float scale_log2;             // softmax_scale * log2(e)
};

struct CombineParams {
  const int32_t* num_splits;
  const int32_t* seqlens;       // [b]: a sequence longer than its block table merges as empty
  const float* part_o;
  const float* part_lse;
  const int* seq_done;          // [b][h_kv][n_rg]: 2 signals per finished split piece
  int* err;                     // device error word
  uint16_t* o;
  float* lse;
  int batch, s_q, h_q, h_kv, hpk, R, n_rg, num_parts, max_pages;
};

struct AppendParams {
  const uint16_t* new_kv;       // [b][s_new][h_kv][576]
  const int32_t* block_table;   // [b][max_pages]
  const int32_t* seqlens;       // [b], lengths before the append
  uint16_t* kvcache;            // [num_pages][64][h_kv][576]
  int32_t* new_seqlens;         // [b] or null: seqlens + s_new
  int* err;                     // device error word
  int batch, s_new, h_kv, max_pages, num_pages;
};

struct ProjParams {
  const uint16_t* a;            // absorb: q^C [T][H][128]; project: o^lat [T][H][512]
  const uint16_t* rope;         // absorb: q^R [T][H][64] (copied to columns 512..575)
  const uint16_t* w;            // W^UK or W^UV [H][128][512]
  uint16_t* out;                // absorb: q [T][H][576]; project: o [T][H][128]
  int* err;                     // device error word
  int tokens, heads;
};

// Workspace layout of one decode call: split partials o (chunk-major fp32),
// their lse, and the per-(sequence, KV head, row group) completion counters the
// merge kernel waits on.  Returns the total size.
struct WorkspaceLayout {
  size_t lse_off, done_off, done_count, bytes;
};
WorkspaceLayout workspace_layout(int batch, int R, int h_kv, int num_parts);

// Host launchers (each returns the CUDA error of its launch).
// Parts [0, num_main) weigh kPartWeightFull, the others kPartWeightAux.
cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_parts, int num_main, int32_t* meta,
                            int32_t* num_splits, cudaStream_t stream);
cudaError_t decode_prepare(int device);  // one-time per-device kernel attributes
// Clusters of the decode kernel resident at once: 2-CTA clusters (pair = false,
// one per 128-row group) or 4-CTA clusters (pair = true, one per two row groups).
int decode_max_active_clusters(int device, bool pair, int* out);
// The 4-CTA variant is used when a KV head has two or more row groups.
inline bool decode_uses_pairs(int n_rg) { return n_rg >= 2; }
// Launches the clusters of parts [p.part0, p.part0 + parts).
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_kv, const CUtensorMap& tmap_q,
                          const CUtensorMap& tmap_v, const CUtensorMap& tmap_kv2, bool pair, int parts,
                          cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);
cudaError_t launch_clear_counters(int* ctr, int n, cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);
cudaError_t launch_proj(const ProjParams& p, bool absorb, const CUtensorMap& tmap_a, const CUtensorMap& tmap_w,
                        const CUtensorMap& tmap_out, cudaStream_t stream);
size_t decode_smem_bytes();

// Records the message pmla_last_error() returns on this host thread.
void set_last_error(const char* msg);

}  // namespace pmla
