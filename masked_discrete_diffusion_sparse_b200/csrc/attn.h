// Host-side interface of the attention kernels (see attn.cu).
#pragma once
#include "kernels.cuh"

namespace smdm {

// A contiguous run of query rows that belong to one sequence.
struct AttnSeg {
  int seq;      // sequence slot (selects the KV cache)
  int row0;     // first forward row
  int rows;     // number of rows
  int nkeys;    // keys to scan: max kvlen over the rows (prefix mode) or n (label mode)
  int tile0;    // filled in by the launcher
};

struct AttnCall {
  int mode;                 // 0 = prefix (kvlen per row), 1 = label (step-causal predicate)
  int bound;                // label mode: kvlen[row] bounds the row's keys, and each 128-row
                            // query tile scans only the key tiles listed for it
  const int* tile_list;     // [query tile][n_ktiles] key tiles (ascending), bounded mode
  const int* tile_count;    // [query tile] number of listed key tiles
  int n_ktiles;
  int H, dh, d_model, layer;
  int n_seg;
  AttnSeg seg[kMaxBatch];
  const int* kvlen;
  const int* type;
  const int* label;
  // 3-D head-tile maps {64, rows, row elements / 64}, box {64, 128, d_head / 64} (one copy per
  // 128-row tile):
  const CUtensorMap* tmQ;   // q [rows][d_model] fp16 (chunk coordinate = head * d_head / 64)
  const CUtensorMap* tmK;   // K cache [cache rows][d_head] fp16
  const CUtensorMap* tmV;   // V cache, same layout
  long long cache_rows_per_seq;
  int cap;
  void* out;                // [rows][d_model] fp16
  uint32_t* status;
  // split-KV: partial results of `nsplit` key ranges, merged by a combine kernel
  float* part_o;            // [nsplit][rows][d_model] fp32 (unnormalised)
  float* part_ml;           // [nsplit][rows][H][2] (reference max in the exp2 domain, sum)
  size_t part_bytes;        // capacity of part_o + part_ml
  int num_sms;
  int rows_total;
};

struct AttnSimtArgs {
  int mode;
  int rows, H, dh, d_model, layer;
  int nkeys;                // label mode
  const int* row_seq;
  const int* kvlen;
  const int* type;
  const int* label;
  float scale;              // 1/sqrt(dh)
};

cudaError_t attn_tc_set_smem_attr();
// Number of key splits the launcher will use for this call (1 = no combine pass).
int attn_tc_splits(const AttnCall& c);
cudaError_t launch_attn_tc(const AttnCall& c, cudaStream_t stream);
template <typename T>
cudaError_t launch_attn_simt(const T* q, T* out, const KVAddr& kv, const AttnSimtArgs& a,
                             cudaStream_t stream);

}  // namespace smdm
