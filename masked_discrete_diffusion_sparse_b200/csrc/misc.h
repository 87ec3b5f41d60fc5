// Host-side interface of the pack / norm / unmask kernels (see misc.cu).
#pragma once
#include "kernels.cuh"

namespace smdm {

struct PackSeq {
  int seq;          // sequence slot
  int row0;         // first forward row of this sequence
  int n_new, n_q, n_reg;
  int ctx;          // cache length before this step
  int P, Lg;
  int label;        // step number k
  int qbase;        // first logit row of this sequence
  int block_lo, block_hi;   // block mode (qpos == nullptr)
  const int* qpos;  // explicit decode set or nullptr
  const int* grid;  // [Lg]
  const int* newpos;// [n_new] positions decoded at the previous step
};

struct PackArgs {
  int n_seq;
  PackSeq s[kMaxBatch];
  int vocab;
  int len_token;    // 1: the one tail row is [LEN] (id vocab+1) instead of REG_0 (vocab+2)
  Rows rows;
  uint32_t* status;
};

enum { kPackPrefill = 0, kPackDense = 1, kPackTrain = 2, kPackPrefillGiven = 3 };

// One sampling step of one sequence under the speed switches of the Table-6 ablation (cache the
// prompt, cache decoded tokens, truncate the other masks).  Cache slots: the prompt at
// [0, P), decoded tokens in decode order from P on, then this step's masks and tail rows.
// Rows, in label order: recomputed prompt (!cache_prompt), decoded tokens (the new-cache rows,
// or with !cache_res every decoded token), the decode set C, the other masks (!truncate), the
// tail rows.  Every row sees a key prefix of that layout.
struct PackSwArgs {
  int seq, P, Lg;
  int label;         // step number k
  int vocab, n_tail, len_token;
  int cache_prompt, cache_res, truncate;
  int n_new;         // tokens committed at step k-1 (this step's new-cache rows)
  int dec_prev;      // tokens decoded before step k-1
  int n_q, n_extra;  // decode set; other still-masked positions (!truncate)
  const int* qpos;   // [n_q] decode set positions
  const int* newpos; // [n_new]
  const int* prompt; // [P]
  const int* grid;   // [Lg]
  int* dec_pos;      // [Lg] decoded positions in decode order (appended here)
  int* dec_lab;      // [Lg] the step each was decoded at
  int* qmark;        // [Lg] the last step that queried the position (0 = never)
  Rows rows;
  uint32_t* status;
};

struct LinearPackArgs {
  int mode;
  int n;            // rows
  int seq;
  int P;
  int Lg;           // prefill with given tokens: generation length
  int vocab, emb_rows, max_pos;
  const int* prompt;    // prefill / dense
  const int* grid;      // dense
  const int* given_pos; // prefill with given generation tokens: rows P.. are these
  const int* given_tok;
  int* grid_out;        // ... and their tokens are written into this grid
  const int* ids;       // training form
  const int* pos;
  const int* type;
  const int* label;
  Rows rows;
  uint32_t* status;
};

struct NormArgs {
  float* x;           // fp32 residual rows [*][d]
  const void* gain;   // [d], weight dtype
  void* out;          // [rows][d], activation dtype
  const int* gather;  // optional: out row r normalises x row gather[r]
  const void* emb;    // optional: x[src] = emb[ids[src]] first
  const int* ids;
  int d;
  float eps;
};

struct UnmaskSeq {
  int qbase, n_q;     // this sequence's decode-set rows: qbase .. qbase + n_q - 1
  int lbase;          // first LM-head row of this sequence
  int dense;          // LM-head row of decode row j = qpos - P - 1 (dense comparator)
  int policy, n_commit;
  int P, Lg;
  int* grid;
  int* newpos;        // committed positions in row order (next step's new-cache rows)
};

struct UnmaskArgs {
  int n_seq;
  UnmaskSeq s[kMaxBatch];
  int n_vt;           // vocab tiles of 128
  const float* pmax;
  const float* psum;
  const int* parg;
  const int* qpos_of; // decode row -> position
  int* tok_out;       // optional
  float* conf_out;    // optional
  uint32_t* status;
};


cudaError_t launch_pack_step(const PackArgs& a, cudaStream_t st);
cudaError_t launch_pack_linear(const LinearPackArgs& a, cudaStream_t st);
cudaError_t launch_pack_switched(const PackSwArgs& a, cudaStream_t st);
// fp16 copy of a bf16 tensor of n elements (kStatusRange in *status for a value beyond 65504).
cudaError_t launch_convert_bf16_f16(const __nv_bfloat16* src, __half* dst, size_t n,
                                    uint32_t* status, cudaStream_t st);
cudaError_t launch_gather_rows(const int* src, int n, int n_fwd, int* qrow, uint32_t* status,
                               cudaStream_t st);
// Training form: per-row key bounds of the step-causal rule into kvlen (see misc.cu);
// scratch: 3 * (n + 1) + 1 ints.
cudaError_t launch_label_bounds(const int* type, const int* label, int n, int* scratch,
                                int* kvlen, cudaStream_t st);
// Training form: per 128-row query tile, the key tiles that may hold a visible key (see
// misc.cu).  scratch: 5 * T + T * T ints, T = ceil(n / 128); returns the list and count arrays.
cudaError_t launch_tile_lists(const int* type, const int* label, int n, int* scratch,
                              int** lists, int** counts, cudaStream_t st);
// T: the gain / embedding dtype (bf16 or fp32); OutT: the output dtype (fp16 for bf16 models).
template <typename T, typename OutT>
cudaError_t launch_rmsnorm(const NormArgs& a, int rows, cudaStream_t st);
cudaError_t launch_unmask(const UnmaskArgs& a, int max_nq, cudaStream_t st);
cudaError_t launch_debug_mask(const int* type, const int* label, int n, uint32_t* bitmap,
                              cudaStream_t st);
cudaError_t launch_fill_i32(int* p, int n, int v, cudaStream_t st);

}  // namespace smdm
