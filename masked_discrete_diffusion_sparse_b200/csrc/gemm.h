// Host-side interface of the GEMM kernels (see gemm.cu).
#pragma once
#include "kernels.cuh"

namespace smdm {

struct GemmCall {
  const CUtensorMap* tmA;   // weights [n_out][K] fp16, box {64, 128} (SwiGLU: gate, box {64, 64})
  const CUtensorMap* tmA2;  // SwiGLU: up weights, box {64, 64} (split layout)
                            // interleaved layout: tmA = 3-D map {d, 2 (gate/up), ffn}, box
                            // {64, 2, 64}: A-tile row 2i / 2i+1 = gate / up row f0 + i
  const CUtensorMap* tmB;   // activations [*][K] fp16, box {64, gemm_tc_box_rows(rows, pair, mrb)}
  const CUtensorMap* tmOut; // epilogue output, rows = `rows` (no swizzle), box {w, 32}:
                            //   store: out fp16 [rows][n_out], w 128;  QKV: q fp16 [rows][d], w 128;
                            //   SwiGLU: act fp16 [rows][ffn], w 64;  residual: x fp32 [rows][d],
                            //   w 128 (reduce-add);  LM head: logits fp32 [rows][V], w 128 (or any
                            //   valid map when no logits are written)
  int K;
  int n_out;                // output features (SwiGLU: ffn)
  int rows;                 // activation rows
  int row0;                 // first activation row in tmB
  int swiglu;               // 1: gate/up tiles with the SwiGLU epilogue
  int swiglu_il;            // SwiGLU: tmA is the interleaved gate/up map (tmA2 unused)
  int a_interleave;         // 0, or d_head: tmA is the rotary-interleaved 4-D/5-D QKV map
  int num_ctas;             // persistent grid size (one CTA per SM)
  int pair;                 // 1: one CTA per tile; 2: CTA pairs (M=256 MMAs, half the
                            // activation rows per CTA); gemm_tc_pair() picks it
  int max_stages;           // 0 = as many as fit
  int producers;            // TMA-issuing threads, 1 or 2 (0 = default)
  int sched;                // 0: whole tiles per CTA when the tile count is 40-100% of the grid,
                            // else stream-K; 1: whole tiles whenever they fit; 2: stream-K
  int min_row_blocks;       // gemm_tc_min_row_blocks(); the B map's box must match
  float* partial;           // split-K scratch: [num_ctas][2][128][row_tile rounded to 32] fp32
  size_t partial_bytes;
  unsigned* counters;       // [max_tiles], zero-initialised; restored to zero by the kernel
  int max_tiles;
  uint32_t* status;
  EpiParams epi;
};

// Activation rows per row block; min_blocks > 1 splits the rows into at least that many
// blocks (multiples of 32 rows).
int gemm_tc_row_tile(int rows, int min_blocks = 1);
int gemm_tc_box_rows(int rows, int pair, int min_blocks = 1);
// Row blocks to ask for: 2 for an LM head whose tiles would occupy at most half of the SMs
// (its epilogue, not its weights, sets its time there), else 1.
int gemm_tc_min_row_blocks(int n_out, int rows, int epi_kind, int sms);
// CTA-pair mode (2) or single-CTA mode (1) for a tensor-core GEMM of this shape.
int gemm_tc_pair(int n_out, int swiglu, int rows, int epi_kind);
cudaError_t gemm_tc_set_smem_attr();
cudaError_t launch_gemm_tc(const GemmCall& c, cudaStream_t stream);
cudaError_t launch_gemm_simt(const float* W, const float* W2, const float* X, int ldx, int K,
                             int n_out, int rows, int swiglu, const EpiParams& ep,
                             cudaStream_t stream);

}  // namespace smdm
