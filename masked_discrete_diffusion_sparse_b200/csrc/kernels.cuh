// Device-side structures shared by the kernels of the sparse sampling step, the step-causal
// predicate, and the GEMM epilogues (applied to a staged 16-row x 128-feature fp32 tile).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ptx.cuh"

namespace smdm {

constexpr int kMaxBatch = 8;
constexpr int kTypePrompt = 0, kTypeClean = 1, kTypeMask = 2, kTypeReg = 3;

template <typename T> SMDM_DEV float to_f(T v);
template <> SMDM_DEV float to_f<float>(float v) { return v; }
template <> SMDM_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> SMDM_DEV T from_f(float v);
template <> SMDM_DEV float from_f<float>(float v) { return v; }
template <> SMDM_DEV __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Step-causal visibility (Sparse-LaViDa Sec. 3.3 / Appendix 7.3; Figure-3 example): clean rows
// (prompt = block 0, clean block = the step the token was decoded at) see clean rows of the same
// or an earlier block; mask and register rows of block s see clean rows of blocks < s and the
// mask/register rows of block s; clean rows never see mask or register rows.
SMDM_DEV bool step_causal_allowed(int tq, int lq, int tk, int lk) {
  const bool qc = (tq == kTypePrompt) || (tq == kTypeClean);
  const bool kc = (tk == kTypePrompt) || (tk == kTypeClean);
  if (kc) return qc ? (lk <= lq) : (lk < lq);
  if (qc) return false;
  return lq == lk;
}

// Per-row metadata of the current forward (device arrays of length max_rows).
struct Rows {
  int* ids;
  int* pos;
  int* type;
  int* label;
  int* seq;     // sequence slot of the row
  int* slot;    // index in that sequence's KV cache where the row's K/V are written
  int* kvlen;   // prefix-mode attention: the row sees keys [0, kvlen)
  int* qrow;    // logit row j -> forward row
  int* qpos;    // logit row j -> position
};

// KV cache addressing: element (seq, layer, head, slot, i) of K (or V) lives at
// base + seq*seq_stride + layer*layer_stride + head*head_stride + slot*d_head + i.
struct KVAddr {
  void* k;
  void* v;
  long long seq_stride;
  long long layer_stride;
  long long head_stride;
  int cap;    // slots per (seq, layer, head)
};

enum EpiKind : int { kEpiStore = 0, kEpiQKV = 1, kEpiResid = 2, kEpiSwiGLU = 3, kEpiLMHead = 4 };

struct EpiParams {
  int kind;
  int rows;       // valid activation rows
  int n_valid;    // valid output features (V for the LM head; ffn for SwiGLU; N otherwise)
  // kEpiStore: out[r][n]
  void* out;
  int ld_out;
  // kEpiQKV
  void* q_out;    // [rows][d]
  int d_model, d_head, layer;
  KVAddr kv;
  const int* row_seq;
  const int* row_slot;
  const int* row_pos;
  const float2* rope;   // [pos][d_head/2] (cos, sin)
  // kEpiResid: x[r][n] += acc (fp32 residual stream)
  float* x;
  int ld_x;
  // kEpiSwiGLU: act[r][f] = silu(gate) * up; tile = 64 gate rows then 64 up rows
  void* act;
  int ld_act;
  // kEpiLMHead
  float* logits;     // optional [rows][ld_logits]
  int ld_logits;
  float* pmax;       // [rows][n_vt]
  float* psum;
  int* parg;
  int n_vt;
};

SMDM_DEV float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Apply the epilogue to a staged tile S[16][128] (S[j][m] = accumulator for activation row
// r0 + j and output feature n0 + m; for SwiGLU m < 64 are gate rows f0 + m and m >= 64 the up
// rows f0 + m - 64 with f0 = n0 / 2).  Called by 128 threads; m = feature lane of this thread.
// atomic_resid: the tile is one of several K segments, so the residual add must be atomic.
template <typename T>
SMDM_DEV void epilogue_tile(const EpiParams& p, const float (*S)[128], int n0, int r0, int m,
                            bool atomic_resid) {
  const int nrows = min(16, p.rows - r0);
  if (nrows <= 0) return;
  switch (p.kind) {
    case kEpiStore: {
      const int n = n0 + m;
      if (n < p.n_valid) {
        T* o = reinterpret_cast<T*>(p.out);
        for (int j = 0; j < nrows; ++j) o[(size_t)(r0 + j) * p.ld_out + n] = from_f<T>(S[j][m]);
      }
      break;
    }
    case kEpiResid: {
      const int n = n0 + m;
      if (n < p.n_valid) {
        if (atomic_resid) {
          for (int j = 0; j < nrows; ++j) atomicAdd(&p.x[(size_t)(r0 + j) * p.ld_x + n], S[j][m]);
        } else {
          for (int j = 0; j < nrows; ++j) p.x[(size_t)(r0 + j) * p.ld_x + n] += S[j][m];
        }
      }
      break;
    }
    case kEpiSwiGLU: {
      // 128 threads: feature i = m & 63, rows split in two halves by m >> 6.
      const int i = m & 63;
      const int f = (n0 >> 1) + i;
      if (f < p.n_valid) {
        T* a = reinterpret_cast<T*>(p.act);
        const int jb = (m >> 6) * 8;
        for (int j = jb; j < min(jb + 8, nrows); ++j) {
          const float g = S[j][i], u = S[j][64 + i];
          a[(size_t)(r0 + j) * p.ld_act + f] = from_f<T>(silu_f(g) * u);
        }
      }
      break;
    }
    case kEpiQKV: {
      const int n = n0 + m;
      const int region = n / p.d_model;          // 0 = q, 1 = k, 2 = v
      const int nn = n - region * p.d_model;
      const int h = nn / p.d_head, i = nn % p.d_head;
      const int half = p.d_head >> 1;
      const int partner = (i < half) ? m + half : m - half;
      T* kc = reinterpret_cast<T*>(p.kv.k);
      T* vc = reinterpret_cast<T*>(p.kv.v);
      T* qo = reinterpret_cast<T*>(p.q_out);
      for (int j = 0; j < nrows; ++j) {
        const int r = r0 + j;
        float val = S[j][m];
        if (region < 2) {
          const float2 cs = p.rope[(size_t)p.row_pos[r] * half + (i % half)];
          const float other = S[j][partner];
          val = (i < half) ? (val * cs.x - other * cs.y) : (other * cs.y + val * cs.x);
        }
        if (region == 0) {
          qo[(size_t)r * p.d_model + nn] = from_f<T>(val);
        } else {
          const long long off = (long long)p.row_seq[r] * p.kv.seq_stride +
                                (long long)p.layer * p.kv.layer_stride +
                                (long long)h * p.kv.head_stride +
                                (long long)p.row_slot[r] * p.d_head + i;
          (region == 1 ? kc : vc)[off] = from_f<T>(val);
        }
      }
      break;
    }
    case kEpiLMHead: {
      // Optional logits; per (row, 128-wide vocab tile) max / first argmax / sum exp(l - max).
      const int n = n0 + m;
      if (p.logits && n < p.n_valid)
        for (int j = 0; j < nrows; ++j) p.logits[(size_t)(r0 + j) * p.ld_logits + n] = S[j][m];
      const int warp = m >> 5, lane = m & 31;
      const int vt = n0 >> 7;
      for (int j = warp * 4; j < min(warp * 4 + 4, nrows); ++j) {
        float best = -INFINITY;
        int arg = 0x7fffffff;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int f = lane + 32 * t;
          const float v = (n0 + f < p.n_valid) ? S[j][f] : -INFINITY;
          if (v > best) { best = v; arg = n0 + f; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, o);
          const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
          if (ob > best || (ob == best && oa < arg)) { best = ob; arg = oa; }
        }
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int f = lane + 32 * t;
          if (n0 + f < p.n_valid) s += __expf(S[j][f] - best);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) {
          const size_t idx = (size_t)(r0 + j) * p.n_vt + vt;
          p.pmax[idx] = best;
          p.parg[idx] = arg;
          p.psum[idx] = s;
        }
      }
      break;
    }
  }
}

}  // namespace smdm
