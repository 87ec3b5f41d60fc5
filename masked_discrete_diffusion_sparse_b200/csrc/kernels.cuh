// Device-side structures shared by the kernels of the sparse sampling step, the step-causal
// predicate, the launch helper (programmatic dependent launch) and the GEMM epilogues (a staged
// 16-row tile for the fp32 SIMT GEMM; 32-row TMEM blocks written with TMA copies for tcgen05).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <utility>

#include "ptx.cuh"

namespace smdm {

// Launch `kern` with programmatic stream serialization (and a cluster of cluster_x CTAs when
// > 1).  Every kernel launched this way calls griddep_wait() before it touches data that an
// earlier kernel produces or consumes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

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
  // kEpiSwiGLU: act[r][f] = silu(gate) * up; tile = 64 gate rows then 64 up rows, or with
  // swiglu_il the gate and up rows of feature f0 + i on lanes 2i and 2i + 1 (swapped when
  // swiglu_up_first)
  void* act;
  int ld_act;
  int swiglu_il, swiglu_up_first;
  // kEpiLMHead
  float* logits;     // optional [rows][ld_logits]
  int ld_logits;
  float* pmax;       // [rows][n_vt]
  float* psum;
  int* parg;
  int n_vt;
};

// silu(g) = g * sigmoid(g) with the fast division (a full-precision division takes a slow
// software path)
SMDM_DEV float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

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
        float* __restrict__ x = p.x + (size_t)r0 * p.ld_x + n;
        if (atomic_resid) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nrows) atomicAdd(x + (size_t)j * p.ld_x, S[j][m]);
        } else {
          // all loads first, then all stores: the rows are independent
          float old[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) old[j] = (j < nrows) ? x[(size_t)j * p.ld_x] : 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nrows) x[(size_t)j * p.ld_x] = old[j] + S[j][m];
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
      T* __restrict__ kc = reinterpret_cast<T*>(p.kv.k);
      T* __restrict__ vc = reinterpret_cast<T*>(p.kv.v);
      T* __restrict__ qo = reinterpret_cast<T*>(p.q_out);
      // metadata for the 16 rows first (independent loads), then the rotary table, then stores
      int pos[16], seq[16], slot[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = r0 + min(j, nrows - 1);
        pos[j] = __ldg(p.row_pos + r);
        seq[j] = __ldg(p.row_seq + r);
        slot[j] = __ldg(p.row_slot + r);
      }
      float val[16];
      if (region < 2) {
        float2 cs[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) cs[j] = __ldg(p.rope + (size_t)pos[j] * half + (i % half));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float a = S[j][m], b = S[j][partner];
          val[j] = (i < half) ? (a * cs[j].x - b * cs[j].y) : (b * cs[j].y + a * cs[j].x);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) val[j] = S[j][m];
      }
      if (region == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < nrows) qo[(size_t)(r0 + j) * p.d_model + nn] = from_f<T>(val[j]);
      } else {
        T* __restrict__ base = (region == 1 ? kc : vc) + (long long)p.layer * p.kv.layer_stride +
                               (long long)h * p.kv.head_stride + i;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < nrows)
            base[(long long)seq[j] * p.kv.seq_stride + (long long)slot[j] * p.d_head] =
                from_f<T>(val[j]);
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

// ------------------------------------------------------------------------------------------
// Epilogue of the tcgen05 GEMM: TMEM lane m holds A-tile row m (an output feature) and TMEM
// columns are activation rows.
//   - QKV tiles are loaded with rotary partners interleaved (A-tile row 2i <- weight row i of
//     the first half of a head, row 2i + 1 <- row i of the second half), so the rotation needs
//     only a lane exchange with lane m ^ 1.
//   - meta_pos / meta_kv: per-row position and K/V cache offset of the tile's rows (shared
//     memory, filled once per tile), indexed by row - meta_r0.
// ------------------------------------------------------------------------------------------
SMDM_DEV int qkv_lane_feature(int m, int d_head) {
  if (d_head == 128) return (m & 1) * 64 + (m >> 1);
  return (m >> 6) * 64 + (m & 1) * 32 + ((m >> 1) & 31);     // d_head == 64
}

// Epilogue of one block of 32 activation rows, written out through shared memory with TMA
// stores (one copy per block instead of hundreds of per-thread stores).  v[j]: accumulator of
// activation row r0 + j for A-tile row m (TMEM lane m).  buf: the block's 16 KB staging buffer;
// callers alternate two, and since et == 0 waits for its earlier copies to finish reading
// shared memory before the block's barrier, a buffer is free again two blocks later.  All 128
// epilogue threads call this (et = 0..127); et == 0 issues the copies.  tm_out: the call's
// output tensor map (fp16 out / q / act boxes of 32 rows, fp32 x / logits boxes of 32 rows);
// K/V cache rows of QKV tiles go out as 16-byte stores of all epilogue threads.
// Output rows at or beyond the map's row count are clipped by the TMA unit.
template <typename T>
SMDM_DEV void epilogue_block(const EpiParams& p, const CUtensorMap* tm_out, float* v, uint8_t* buf,
                             int n0, int r0, int m, int et, int nrows, const int* meta_pos,
                             const long long* meta_kv, int meta_r0) {
  auto publish = [&]() {   // staged data visible to the async proxy; earlier copies done reading
    fence_proxy_async_smem();
    if (et == 0) bulk_wait_read<0>();
    named_bar_sync(1, 128);
  };
  switch (p.kind) {
    case kEpiQKV: {
      const int dh = p.d_head, half = dh >> 1;
      const int f = qkv_lane_feature(m, dh);
      const int region = n0 / p.d_model;
      const int nn0 = n0 - region * p.d_model;
      if (region < 2) {
        const int ih = (f % dh) % half;
        const bool second = (m & 1) != 0;
        // all 32 rows' (cos, sin) requested before any is used: one memory round trip per
        // block instead of one per few rows
        float2 cs[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int jj = min(j, nrows - 1);
          cs[j] = __ldg(p.rope + (size_t)meta_pos[r0 + jj - meta_r0] * half + ih);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = v[j];
          const float b = __shfl_xor_sync(0xffffffffu, a, 1);
          v[j] = second ? (b * cs[j].y + a * cs[j].x) : (a * cs[j].x - b * cs[j].y);
        }
      }
      // q: [32 rows][128 features]; k / v: [head within the tile][32 rows][d_head].  The
      // attention operands are fp16 (3 more mantissa bits than bf16; the attention's MMAs take
      // both of their operands in fp16)
      __half* Sb = reinterpret_cast<__half*>(buf);
      const int hh = f / dh;
      __half* dst = (region == 0) ? Sb + f : Sb + hh * 32 * dh + (f - hh * dh);
      const int stride = (region == 0) ? 128 : dh;
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[j * stride] = __float2half_rn(v[j]);
      publish();
      if (region == 0) {
        if (et == 0) {
          tma_store_2d(tm_out, Sb, nn0, r0);
          bulk_commit();
        }
      } else {
        // K / V rows go to their cache slots, which follow the positions (scattered at a
        // sampling step): 16-byte stores by all 128 threads, two rows per warp instruction.
        // (One bulk copy per row issued by a single thread serialised the block.)  The staging
        // buffer is read synchronously here, so it is free again two blocks later as well.
        const long long base = (long long)p.layer * p.kv.layer_stride +
                               (long long)(nn0 / dh) * p.kv.head_stride;
        __half* cache = reinterpret_cast<__half*>(region == 1 ? p.kv.k : p.kv.v) + base;
        const int cpr = dh / 8;                  // 16-byte chunks per row of one head
        const int per_head = nrows * cpr;
        const int total = (128 / dh) * per_head;
        for (int i = et; i < total; i += 128) {
          const int hh2 = i / per_head, rem = i - hh2 * per_head;
          const int rr = rem / cpr, c = rem - rr * cpr;
          const long long o0 = meta_kv[r0 + rr - meta_r0];
          const uint4 v4 = *reinterpret_cast<const uint4*>(Sb + (hh2 * 32 + rr) * dh + c * 8);
          *reinterpret_cast<uint4*>(cache + (long long)hh2 * p.kv.head_stride + o0 + c * 8) = v4;
        }
      }
      break;
    }
    case kEpiStore: {
      __half* Sb = reinterpret_cast<__half*>(buf);
#pragma unroll
      for (int j = 0; j < 32; ++j) Sb[j * 128 + m] = __float2half_rn(v[j]);
      publish();
      if (et == 0) {
        tma_store_2d(tm_out, Sb, n0, r0);
        bulk_commit();
      }
      break;
    }
    case kEpiResid: {
      float* S = reinterpret_cast<float*>(buf);
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j * 128 + m] = v[j];
      publish();
      if (et == 0) {
        tma_reduce_add_2d(tm_out, S, n0, r0);   // x += block (fp32, element-wise atomic)
        bulk_commit();
      }
      break;
    }
    case kEpiSwiGLU: {
      if (p.swiglu_il) {
        // the partner lane m ^ 1 holds the other half of the pair; lane parity picks the rows
        // (even lanes even rows) so that the work splits evenly, with no shared-memory exchange
        __half* Ob = reinterpret_cast<__half*>(buf);   // [32][64] fp16
        const int i = m >> 1, h = m & 1;
        const bool mine_is_gate = (h == (p.swiglu_up_first ? 1 : 0));
#pragma unroll
        for (int j = 0; j < 32; j += 2) {   // even lanes take row j, odd lanes row j + 1
          const float o0 = __shfl_xor_sync(0xffffffffu, v[j], 1);
          const float o1 = __shfl_xor_sync(0xffffffffu, v[j + 1], 1);
          const float mine = h ? v[j + 1] : v[j];
          const float other = h ? o1 : o0;
          const float gate = mine_is_gate ? mine : other;
          const float up = mine_is_gate ? other : mine;
          Ob[(j + h) * 64 + i] = __float2half_rn(silu_f(gate) * up);
        }
        publish();
        if (et == 0) {
          tma_store_2d(tm_out, Ob, n0 >> 1, r0);
          bulk_commit();
        }
        break;
      }
      // lanes 0..63: gate rows f0 + m; lanes 64..127: up rows f0 + m - 64 (f0 = n0 / 2)
      float* U = reinterpret_cast<float*>(buf);                               // [32][64] fp32
      __half* Ob = reinterpret_cast<__half*>(buf + 32 * 64 * 4);  // [32][64] fp16
      if (m >= 64) {
#pragma unroll
        for (int j = 0; j < 32; ++j) U[j * 64 + (m - 64)] = v[j];
      }
      named_bar_sync(1, 128);
      if (m < 64) {
#pragma unroll
        for (int j = 0; j < 32; ++j) Ob[j * 64 + m] = __float2half_rn(silu_f(v[j]) * U[j * 64 + m]);
      }
      publish();
      if (et == 0) {
        tma_store_2d(tm_out, Ob, n0 >> 1, r0);
        bulk_commit();
      }
      break;
    }
    case kEpiLMHead: {
      float* S = reinterpret_cast<float*>(buf);
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j * 128 + m] = v[j];
      publish();
      if (p.logits && et == 0) {
        tma_store_2d(tm_out, S, n0, r0);
        bulk_commit();
      }
      // Per row: max, first argmax and sum exp(l - max) over the tile's 128 columns.  Four
      // threads per row (et >> 2 = row, et & 3 = a quarter of 32 columns), each walking its
      // columns in an order rotated by et so that the 32 lanes of a warp read 32 different
      // banks.  Three passes (the row maximum, the lowest column holding it, the sum), each a
      // short loop of four independent chains: compact code, no 32-long dependent chain.
      const int vt = n0 >> 7;
      const int j = et >> 2, qq = et & 3;
      const float* Srow = S + j * 128 + qq * 32;
      const int col0 = n0 + qq * 32;
      const int nv = min(32, max(0, p.n_valid - col0));   // valid columns of this quarter
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
      for (int c0 = 0; c0 < 32; c0 += 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int cc = (c0 + i + et) & 31;
          if (cc < nv) m4[i & 3] = fmaxf(m4[i & 3], Srow[cc]);
        }
      }
      float best = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
      int a4[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int c0 = 0; c0 < 32; c0 += 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int cc = (c0 + i + et) & 31;
          if (cc < nv) {
            const float x = Srow[cc];
            if (x == best) a4[i & 3] = min(a4[i & 3], col0 + cc);
            s4[i & 3] += __expf(x - best);
          }
        }
      }
      int arg = min(min(a4[0], a4[1]), min(a4[2], a4[3]));
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) arg = min(arg, __shfl_xor_sync(0xffffffffu, arg, o));
      float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (qq == 0 && j < nrows) {
        const size_t idx = (size_t)(r0 + j) * p.n_vt + vt;
        p.pmax[idx] = best;
        p.parg[idx] = arg;
        p.psum[idx] = sum;
      }
      break;
    }
  }
}

}  // namespace smdm
