// C ABI of the sparse sampling library: handle, workspace carving, TMA descriptors and the
// forward driver that chains the kernels of one step (pack -> [QKV+RoPE+KV append ->
// step-causal attention -> O-proj+residual -> RMSNorm -> gate/up+SwiGLU -> down+residual ->
// RMSNorm] x layers -> LM head over the decode set -> unmask), plus the switched step, the
// training form and the allocation-free entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "attn.h"
#include "gemm.h"
#include "misc.h"
#include "smdm.h"

using namespace smdm;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D fp16 tensor map: `inner` contiguous elements per row, `outer` rows, 128-byte swizzle (the
// GEMMs' operands: the fp16 weight copies and the fp16 activations).
bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Interleaved gate/up view for the SwiGLU GEMM's A tiles: one 3-D map {d, 2, ffn} over both
// weight tensors (the second dimension steps from the lower of the two base addresses to the
// higher), box {64, 2, 64}, so that a 16 KB tile holds gate row f0 + i and up row f0 + i on
// adjacent rows 2i, 2i + 1.  Returns 0 when the address gap is unusable as a TMA stride (then
// the two-box layout is used), 1 when gate comes first, 2 when up comes first.
int encode_gateup_interleaved(CUtensorMap* m, const void* gate, const void* up, uint64_t d,
                              uint64_t f) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return 0;
  const uintptr_t g = reinterpret_cast<uintptr_t>(gate), u = reinterpret_cast<uintptr_t>(up);
  const bool up_first = u < g;
  const uint64_t delta = up_first ? g - u : u - g;
  if (delta == 0 || delta % 16 || delta >= (1ull << 40)) return 0;
  cuuint64_t dims[3] = {d, 2, f};
  cuuint64_t strides[2] = {delta, d * 2};
  cuuint32_t box[3] = {64, 2, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void*>(up_first ? up : gate), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return 0;
  return up_first ? 2 : 1;
}

// Head-tile view for the attention kernel (q, K and V are fp16): rows of `row_elems` split into
// 64-element
// (128-byte) chunks, dims {64, rows, row_elems / 64}, box {64, 128, nsub}: one copy brings a
// 128-row tile of nsub chunks, landing as nsub swizzled [128][64] sub-tiles.
bool encode_head_tiles(CUtensorMap* m, const void* base, uint64_t row_elems, uint64_t rows,
                       uint32_t nsub) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || row_elems % 64) return false;
  cuuint64_t dims[3] = {64, rows, row_elems / 64};
  cuuint64_t strides[2] = {row_elems * 2, 128};
  cuuint32_t box[3] = {64, 128, nsub};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D output map for the GEMM epilogue's TMA stores: `cols` x `rows` elements (fp32 or fp16),
// row pitch `ld` elements, box {box_cols, 32}, no swizzle.
bool encode_out(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols,
                uint64_t rows, uint64_t ld, uint32_t box_cols) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || !base || rows == 0) return false;
  const bool f32 = dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {box_cols, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Rotary-interleaved view of W_qkv [3d][d] for the GEMM's A tiles: a 128-row tile is loaded so
// that A-tile row 2i holds weight row i of the first half of a head and row 2i + 1 the matching
// row of the second half (the RoPE partner), putting the two on adjacent TMEM lanes.
//   d_head 128: dims {d, 2 (half, 64 rows), 64 (i, 1 row), 3d/128 (tile, 128 rows)}
//   d_head  64: dims {d, 2 (half, 32 rows), 32 (i, 1 row), 2 (head in tile, 64 rows), tiles}
bool encode_qkv_interleaved(CUtensorMap* m, const void* w, uint64_t d, int d_head) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const uint64_t rb = d * 2;   // bytes per weight row
  const uint64_t tiles = 3 * d / 128;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r;
  if (d_head == 128) {
    cuuint64_t dims[4] = {d, 2, 64, tiles};
    cuuint64_t strides[3] = {64 * rb, rb, 128 * rb};
    cuuint32_t box[4] = {64, 2, 64, 1};
    r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(w), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    cuuint64_t dims[5] = {d, 2, 32, 2, tiles};
    cuuint64_t strides[4] = {32 * rb, rb, 64 * rb, 128 * rb};
    cuuint32_t box[5] = {64, 2, 32, 2, 1};
    r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(w), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  size_t w16, w16_layer, w16_qkv, w16_o, w16_gu, w16_down, w16_lm;   // fp16 weight copies
  size_t kc, vc, kscr, vscr, x, h, q, ao, act, hq, pmax, psum, parg, rows, rope, partial,
      counters, status, newpos, prompts, aux, attn_part, lbound, tlist, sw, total;
  size_t attn_part_bytes;
  int cap, max_pos, n_vt, rt_max, max_tiles, n_sms;
  size_t partial_bytes;
};

// Rows that close every sampling step: n_reg registers, or with n_reg == SMDM_REG_LEN a single
// [LEN] row (the length-token variant, no registers).
int tail_rows(const smdm_config* c) { return c->n_reg == SMDM_REG_LEN ? 1 : c->n_reg; }
// Embedding rows: content ids, [MASK], [LEN] and the registers.
int emb_rows(const smdm_config* c) { return c->vocab + 2 + std::max(c->n_reg, 0); }

bool config_ok(const smdm_config* c, std::string* why) {
  auto fail = [&](const char* s) {
    if (why) *why = s;
    return false;
  };
  if (!c) return fail("null config");
  if (c->n_layers < 1 || c->d_model < 1 || c->n_heads < 1 || c->d_head < 1 || c->d_ffn < 1 ||
      c->vocab < 1 || c->n_reg < SMDM_REG_LEN)
    return fail("non-positive model dimension");
  if (c->n_heads * c->d_head != c->d_model) return fail("n_heads * d_head != d_model");
  if (c->d_head % 2) return fail("d_head must be even (rotary pairs)");
  if (c->d_model > 8192) return fail("d_model > 8192 is not supported");
  if (c->max_batch < 1 || c->max_batch > SMDM_MAX_BATCH) return fail("max_batch out of range");
  if (c->max_len < 1 || c->max_step_rows < 1 || c->max_rows < 1) return fail("bad capacity");
  // positions, cache slots and row indices are 32-bit on the device
  if ((long long)c->max_len + c->max_step_rows + tail_rows(c) + 8 > (1LL << 30) ||
      c->max_rows > (1 << 24) || c->n_reg > (1 << 16))
    return fail("capacity too large");
  if (c->dtype == SMDM_BF16) {
    if (c->d_model % 128) return fail("bf16 models need d_model % 128 == 0");
    if (c->d_head != 64 && c->d_head != 128) return fail("bf16 models need d_head 64 or 128");
    if (c->d_ffn % 64) return fail("bf16 models need d_ffn % 64 == 0");
    if (c->vocab % 4) return fail("bf16 models need vocab % 4 == 0");
  } else if (c->dtype == SMDM_F32) {
    if (c->d_head % 32 || c->d_head > 128) return fail("fp32 models need d_head % 32 == 0, <= 128");
  } else {
    return fail("unknown dtype");
  }
  return true;
}

int query_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// extras: the buffers of sampling sequences (KV caches, new-cache lists, prompt copies,
// switched-step lists); the allocation-free training form needs none of them and lays its
// scratch out with extras = false.
Layout make_layout(const smdm_config* c, int n_sms, bool extras = true) {
  Layout L{};
  const size_t es = c->dtype == SMDM_BF16 ? 2 : 4;
  const size_t d = c->d_model, H = c->n_heads, dh = c->d_head;
  L.cap = (int)align_up((size_t)c->max_len + c->max_step_rows, 8);
  L.max_pos = c->max_len + tail_rows(c) + 2;
  L.n_vt = (c->vocab + 127) / 128;
  L.n_sms = n_sms;
  const size_t MR = align_up((size_t)c->max_rows, 256);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  // bf16 models: fp16 copies of every weight matrix, per layer [qkv 3d x d | o d x d |
  // gate ffn x d | up ffn x d | down d x ffn], then the LM head [V][d]
  if (c->dtype == SMDM_BF16) {
    const size_t f = c->d_ffn;
    L.w16_qkv = 0;
    L.w16_o = 3 * d * d * 2;
    L.w16_gu = L.w16_o + d * d * 2;
    L.w16_down = L.w16_gu + 2 * f * d * 2;
    L.w16_layer = align_up(L.w16_down + d * f * 2, 1024);
    L.w16_lm = L.w16_layer * c->n_layers;
    L.w16 = take(L.w16_lm + (size_t)c->vocab * d * 2);
  }
  const size_t cache_elems = extras ? (size_t)c->max_batch * c->n_layers * H * L.cap * dh : 0;
  L.kc = take(cache_elems * es);
  L.vc = take(cache_elems * es);
  L.kscr = take(H * MR * dh * es);
  L.vscr = take(H * MR * dh * es);
  L.x = take(MR * d * 4);
  L.h = take(MR * d * es);
  L.q = take(MR * d * es);
  L.ao = take(MR * d * es);
  L.act = take(MR * c->d_ffn * es);
  L.hq = take(MR * d * es);
  L.pmax = take(MR * L.n_vt * 4);
  L.psum = take(MR * L.n_vt * 4);
  L.parg = take(MR * L.n_vt * 4);
  L.rows = take(9 * MR * 4);
  L.aux = take(9 * MR * 4);
  L.rope = take((size_t)L.max_pos * (dh / 2) * 8);
  L.rt_max = c->max_rows > 256 ? 512 : (int)align_up(c->max_rows, 32);
  L.partial_bytes = (size_t)n_sms * 2 * L.rt_max * 128 * 4;
  L.partial = take(L.partial_bytes);
  int max_nt = 3 * c->d_model / 128 + 1;
  max_nt = std::max(max_nt, c->d_ffn / 64 + 1);
  max_nt = std::max(max_nt, (c->vocab + 127) / 128);
  const int rb = c->max_rows > 512 ? (c->max_rows + 255) / 256 : 2;   // (2: the split LM head)
  L.max_tiles = max_nt * rb;
  L.counters = take((size_t)L.max_tiles * 4);
  L.status = take(256);
  L.newpos = take(extras ? (size_t)c->max_batch * c->max_step_rows * 4 : 0);
  L.prompts = take(extras ? (size_t)c->max_batch * c->max_len * 4 : 0);
  // split-KV partials for up to 16 key splits of a sampling step's rows
  const size_t step_rows = std::min((size_t)c->max_rows, (size_t)c->max_batch * c->max_step_rows);
  L.attn_part_bytes = 16 * step_rows * ((size_t)d * 4 + H * 8);
  L.attn_part = take(L.attn_part_bytes);
  // training form with key bounds: per-label last indices, their prefix maximum, a flag
  L.lbound = take((3 * (MR + 1) + 1) * 4);
  {
    const size_t T = MR / 128;   // query / key tiles of a training-form forward
    L.tlist = take((5 * T + T * T) * 4);
  }
  // switched steps: per sequence, decoded positions, their steps and the query marks
  L.sw = take(extras ? (size_t)c->max_batch * 3 * c->max_len * 4 : 0);
  L.total = off + 1024;
  return L;
}

struct SeqState {
  bool active = false;
  bool dense = false;
  int P = 0, Lg = 0;
  int n0 = 0;      // block-0 rows (prompt and given tokens)
  int ctx = 0;     // KV cache length (prompt + cached clean tokens)
  int n_new = 0;   // tokens committed at the previous step
  int k = 0;       // steps taken
  int sw = -1;     // switches of smdm_step_switched (fixed at its first step), -1 = not used
  int dec = 0;     // switched steps: tokens decoded before the previous step
  int32_t* grid = nullptr;
};

}  // namespace

struct Profiler {
  bool on = false, timed = false;
  unsigned long long launches = 0;
  unsigned long long class_launches[SMDM_K_CLASSES] = {};
  std::vector<cudaEvent_t> ev;   // pairs
  std::vector<int> cls;
  size_t used = 0;
};

struct smdm_handle {
  smdm_config cfg;
  Profiler prof;
  Layout L;
  bool bf16;
  const void* emb;
  const void* final_norm;
  const void* lm_head;
  std::vector<const void*> attn_norm, w_qkv, w_o, mlp_norm, w_gate, w_up, w_down;
  uint8_t* ws;
  Rows rows, aux;
  std::vector<CUtensorMap> tm_qkv, tm_o, tm_gate, tm_up, tm_down, tm_gu;
  std::vector<int> gu_il;   // per layer: 0 two-box gate/up tiles, 1/2 interleaved (tm_gu)
  CUtensorMap tm_lm, tm_kc, tm_vc, tm_kscr, tm_vscr, tm_q;
  std::string err;
  SeqState seq[SMDM_MAX_BATCH];
  int last_rows = 0;

  template <typename P> P* at(size_t off) { return reinterpret_cast<P*>(ws + off); }
  uint32_t* status() { return at<uint32_t>(L.status); }
  int* newpos(int s) { return at<int>(L.newpos) + (size_t)s * cfg.max_step_rows; }
  int* prompt(int s) { return at<int>(L.prompts) + (size_t)s * cfg.max_len; }
  int* sw_arrays(int s) { return at<int>(L.sw) + (size_t)s * 3 * cfg.max_len; }
  size_t es() const { return bf16 ? 2 : 4; }
};

namespace {

smdm_status fail(smdm_handle* h, smdm_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  return st;
}

#define CK(call)                                                                    \
  do {                                                                              \
    cudaError_t e_ = (call);                                                        \
    if (e_ != cudaSuccess)                                                          \
      return fail(h, SMDM_ECUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

// Launch bookkeeping: every kernel launch of the library goes through Launch{h, class, stream}.
struct Launch {
  smdm_handle* h;
  cudaStream_t st;
  Launch(smdm_handle* h_, int cls, cudaStream_t st_) : h(h_), st(st_) {
    Profiler& p = h->prof;
    p.launches++;
    p.class_launches[cls]++;
    if (p.on && p.timed) {
      if (p.used * 2 + 2 > p.ev.size()) {
        cudaEvent_t a, b;
        cudaEventCreate(&a);
        cudaEventCreate(&b);
        p.ev.push_back(a);
        p.ev.push_back(b);
      }
      p.cls.resize(p.used + 1);
      p.cls[p.used] = cls;
      record(p.ev[p.used * 2]);
    }
  }
  // Under stream capture a plain record only marks a point for cross-stream waits; the
  // external flag turns it into an event-record node whose time the replay fills in.
  void record(cudaEvent_t e) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    else cudaEventRecord(e, st);
  }
  ~Launch() {
    Profiler& p = h->prof;
    if (p.on && p.timed) {
      record(p.ev[p.used * 2 + 1]);
      p.used++;
    }
  }
};

Rows rows_at(smdm_handle* h, size_t off) {
  const size_t MR = align_up((size_t)h->cfg.max_rows, 256);
  int* b = h->at<int>(off);
  Rows r;
  r.ids = b;
  r.pos = b + MR;
  r.type = b + 2 * MR;
  r.label = b + 3 * MR;
  r.seq = b + 4 * MR;
  r.slot = b + 5 * MR;
  r.kvlen = b + 6 * MR;
  r.qrow = b + 7 * MR;
  r.qpos = b + 8 * MR;
  return r;
}

KVAddr cache_addr(smdm_handle* h) {
  const smdm_config& c = h->cfg;
  KVAddr kv;
  kv.k = h->at<uint8_t>(h->L.kc);
  kv.v = h->at<uint8_t>(h->L.vc);
  kv.cap = h->L.cap;
  kv.head_stride = (long long)h->L.cap * c.d_head;
  kv.layer_stride = kv.head_stride * c.n_heads;
  kv.seq_stride = kv.layer_stride * c.n_layers;
  return kv;
}

KVAddr scratch_addr(smdm_handle* h) {
  const smdm_config& c = h->cfg;
  const long long MR = (long long)align_up((size_t)c.max_rows, 256);
  KVAddr kv;
  kv.k = h->at<uint8_t>(h->L.kscr);
  kv.v = h->at<uint8_t>(h->L.vscr);
  kv.cap = (int)MR;
  kv.head_stride = MR * c.d_head;
  kv.layer_stride = 0;
  kv.seq_stride = 0;
  return kv;
}

// What one forward needs beyond the row arrays.
struct FwdSpec {
  int R;                      // rows
  int attn_mode;              // 0 prefix, 1 label
  bool scratch_kv;            // training form: K/V into the scratch, not a sequence cache
  int n_seg;
  AttnSeg seg[SMDM_MAX_BATCH];
  int n_logit;                // decode-set rows (0 = no LM head)
  float* logits;              // optional [n_logit][V]
  bool attn_bound;            // label mode: rows.kvlen holds per-row key bounds and
  const int* tile_list;       // tile_list / tile_count the key tiles of each query tile
  const int* tile_count;
};

smdm_status gemm(smdm_handle* h, int cls, const CUtensorMap* tmA, const CUtensorMap* tmA2,
                 const void* W, const void* W2, void* X, int K, int n_out, int rows, int swiglu,
                 const EpiParams& ep, cudaStream_t st, int a_interleave = 0, int sched = 0) {
  if (rows <= 0) return SMDM_OK;
  Launch lg(h, cls, st);
  constexpr CUtensorMapDataType F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (h->bf16) {
    CUtensorMap tmB;
    const size_t MR = align_up((size_t)h->cfg.max_rows, 256);
    const int pair = gemm_tc_pair(n_out, swiglu, rows, ep.kind);
    const int mrb = gemm_tc_min_row_blocks(n_out, rows, ep.kind, h->L.n_sms);
    if (!encode_2d(&tmB, X, K, MR, (uint64_t)K * 2, 64, gemm_tc_box_rows(rows, pair, mrb)))
      return fail(h, SMDM_ECUDA, "cuTensorMapEncodeTiled failed for an activation operand");
    CUtensorMap tmOut;
    bool ok_out = false;
    switch (ep.kind) {
      case kEpiStore: ok_out = encode_out(&tmOut, ep.out, F16, ep.n_valid, rows, ep.ld_out, 128); break;
      case kEpiQKV: ok_out = encode_out(&tmOut, ep.q_out, F16, ep.d_model, rows, ep.d_model, 128); break;
      case kEpiSwiGLU: ok_out = encode_out(&tmOut, ep.act, F16, ep.n_valid, rows, ep.ld_act, 64); break;
      case kEpiResid: ok_out = encode_out(&tmOut, ep.x, F32, ep.n_valid, rows, ep.ld_x, 128); break;
      case kEpiLMHead:
        // without logits the map is never used: any valid fp32 map will do
        ok_out = ep.logits ? encode_out(&tmOut, ep.logits, F32, ep.n_valid, rows, ep.ld_logits, 128)
                           : encode_out(&tmOut, ep.pmax, F32, 128, 32, 128, 128);
        break;
    }
    if (!ok_out) return fail(h, SMDM_ECUDA, "cuTensorMapEncodeTiled failed for a GEMM output");
    GemmCall c{};
    c.tmOut = &tmOut;
    c.pair = pair;
    c.tmA = tmA;
    c.tmA2 = tmA2;
    c.tmB = &tmB;
    c.K = K;
    c.n_out = n_out;
    c.rows = rows;
    c.row0 = 0;
    c.swiglu = swiglu;
    c.swiglu_il = swiglu && ep.swiglu_il;
    c.a_interleave = a_interleave;
    c.sched = sched;
    c.min_row_blocks = mrb;
    c.num_ctas = h->L.n_sms;
    c.partial = h->at<float>(h->L.partial);
    c.partial_bytes = h->L.partial_bytes;
    c.counters = h->at<unsigned>(h->L.counters);
    c.max_tiles = h->L.max_tiles;
    c.status = h->status();
    c.epi = ep;
    CK(launch_gemm_tc(c, st));
  } else {
    CK(launch_gemm_simt(static_cast<const float*>(W), static_cast<const float*>(W2),
                        static_cast<const float*>(X), K, K, n_out, rows, swiglu, ep, st));
  }
  return SMDM_OK;
}

smdm_status norm(smdm_handle* h, float* x, const void* gain, void* out, const int* gather,
                 const void* emb, const int* ids, int rows, cudaStream_t st) {
  NormArgs a;
  a.x = x;
  a.gain = gain;
  a.out = out;
  a.gather = gather;
  a.emb = emb;
  a.ids = ids;
  a.d = h->cfg.d_model;
  a.eps = h->cfg.rms_eps;
  Launch lg(h, SMDM_K_NORM, st);
  if (h->bf16) CK((launch_rmsnorm<__nv_bfloat16, __half>(a, rows, st)));
  else CK((launch_rmsnorm<float, float>(a, rows, st)));
  return SMDM_OK;
}

smdm_status forward(smdm_handle* h, const FwdSpec& f, cudaStream_t st) {
  const smdm_config& c = h->cfg;
  const int d = c.d_model, R = f.R;
  smdm_status s;
  float* x = h->at<float>(h->L.x);
  void* hb = h->at<uint8_t>(h->L.h);
  void* q = h->at<uint8_t>(h->L.q);
  void* ao = h->at<uint8_t>(h->L.ao);
  void* act = h->at<uint8_t>(h->L.act);
  void* hq = h->at<uint8_t>(h->L.hq);
  const KVAddr kv = f.scratch_kv ? scratch_addr(h) : cache_addr(h);
  const Rows& rw = h->rows;
  h->last_rows = R;

  // The RMSNorms run as their own kernel between the GEMMs.  (Run inside the consuming GEMM,
  // every CTA of that GEMM would have to wait for the rows of every other CTA at a grid-wide
  // barrier; the separate kernel's small CTAs sit beside the previous GEMM's and start the
  // moment it completes, while the next GEMM is already streaming its first weight stages.)
  if ((s = norm(h, x, h->attn_norm[0], hb, nullptr, h->emb, rw.ids, R, st))) return s;
  for (int l = 0; l < c.n_layers; ++l) {
    EpiParams ep{};
    ep.rows = R;
    // QKV + RoPE + KV append
    ep.kind = kEpiQKV;
    ep.n_valid = 3 * d;
    ep.q_out = q;
    ep.d_model = d;
    ep.d_head = c.d_head;
    ep.layer = f.scratch_kv ? 0 : l;
    ep.kv = kv;
    ep.row_seq = rw.seq;
    ep.row_slot = rw.slot;
    ep.row_pos = rw.pos;
    ep.rope = h->at<float2>(h->L.rope);
    if ((s = gemm(h, SMDM_K_GEMM_QKV, h->bf16 ? &h->tm_qkv[l] : nullptr, nullptr,
                  h->w_qkv[l], nullptr, hb, d, 3 * d, R, 0, ep, st, c.d_head)))
      return s;
    // step-causal attention
    if (h->bf16) {
      AttnCall a{};
      a.mode = f.attn_mode;
      a.bound = f.attn_bound ? 1 : 0;
      a.tile_list = f.tile_list;
      a.tile_count = f.tile_count;
      a.n_ktiles = (R + 127) / 128;
      a.H = c.n_heads;
      a.dh = c.d_head;
      a.d_model = d;
      a.layer = f.scratch_kv ? 0 : l;
      a.n_seg = f.n_seg;
      for (int i = 0; i < f.n_seg; ++i) a.seg[i] = f.seg[i];
      a.kvlen = rw.kvlen;
      a.type = rw.type;
      a.label = rw.label;
      a.tmQ = &h->tm_q;
      a.tmK = f.scratch_kv ? &h->tm_kscr : &h->tm_kc;
      a.tmV = f.scratch_kv ? &h->tm_vscr : &h->tm_vc;
      a.cache_rows_per_seq = f.scratch_kv ? 0 : (long long)c.n_layers * c.n_heads * h->L.cap;
      a.cap = kv.cap;
      a.out = ao;
      a.status = h->status();
      a.part_o = h->at<float>(h->L.attn_part);
      a.part_bytes = h->L.attn_part_bytes;
      a.num_sms = h->L.n_sms;
      a.rows_total = R;
      Launch lg(h, SMDM_K_ATTN, st);
      CK(launch_attn_tc(a, st));
    } else {
      AttnSimtArgs a{};
      a.mode = f.attn_mode;
      a.rows = R;
      a.H = c.n_heads;
      a.dh = c.d_head;
      a.d_model = d;
      a.layer = f.scratch_kv ? 0 : l;
      a.nkeys = R;
      a.row_seq = rw.seq;
      a.kvlen = rw.kvlen;
      a.type = rw.type;
      a.label = rw.label;
      a.scale = 1.0f / sqrtf((float)c.d_head);
      Launch lg(h, SMDM_K_ATTN, st);
      CK(launch_attn_simt<float>(static_cast<const float*>(q), static_cast<float*>(ao), kv, a, st));
    }
    // O-projection + residual
    EpiParams eo{};
    eo.kind = kEpiResid;
    eo.rows = R;
    eo.n_valid = d;
    eo.x = x;
    eo.ld_x = d;
    if ((s = gemm(h, SMDM_K_GEMM_O, h->bf16 ? &h->tm_o[l] : nullptr, nullptr, h->w_o[l], nullptr, ao, d, d, R,
                  0, eo, st)))
      return s;
    if ((s = norm(h, x, h->mlp_norm[l], hb, nullptr, nullptr, nullptr, R, st))) return s;
    // gate/up + SwiGLU
    EpiParams eg{};
    eg.kind = kEpiSwiGLU;
    eg.rows = R;
    eg.n_valid = c.d_ffn;
    eg.act = act;
    eg.ld_act = c.d_ffn;
    const bool il = h->bf16 && h->gu_il[l] != 0;
    eg.swiglu_il = il ? 1 : 0;
    eg.swiglu_up_first = (il && h->gu_il[l] == 2) ? 1 : 0;
    if ((s = gemm(h, SMDM_K_GEMM_GATEUP, h->bf16 ? (il ? &h->tm_gu[l] : &h->tm_gate[l]) : nullptr,
                  h->bf16 ? &h->tm_up[l] : nullptr,
                  h->w_gate[l], h->w_up[l], hb, d, c.d_ffn, R, 1, eg, st)))
      return s;
    // down + residual
    EpiParams ed = eo;
    if ((s = gemm(h, SMDM_K_GEMM_DOWN, h->bf16 ? &h->tm_down[l] : nullptr, nullptr, h->w_down[l], nullptr, act,
                  c.d_ffn, d, R, 0, ed, st)))
      return s;
    if (l + 1 < c.n_layers)
      if ((s = norm(h, x, h->attn_norm[l + 1], hb, nullptr, nullptr, nullptr, R, st))) return s;
  }
  if (f.n_logit > 0) {
    if ((s = norm(h, x, h->final_norm, hq, rw.qrow, nullptr, nullptr, f.n_logit, st))) return s;
    EpiParams el{};
    el.kind = kEpiLMHead;
    el.rows = f.n_logit;
    el.n_valid = c.vocab;
    el.logits = f.logits;
    el.ld_logits = c.vocab;
    el.pmax = h->at<float>(h->L.pmax);
    el.psum = h->at<float>(h->L.psum);
    el.parg = h->at<int>(h->L.parg);
    el.n_vt = h->L.n_vt;
    if ((s = gemm(h, SMDM_K_GEMM_LMHEAD, h->bf16 ? &h->tm_lm : nullptr, nullptr, h->lm_head, nullptr, hq, d, c.vocab,
                  f.n_logit, 0, el, st)))
      return s;
  }
  return SMDM_OK;
}

// bf16 models compute in fp16 (fp32 accumulation): every weight matrix is re-encoded once into
// an fp16 copy in the workspace (exact for magnitudes in [2^-14, 65504]; smaller ones round at
// 2^-24 absolute; a larger one sets kStatusRange), and the GEMMs' tensor maps point at the
// copies.  fp16 carries three more mantissa bits than bf16 at the same bytes and the same MMA
// rate, so the activations that feed the GEMMs (normalised rows, attention output, SwiGLU
// output) keep them too.  Asynchronous on `st`.
bool prepare_weights16(smdm_handle* h, const smdm_weights* w, cudaStream_t st) {
  const smdm_config& c = h->cfg;
  const size_t d = c.d_model, f = c.d_ffn;
  const int nl = c.n_layers, dh = c.d_head;
  uint8_t* base = h->at<uint8_t>(h->L.w16);
  auto conv = [&](const void* src, uint8_t* dst, size_t n) {
    return launch_convert_bf16_f16(static_cast<const __nv_bfloat16*>(src),
                                   reinterpret_cast<__half*>(dst), n, h->status(), st) ==
           cudaSuccess;
  };
  bool ok = true;
  h->tm_qkv.resize(nl);
  h->tm_o.resize(nl);
  h->tm_gate.resize(nl);
  h->tm_up.resize(nl);
  h->tm_gu.resize(nl);
  h->gu_il.assign(nl, 0);
  h->tm_down.resize(nl);
  for (int l = 0; l < nl; ++l) {
    uint8_t* lb = base + (size_t)l * h->L.w16_layer;
    uint8_t* qkv = lb + h->L.w16_qkv;
    uint8_t* o = lb + h->L.w16_o;
    uint8_t* gate = lb + h->L.w16_gu;
    uint8_t* up = gate + f * d * 2;
    uint8_t* down = lb + h->L.w16_down;
    ok &= conv(w->w_qkv[l], qkv, 3 * d * d) && conv(w->w_o[l], o, d * d) &&
          conv(w->w_gate[l], gate, f * d) && conv(w->w_up[l], up, f * d) &&
          conv(w->w_down[l], down, d * f);
    ok &= encode_qkv_interleaved(&h->tm_qkv[l], qkv, d, dh);
    ok &= encode_2d(&h->tm_o[l], o, d, d, d * 2, 64, 128);
    ok &= encode_2d(&h->tm_gate[l], gate, d, f, d * 2, 64, 64);
    ok &= encode_2d(&h->tm_up[l], up, d, f, d * 2, 64, 64);
    h->gu_il[l] = encode_gateup_interleaved(&h->tm_gu[l], gate, up, d, f);
    ok &= encode_2d(&h->tm_down[l], down, f, d, f * 2, 64, 128);
  }
  uint8_t* lm = base + h->L.w16_lm;
  ok &= conv(w->lm_head, lm, (size_t)c.vocab * d);
  ok &= encode_2d(&h->tm_lm, lm, d, c.vocab, d * 2, 64, 128);
  return ok;
}

smdm_status check_seq(smdm_handle* h, int seq) {
  if (seq < 0 || seq >= h->cfg.max_batch)
    return fail(h, SMDM_EINVAL, "sequence slot %d out of range [0, %d)", seq, h->cfg.max_batch);
  return SMDM_OK;
}

// Validate a step descriptor against the sequence state; returns n_query and R.
smdm_status check_desc(smdm_handle* h, const smdm_step_desc& d, bool dense) {
  smdm_status s;
  if ((s = check_seq(h, d.seq))) return s;
  const SeqState& q = h->seq[d.seq];
  if (!q.active) return fail(h, SMDM_ESTATE, "sequence %d has not been prefilled", d.seq);
  if (q.dense != dense)
    return fail(h, SMDM_ESTATE, "sequence %d mixes sparse and dense steps", d.seq);
  if (q.sw >= 0)
    return fail(h, SMDM_ESTATE, "sequence %d runs switched steps (smdm_step_switched)", d.seq);
  if (d.n_query < 1) return fail(h, SMDM_EINVAL, "empty decode set");
  if (d.policy != SMDM_POLICY_ALL && d.policy != SMDM_POLICY_TOPN)
    return fail(h, SMDM_EINVAL, "unknown policy %d", d.policy);
  if (d.policy == SMDM_POLICY_TOPN && d.n_commit < 1)
    return fail(h, SMDM_EINVAL, "TOPN needs n_commit >= 1");
  if (!d.d_query_pos) {
    const int lo = q.P + 1, hi = q.P + q.Lg + 1;
    if (d.block_lo < lo || d.block_hi > hi || d.block_lo >= d.block_hi)
      return fail(h, SMDM_EINVAL, "block [%d, %d) outside the generated span [%d, %d)",
                  d.block_lo, d.block_hi, lo, hi);
    if (d.n_query > d.block_hi - d.block_lo)
      return fail(h, SMDM_EINVAL, "n_query larger than the block");
  }
  if (d.n_query > q.Lg) return fail(h, SMDM_EINVAL, "n_query larger than Lgen");
  if (!dense) {
    const int R = q.n_new + d.n_query + tail_rows(&h->cfg);
    if (R > h->cfg.max_step_rows)
      return fail(h, SMDM_ESHAPE, "step rows %d exceed max_step_rows %d", R, h->cfg.max_step_rows);
    if (q.ctx + R > h->L.cap) return fail(h, SMDM_ESHAPE, "KV cache capacity exceeded");
  }
  return SMDM_OK;
}

int committed(const smdm_step_desc& d) {
  return d.policy == SMDM_POLICY_ALL ? d.n_query : std::min(d.n_commit, d.n_query);
}

}  // namespace

// ==============================================================================================
// C ABI
// ==============================================================================================
extern "C" {

size_t smdm_workspace_bytes(const smdm_config* cfg) {
  if (!config_ok(cfg, nullptr)) return 0;
  return make_layout(cfg, query_sms()).total;
}

smdm_status smdm_create(const smdm_config* cfg, const smdm_weights* w, void* d_workspace,
                        size_t bytes, smdm_handle** out) {
  if (!out) return SMDM_EINVAL;
  *out = nullptr;
  std::string why;
  if (!config_ok(cfg, &why)) return SMDM_ESHAPE;
  if (!w || !d_workspace || !w->emb || !w->final_norm || !w->lm_head || !w->attn_norm ||
      !w->w_qkv || !w->w_o || !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down)
    return SMDM_EINVAL;
  if (reinterpret_cast<uintptr_t>(d_workspace) % 256) return SMDM_EINVAL;
  smdm_handle* h = new smdm_handle();
  h->cfg = *cfg;
  h->bf16 = cfg->dtype == SMDM_BF16;
  h->L = make_layout(cfg, query_sms());
  if (bytes < h->L.total) {
    delete h;
    return SMDM_ENOMEM;
  }
  h->ws = static_cast<uint8_t*>(d_workspace);
  h->emb = w->emb;
  h->final_norm = w->final_norm;
  h->lm_head = w->lm_head;
  const int nl = cfg->n_layers;
  for (int l = 0; l < nl; ++l) {
    if (!w->attn_norm[l] || !w->w_qkv[l] || !w->w_o[l] || !w->mlp_norm[l] || !w->w_gate[l] ||
        !w->w_up[l] || !w->w_down[l]) {
      delete h;
      return SMDM_EINVAL;
    }
    h->attn_norm.push_back(w->attn_norm[l]);
    h->w_qkv.push_back(w->w_qkv[l]);
    h->w_o.push_back(w->w_o[l]);
    h->mlp_norm.push_back(w->mlp_norm[l]);
    h->w_gate.push_back(w->w_gate[l]);
    h->w_up.push_back(w->w_up[l]);
    h->w_down.push_back(w->w_down[l]);
  }
  h->rows = rows_at(h, h->L.rows);
  h->aux = rows_at(h, h->L.aux);
  auto cuda_fail = [&](cudaError_t e) {
    delete h;
    (void)e;
    return SMDM_ECUDA;
  };
  cudaError_t e = cudaMemset(d_workspace, 0, h->L.total);
  if (e != cudaSuccess) return cuda_fail(e);
  // RoPE table: angle = pos * theta^(-2i/d_head), computed in double, stored (cos, sin) fp32.
  {
    const int half = cfg->d_head / 2;
    std::vector<float2> tab((size_t)h->L.max_pos * half);
    for (int p = 0; p < h->L.max_pos; ++p)
      for (int i = 0; i < half; ++i) {
        const double inv = std::pow((double)cfg->rope_theta, -2.0 * i / cfg->d_head);
        const double ang = (double)p * inv;
        tab[(size_t)p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    e = cudaMemcpy(h->at<float2>(h->L.rope), tab.data(), tab.size() * sizeof(float2),
                   cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (h->bf16) {
    const int d = cfg->d_model, H = cfg->n_heads, dh = cfg->d_head;
    bool ok = prepare_weights16(h, w, 0);
    const size_t MR = align_up((size_t)cfg->max_rows, 256);
    const uint64_t cache_rows = (uint64_t)cfg->max_batch * nl * H * h->L.cap;
    ok &= encode_head_tiles(&h->tm_kc, h->at<uint8_t>(h->L.kc), dh, cache_rows, dh / 64);
    ok &= encode_head_tiles(&h->tm_vc, h->at<uint8_t>(h->L.vc), dh, cache_rows, dh / 64);
    ok &= encode_head_tiles(&h->tm_kscr, h->at<uint8_t>(h->L.kscr), dh, (uint64_t)H * MR, dh / 64);
    ok &= encode_head_tiles(&h->tm_vscr, h->at<uint8_t>(h->L.vscr), dh, (uint64_t)H * MR, dh / 64);
    ok &= encode_head_tiles(&h->tm_q, h->at<uint8_t>(h->L.q), d, MR, dh / 64);
    if (!ok) {
      delete h;
      return SMDM_ECUDA;
    }
    if (gemm_tc_set_smem_attr() != cudaSuccess || attn_tc_set_smem_attr() != cudaSuccess) {
      delete h;
      return SMDM_ECUDA;
    }
  }
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  if (h->bf16) {   // a weight beyond the fp16 range (set by the conversion)
    uint32_t bits = 0;
    e = cudaMemcpy(&bits, h->status(), 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (bits & kStatusRange) {
      delete h;
      return SMDM_EINVAL;
    }
  }
  *out = h;
  return SMDM_OK;
}

void smdm_destroy(smdm_handle* h) {
  if (!h) return;
  for (cudaEvent_t e : h->prof.ev) cudaEventDestroy(e);
  delete h;
}

const char* smdm_last_error(const smdm_handle* h) { return h ? h->err.c_str() : "null handle"; }

int smdm_context_length(const smdm_handle* h, int seq) {
  if (!h || seq < 0 || seq >= h->cfg.max_batch) return -1;
  return h->seq[seq].ctx;
}

// Block 0 of a sequence: the prompt and (bidirectional tasks) any given generation tokens.
static smdm_status prefill_block0(smdm_handle* h, int seq, const int32_t* d_prompt, int P,
                                  int Lgen, const int32_t* d_given_pos,
                                  const int32_t* d_given_tok, int n_given, int32_t* d_grid,
                                  cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  smdm_status s;
  if ((s = check_seq(h, seq))) return s;
  if (P < 0 || Lgen < 1 || P + Lgen > h->cfg.max_len)
    return fail(h, SMDM_ESHAPE, "P=%d, Lgen=%d outside max_len %d", P, Lgen, h->cfg.max_len);
  if (n_given < 0 || n_given >= Lgen)
    return fail(h, SMDM_EINVAL, "n_given=%d must leave generation positions to decode", n_given);
  if (P + n_given > h->cfg.max_rows)
    return fail(h, SMDM_ESHAPE, "prompt and given tokens longer than max_rows");
  if (!d_grid || (P > 0 && !d_prompt)) return fail(h, SMDM_EINVAL, "null prompt or grid");
  if (n_given > 0 && (!d_given_pos || !d_given_tok))
    return fail(h, SMDM_EINVAL, "null given positions or tokens");
  { Launch lg_(h, SMDM_K_OTHER, st); CK(launch_fill_i32(d_grid, Lgen, -1, st)); }
  if (P > 0)
    CK(cudaMemcpyAsync(h->prompt(seq), d_prompt, (size_t)P * 4, cudaMemcpyDeviceToDevice, st));
  SeqState& q = h->seq[seq];
  q = SeqState();
  q.P = P;
  q.Lg = Lgen;
  q.grid = d_grid;
  const int n0 = P + n_given;   // rows of block 0
  if (n0 > 0) {
    LinearPackArgs a{};
    a.mode = n_given > 0 ? kPackPrefillGiven : kPackPrefill;
    a.n = n0;
    a.seq = seq;
    a.P = P;
    a.Lg = Lgen;
    a.vocab = h->cfg.vocab;
    a.emb_rows = emb_rows(&h->cfg);
    a.max_pos = h->L.max_pos;
    a.prompt = h->prompt(seq);
    a.given_pos = d_given_pos;
    a.given_tok = d_given_tok;
    a.grid_out = d_grid;
    a.rows = h->rows;
    a.status = h->status();
    { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_linear(a, st)); }
    FwdSpec f{};
    f.R = n0;
    f.attn_mode = 0;
    f.n_seg = 1;
    f.seg[0] = AttnSeg{seq, 0, n0, n0, 0};
    if ((s = forward(h, f, st))) return s;
  }
  q.active = true;
  q.n0 = n0;
  q.ctx = n0;
  return SMDM_OK;
}

smdm_status smdm_prefill(smdm_handle* h, int seq, const int32_t* d_prompt, int P, int Lgen,
                         int32_t* d_grid, cudaStream_t st) {
  return prefill_block0(h, seq, d_prompt, P, Lgen, nullptr, nullptr, 0, d_grid, st);
}

smdm_status smdm_prefill_given(smdm_handle* h, int seq, const int32_t* d_prompt, int P, int Lgen,
                               const int32_t* d_given_pos, const int32_t* d_given_tok,
                               int n_given, int32_t* d_grid, cudaStream_t st) {
  return prefill_block0(h, seq, d_prompt, P, Lgen, d_given_pos, d_given_tok, n_given, d_grid,
                        st);
}

smdm_status smdm_step(smdm_handle* h, int n_seq, const smdm_step_desc* hd, float* d_logits,
                      int32_t* d_tok, float* d_conf, cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  if (n_seq < 1 || n_seq > h->cfg.max_batch || !hd) return fail(h, SMDM_EINVAL, "bad batch");
  smdm_status s;
  int R = 0, NQ = 0;
  for (int i = 0; i < n_seq; ++i) {
    if ((s = check_desc(h, hd[i], false))) return s;
    for (int j = 0; j < i; ++j)
      if (hd[j].seq == hd[i].seq) return fail(h, SMDM_EINVAL, "sequence %d twice in a batch", hd[i].seq);
    R += h->seq[hd[i].seq].n_new + hd[i].n_query + tail_rows(&h->cfg);
    NQ += hd[i].n_query;
  }
  if (R > h->cfg.max_rows) return fail(h, SMDM_ESHAPE, "batched rows %d exceed max_rows", R);
  PackArgs pa{};
  pa.n_seq = n_seq;
  pa.vocab = h->cfg.vocab;
  pa.len_token = h->cfg.n_reg == SMDM_REG_LEN;
  pa.rows = h->rows;
  pa.status = h->status();
  FwdSpec f{};
  f.R = R;
  f.attn_mode = 0;
  f.n_seg = n_seq;
  f.n_logit = NQ;
  f.logits = d_logits;
  UnmaskArgs ua{};
  ua.n_seq = n_seq;
  int row0 = 0, qbase = 0, max_nq = 0;
  for (int i = 0; i < n_seq; ++i) {
    const smdm_step_desc& d = hd[i];
    SeqState& q = h->seq[d.seq];
    const int Rs = q.n_new + d.n_query + tail_rows(&h->cfg);
    PackSeq& p = pa.s[i];
    p.seq = d.seq;
    p.row0 = row0;
    p.n_new = q.n_new;
    p.n_q = d.n_query;
    p.n_reg = tail_rows(&h->cfg);
    p.ctx = q.ctx;
    p.P = q.P;
    p.Lg = q.Lg;
    p.label = q.k + 1;
    p.qbase = qbase;
    p.block_lo = d.block_lo;
    p.block_hi = d.block_hi;
    p.qpos = d.d_query_pos;
    p.grid = q.grid;
    p.newpos = h->newpos(d.seq);
    f.seg[i] = AttnSeg{d.seq, row0, Rs, q.ctx + Rs, 0};
    UnmaskSeq& u = ua.s[i];
    u.qbase = qbase;
    u.n_q = d.n_query;
    u.lbase = 0;
    u.dense = 0;
    u.policy = d.policy;
    u.n_commit = d.policy == SMDM_POLICY_ALL ? d.n_query : d.n_commit;
    u.P = q.P;
    u.Lg = q.Lg;
    u.grid = q.grid;
    u.newpos = h->newpos(d.seq);
    row0 += Rs;
    qbase += d.n_query;
    max_nq = std::max(max_nq, d.n_query);
  }
  { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_step(pa, st)); }
  if ((s = forward(h, f, st))) return s;
  ua.n_vt = h->L.n_vt;
  ua.pmax = h->at<float>(h->L.pmax);
  ua.psum = h->at<float>(h->L.psum);
  ua.parg = h->at<int>(h->L.parg);
  ua.qpos_of = h->rows.qpos;
  ua.tok_out = d_tok;
  ua.conf_out = d_conf;
  ua.status = h->status();
  { Launch lg_(h, SMDM_K_UNMASK, st); CK(launch_unmask(ua, max_nq, st)); }
  for (int i = 0; i < n_seq; ++i) {
    SeqState& q = h->seq[hd[i].seq];
    q.ctx += q.n_new;
    q.n_new = committed(hd[i]);
    q.k += 1;
  }
  return SMDM_OK;
}

smdm_status smdm_step_switched(smdm_handle* h, const smdm_step_desc* hd, int switches,
                               float* d_logits, int32_t* d_tok, float* d_conf, cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  if (!hd) return fail(h, SMDM_EINVAL, "null step descriptor");
  if (switches < 0 || switches > SMDM_SW_ALL) return fail(h, SMDM_EINVAL, "bad switches %d", switches);
  const smdm_step_desc& d = *hd;
  smdm_status s;
  if ((s = check_seq(h, d.seq))) return s;
  SeqState& q = h->seq[d.seq];
  if (!q.active) return fail(h, SMDM_ESTATE, "sequence %d has not been prefilled", d.seq);
  if (q.dense) return fail(h, SMDM_ESTATE, "sequence %d runs dense steps", d.seq);
  if (q.sw != switches && (q.k > 0 || q.sw >= 0))
    return fail(h, SMDM_ESTATE, "sequence %d keeps one set of switches for its whole run", d.seq);
  if (q.n0 != q.P)
    return fail(h, SMDM_EINVAL, "switched steps need a prompt-only prefill (no given tokens)");
  if (!d.d_query_pos) return fail(h, SMDM_EINVAL, "switched steps take explicit query positions");
  if (d.policy != SMDM_POLICY_ALL && d.policy != SMDM_POLICY_TOPN)
    return fail(h, SMDM_EINVAL, "unknown policy %d", d.policy);
  if (d.policy == SMDM_POLICY_TOPN && d.n_commit < 1)
    return fail(h, SMDM_EINVAL, "TOPN needs n_commit >= 1");
  const int masked = q.Lg - q.dec - q.n_new;   // still masked before this step commits
  if (d.n_query < 1 || d.n_query > masked)
    return fail(h, SMDM_EINVAL, "n_query %d outside [1, %d masked positions]", d.n_query, masked);
  const bool cp = switches & SMDM_SW_CACHE_PROMPT, cr = switches & SMDM_SW_CACHE_RES,
             tr = switches & SMDM_SW_TRUNCATE;
  const int n_tail = tail_rows(&h->cfg);
  const int n_extra = tr ? 0 : masked - d.n_query;
  const int n_dec = q.dec + q.n_new;
  const int R = (cp ? 0 : q.P) + (cr ? q.n_new : n_dec) + d.n_query + n_extra + n_tail;
  const int keys = q.P + n_dec + d.n_query + n_extra + n_tail;
  if (R > h->cfg.max_step_rows || R > h->cfg.max_rows)
    return fail(h, SMDM_ESHAPE, "switched step needs %d rows (max_step_rows %d, max_rows %d)", R,
                h->cfg.max_step_rows, h->cfg.max_rows);
  if (keys > h->L.cap) return fail(h, SMDM_ESHAPE, "KV cache capacity exceeded");
  int* dec_pos = h->sw_arrays(d.seq);
  int* dec_lab = dec_pos + h->cfg.max_len;
  int* qmark = dec_lab + h->cfg.max_len;
  if (q.sw < 0) {   // first switched step of the sequence: no position has been queried yet
    Launch lg_(h, SMDM_K_OTHER, st);
    CK(launch_fill_i32(qmark, q.Lg, 0, st));
  }
  PackSwArgs pa{};
  pa.seq = d.seq;
  pa.P = q.P;
  pa.Lg = q.Lg;
  pa.label = q.k + 1;
  pa.vocab = h->cfg.vocab;
  pa.n_tail = n_tail;
  pa.len_token = h->cfg.n_reg == SMDM_REG_LEN;
  pa.cache_prompt = cp;
  pa.cache_res = cr;
  pa.truncate = tr;
  pa.n_new = q.n_new;
  pa.dec_prev = q.dec;
  pa.n_q = d.n_query;
  pa.n_extra = n_extra;
  pa.qpos = d.d_query_pos;
  pa.newpos = h->newpos(d.seq);
  pa.prompt = h->prompt(d.seq);
  pa.grid = q.grid;
  pa.dec_pos = dec_pos;
  pa.dec_lab = dec_lab;
  pa.qmark = qmark;
  pa.rows = h->rows;
  pa.status = h->status();
  { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_switched(pa, st)); }
  FwdSpec f{};
  f.R = R;
  f.attn_mode = 0;
  f.n_seg = 1;
  f.seg[0] = AttnSeg{d.seq, 0, R, keys, 0};
  f.n_logit = d.n_query;
  f.logits = d_logits;
  if ((s = forward(h, f, st))) return s;
  UnmaskArgs ua{};
  ua.n_seq = 1;
  UnmaskSeq& u = ua.s[0];
  u.qbase = 0;
  u.n_q = d.n_query;
  u.lbase = 0;
  u.dense = 0;
  u.policy = d.policy;
  u.n_commit = d.policy == SMDM_POLICY_ALL ? d.n_query : d.n_commit;
  u.P = q.P;
  u.Lg = q.Lg;
  u.grid = q.grid;
  u.newpos = h->newpos(d.seq);
  ua.n_vt = h->L.n_vt;
  ua.pmax = h->at<float>(h->L.pmax);
  ua.psum = h->at<float>(h->L.psum);
  ua.parg = h->at<int>(h->L.parg);
  ua.qpos_of = h->rows.qpos;
  ua.tok_out = d_tok;
  ua.conf_out = d_conf;
  ua.status = h->status();
  { Launch lg_(h, SMDM_K_UNMASK, st); CK(launch_unmask(ua, d.n_query, st)); }
  q.sw = switches;
  if (cr) q.ctx += q.n_new;    // decoded tokens stay in the cache only when it is on
  q.dec += q.n_new;
  q.n_new = committed(d);
  q.k += 1;
  return SMDM_OK;
}

smdm_status smdm_dense_step(smdm_handle* h, const smdm_step_desc* d, float* d_logits,
                            int32_t* d_tok, float* d_conf, cudaStream_t st) {
  if (!h || !d) return SMDM_EINVAL;
  smdm_status s;
  if ((s = check_seq(h, d->seq))) return s;
  SeqState& q = h->seq[d->seq];
  if (q.active && q.k == 0) q.dense = true;   // a freshly prefilled sequence may go dense
  if ((s = check_desc(h, *d, true))) return s;
  const int L = q.P + q.Lg;
  if (L > h->cfg.max_rows) return fail(h, SMDM_ESHAPE, "P + Lgen exceeds max_rows");
  // decode set -> aux.qpos
  PackArgs pa{};
  pa.n_seq = 1;
  pa.vocab = h->cfg.vocab;
  pa.rows = h->aux;
  pa.status = h->status();
  PackSeq& p = pa.s[0];
  p.seq = d->seq;
  p.row0 = 0;
  p.n_new = 0;
  p.n_q = d->n_query;
  p.n_reg = 0;
  p.ctx = 0;
  p.P = q.P;
  p.Lg = q.Lg;
  p.label = q.k + 1;
  p.qbase = 0;
  p.block_lo = d->block_lo;
  p.block_hi = d->block_hi;
  p.qpos = d->d_query_pos;
  p.grid = q.grid;
  p.newpos = h->newpos(d->seq);
  { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_step(pa, st)); }
  LinearPackArgs a{};
  a.mode = kPackDense;
  a.n = L;
  a.seq = d->seq;
  a.P = q.P;
  a.vocab = h->cfg.vocab;
  a.emb_rows = emb_rows(&h->cfg);
  a.max_pos = h->L.max_pos;
  a.prompt = h->prompt(d->seq);
  a.grid = q.grid;
  a.rows = h->rows;
  a.status = h->status();
  { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_linear(a, st)); }
  FwdSpec f{};
  f.R = L;
  f.attn_mode = 0;
  f.n_seg = 1;
  f.seg[0] = AttnSeg{d->seq, 0, L, L, 0};
  f.n_logit = q.Lg;
  f.logits = d_logits;
  if ((s = forward(h, f, st))) return s;
  UnmaskArgs ua{};
  ua.n_seq = 1;
  UnmaskSeq& u = ua.s[0];
  u.qbase = 0;
  u.n_q = d->n_query;
  u.lbase = 0;
  u.dense = 1;
  u.policy = d->policy;
  u.n_commit = d->policy == SMDM_POLICY_ALL ? d->n_query : d->n_commit;
  u.P = q.P;
  u.Lg = q.Lg;
  u.grid = q.grid;
  u.newpos = nullptr;
  ua.n_vt = h->L.n_vt;
  ua.pmax = h->at<float>(h->L.pmax);
  ua.psum = h->at<float>(h->L.psum);
  ua.parg = h->at<int>(h->L.parg);
  ua.qpos_of = h->aux.qpos;
  ua.tok_out = d_tok;
  ua.conf_out = d_conf;
  ua.status = h->status();
  { Launch lg_(h, SMDM_K_UNMASK, st); CK(launch_unmask(ua, d->n_query, st)); }
  q.k += 1;
  return SMDM_OK;
}

smdm_status smdm_generate(smdm_handle* h, int batch, const int32_t* d_prompts, int P, int Lgen,
                          const smdm_plan* plans, int mode, int32_t* d_grids, cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  if (batch < 1 || batch > h->cfg.max_batch || !plans || !d_grids || (P > 0 && !d_prompts))
    return fail(h, SMDM_EINVAL, "bad generate arguments");
  if (mode != SMDM_MODE_SPARSE && mode != SMDM_MODE_DENSE)
    return fail(h, SMDM_EINVAL, "unknown mode %d", mode);
  const int K = plans[0].n_steps;
  if (P < 0 || Lgen < 1 || (long long)P + Lgen > h->cfg.max_len)
    return fail(h, SMDM_ESHAPE, "P=%d, Lgen=%d outside max_len %d", P, Lgen, h->cfg.max_len);
  if (K < 1 || K > Lgen) return fail(h, SMDM_EINVAL, "step count %d outside [1, Lgen]", K);
  // Whole-plan checks before any work, so that a bad plan leaves every sequence untouched.
  // Rows of sparse step k for one sequence: the tokens committed at step k-1 (new-cache rows),
  // the decode set and the registers; they must fit max_step_rows, and a batched step's rows
  // summed over the sequences must fit max_rows (the checks smdm_step makes per step).
  std::vector<long long> batch_rows(K, 0);
  for (int b = 0; b < batch; ++b) {
    const smdm_plan& p = plans[b];
    if (p.n_steps != K || K < 1) return fail(h, SMDM_EINVAL, "plans need the same step count");
    if (p.kind == SMDM_PLAN_ORDER) {
      if (!p.h_n_per_step || !p.d_order) return fail(h, SMDM_EINVAL, "ORDER plan needs order + sizes");
      long long tot = 0;
      for (int k = 0; k < K; ++k) {
        if (p.h_n_per_step[k] < 1) return fail(h, SMDM_EINVAL, "empty step in plan");
        tot += p.h_n_per_step[k];
      }
      if (tot != Lgen) return fail(h, SMDM_EINVAL, "plan sizes sum to %lld, not Lgen %d", tot, Lgen);
    } else if (p.kind == SMDM_PLAN_SEMIAR) {
      if (p.block < 1 || p.commit < 1 || p.steps_per_block < 1 || Lgen % p.block ||
          p.block != p.steps_per_block * p.commit || K != (Lgen / p.block) * p.steps_per_block)
        return fail(h, SMDM_EINVAL, "inconsistent SEMIAR plan");
      if (p.h_block_order) {
        const int nb = Lgen / p.block;
        std::vector<char> seen(nb, 0);
        for (int i = 0; i < nb; ++i) {
          const int v = p.h_block_order[i];
          if (v < 0 || v >= nb || seen[v])
            return fail(h, SMDM_EINVAL, "block order of plan %d is not a permutation", b);
          seen[v] = 1;
        }
      }
    } else {
      return fail(h, SMDM_EINVAL, "unknown plan kind");
    }
    for (int k = 0; k < K; ++k) {
      long long n_new, n_q;
      if (p.kind == SMDM_PLAN_ORDER) {
        n_new = k ? p.h_n_per_step[k - 1] : 0;
        n_q = p.h_n_per_step[k];
      } else {
        n_new = k ? p.commit : 0;
        n_q = p.block - (long long)(k % p.steps_per_block) * p.commit;
      }
      const long long rows = n_new + n_q + tail_rows(&h->cfg);
      if (mode == SMDM_MODE_SPARSE && rows > h->cfg.max_step_rows)
        return fail(h, SMDM_ESHAPE, "plan %d step %d needs %lld rows, max_step_rows is %d", b,
                    k + 1, rows, h->cfg.max_step_rows);
      batch_rows[k] += rows;
    }
  }
  if (mode == SMDM_MODE_SPARSE)
    for (int k = 0; k < K; ++k)
      if (batch_rows[k] > h->cfg.max_rows)
        return fail(h, SMDM_ESHAPE, "batched step %d needs %lld rows, max_rows is %d", k + 1,
                    batch_rows[k], h->cfg.max_rows);
  smdm_status s;
  for (int b = 0; b < batch; ++b)
    if ((s = smdm_prefill(h, b, d_prompts + (size_t)b * P, P, Lgen, d_grids + (size_t)b * Lgen, st)))
      return s;
  std::vector<long long> off(batch, 0);
  for (int k = 1; k <= K; ++k) {
    smdm_step_desc desc[SMDM_MAX_BATCH];
    for (int b = 0; b < batch; ++b) {
      const smdm_plan& p = plans[b];
      smdm_step_desc& d = desc[b];
      d = smdm_step_desc{};
      d.seq = b;
      if (p.kind == SMDM_PLAN_ORDER) {
        d.d_query_pos = p.d_order + off[b];
        d.n_query = p.h_n_per_step[k - 1];
        d.policy = SMDM_POLICY_ALL;
        d.n_commit = d.n_query;
        off[b] += d.n_query;
      } else {
        const int nth = (k - 1) / p.steps_per_block, j = (k - 1) % p.steps_per_block;
        const int blk = p.h_block_order ? p.h_block_order[nth] : nth;
        d.d_query_pos = nullptr;
        d.block_lo = P + 1 + blk * p.block;
        d.block_hi = d.block_lo + p.block;
        d.n_query = p.block - j * p.commit;
        d.policy = SMDM_POLICY_TOPN;
        d.n_commit = p.commit;
      }
    }
    if (mode == SMDM_MODE_SPARSE) {
      if ((s = smdm_step(h, batch, desc, nullptr, nullptr, nullptr, st))) return s;
    } else {
      for (int b = 0; b < batch; ++b)
        if ((s = smdm_dense_step(h, &desc[b], nullptr, nullptr, nullptr, st))) return s;
    }
  }
  return SMDM_OK;
}

smdm_status smdm_forward_stepcausal(smdm_handle* h, const int32_t* d_ids, const int32_t* d_pos,
                                    const int32_t* d_type, const int32_t* d_label, int n,
                                    const int32_t* d_logit_rows, int n_rows, float* d_logits,
                                    cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  if (!d_ids || !d_pos || !d_type || !d_label || !d_logit_rows || !d_logits)
    return fail(h, SMDM_EINVAL, "null argument");
  if (n < 1 || n > h->cfg.max_rows || n_rows < 1 || n_rows > h->cfg.max_rows)
    return fail(h, SMDM_ESHAPE, "n=%d / n_rows=%d outside [1, max_rows]", n, n_rows);
  LinearPackArgs a{};
  a.mode = kPackTrain;
  a.n = n;
  a.seq = 0;
  a.vocab = h->cfg.vocab;
  a.emb_rows = emb_rows(&h->cfg);
  a.max_pos = h->L.max_pos;
  a.ids = d_ids;
  a.pos = d_pos;
  a.type = d_type;
  a.label = d_label;
  a.rows = h->rows;
  a.status = h->status();
  { Launch lg_(h, SMDM_K_PACK, st); CK(launch_pack_linear(a, st)); }
  { Launch lg_(h, SMDM_K_OTHER, st); CK(launch_gather_rows(d_logit_rows, n_rows, n, h->rows.qrow, h->status(), st)); }
  // bf16 models: per-row key bounds and per-query-tile key-tile lists, so the attention skips
  // the 128-key tiles in which no key is visible to a query tile
  const bool bound = h->bf16;
  int* tile_list = nullptr;
  int* tile_count = nullptr;
  if (bound) {
    Launch lg_(h, SMDM_K_OTHER, st);
    CK(launch_label_bounds(h->rows.type, h->rows.label, n, h->at<int>(h->L.lbound),
                           h->rows.kvlen, st));
    CK(launch_tile_lists(h->rows.type, h->rows.label, n, h->at<int>(h->L.tlist), &tile_list,
                         &tile_count, st));
  }
  FwdSpec f{};
  f.R = n;
  f.attn_mode = 1;
  f.attn_bound = bound;
  f.tile_list = tile_list;
  f.tile_count = tile_count;
  f.scratch_kv = true;
  f.n_seg = 1;
  f.seg[0] = AttnSeg{0, 0, n, n, 0};
  f.n_logit = n_rows;
  f.logits = d_logits;
  return forward(h, f, st);
}

smdm_status smdm_debug_mask(smdm_handle* h, const int32_t* d_type, const int32_t* d_label, int n,
                            uint32_t* d_bitmap, cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  if (!d_type || !d_label || !d_bitmap || n < 1) return fail(h, SMDM_EINVAL, "bad arguments");
  { Launch lg_(h, SMDM_K_OTHER, st); CK(launch_debug_mask(d_type, d_label, n, d_bitmap, st)); }
  return SMDM_OK;
}

smdm_status smdm_debug_rows(smdm_handle* h, int32_t* d_ids, int32_t* d_pos, int32_t* d_type,
                            int32_t* d_label, int* h_n, cudaStream_t st) {
  if (!h || !h_n) return SMDM_EINVAL;
  const int n = h->last_rows;
  *h_n = n;
  const size_t b = (size_t)n * 4;
  if (n > 0) {
    if (d_ids) CK(cudaMemcpyAsync(d_ids, h->rows.ids, b, cudaMemcpyDeviceToDevice, st));
    if (d_pos) CK(cudaMemcpyAsync(d_pos, h->rows.pos, b, cudaMemcpyDeviceToDevice, st));
    if (d_type) CK(cudaMemcpyAsync(d_type, h->rows.type, b, cudaMemcpyDeviceToDevice, st));
    if (d_label) CK(cudaMemcpyAsync(d_label, h->rows.label, b, cudaMemcpyDeviceToDevice, st));
  }
  return SMDM_OK;
}

smdm_status smdm_profile_begin(smdm_handle* h, int timed) {
  if (!h) return SMDM_EINVAL;
  Profiler& p = h->prof;
  p.on = true;
  p.timed = timed != 0;
  p.launches = 0;
  for (int i = 0; i < SMDM_K_CLASSES; ++i) p.class_launches[i] = 0;
  p.used = 0;
  return SMDM_OK;
}

smdm_status smdm_profile_end(smdm_handle* h, smdm_profile* out, cudaStream_t st) {
  if (!h || !out) return SMDM_EINVAL;
  Profiler& p = h->prof;
  CK(cudaStreamSynchronize(st));
  std::memset(out, 0, sizeof(*out));
  out->launches = p.launches;
  for (int i = 0; i < SMDM_K_CLASSES; ++i) out->class_launches[i] = p.class_launches[i];
  if (p.timed) {
    for (size_t i = 0; i < p.used; ++i) {
      float ms = 0.f;
      CK(cudaEventElapsedTime(&ms, p.ev[2 * i], p.ev[2 * i + 1]));
      out->class_ms[p.cls[i]] += ms;
    }
  }
  p.on = false;
  p.timed = false;
  p.used = 0;
  return SMDM_OK;
}

smdm_status smdm_device_status(smdm_handle* h, unsigned* h_bits, cudaStream_t st) {
  if (!h) return SMDM_EINVAL;
  uint32_t bits = 0;
  CK(cudaMemcpyAsync(&bits, h->status(), 4, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  CK(cudaMemsetAsync(h->status(), 0, 4, st));
  CK(cudaStreamSynchronize(st));
  if (h_bits) *h_bits = bits;
  if (bits & kStatusTimeout) return fail(h, SMDM_ETIMEOUT, "a device-side wait timed out");
  if (bits & kStatusBounds) return fail(h, SMDM_EDEVICE, "a device-side bounds check failed");
  return SMDM_OK;
}

}  // extern "C"

// ==============================================================================================
// Allocation-free training-form forward.
//
// Some callers cannot allocate device memory at the point where they need a forward pass: code
// running under an allocator that forbids new device allocations after start-up, a plug-in
// that only receives pointers from its host application, or a caller that is recording into a
// stream while a memory pool is frozen.  They cannot create a handle (its workspace is caller
// memory), so this entry point keeps all of its scratch — activations, the KV rows of the
// forward, the split-K partial sums and tile counters of the GEMMs, the LM-head statistics and
// the RoPE table — in one statically sized device array that the library carries with it.
// ==============================================================================================

#define SMDM_NOALLOC_SCRATCH_BYTES (16u << 20)   /* 16 MiB, held by every GPU that loads the library */
#define SMDM_NOALLOC_GEMM_CTAS 32                /* split-K width; bounds the partial-sum scratch */
#define SMDM_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char g_noalloc_scratch[SMDM_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoAllocDevice {
  bool ready = false;
  void* scratch = nullptr;          // device address of g_noalloc_scratch on this device
  smdm_handle* handle = nullptr;    // host-side bookkeeping reused by every call
};
NoAllocDevice g_noalloc[SMDM_NOALLOC_MAX_DEVICES];

__global__ void noalloc_rope_kernel(float2* tab, int max_pos, int half, double theta, int d_head) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)max_pos * half) return;
  const int p = (int)(i / half), j = (int)(i % half);
  const double ang = (double)p * pow(theta, -2.0 * j / d_head);
  double s, c;
  sincos(ang, &s, &c);
  tab[i] = make_float2((float)c, (float)s);
}

}  // namespace

extern "C" smdm_status smdm_forward_stepcausal_noalloc(
    const smdm_config* cfg, const smdm_weights* w, const int32_t* d_ids, const int32_t* d_pos,
    const int32_t* d_type, const int32_t* d_label, int n, const int32_t* d_logit_rows,
    int n_rows, float* d_logits, cudaStream_t st) {
  if (!config_ok(cfg, nullptr)) return SMDM_ESHAPE;
  if (!w || !w->emb || !w->final_norm || !w->lm_head || !w->attn_norm || !w->w_qkv || !w->w_o ||
      !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down)
    return SMDM_EINVAL;
  if (!d_ids || !d_pos || !d_type || !d_label || !d_logit_rows || !d_logits || n < 1 ||
      n_rows < 1)
    return SMDM_EINVAL;
  // every layer's weights, as smdm_create checks them (a null norm gain would otherwise reach
  // a kernel as a device address)
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!w->attn_norm[l] || !w->w_qkv[l] || !w->w_o[l] || !w->mlp_norm[l] || !w->w_gate[l] ||
        !w->w_up[l] || !w->w_down[l])
      return SMDM_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= SMDM_NOALLOC_MAX_DEVICES)
    return SMDM_ECUDA;
  NoAllocDevice& D = g_noalloc[dev];
  if (!D.ready) {
    // Once per device, with that device current: the host-side name of the array is only a
    // stand-in, so fetch its real device address.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SMDM_ECUDA;
    if (gemm_tc_set_smem_attr() != cudaSuccess || attn_tc_set_smem_attr() != cudaSuccess)
      return SMDM_ECUDA;
    D.scratch = p;
    D.handle = new smdm_handle();
    D.ready = true;
  }
  // The scratch is laid out like a one-sequence handle sized for exactly this call.
  smdm_config vc = *cfg;
  vc.max_batch = 1;
  vc.max_step_rows = 1;
  vc.max_rows = std::max(n, n_rows);
  const Layout L = make_layout(&vc, SMDM_NOALLOC_GEMM_CTAS, false);
  if (L.total > SMDM_NOALLOC_SCRATCH_BYTES) return SMDM_ESHAPE;
  smdm_handle* h = D.handle;
  h->cfg = vc;
  h->L = L;
  h->bf16 = vc.dtype == SMDM_BF16;
  h->ws = static_cast<uint8_t*>(D.scratch);
  h->emb = w->emb;
  h->final_norm = w->final_norm;
  h->lm_head = w->lm_head;
  const int nl = vc.n_layers;
  h->attn_norm.assign(w->attn_norm, w->attn_norm + nl);
  h->w_qkv.assign(w->w_qkv, w->w_qkv + nl);
  h->w_o.assign(w->w_o, w->w_o + nl);
  h->mlp_norm.assign(w->mlp_norm, w->mlp_norm + nl);
  h->w_gate.assign(w->w_gate, w->w_gate + nl);
  h->w_up.assign(w->w_up, w->w_up + nl);
  h->w_down.assign(w->w_down, w->w_down + nl);
  h->rows = rows_at(h, L.rows);
  h->aux = rows_at(h, L.aux);
  h->err.clear();
  // Every call starts from zero: tile counters, status word and the KV rows.
  if (cudaMemsetAsync(D.scratch, 0, L.total, st) != cudaSuccess) return SMDM_ECUDA;
  {
    const int half = vc.d_head / 2;
    const long long cnt = (long long)L.max_pos * half;
    noalloc_rope_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, st>>>(
        h->at<float2>(L.rope), L.max_pos, half, (double)vc.rope_theta, vc.d_head);
    if (cudaGetLastError() != cudaSuccess) return SMDM_ECUDA;
  }
  if (h->bf16) {
    const int d = vc.d_model, H = vc.n_heads, dh = vc.d_head;
    bool ok = prepare_weights16(h, w, st);
    const size_t MR = align_up((size_t)vc.max_rows, 256);
    ok &= encode_head_tiles(&h->tm_kscr, h->at<uint8_t>(L.kscr), dh, (uint64_t)H * MR, dh / 64);
    ok &= encode_head_tiles(&h->tm_vscr, h->at<uint8_t>(L.vscr), dh, (uint64_t)H * MR, dh / 64);
    ok &= encode_head_tiles(&h->tm_q, h->at<uint8_t>(L.q), d, MR, dh / 64);
    if (!ok) return SMDM_ECUDA;
  }
  return smdm_forward_stepcausal(h, d_ids, d_pos, d_type, d_label, n, d_logit_rows, n_rows,
                                 d_logits, st);
}
