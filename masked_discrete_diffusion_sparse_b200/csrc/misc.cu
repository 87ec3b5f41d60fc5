// The non-contraction kernels of the sparse sampling step:
//   pack        — builds the step's sparse row set (Sparse-LaViDa Sec. 3.1 / Appendix 7.2:
//                 |A| + |C| + m rows) and the per-row attention prefixes;
//   rmsnorm     — RMSNorm of fp32 models (optionally gathering the embedding rows first, or the
//                 decode-set rows for the LM head); bf16 models run it inside the GEMMs;
//   unmask      — confidence/argmax from the LM-head partials, top-n selection and the
//                 scatter of committed tokens into the grid (Figure-3 example, Sec. 3.2);
//   debug_mask  — the device step-causal predicate as a bitmap (test hook);
//   pack_switched — the row set of a step under the Table-6 speed switches;
//   label bounds, tile lists — the training form's key skipping (bf16 models);
#include <climits>

#include "misc.h"

namespace smdm {

// ------------------------------------------------------------------------------------------
// pack: one CTA per sequence of a sampling step.  Rows of sequence s, in order:
//   new cache  (tokens decoded at step k-1; id from the grid; CLEAN, label k-1),
//   queries    (the decode set C_k; id [MASK]; MASK, label k),
//   registers  (ids V+2+j, positions L+1+j; REG, label k), or in the length-token variant one
//              [LEN] row (id V+1, position L+1; REG, label k).
// kvlen: new-cache rows see the cache plus the new-cache rows; query and register rows see
// every row of the step.  slot: K/V of row i go to cache slot ctx + i.
// ------------------------------------------------------------------------------------------
__global__ void pack_step_kernel(PackArgs a) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const PackSeq& s = a.s[blockIdx.x];
  __shared__ int qbuf_count;
  __shared__ int warp_counts[32];
  const int tid = threadIdx.x;
  const int L = s.P + s.Lg;
  const int R = s.n_new + s.n_q + s.n_reg;
  const int q0 = s.row0 + s.n_new;
  if (s.qpos == nullptr) {
    // Block mode: C = every still-masked position of [block_lo, block_hi), in position order.
    if (tid == 0) qbuf_count = 0;
    __syncthreads();
    for (int base = s.block_lo; base < s.block_hi; base += blockDim.x) {
      const int p = base + tid;
      const bool masked = (p < s.block_hi) && (s.grid[p - s.P - 1] < 0);
      const unsigned ballot = __ballot_sync(0xffffffffu, masked);
      const int lane = tid & 31, w = tid >> 5;
      if (lane == 0) warp_counts[w] = __popc(ballot);
      __syncthreads();
      int before = 0;
      for (int i = 0; i < w; ++i) before += warp_counts[i];
      const int idx = qbuf_count + before + __popc(ballot & ((1u << lane) - 1u));
      if (masked && idx < s.n_q) {
        const int r = q0 + idx;
        a.rows.pos[r] = p;
        a.rows.qpos[s.qbase + idx] = p;
      }
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += warp_counts[i];
        qbuf_count += tot;
      }
      __syncthreads();
    }
    if (tid == 0 && qbuf_count != s.n_q) atomicOr(a.status, kStatusBounds);
  }
  for (int i = tid; i < R; i += blockDim.x) {
    const int r = s.row0 + i;
    int id, pos, type, label, kvlen;
    if (i < s.n_new) {
      pos = s.newpos[i];
      const bool ok = pos > s.P && pos <= L;
      id = ok ? s.grid[pos - s.P - 1] : 0;
      if (!ok || id < 0) {
        atomicOr(a.status, kStatusBounds);
        id = 0;
      }
      type = kTypeClean;
      label = s.label - 1;
      kvlen = s.ctx + s.n_new;
    } else if (i < s.n_new + s.n_q) {
      const int j = i - s.n_new;
      if (s.qpos != nullptr) {
        pos = s.qpos[j];
        a.rows.pos[r] = pos;
        a.rows.qpos[s.qbase + j] = pos;
      } else {
        pos = -1;   // written by the scan above
      }
      id = a.vocab;   // [MASK]
      type = kTypeMask;
      label = s.label;
      kvlen = s.ctx + R;
      a.rows.qrow[s.qbase + j] = r;
    } else {
      const int j = i - s.n_new - s.n_q;
      pos = L + 1 + j;
      id = a.vocab + 2 + j - a.len_token;
      type = kTypeReg;
      label = s.label;
      kvlen = s.ctx + R;
    }
    a.rows.ids[r] = id;
    if (pos >= 0) a.rows.pos[r] = pos;
    a.rows.type[r] = type;
    a.rows.label[r] = label;
    a.rows.seq[r] = s.seq;
    a.rows.slot[r] = s.ctx + i;
    a.rows.kvlen[r] = kvlen;
  }
  if (s.qpos != nullptr) {
    // checked: every explicit query position lies in the generated part and is still masked
    for (int j = tid; j < s.n_q; j += blockDim.x) {
      const int p = s.qpos[j];
      if (p <= s.P || p > L || s.grid[p - s.P - 1] >= 0) atomicOr(a.status, kStatusBounds);
    }
  }
}

// ------------------------------------------------------------------------------------------
// pack_switched: one CTA for one sequence (see PackSwArgs).  Slots and key prefixes:
//   prompt rows          slot i (rewrites the prompt's K/V), keys [0, P)
//   decoded rows, cached  the new-cache rows at slot P + dec_prev + i, keys [0, P + dec_prev + n_new)
//   decoded rows, not cached  every decoded token j at slot P + j, keys [0, P + (first j' whose
//                        step is later than j's))
//   C, other masks, tail rows  slots from base = P + dec_prev + n_new on, keys: all of them.
// ------------------------------------------------------------------------------------------
__global__ void pack_switched_kernel(PackSwArgs a) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  __shared__ int warp_counts[32];
  __shared__ int found;
  const int tid = threadIdx.x, nth = blockDim.x;
  const int P = a.P, L = a.P + a.Lg, k = a.label;
  const int n_dec = a.dec_prev + a.n_new;
  const int n_p = a.cache_prompt ? 0 : P;
  const int n_d = a.cache_res ? a.n_new : n_dec;
  const int r_c = n_p + n_d, r_e = r_c + a.n_q, r_t = r_e + a.n_extra;
  const int base = P + n_dec;
  const int all_keys = base + a.n_q + a.n_extra + a.n_tail;
  Rows rw = a.rows;
  auto put = [&](int r, int id, int pos, int type, int label, int slot, int kvlen) {
    rw.ids[r] = id;
    rw.pos[r] = pos;
    rw.type[r] = type;
    rw.label[r] = label;
    rw.seq[r] = a.seq;
    rw.slot[r] = slot;
    rw.kvlen[r] = kvlen;
  };
  auto token_at = [&](int pos) {
    const bool ok = pos > P && pos <= L;
    const int id = ok ? a.grid[pos - P - 1] : -1;
    if (id < 0) {
      atomicOr(a.status, kStatusBounds);
      return 0;
    }
    return id;
  };
  // the tokens committed at step k-1 join the decoded list; the decode set is marked
  for (int i = tid; i < a.n_new; i += nth) {
    a.dec_pos[a.dec_prev + i] = a.newpos[i];
    a.dec_lab[a.dec_prev + i] = k - 1;
  }
  for (int j = tid; j < a.n_q; j += nth) {
    const int p = a.qpos[j];
    if (p <= P || p > L || a.grid[p - P - 1] >= 0) {
      atomicOr(a.status, kStatusBounds);
    } else {
      a.qmark[p - P - 1] = k;
    }
  }
  if (tid == 0) found = 0;
  __syncthreads();
  for (int i = tid; i < n_p; i += nth) put(i, a.prompt[i], i + 1, kTypePrompt, 0, i, P);
  if (a.cache_res) {
    for (int i = tid; i < a.n_new; i += nth) {
      const int pos = a.dec_pos[a.dec_prev + i];
      put(n_p + i, token_at(pos), pos, kTypeClean, k - 1, P + a.dec_prev + i, base);
    }
  } else {
    for (int j = tid; j < n_dec; j += nth) {
      const int lab = a.dec_lab[j];
      int lo = j + 1, hi = n_dec;          // first entry decoded after step `lab`
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a.dec_lab[mid] <= lab) lo = mid + 1; else hi = mid;
      }
      const int pos = a.dec_pos[j];
      put(n_p + j, token_at(pos), pos, kTypeClean, lab, P + j, P + lo);
    }
  }
  for (int j = tid; j < a.n_q; j += nth) {
    const int pos = a.qpos[j];
    put(r_c + j, a.vocab, pos, kTypeMask, k, base + j, all_keys);
    rw.qrow[j] = r_c + j;
    rw.qpos[j] = pos;
  }
  for (int t = tid; t < a.n_tail; t += nth)
    put(r_t + t, a.vocab + 2 + t - a.len_token, L + 1 + t, kTypeReg, k,
        base + a.n_q + a.n_extra + t, all_keys);
  if (!a.truncate) {
    // every other still-masked position, in position order (block-wide stream compaction)
    const int lane = tid & 31, w = tid >> 5, nw = nth >> 5;
    for (int b0 = 0; b0 < a.Lg; b0 += nth) {
      const int i = b0 + tid;
      const bool extra = i < a.Lg && a.grid[i] < 0 && a.qmark[i] != k;
      const unsigned ballot = __ballot_sync(0xffffffffu, extra);
      if (lane == 0) warp_counts[w] = __popc(ballot);
      __syncthreads();
      int before = found;
      for (int x = 0; x < w; ++x) before += warp_counts[x];
      const int idx = before + __popc(ballot & ((1u << lane) - 1u));
      if (extra && idx < a.n_extra)
        put(r_e + idx, a.vocab, P + 1 + i, kTypeMask, k, base + a.n_q + idx, all_keys);
      __syncthreads();
      if (tid == 0)
        for (int x = 0; x < nw; ++x) found += warp_counts[x];
      __syncthreads();
    }
    if (tid == 0 && found != a.n_extra) atomicOr(a.status, kStatusBounds);
  }
}

// ------------------------------------------------------------------------------------------
// Training form, key bounds: kvlen[r] = 1 + the last key index row r may see under the
// step-causal rule, exact for any row order (rows grouped by step make the bounds triangular,
// so the attention kernel skips the key tiles after a query tile's last visible key).
//   lastc[l] / lastm[l]: last index of a clean / mask-or-register row with label l;
//   a clean query sees clean keys with label <= own: max over l' <= lq of lastc[l'];
//   a mask or register query: max(max over l' < lq of lastc[l'], lastm[lq]).
// Scratch: lastc, lastm, prefix (n + 1 each) and a flag, all -1 on entry; a label outside
// [0, n] sets the flag and every bound stays n.
// ------------------------------------------------------------------------------------------
__global__ void label_last_kernel(const int* type, const int* label, int n, int* lastc,
                                  int* lastm, int* flag) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int l = label[j], t = type[j];
  if (l < 0 || l > n) {
    atomicMax(flag, 1);
    return;
  }
  atomicMax((t == kTypePrompt || t == kTypeClean) ? &lastc[l] : &lastm[l], j);
}

// prefix[l] = max(lastc[0..l]); one CTA, block-wide scan in chunks with a running carry.
__global__ void label_prefix_kernel(const int* lastc, int n_labels, int* prefix) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  __shared__ int wmax[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) carry = -1;
  __syncthreads();
  for (int b0 = 0; b0 < n_labels; b0 += blockDim.x) {
    const int i = b0 + tid;
    int v = i < n_labels ? lastc[i] : -1;
    for (int o = 1; o < 32; o <<= 1) {              // inclusive warp scan (max)
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v = max(v, u);
    }
    if (lane == 31) wmax[w] = v;
    __syncthreads();
    int before = carry;
    for (int x = 0; x < w; ++x) before = max(before, wmax[x]);
    v = max(v, before);
    if (i < n_labels) prefix[i] = v;
    __syncthreads();
    if (tid == 0) {
      int c = carry;
      for (int x = 0; x < nw; ++x) c = max(c, wmax[x]);
      carry = c;
    }
    __syncthreads();
  }
}

__global__ void label_bound_kernel(const int* type, const int* label, int n, const int* lastm,
                                   const int* prefix, const int* flag, int* kvlen) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n) return;
  if (*flag > 0) {
    kvlen[r] = n;
    return;
  }
  const int l = label[r], t = type[r];
  const int hi = (t == kTypePrompt || t == kTypeClean)
                     ? prefix[l]
                     : max(l > 0 ? prefix[l - 1] : -1, lastm[l]);
  kvlen[r] = min(n, max(hi + 1, r + 1));   // every row sees itself
}

// ------------------------------------------------------------------------------------------
// Training form, key-tile lists: for every 128-row query tile, the 128-row key tiles that may
// hold a key visible to one of its rows (the keys are the forward's own rows).  A tile is
// summarised by the label ranges of its clean rows [cmin, cmax] and of its mask/register rows
// [mmin, mmax] (empty: INT_MAX / INT_MIN).  Key tile T may matter to query tile Q when
//   Q has clean rows and T a clean key with label <= Q's largest clean label, or
//   Q has mask/register rows and T a clean key with label < Q's largest such label, or T's
//   mask/register labels overlap Q's —
// a superset of the tiles the step-causal rule needs (each visible pair satisfies one of them).
// ------------------------------------------------------------------------------------------
__global__ void tile_summary_kernel(const int* type, const int* label, int n, int4* summary) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  __shared__ int s[4];
  if (threadIdx.x == 0) {
    s[0] = INT_MAX;
    s[1] = INT_MIN;
    s[2] = INT_MAX;
    s[3] = INT_MIN;
  }
  __syncthreads();
  const int r = blockIdx.x * 128 + threadIdx.x;
  if (r < n) {
    const int l = label[r], t = type[r];
    if (t == kTypePrompt || t == kTypeClean) {
      atomicMin(&s[0], l);
      atomicMax(&s[1], l);
    } else {
      atomicMin(&s[2], l);
      atomicMax(&s[3], l);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) summary[blockIdx.x] = make_int4(s[0], s[1], s[2], s[3]);
}

__global__ void tile_list_kernel(const int4* summary, int n_tiles, int* lists, int* counts) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  __shared__ int warp_counts[4];
  __shared__ int found;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int4 q = summary[blockIdx.x];
  int* list = lists + (size_t)blockIdx.x * n_tiles;
  if (tid == 0) found = 0;
  __syncthreads();
  for (int b0 = 0; b0 < n_tiles; b0 += 128) {
    const int t = b0 + tid;
    bool vis = false;
    if (t < n_tiles) {
      const int4 k = summary[t];
      vis = (k.x <= q.y) ||                                   // clean query, clean key
            (k.x < q.w) ||                                    // mask/register query, clean key
            (max(k.z, q.z) <= min(k.w, q.w));                 // same mask/register label
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, vis);
    if (lane == 0) warp_counts[w] = __popc(ballot);
    __syncthreads();
    int before = found;
    for (int x = 0; x < w; ++x) before += warp_counts[x];
    if (vis) list[before + __popc(ballot & ((1u << lane) - 1u))] = t;
    __syncthreads();
    if (tid == 0) found += warp_counts[0] + warp_counts[1] + warp_counts[2] + warp_counts[3];
    __syncthreads();
  }
  if (tid == 0) counts[blockIdx.x] = found;
}

// ------------------------------------------------------------------------------------------
// Prefill / dense / training-form rows: one thread per row.
__global__ void pack_linear_kernel(LinearPackArgs a) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n) return;
  int id, pos, type, label;
  if (a.mode == kPackPrefill || (a.mode == kPackPrefillGiven && i < a.P)) {
    id = a.prompt[i];
    pos = i + 1;
    type = kTypePrompt;
    label = 0;
  } else if (a.mode == kPackPrefillGiven) {
    // a given generation token: clean, block 0, computed and cached with the prompt
    id = a.given_tok[i - a.P];
    pos = a.given_pos[i - a.P];
    type = kTypeClean;
    label = 0;
    if (pos <= a.P || pos > a.P + a.Lg || id < 0 || id >= a.vocab) {
      atomicOr(a.status, kStatusBounds);
    } else {
      a.grid_out[pos - a.P - 1] = id;
    }
  } else if (a.mode == kPackDense) {
    pos = i + 1;
    if (i < a.P) {
      id = a.prompt[i];
      type = kTypePrompt;
    } else {
      const int g = a.grid[i - a.P];
      id = g < 0 ? a.vocab : g;
      type = g < 0 ? kTypeMask : kTypeClean;
      a.rows.qrow[i - a.P] = i;
      a.rows.qpos[i - a.P] = pos;
    }
    label = 0;
  } else {
    id = a.ids[i];
    pos = a.pos[i];
    type = a.type[i];
    label = a.label[i];
  }
  if (id < 0 || id >= a.emb_rows || pos < 0 || pos >= a.max_pos) {
    atomicOr(a.status, kStatusBounds);
    id = 0;
    pos = 0;
  }
  a.rows.ids[i] = id;
  a.rows.pos[i] = pos;
  a.rows.type[i] = type;
  a.rows.label[i] = label;
  a.rows.seq[i] = a.seq;
  a.rows.slot[i] = i;
  a.rows.kvlen[i] = a.n;
}

// Logit row j -> forward row src_rows[j]; a row index outside [0, n_fwd) is flagged in the
// status word and replaced by row 0, so that no later kernel reads outside the activations.
__global__ void gather_rows_kernel(const int* __restrict__ src_rows, int n, int n_fwd,
                                   int* __restrict__ qrow, uint32_t* status) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int r = src_rows[i];
  if (r < 0 || r >= n_fwd) {
    atomicOr(status, kStatusBounds);
    r = 0;
  }
  qrow[i] = r;
}

// ------------------------------------------------------------------------------------------
// RMSNorm: out[r] = x[src] / sqrt(mean(x[src]^2) + eps) * g.  With emb != nullptr the source
// row is first gathered from the embedding table into the fp32 residual stream x.
// ------------------------------------------------------------------------------------------
template <typename T> struct Vec4;
template <> struct Vec4<float> {
  using type = float4;
  static SMDM_DEV float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static SMDM_DEV void store(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
};
template <> struct Vec4<__nv_bfloat16> {
  static SMDM_DEV float4 load(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
  static SMDM_DEV void store(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

template <> struct Vec4<__half> {
  static SMDM_DEV void store(__half* p, float4 v) {
    __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

// One CTA of 256 threads per row; the row stays in registers (d <= 8192, d % 4 == 0).  T: gain
// and embedding dtype; OutT: output dtype.
template <typename T, typename OutT>
__global__ void __launch_bounds__(256) rmsnorm_kernel(NormArgs a) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  constexpr int kMaxV = 8;
  const int r = blockIdx.x;
  const int src = a.gather ? a.gather[r] : r;
  float* xr = a.x + (size_t)src * a.d;
  const T* g = reinterpret_cast<const T*>(a.gain);
  __shared__ float red[8];
  const int d4 = a.d >> 2;
  float4 v[kMaxV];
  float ss = 0.f;
  const T* e = a.emb ? reinterpret_cast<const T*>(a.emb) + (size_t)a.ids[src] * a.d : nullptr;
#pragma unroll
  for (int t = 0; t < kMaxV; ++t) {
    const int i4 = threadIdx.x + t * 256;
    if (i4 < d4) {
      if (e) {
        v[t] = Vec4<T>::load(e + 4 * i4);
        *reinterpret_cast<float4*>(xr + 4 * i4) = v[t];
      } else {
        v[t] = *reinterpret_cast<const float4*>(xr + 4 * i4);
      }
      ss += v[t].x * v[t].x + v[t].y * v[t].y + v[t].z * v[t].z + v[t].w * v[t].w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += red[i];
  const float rstd = rsqrtf(tot / (float)a.d + a.eps);
  OutT* out = reinterpret_cast<OutT*>(a.out) + (size_t)r * a.d;
#pragma unroll
  for (int t = 0; t < kMaxV; ++t) {
    const int i4 = threadIdx.x + t * 256;
    if (i4 < d4) {
      const float4 gg = Vec4<T>::load(g + 4 * i4);
      Vec4<OutT>::store(out + 4 * i4, make_float4(v[t].x * rstd * gg.x, v[t].y * rstd * gg.y,
                                               v[t].z * rstd * gg.z, v[t].w * rstd * gg.w));
    }
  }
}

// ------------------------------------------------------------------------------------------
// unmask: one CTA per sequence.
// ------------------------------------------------------------------------------------------
__global__ void unmask_kernel(UnmaskArgs a) {
  griddep_launch();
  griddep_wait();   // launched with programmatic dependent launch
  const UnmaskSeq& s = a.s[blockIdx.x];
  extern __shared__ float sh[];
  float* conf = sh;                                     // [n_q]
  int* tok = reinterpret_cast<int*>(sh + s.n_q);        // [n_q]
  int* commit = tok + s.n_q;                            // [n_q]
  const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  constexpr int kPer = 8;   // partials per lane held in registers (n_vt <= 256: V <= 32768)
  for (int j = threadIdx.x >> 5; j < s.n_q; j += nwarps) {
    const int lr = s.dense ? (a.qpos_of[s.qbase + j] - s.P - 1) : (s.qbase + j);
    const float* pm = a.pmax + (size_t)(s.lbase + lr) * a.n_vt;
    const float* ps = a.psum + (size_t)(s.lbase + lr) * a.n_vt;
    const int* pa = a.parg + (size_t)(s.lbase + lr) * a.n_vt;
    float M = -INFINITY;
    int arg = 0x7fffffff;
    float z = 0.f;
    if (a.n_vt <= 32 * kPer) {
      // every load of the row in flight at once (one round trip), then reduce from registers
      float vm[kPer], vs[kPer];
      int va[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int t = lane + 32 * i;
        const bool ok = t < a.n_vt;
        vm[i] = ok ? pm[t] : -INFINITY;
        vs[i] = ok ? ps[t] : 0.f;
        va[i] = ok ? pa[t] : 0x7fffffff;
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (vm[i] > M) { M = vm[i]; arg = va[i]; }   // tiles in vocab order: first max = lowest id
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oM = __shfl_xor_sync(0xffffffffu, M, o);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
        if (oM > M || (oM == M && oa < arg)) { M = oM; arg = oa; }
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (vs[i] > 0.f) z += vs[i] * __expf(vm[i] - M);
    } else {
      for (int t = lane; t < a.n_vt; t += 32) {
        const float v = pm[t];
        if (v > M) { M = v; arg = pa[t]; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oM = __shfl_xor_sync(0xffffffffu, M, o);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
        if (oM > M || (oM == M && oa < arg)) { M = oM; arg = oa; }
      }
      for (int t = lane; t < a.n_vt; t += 32) z += ps[t] * __expf(pm[t] - M);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) {
      conf[j] = 1.f / z;
      tok[j] = arg;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < s.n_q; j += blockDim.x) {
    int c = 1;
    if (s.policy == 1) {
      int rank = 0;
      const float cj = conf[j];
      for (int i = 0; i < s.n_q; ++i) rank += (conf[i] > cj) || (conf[i] == cj && i < j);
      c = rank < s.n_commit;
    }
    commit[j] = c;
    if (a.tok_out) a.tok_out[s.qbase + j] = tok[j];
    if (a.conf_out) a.conf_out[s.qbase + j] = conf[j];
  }
  __syncthreads();
  // Committed rows keep their row order: index = number of committed rows before them
  // (block-wide exclusive scan over the commit flags, one tile of blockDim rows at a time).
  __shared__ int warp_sums[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < s.n_q; base += blockDim.x) {
    const int j = base + threadIdx.x;
    const int c = (j < s.n_q) ? commit[j] : 0;
    const unsigned ballot = __ballot_sync(0xffffffffu, c);
    if (lane == 0) warp_sums[threadIdx.x >> 5] = __popc(ballot);
    __syncthreads();
    int before = carry;
    for (int w = 0; w < (int)(threadIdx.x >> 5); ++w) before += warp_sums[w];
    before += __popc(ballot & ((1u << lane) - 1u));
    if (c) {
      const int p = a.qpos_of[s.qbase + j];
      if (p <= s.P || p > s.P + s.Lg) {
        atomicOr(a.status, kStatusBounds);
      } else {
        s.grid[p - s.P - 1] = tok[j];
        if (s.newpos) s.newpos[before] = p;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int w = 0; w < nwarps; ++w) t += warp_sums[w];
      carry += t;
    }
    __syncthreads();
  }
}

__global__ void debug_mask_kernel(const int* type, const int* label, int n, uint32_t* bitmap) {
  const int i = blockIdx.x;
  const int words = (n + 31) / 32;
  for (int w = threadIdx.x; w < words; w += blockDim.x) {
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int j = w * 32 + b;
      if (j < n && step_causal_allowed(type[i], label[i], type[j], label[j])) bits |= 1u << b;
    }
    bitmap[(size_t)i * words + w] = bits;
  }
}

__global__ void fill_i32_kernel(int* p, int n, int v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
cudaError_t launch_pack_step(const PackArgs& a, cudaStream_t st) {
  return launch_pdl(pack_step_kernel, dim3(a.n_seq), dim3(256), 0, st, 1, a);
}
cudaError_t launch_pack_linear(const LinearPackArgs& a, cudaStream_t st) {
  if (a.n <= 0) return cudaSuccess;
  return launch_pdl(pack_linear_kernel, dim3((a.n + 255) / 256), dim3(256), 0, st, 1, a);
}
cudaError_t launch_pack_switched(const PackSwArgs& a, cudaStream_t st) {
  return launch_pdl(pack_switched_kernel, dim3(1), dim3(512), 0, st, 1, a);
}
cudaError_t launch_label_bounds(const int* type, const int* label, int n, int* scratch,
                                int* kvlen, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  int* lastc = scratch;
  int* lastm = lastc + (n + 1);
  int* prefix = lastm + (n + 1);
  int* flag = prefix + (n + 1);
  cudaError_t e = launch_fill_i32(scratch, 3 * (n + 1) + 1, -1, st);
  if (e != cudaSuccess) return e;
  e = launch_pdl(label_last_kernel, dim3((n + 255) / 256), dim3(256), 0, st, 1, type, label, n,
                 lastc, lastm, flag);
  if (e != cudaSuccess) return e;
  e = launch_pdl(label_prefix_kernel, dim3(1), dim3(1024), 0, st, 1, (const int*)lastc, n + 1,
                 prefix);
  if (e != cudaSuccess) return e;
  return launch_pdl(label_bound_kernel, dim3((n + 255) / 256), dim3(256), 0, st, 1, type, label,
                    n, (const int*)lastm, (const int*)prefix, (const int*)flag, kvlen);
}
cudaError_t launch_tile_lists(const int* type, const int* label, int n, int* scratch,
                              int** lists, int** counts, cudaStream_t st) {
  const int T = (n + 127) / 128;
  int4* summary = reinterpret_cast<int4*>(scratch);
  *counts = scratch + 4 * T;
  *lists = *counts + T;
  if (n <= 0) return cudaSuccess;
  cudaError_t e = launch_pdl(tile_summary_kernel, dim3(T), dim3(128), 0, st, 1, type, label, n,
                             summary);
  if (e != cudaSuccess) return e;
  return launch_pdl(tile_list_kernel, dim3(T), dim3(128), 0, st, 1, (const int4*)summary, T,
                    *lists, *counts);
}
cudaError_t launch_gather_rows(const int* src, int n, int n_fwd, int* qrow, uint32_t* status,
                               cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(gather_rows_kernel, dim3((n + 255) / 256), dim3(256), 0, st, 1, src, n, n_fwd, qrow,
                    status);
}
template <typename T, typename OutT>
cudaError_t launch_rmsnorm(const NormArgs& a, int rows, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_pdl(rmsnorm_kernel<T, OutT>, dim3(rows), dim3(256), 0, st, 1, a);
}
template cudaError_t launch_rmsnorm<float, float>(const NormArgs&, int, cudaStream_t);
template cudaError_t launch_rmsnorm<__nv_bfloat16, __half>(const NormArgs&, int, cudaStream_t);

// bf16 -> fp16, 8 elements per thread when the pointers allow 16-byte accesses
__global__ void convert_bf16_f16_kernel(const __nv_bfloat16* __restrict__ src,
                                        __half* __restrict__ dst, size_t n, uint32_t* status) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  bool over = false;
  if (i + 8 <= n && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0) {
    const uint4 u = *reinterpret_cast<const uint4*>(src + i);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint4 o;
    __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b[k]);
      over |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
      h[k] = __floats2half2_rn(f.x, f.y);
    }
    *reinterpret_cast<uint4*>(dst + i) = o;
  } else {
    for (size_t j = i; j < n && j < i + 8; ++j) {
      const float f = __bfloat162float(src[j]);
      over |= fabsf(f) > 65504.f;
      dst[j] = __float2half_rn(f);
    }
  }
  if (over) atomicOr(status, kStatusRange);
}

cudaError_t launch_convert_bf16_f16(const __nv_bfloat16* src, __half* dst, size_t n,
                                    uint32_t* status, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t threads = (n + 7) / 8;
  convert_bf16_f16_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(src, dst, n, status);
  return cudaGetLastError();
}

cudaError_t launch_unmask(const UnmaskArgs& a, int max_nq, cudaStream_t st) {
  const size_t smem = (size_t)max_nq * 12;
  return launch_pdl(unmask_kernel, dim3(a.n_seq), dim3(1024), smem, st, 1, a);
}
cudaError_t launch_debug_mask(const int* type, const int* label, int n, uint32_t* bitmap,
                              cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  debug_mask_kernel<<<n, 128, 0, st>>>(type, label, n, bitmap);
  return cudaGetLastError();
}
cudaError_t launch_fill_i32(int* p, int n, int v, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  fill_i32_kernel<<<(n + 255) / 256, 256, 0, st>>>(p, n, v);
  return cudaGetLastError();
}

}  // namespace smdm
