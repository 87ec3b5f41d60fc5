// Step-causal attention of the sparse sampling step (Sparse-LaViDa Figure-3 example and
// Sec. 3.3).  Two ways of stating which keys a query row sees:
//   prefix mode — the row sees keys [0, kvlen[row]) of its sequence's KV cache.  At a sampling
//     step the cache holds [prompt + clean tokens | new-cache rows | masks | registers], so the
//     step-causal rule is exactly a per-row prefix: new-cache rows stop after the new-cache
//     rows, mask and register rows see everything.  Prefill and the dense comparator use a
//     common prefix for all rows.
//   label mode — the training-form rule evaluated per (query, key) from row types and step
//     labels; keys are the rows of the same forward.
//
// bf16 models (fp16 operands): one CTA per (sequence, 128-row query tile, head, key split).  Warp 0 streams Q and
// K/V tiles with TMA (one copy per 128-row head tile), warp 1 issues tcgen05.mma (S = Q K^T
// into one of two TMEM buffers, O += P V into a TMEM accumulator), warps 2-5 own one query row
// per thread: masking, online softmax in the exp2 domain, P (fp16) written into tensor memory
// over the columns of the S buffer it came from (the P V product reads its A operand from
// TMEM), final 1/l scaling (or the unnormalised partial for the combine).  The running maximum is
// only moved (and O rescaled) when it grows by more than 2^8, so most tiles skip the rescale;
// the result is exact because numerator and denominator share the reference maximum.
// The bounded label-mode instantiation (the training form of bf16 models) scans only the key
// tiles listed for each query tile.
// fp32 path: one warp per (row, head), SIMT.
#include <algorithm>

#include "attn.h"

namespace smdm {

constexpr int kAttnThreads = 320;   // warp 0 loads, warp 1 MMA, warps 2-9 two softmax groups

struct AttnDev {
  int mode;        // 0 prefix, 1 label
  int H, dh, d_model, layer;
  int n_seg;
  AttnSeg seg[kMaxBatch];         // seg[s].tile0 = first grid block of segment s
  const int* kvlen;
  const int* type;
  const int* label;
  long long cache_rows_per_seq;   // rows of the 2-D cache map per sequence (n_layers*H*cap)
  int cap;
  float scale_log2;               // log2(e) / sqrt(dh)
  int nstages;
  int q_off, k_off, v_off, bar_off, stage_bytes;
  void* out;                      // [rows][d_model] fp16
  uint32_t* status;
  int nsplit;                     // key splits per query tile
  int rows_total;
  float* part_o;                  // [nsplit][rows_total][d_model]
  float* part_ml;                 // [nsplit][rows_total][H][2]
  const int* tile_list;           // bounded label mode: [query tile][n_ktiles] key tiles
  const int* tile_count;          // [query tile] listed key tiles
  int n_ktiles;
};

// 2^x with the hardware approximation (PTX ex2.approx.ftz.f32).
SMDM_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

SMDM_DEV uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// DH: head dim (64 or 128) as a compile-time constant so that every MMA issue sequence is
// straight-line code (control flow between tcgen05.mma instructions stalls the issue).
// kBound (label mode, training form from row 0): kvlen[row] bounds the keys a row may see, and
// a query tile scans only the key tiles listed for it (tile_list / tile_count).
//
// Two softmax groups take the key tiles in turn (group g: tiles g, g + 2, ...), each with its
// own S/P buffer (tensor-memory columns [128 g, 128 g + 128)), its own O accumulator (columns
// 256 + g DH ...) and its own running maximum and sum, so that one group's exponentials overlap
// the other's and the tensor core's work.  At the end the two partial results of every row are
// merged exactly as two key splits are: O = 2^(m0 - M) O0 + 2^(m1 - M) O1 over the same sum.
template <int DH, bool kBound = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnDev a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* Qs = smem + a.q_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  const int NS = a.nstages;
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* k_empty = v_full + NS;    // [NS] K stage free: the S = Q K^T product completed
  uint64_t* v_empty = k_empty + NS;   // [NS] V stage free: the P V product completed
  uint64_t* s_full = v_empty + NS;    // [2] per group: S of its current tile is in its buffer
  uint64_t* s_free = s_full + 2;      // [2] per group: S read (the buffer may take the next S
                                      //     once the group's P V product has been issued)
  uint64_t* p_full = s_free + 2;      // [2] per group: P of its current tile written
  uint64_t* pv_done = p_full + 2;     // [2] per group: the P V product of its tile completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(pv_done + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x / a.nsplit, split = blockIdx.x % a.nsplit, h = blockIdx.y;
  int si = 0;
  while (si + 1 < a.n_seg && a.seg[si + 1].tile0 <= blk) ++si;
  const AttnSeg sg = a.seg[si];
  const int tile = blk - sg.tile0;
  const int qrow0 = sg.row0 + tile * 128;            // first forward row of this tile
  const int nq = min(128, sg.rows - tile * 128);     // valid query rows
  const int nkeys = sg.nkeys;
  // key tiles to scan: all of [0, nkeys), or with kBound the listed ones of this query tile
  const int* tlist = nullptr;
  int nkv_all = (nkeys + 127) / 128;
  if constexpr (kBound) {
    griddep_wait();   // the lists come from earlier kernels
    const int tq = qrow0 >> 7;   // training form: one segment starting at row 0
    tlist = a.tile_list + (size_t)tq * a.n_ktiles;
    nkv_all = a.tile_count[tq];
  }
  const int j0 = split * nkv_all / a.nsplit, j1 = (split + 1) * nkv_all / a.nsplit;
  const int nkv = j1 - j0;                           // key tiles of this split
  constexpr int dh = DH;
  if (nkv == 0) {
    griddep_launch();
    griddep_wait();
    // empty split: contribute nothing to the combine
    for (int r = threadIdx.x; r < nq; r += blockDim.x) {
      float* ml = a.part_ml + (((size_t)split * a.rows_total + qrow0 + r) * a.H + h) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
    return;
  }
  constexpr int nsub = dh / 64;                      // 64-wide chunks of the head dim
  const long long cache_base = (long long)sg.seq * a.cache_rows_per_seq +
                               ((long long)a.layer * a.H + h) * a.cap;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&pv_done[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const uint32_t t_o0 = tbase + 256;   // O accumulator of group g: columns [256 + g dh, ...)
  griddep_launch();
  griddep_wait();   // q, the KV cache and the row metadata come from earlier kernels

  if (warp == 0) {
    // Two producer lanes fill the K and the V ring independently: a K stage is free again as
    // soon as its S = Q K^T product completes, a V stage only after the P V product, so K loads
    // run ahead of V loads.
    if (lane < 2) {
      const bool is_k = lane == 0;
      const uint64_t pol_kv = policy_evict_last();
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      uint64_t* full_b = is_k ? k_full : v_full;
      uint64_t* empty_b = is_k ? k_empty : v_empty;
      const int off = is_k ? a.k_off : a.v_off;
      if (is_k) {
        mbar_arrive_expect_tx(q_full, 128 * dh * 2);
        tma_load_3d(Qs, &tmQ, q_full, 0, qrow0, h * nsub, policy_evict_normal());   // nsub [128][64] sub-tiles
      }
      auto tile_y = [&](int jj) {
        const int kt = kBound ? tlist[j0 + jj] : (j0 + jj);
        return (int)(cache_base + (long long)kt * 128);
      };
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&empty_b[stage], phase ^ 1, abort_flag, a.status)) break;
        uint8_t* dst = smem + off + stage * a.stage_bytes;
        mbar_arrive_expect_tx(&full_b[stage], 128 * dh * 2);
        tma_load_3d(dst, tm, &full_b[stage], 0, tile_y(j), 0, pol_kv);
        if (++stage == NS) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16(128, 128, 0, 0);   // q, K fp16
      const uint32_t idesc_o = idesc_f16(128, dh, 0, 1);   // P, V fp16; V is MN-major
      const uint32_t q_addr = smem_u32(Qs);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.status);
      int stage = 0;
      uint32_t phase = 0;
      int pstage = 0;
      uint32_t pphase = 0;
      // S(j) = Q K(j)^T into the buffer of group j & 1, once that group has read S(j - 2)
      auto issue_s = [&](int j) -> bool {
        const int b = j & 1;
        if (!mbar_wait(&k_full[stage], phase, abort_flag, a.status)) return false;
        if (!mbar_wait(&s_free[b], ((j >> 1) & 1) ^ 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + a.k_off + stage * a.stage_bytes);
#pragma unroll
        for (int kk = 0; kk < dh / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16(tbase + b * 128, sdesc_sw128(q_addr + off, 16, 1024),
                   sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[b]);
        umma_commit(&k_empty[stage]);
        if (++stage == NS) { stage = 0; phase ^= 1; }
        return true;
      };
      // Issue order follows the order in which the groups finish their tiles: after group g
      // publishes P(j), its product O_g += P(j) V(j) and then its next score tile S(j + 2).
      // (Issuing S(j) before P(j - 1) V(j - 1) made each group wait for the other's softmax,
      // so the two never overlapped.)
      if (ok) ok = issue_s(0);
      if (ok && nkv > 1) ok = issue_s(1);
      for (int j = 0; ok && j < nkv; ++j) {
        // O_g += P_j V_j (g = j & 1), P from tensor memory: it occupies the first 64 columns of
        // the group's S buffer (two fp16 keys per column); the next S written there is issued
        // after this product and the tensor core keeps issue order
        const int pb = j & 1;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1, abort_flag, a.status)) break;
        if (!mbar_wait(&v_full[pstage], pphase, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + a.v_off + pstage * a.stage_bytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_ts(t_o0 + pb * dh, tbase + pb * 128 + kk * 8,
                      sdesc_sw128(v_addr + kk * 2048, 16384, 1024), idesc_o,
                      (j >= 2 || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[pstage]);
        umma_commit(&pv_done[pb]);
        if (++pstage == NS) { pstage = 0; pphase ^= 1; }
        if (j + 2 < nkv && !issue_s(j + 2)) break;
      }
    }
  } else {
    // Softmax groups: warps 2-5 (g = 0) and 6-9 (g = 1); a thread owns query row em of the tile
    // (TMEM lane quarter = warp % 4).
    const int g = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int em = q4 * 32 + lane;
    const int row = qrow0 + em;
    const bool valid = em < nq;
    const uint32_t lane_off = uint32_t(q4 * 32) << 16;
    const uint32_t t_s = tbase + lane_off + g * 128;   // this group's S / P buffer
    const uint32_t t_og = t_o0 + lane_off + g * dh;    // this group's O accumulator
    int kv_lim = 0, tq = 0, lq = 0;
    if (valid) {
      if (a.mode == 0) kv_lim = a.kvlen[row];
      else { tq = a.type[row]; lq = a.label[row]; kv_lim = kBound ? a.kvlen[row] : nkeys; }
    }
    float m_ref = -INFINITY, l = 0.f;
    const bool warp_any = __any_sync(0xffffffffu, valid);
    const int n_mine = (nkv - g + 1) >> 1;             // tiles g, g + 2, ... below nkv
    for (int it = 0; it < n_mine; ++it) {
      const int j = g + 2 * it;
      if (!mbar_wait(&s_full[g], it & 1, abort_flag, a.status)) break;
      tc_fence_after();
      if (!warp_any) {
        // no valid query row in this warp: keep the barrier protocol, skip the math
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[g]);
        // signal P only once the P buffer is free (the group's previous product completed), so
        // that no arrival can land in a later phase of p_full (these P rows are never read back)
        if (it >= 1 && !mbar_wait(&pv_done[g], (it - 1) & 1, abort_flag, a.status)) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g]);
        continue;
      }
      const int key0 = (kBound ? tlist[j0 + j] : (j0 + j)) * 128;
      // visibility of the 128 keys as four 32-bit masks (registers only, no local arrays)
      uint32_t mw[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int kb = key0 + w * 32;
        uint32_t bits;
        if (a.mode == 0) {
          const int n_ok = min(max(kv_lim - kb, 0), 32);
          bits = n_ok == 32 ? 0xffffffffu : ((1u << n_ok) - 1u);
        } else {
          bits = 0;
          for (int bb = 0; bb < 32; ++bb) {
            const int key = kb + bb;
            if (key < kv_lim && step_causal_allowed(tq, lq, a.type[key], a.label[key]))
              bits |= 1u << bb;
          }
        }
        mw[w] = valid ? bits : 0xffffffffu;   // rows past the tile's end: results unused
      }
      // Most tiles are visible to every row of the warp: then the per-key tests drop out of
      // both passes (the softmax is bound by its instruction count, not by latency).
      const bool full = __all_sync(0xffffffffu, (mw[0] & mw[1] & mw[2] & mw[3]) == 0xffffffffu);
      // pass 1: row maximum over the visible keys (two 64-column halves) with eight
      // independent partial maxima (no 128-long dependent chain)
      float mxp[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mxp[t] = -INFINITY;
      // the two halves as a loop, not unrolled: every CTA runs its first tile from a cold
      // instruction cache (measured ≈4 µs of the first tile), so half the code costs less
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float sv[64];
        tmem_ld64(t_s + hh * 64, sv);
        if (full) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mxp[c & 7] = fmaxf(mxp[c & 7], sv[c]);
        } else {
          const uint32_t w0 = hh ? mw[2] : mw[0], w1 = hh ? mw[3] : mw[1];
#pragma unroll
          for (int c = 0; c < 64; ++c)
            mxp[c & 7] = fmaxf(mxp[c & 7], (((c < 32 ? w0 : w1) >> (c & 31)) & 1u) ? sv[c] : -INFINITY);
        }
      }
      float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                       fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      mx *= a.scale_log2;
      float alpha = 1.f;
      if (mx > m_ref + 8.f) {          // move the reference maximum (also the first time)
        alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mx);
        m_ref = mx;
      }
      // the P buffer (and O_g) were last used by the group's previous P V product
      if (it >= 1 && !mbar_wait(&pv_done[g], (it - 1) & 1, abort_flag, a.status)) break;
      tc_fence_after();
      if (__any_sync(0xffffffffu, alpha != 1.f) && it >= 1) {
        for (int c = 0; c < dh / 16; ++c) {
          float o[16];
          tmem_ld16(t_og + c * 16, o);
#pragma unroll
          for (int t = 0; t < 16; ++t) o[t] *= alpha;
          tmem_st16(t_og + c * 16, o);
        }
      }
      // pass 2: P = 2^(s*scale - m_ref) in fp16, two keys per 32-bit column, over the first 64
      // columns of the S buffer (half hh -> columns 32 hh .. 32 hh + 31, after the S columns
      // 64 hh .. 64 hh + 63 it replaces have been read)
      const float mref_eff = (m_ref == -INFINITY) ? 0.f : m_ref;
      float rsp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // partial sums of P
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float sv[64];
        tmem_ld64(t_s + hh * 64, sv);
        uint32_t pk[32];
        if (full) {
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            float p2[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              p2[t] = ex2_approx(fmaf(sv[c2 * 2 + t], a.scale_log2, -mref_eff));
              rsp[(c2 & 3) * 2 + t] += p2[t];
            }
            pk[c2] = pack_f16x2(p2[0], p2[1]);
          }
        } else {
          const uint32_t w0 = hh ? mw[2] : mw[0], w1 = hh ? mw[3] : mw[1];
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            float p2[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int c = c2 * 2 + t;
              const bool vis = (((c < 32 ? w0 : w1) >> (c & 31)) & 1u) != 0;
              p2[t] = vis ? ex2_approx(fmaf(sv[c], a.scale_log2, -mref_eff)) : 0.f;
              rsp[(c2 & 3) * 2 + t] += p2[t];
            }
            pk[c2] = pack_f16x2(p2[0], p2[1]);
          }
        }
        tmem_st32_nowait(t_s + hh * 32, pk);
      }
      tmem_wait_st();
      const float rs = ((rsp[0] + rsp[1]) + (rsp[2] + rsp[3])) + ((rsp[4] + rsp[5]) + (rsp[6] + rsp[7]));
      l = l * alpha + rs;
      // S read and P written (tcgen05.st completed)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[g]);
        mbar_arrive(&p_full[g]);
      }
    }
    // The group's last product; after the barrier below every product of the CTA has completed
    // (the group holding the final tile waited for it, and a commit covers all earlier MMAs),
    // so the Q tile's shared memory is free for the exchange of (m, l).
    if (n_mine > 0) mbar_wait(&pv_done[g], (n_mine - 1) & 1, abort_flag, a.status);
    named_bar_sync(1, 256);
    tc_fence_after();
    float* xch = reinterpret_cast<float*>(Qs);   // [group][row][m, l]
    xch[(g * 128 + em) * 2 + 0] = m_ref;
    xch[(g * 128 + em) * 2 + 1] = l;
    named_bar_sync(2, 256);
    const float m_x = xch[((g ^ 1) * 128 + em) * 2 + 0];
    const float l_x = xch[((g ^ 1) * 128 + em) * 2 + 1];
    const float m0 = g ? m_x : m_ref, l0 = g ? l_x : l;
    const float m1 = g ? m_ref : m_x, l1 = g ? l : l_x;
    const float M = fmaxf(m0, m1);
    const float a0 = (M == -INFINITY || m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
    const float a1 = (M == -INFINITY || m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
    const float L = a0 * l0 + a1 * l1;
    // a group without tiles never wrote its accumulator: leave it out (its a is 0)
    const bool use1 = nkv >= 2;
    // group g writes the head-dim columns [g dh/2, (g + 1) dh/2) of the merged row
    constexpr int half = dh / 2;
    const uint32_t t_c0 = t_o0 + lane_off + g * half;
    if (a.nsplit == 1) {
      const float inv = (L > 0.f) ? 1.f / L : 0.f;
      const float f0 = a0 * inv, f1 = a1 * inv;
      __half* out = reinterpret_cast<__half*>(a.out) + (size_t)row * a.d_model + h * dh + g * half;
      for (int c = 0; c < half / 16; ++c) {
        float o[16], o1[16];
        tmem_ld16(t_c0 + c * 16, o);
        if (use1) tmem_ld16(t_c0 + dh + c * 16, o1);
        else {
#pragma unroll
          for (int t = 0; t < 16; ++t) o1[t] = 0.f;
        }
        if (valid) {
          uint32_t w[8];
#pragma unroll
          for (int t = 0; t < 8; ++t)
            w[t] = pack_f16x2(o[2 * t] * f0 + o1[2 * t] * f1, o[2 * t + 1] * f0 + o1[2 * t + 1] * f1);
          reinterpret_cast<uint4*>(out + c * 16)[0] = make_uint4(w[0], w[1], w[2], w[3]);
          reinterpret_cast<uint4*>(out + c * 16)[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    } else {
      float* po = a.part_o + ((size_t)split * a.rows_total + row) * a.d_model + h * dh + g * half;
      for (int c = 0; c < half / 16; ++c) {
        float o[16], o1[16];
        tmem_ld16(t_c0 + c * 16, o);
        if (use1) tmem_ld16(t_c0 + dh + c * 16, o1);
        else {
#pragma unroll
          for (int t = 0; t < 16; ++t) o1[t] = 0.f;
        }
        if (valid) {
#pragma unroll
          for (int t = 0; t < 16; t += 4)
            *reinterpret_cast<float4*>(po + c * 16 + t) =
                make_float4(o[t] * a0 + o1[t] * a1, o[t + 1] * a0 + o1[t + 1] * a1,
                            o[t + 2] * a0 + o1[t + 2] * a1, o[t + 3] * a0 + o1[t + 3] * a1);
        }
      }
      if (valid && g == 0) {
        float* ml = a.part_ml + (((size_t)split * a.rows_total + row) * a.H + h) * 2;
        ml[0] = M;
        ml[1] = L;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Merge the key splits: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.  One warp per
// (row, head).
__global__ void attn_combine_kernel(const float* __restrict__ part_o,
                                    const float* __restrict__ part_ml, int nsplit, int rows,
                                    int H, int dh, int d_model, __half* __restrict__ out) {
  griddep_launch();
  griddep_wait();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows * H) return;
  const int row = w / H, h = w % H;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s)
    M = fmaxf(M, part_ml[(((size_t)s * rows + row) * H + h) * 2]);
  float den = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int per = dh / 32;
  for (int s = 0; s < nsplit; ++s) {
    const float* ml = part_ml + (((size_t)s * rows + row) * H + h) * 2;
    const float m = ml[0];
    if (m == -INFINITY) continue;
    const float wgt = exp2f(m - M);
    den += wgt * ml[1];
    const float* po = part_o + ((size_t)s * rows + row) * d_model + h * dh;
    for (int t = 0; t < per; ++t) acc[t] += wgt * po[lane * per + t];
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int t = 0; t < per; ++t)
    out[(size_t)row * d_model + h * dh + lane * per + t] = __float2half_rn(acc[t] * inv);
}

// ------------------------------------------------------------------------------------------
// SIMT attention (fp32 models): one warp per (row, head); lanes split the head dimension.
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void attn_simt_kernel(const T* __restrict__ q, T* __restrict__ out, KVAddr kv,
                                 AttnSimtArgs a) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int row = warp_global / a.H, h = warp_global % a.H;
  if (row >= a.rows) return;
  const int dh = a.dh;
  const int per = dh / 32;   // dims per lane (1..4)
  float qv[4], acc[4];
  for (int t = 0; t < per; ++t) {
    qv[t] = to_f(q[(size_t)row * a.d_model + h * dh + lane * per + t]) * a.scale;
    acc[t] = 0.f;
  }
  const int seq = a.row_seq[row];
  const T* K = reinterpret_cast<const T*>(kv.k) + seq * kv.seq_stride + a.layer * kv.layer_stride +
               h * kv.head_stride;
  const T* V = reinterpret_cast<const T*>(kv.v) + seq * kv.seq_stride + a.layer * kv.layer_stride +
               h * kv.head_stride;
  int nk;
  int tq = 0, lq = 0;
  if (a.mode == 0) nk = a.kvlen[row];
  else { nk = a.nkeys; tq = a.type[row]; lq = a.label[row]; }
  float m = -INFINITY, l = 0.f;
  for (int key = 0; key < nk; ++key) {
    if (a.mode == 1 && !step_causal_allowed(tq, lq, a.type[key], a.label[key])) continue;
    float d = 0.f;
    for (int t = 0; t < per; ++t) d += qv[t] * to_f(K[(size_t)key * dh + lane * per + t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    const float mn = fmaxf(m, d);
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float p = expf(d - mn);
    l = l * corr + p;
    for (int t = 0; t < per; ++t) acc[t] = acc[t] * corr + p * to_f(V[(size_t)key * dh + lane * per + t]);
    m = mn;
  }
  for (int t = 0; t < per; ++t)
    out[(size_t)row * a.d_model + h * dh + lane * per + t] = from_f<T>(acc[t] / l);
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
// Shared memory: the Q tile, then NS stages of K and NS stages of V (P lives in tensor memory).
static int attn_layout(int dh, AttnDev& d) {
  const int q_bytes = 128 * dh * 2;
  const int kv_bytes = 128 * dh * 2;
  d.q_off = 0;
  d.stage_bytes = kv_bytes;
  const int budget = 227 * 1024 - 1024 - 512;
  int ns = (budget - q_bytes) / (2 * kv_bytes);
  if (ns > 6) ns = 6;   // the 512-byte barrier area holds 1 + 4 * 6 + 8 barriers
  d.nstages = ns;
  d.k_off = q_bytes;
  d.v_off = d.k_off + ns * kv_bytes;
  d.bar_off = d.v_off + ns * kv_bytes;
  return d.bar_off + 512 + 1024;
}

cudaError_t attn_tc_set_smem_attr() {
  const cudaError_t e = cudaFuncSetAttribute(
      attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              227 * 1024);
}

int attn_tc_splits(const AttnCall& c) {
  int qt = 0, nkv = 1;
  for (int s = 0; s < c.n_seg; ++s) {
    qt += (c.seg[s].rows + 127) / 128;
    nkv = std::max(nkv, (c.seg[s].nkeys + 127) / 128);
  }
  const long long base = (long long)qt * c.H;
  const int sms = c.num_sms > 0 ? c.num_sms : 148;
  const size_t per_split = (size_t)c.rows_total * ((size_t)c.d_model * 4 + (size_t)c.H * 8);
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 16; ++s) {
    if (s > 1 && (s * 2 > nkv || (size_t)s * per_split > c.part_bytes || !c.part_o)) break;
    // one CTA per SM: cost ~ waves x (key tiles per split + a CTA's fixed cost) + the combine
    // launch, in periods of one key tile (≈1.4 µs at the 4096-token workload's last step): a
    // CTA's fixed cost (waiting for q, a first tile on a cold instruction cache, the merge and
    // output) is ≈8 of them, and so is the combine (measured: 8 and 8 run the 4096-token
    // workload 1.5 % faster than 2 and 0.5; 12 / 8, 8 / 16 and 10 / 12 within 0.5 % of it)
    const long long ctas = base * s;
    const double waves = (double)((ctas + sms - 1) / sms);
    const double cost = waves * ((nkv + s - 1) / s + 8.0) + (s > 1 ? 8.0 : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_attn_tc(const AttnCall& c, cudaStream_t stream) {
  AttnDev d{};
  d.mode = c.mode;
  d.H = c.H;
  d.dh = c.dh;
  d.d_model = c.d_model;
  d.layer = c.layer;
  d.kvlen = c.kvlen;
  d.type = c.type;
  d.label = c.label;
  d.cache_rows_per_seq = c.cache_rows_per_seq;
  d.cap = c.cap;
  d.scale_log2 = 1.4426950408889634f / sqrtf((float)c.dh);
  d.out = c.out;
  d.status = c.status;
  d.tile_list = c.tile_list;
  d.tile_count = c.tile_count;
  d.n_ktiles = c.n_ktiles;
  if (c.n_seg < 1 || c.n_seg > kMaxBatch) return cudaErrorInvalidValue;
  int nb = 0;
  d.n_seg = c.n_seg;
  for (int s = 0; s < c.n_seg; ++s) {
    d.seg[s] = c.seg[s];
    d.seg[s].tile0 = nb;
    nb += (c.seg[s].rows + 127) / 128;
  }
  if (nb == 0) return cudaSuccess;
  d.nsplit = attn_tc_splits(c);
  d.rows_total = c.rows_total;
  d.part_o = c.part_o;
  d.part_ml = c.part_o ? c.part_o + (size_t)d.nsplit * c.rows_total * c.d_model : nullptr;
  cudaError_t e;
  if (c.bound && c.mode == 1 && c.tile_list && c.tile_count && c.n_seg == 1 &&
             c.seg[0].row0 == 0) {
    // label mode with per-row key bounds (training form over step-grouped rows)
    static bool attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
      // these instantiations hold a few bytes of static shared memory: leave room for them
      e = cudaFuncSetAttribute(attn_tc_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_tc_kernel<64, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    const int smem = attn_layout(c.dh, d);
    dim3 grid(nb * d.nsplit, c.H);
    if (c.dh == 128)
      e = launch_pdl(attn_tc_kernel<128, true>, grid, dim3(kAttnThreads), smem, stream, 1,
                     *c.tmQ, *c.tmK, *c.tmV, d);
    else if (c.dh == 64)
      e = launch_pdl(attn_tc_kernel<64, true>, grid, dim3(kAttnThreads), smem, stream, 1,
                     *c.tmQ, *c.tmK, *c.tmV, d);
    else
      return cudaErrorInvalidValue;
  } else {
    const int smem = attn_layout(c.dh, d);
    dim3 grid(nb * d.nsplit, c.H);
    if (c.dh == 128)
      e = launch_pdl(attn_tc_kernel<128>, grid, dim3(kAttnThreads), smem, stream, 1, *c.tmQ,
                     *c.tmK, *c.tmV, d);
    else if (c.dh == 64)
      e = launch_pdl(attn_tc_kernel<64>, grid, dim3(kAttnThreads), smem, stream, 1, *c.tmQ,
                     *c.tmK, *c.tmV, d);
    else
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || d.nsplit == 1) return e;
  const long long warps = (long long)c.rows_total * c.H;
  return launch_pdl(attn_combine_kernel, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0,
                    stream, 1, (const float*)d.part_o, (const float*)d.part_ml, d.nsplit,
                    c.rows_total, c.H, c.dh, c.d_model, reinterpret_cast<__half*>(c.out));
}

template <typename T>
cudaError_t launch_attn_simt(const T* q, T* out, const KVAddr& kv, const AttnSimtArgs& a,
                             cudaStream_t stream) {
  if (a.rows <= 0) return cudaSuccess;
  const long long warps = (long long)a.rows * a.H;
  const int threads = 128;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  attn_simt_kernel<T><<<(unsigned)blocks, threads, 0, stream>>>(q, out, kv, a);
  return cudaGetLastError();
}

template cudaError_t launch_attn_simt<float>(const float*, float*, const KVAddr&,
                                             const AttnSimtArgs&, cudaStream_t);


}  // namespace smdm
