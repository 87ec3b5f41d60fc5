// Weight-streaming GEMMs of the transformer step: Y[r][n] = sum_k X[r][k] * W[n][k].
//
// bf16 models (tcgen05, fp16 operands: the weights' fp16 copies and fp16 activations, fp32
// accumulation): "swap-AB" tiles — the weight tile (128 output features x 64 of K) is
// the MMA's A operand and the activation rows (up to 512 of them) are its N dimension, so the
// per-step row count of a sparse step (|A| + |C| + registers, usually < 300) never pads the
// 128-row MMA M dimension.  Work is split stream-K style: the (tile, 64-wide K chunk) units are
// divided evenly over one CTA (or 2-CTA cluster) per SM (pair); tiles cut between CTAs are
// finished by whichever CTA contributes last (fp32 partials in L2-resident scratch, summed in a
// fixed order).  The residual epilogues (O-proj, down) instead add every segment into the fp32
// residual stream with TMA reduce-add as it finishes, so their sums — and through them the
// logits — are not bit-reproducible from run to run.  When the tile count is a large enough share of
// the grid, every CTA takes one whole tile instead.  Warp roles: warps 0 and 6 issue TMA loads
// (alternate pipeline stages), warp 1 owns TMEM and issues tcgen05.mma (straight-line per
// 64-wide K chunk), warps 2-5 drain the accumulator through the fused epilogue, which writes
// its 32-row blocks with TMA stores (K/V cache rows, scattered, with 16-byte stores).
//
// fp32 path (SIMT FFMA): the same tiles and epilogues for fp32 models, where a tf32 MMA would
// not hold the 1e-4 tolerance.
#include "gemm.h"

namespace smdm {

constexpr int kGemmThreads = 224;   // 7 warps: 2 producers, MMA, 4 epilogue
constexpr int kATileBytes = 128 * 128;   // 128 rows x 64 fp16
constexpr int kRing = 16;                // max landing slots (16 KB each) for split-K partials

struct SmemLayout {
  int stage_bytes, a_bytes, b_bytes;
  int nstages;
  int stage_off;   // after 1024 alignment
  int staging_off; // 2 x 32 x 128 floats
  int meta_off;    // 512 positions + 512 cache offsets
  int bar_off;
  int total;       // bytes of dynamic smem requested (incl. alignment slack)
};

static SmemLayout gemm_smem_layout(int RT, int max_stages) {
  SmemLayout L;
  L.a_bytes = kATileBytes;
  L.b_bytes = RT * 128;
  L.stage_bytes = L.a_bytes + L.b_bytes;
  const int budget = 227 * 1024 - 1024 /*align*/ - 2 * 32 * 128 * 4 - 6144 /*meta*/ - 512;
  // (the two 16 KB staging buffers serve the split-K partial bulk copies and the epilogues
  //  that combine lanes)
  L.nstages = budget / L.stage_bytes;
  if (L.nstages > max_stages) L.nstages = max_stages;
  L.stage_off = 0;
  L.staging_off = L.nstages * L.stage_bytes;
  L.meta_off = L.staging_off + 2 * 32 * 128 * 4;
  L.bar_off = L.meta_off + 6144;
  L.total = L.bar_off + 512 + 1024;
  return L;
}

struct GemmDev {
  int KC;          // K / 64
  int n_tiles;     // tiles of 128 A rows
  int row_blocks;
  int RT;          // activation rows per row block (multiple of 16; multiple of 32 if > 256)
  int rows;        // valid activation rows
  int row0;        // first activation row (TMA y offset)
  long long units; // n_tiles * row_blocks * KC
  int swiglu;
  int a_mode;      // 0: 2-D box {64,128}; 1: SwiGLU gate+up boxes {64,64}; 4: SwiGLU
                   // interleaved 3-D box {64,2,64};
                   // 2: 4-D rotary interleave (d_head 128); 3: 5-D rotary interleave (d_head 64)
  int RTp;         // partial-sum row stride (RT rounded up to 32)
  int np;          // TMA producer threads (1 or 2; stages alternate between them)
  int nstages, stage_bytes, staging_off, meta_off, bar_off;
  int n_acc, tmem_cols;
  float* partial;
  unsigned* counters;
  uint32_t* status;
};

SMDM_DEV long long cta_start(long long g, long long U, long long G) { return g * U / G; }
// CTA whose unit range contains unit u (inverse of cta_start).
SMDM_DEV long long cta_of(long long u, long long U, long long G) { return ((u + 1) * G - 1) / U; }

// kPair == 1: one CTA per SM.  kPair == 2: clusters of two CTAs on an SM pair running M=256
// tcgen05 MMAs (cta_group::2): each CTA streams its own 128 weight rows but only half of the
// activation rows, which halves the per-SM activation traffic.  The pair's first CTA issues the
// MMAs; both CTAs run their own epilogue on their 128 rows of the accumulator.
// NP: MMA N-parts per k-step (2 when the row tile exceeds 256 activation rows).
template <typename T, int kPair, int NP>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmOut,
                   const GemmDev g, const EpiParams ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float(*staging)[32][128] = reinterpret_cast<float(*)[32][128]>(smem + g.staging_off);
  int* meta_pos = reinterpret_cast<int*>(smem + g.meta_off);
  long long* meta_kv = reinterpret_cast<long long*>(smem + g.meta_off + 2048);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + g.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + g.nstages;
  uint64_t* acc_full = bars + 2 * g.nstages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* io_bar = acc_empty + 2;   // [2] partial bulk loads (staging buffers)
  uint64_t* ring_bar = io_bar + 2;    // [kRing] partial bulk loads landing in the idle stages
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring_bar + kRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (kPair == 2) ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < g.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4 * kPair);
      mbar_init(&io_bar[a], 1);
    }
    for (int r = 0; r < kRing; ++r) mbar_init(&ring_bar[r], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
    if (g.a_mode == 1) tma_prefetch_desc(&tmA2);
  }
  // Pair: both CTAs are running and their barriers initialised before any cross-CTA signal or
  // the pair's joint TMEM allocation (one warp in each CTA allocates collectively).
  if constexpr (kPair == 2) cluster_sync_all();
  if (warp == 1) {
    if constexpr (kPair == 2) {
      tmem_alloc_pair(tmem_holder, g.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, g.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  griddep_launch();   // the next kernel may start its prologue

  // Work is split over pairs (kPair == 2) or CTAs; a tile is kPair * 128 weight rows.
  const long long U = g.units, G = gridDim.x / kPair;
  const long long gp = blockIdx.x / kPair;
  const long long u_begin = cta_start(gp, U, G), u_end = cta_start(gp + 1, U, G);
  const int KC = g.KC;
  const int part_rows = g.RT / NP;                             // MMA N per part
  constexpr int nparts = NP;
  const int b_rows = part_rows / kPair;                        // B rows per part in this CTA
  // barriers that the pair's TMA and epilogue arrivals target live in the first CTA
  auto lead_addr = [&](uint64_t* bar) -> uint32_t {
    return (kPair == 2) ? mapa_shared(smem_u32(bar), 0) : smem_u32(bar);
  };

  if (warp == 0 || warp == 6) {
    // Producers: with np == 2, warp 0 fills the CTA's even units and warp 6 the odd ones (a
    // single thread issuing every TMA copy caps the SM's copy rate well below its bandwidth).
    const int pidx = (warp == 0) ? 0 : 1;
    if (lane == 0 && pidx < g.np) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int np = g.np, NS = g.nstages;
      int stage = pidx % NS;
      uint32_t phase = (uint32_t)((pidx / NS) & 1);
      // incremental (tile, k-chunk) walk: no 64-bit divisions on the per-chunk path
      const long long u_first = u_begin + pidx;
      int tile_i = (int)(u_first / KC), kc = (int)(u_first % KC);
      int nt = tile_i / g.row_blocks, rb = tile_i % g.row_blocks;
      // Activation (B) loads of one stage; the weights (A) do not depend on earlier kernels.
      auto load_b = [&](int st, int rb_, int kc_) {
        uint8_t* B = smem + st * g.stage_bytes + kATileBytes;
        for (int p = 0; p < nparts; ++p) {
          const int y = g.row0 + rb_ * g.RT + p * part_rows + (int)rank * b_rows;
          if constexpr (kPair == 1)
            tma_load_2d(B + p * b_rows * 128, &tmB, &full[st], kc_ * 64, y, pol_x);
          else
            tma_load_2d_pair(B + p * b_rows * 128, &tmB, lead_addr(&full[st]), kc_ * 64, y, pol_x);
        }
      };
      // First round of stages: issue the weight loads before waiting for the previous kernel
      // (programmatic dependent launch) and the activation loads after it.
      int pend_st[8], pend_rb[8], pend_kc[8];
      int npend = 0;
      bool dep_done = false;
      auto finish_dep = [&]() {
        griddep_wait();
        for (int i = 0; i < npend; ++i) load_b(pend_st[i], pend_rb[i], pend_kc[i]);
        npend = 0;
        dep_done = true;
      };
      for (long long u = u_first; u < u_end; u += np) {
        if (!dep_done && (u - u_begin >= NS || npend == 8)) finish_dep();
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, g.status)) break;
        uint8_t* A = smem + stage * g.stage_bytes;
        const int at = nt * kPair + (int)rank;    // this CTA's 128-row A tile
        if constexpr (kPair == 1) {
          mbar_arrive_expect_tx(&full[stage], g.stage_bytes);
          if (g.a_mode == 4) {
            tma_load_3d(A, &tmA, &full[stage], kc * 64, 0, at * 64, pol_w);
          } else if (g.a_mode == 1) {
            tma_load_2d(A, &tmA, &full[stage], kc * 64, at * 64, pol_w);
            tma_load_2d(A + kATileBytes / 2, &tmA2, &full[stage], kc * 64, at * 64, pol_w);
          } else if (g.a_mode == 2) {
            tma_load_4d(A, &tmA, &full[stage], kc * 64, 0, 0, at, pol_w);
          } else if (g.a_mode == 3) {
            tma_load_5d(A, &tmA, &full[stage], kc * 64, 0, 0, 0, at, pol_w);
          } else {
            tma_load_2d(A, &tmA, &full[stage], kc * 64, at * 128, pol_w);
          }
        } else {
          // both CTAs' bytes complete on the first CTA's barrier, which expects them all
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * g.stage_bytes);
          const uint32_t fb = lead_addr(&full[stage]);
          if (g.a_mode == 4) {
            tma_load_3d_pair(A, &tmA, fb, kc * 64, 0, at * 64, pol_w);
          } else if (g.a_mode == 1) {
            tma_load_2d_pair(A, &tmA, fb, kc * 64, at * 64, pol_w);
            tma_load_2d_pair(A + kATileBytes / 2, &tmA2, fb, kc * 64, at * 64, pol_w);
          } else if (g.a_mode == 2) {
            tma_load_4d_pair(A, &tmA, fb, kc * 64, 0, 0, at, pol_w);
          } else if (g.a_mode == 3) {
            tma_load_5d_pair(A, &tmA, fb, kc * 64, 0, 0, 0, at, pol_w);
          } else {
            tma_load_2d_pair(A, &tmA, fb, kc * 64, at * 128, pol_w);
          }
        }
        if (dep_done) {
          load_b(stage, rb, kc);
        } else {
          pend_st[npend] = stage;
          pend_rb[npend] = rb;
          pend_kc[npend] = kc;
          ++npend;
        }
        stage += np;
        while (stage >= NS) { stage -= NS; phase ^= 1; }
        kc += np;
        while (kc >= KC) {
          kc -= KC;
          if (++rb == g.row_blocks) { rb = 0; ++nt; }
        }
      }
      if (!dep_done) finish_dep();
      if constexpr (kPair == 2) {
        // The pair's MMA completions arrive on these barriers from the first CTA: wait for the
        // release of every stage so that no arrival lands after this CTA has exited.
        if (pidx == 0) {
          const long long n = u_end - u_begin;
          for (long long i = n; i < n + NS && !*abort_flag; ++i)
            if (!mbar_wait(&empty[i % NS], (uint32_t)(((i / NS) & 1) ^ 1), abort_flag, g.status)) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_f16(128 * kPair, part_rows, 0, 0);   // fp16 x fp16 -> fp32
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      long long u = u_begin;
      bool ok = true;
      while (u < u_end && ok) {
        const long long tile = u / KC;
        const long long seg_end = min(u_end, (tile + 1) * KC);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, g.status)) break;
        tc_fence_after();
        const uint32_t dcol = tbase + acc * g.RT;
        bool first = true;
        for (; u < seg_end; ++u) {
          if (!mbar_wait(&full[stage], phase, abort_flag, g.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * g.stage_bytes);
          const uint32_t b_addr = a_addr + kATileBytes;
          // Straight-line issue (k-steps and parts fully unrolled): control flow between
          // consecutive tcgen05.mma instructions stalls the issue by tens of cycles each.
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint32_t accum = (first && kk == 0) ? 0u : 1u;
#pragma unroll
            for (int p = 0; p < NP; ++p) {
              const uint64_t bdesc = sdesc_sw128(b_addr + p * b_rows * 128 + kk * 32, 16, 1024);
              const uint32_t d = dcol + p * part_rows;
              if constexpr (kPair == 2) umma_f16_pair(d, adesc, bdesc, idesc, accum);
              else umma_f16(d, adesc, bdesc, idesc, accum);
            }
          }
          if constexpr (kPair == 2) umma_commit_pair(&empty[stage]);
          else umma_commit(&empty[stage]);
          first = false;
          if (++stage == g.nstages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (kPair == 2) umma_commit_pair(&acc_full[acc]);
        else umma_commit(&acc_full[acc]);
        if (g.n_acc == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1;
        } else {
          acc_phase ^= 1;
        }
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    // Epilogue warps 2..5: TMEM lane quarter = warp % 4 -> A-tile row m.
    griddep_wait();   // row metadata, outputs, partial slots and counters follow earlier kernels
    const int q = warp & 3;
    const int m = q * 32 + lane;
    const int et = threadIdx.x - 64;   // 0..127
    // the accumulator is free again once all epilogue warps of the pair (or CTA) are done
    auto acc_release = [&](int a) {
      if constexpr (kPair == 2) mbar_arrive_cluster(lead_addr(&acc_empty[a]));
      else mbar_arrive(&acc_empty[a]);
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    int sbuf = 0;
    uint32_t io_phase[2] = {0u, 0u};
    long long u = u_begin;
    while (u < u_end) {
      const long long tile = u / KC;
      const long long tstart = tile * KC, tend = tstart + KC;
      const long long seg_end = min(u_end, tend);
      const bool full_tile = (u == tstart) && (seg_end == tend);
      const int nt = (int)(tile / g.row_blocks), rb = (int)(tile % g.row_blocks);
      const int at = nt * kPair + (int)rank;             // this CTA's 128-row weight tile
      const long long ctile = tile * kPair + rank;       // its fixup counter
      const int rbase = rb * g.RT;                       // first activation row of the block
      const int nvalid_rows = min(g.RT, g.rows - rbase);
      const int nblk = (nvalid_rows + 31) >> 5;
      u = seg_end;
      // A failed (timed-out) wait only flags the status word: the epilogue threads keep going so
      // that their named barriers stay matched; the results are then garbage but the kernel ends.
      mbar_wait_sleep(&acc_full[acc], acc_phase, abort_flag, g.status);
      tc_fence_after();
      const uint32_t tacc = tbase + (uint32_t(q * 32) << 16) + acc * g.RT;
      // 32 accumulator columns (activation rows b*32..) of this lane
      auto ld_acc = [&](int b, float* v) { tmem_ld32(tacc + b * 32, v); };
      // Residual epilogues are additive: split segments add straight into x (fp32 atomics).
      const bool additive = (ep.kind == kEpiResid);
      const bool from_tmem = full_tile || additive;
      bool do_epi = true;
      long long g_first = 0, g_last = -1;
      // Split tile (non-additive epilogue): every contributing CTA except the last parks its
      // fp32 segment in a slot ([blocks of 32 columns][128 rows], bulk stores); the last one
      // sums all segments in segment order (deterministic) and runs the epilogue.  A CTA that
      // finds every other segment already published (the usual case for the CTA finishing a
      // tile, whose neighbour did its part first) skips parking its own segment and adds it
      // straight from TMEM.
      bool own_in_tmem = false;
      if (!from_tmem) {
        g_first = cta_of(tstart, U, G);
        g_last = cta_of(tend - 1, U, G);
        const unsigned nseg_u = (unsigned)(g_last - g_first + 1);
        if (et == 0) {
          const unsigned done = atomicAdd(&g.counters[ctile], 0u);
          *last_flag = (done == nseg_u - 1) ? 2 : 0;
        }
        named_bar_sync(1, 128);
        if (*last_flag == 2) {
          own_in_tmem = true;
          if (et == 0) {
            __threadfence();
            asm volatile("fence.proxy.async;" ::: "memory");   // partials are read by bulk copies
            g.counters[ctile] = 0u;               // nobody else touches it in this launch
          }
        } else {
          const int slot = (cta_start(gp, U, G) < tstart) ? 1 : 0;
          float* P = g.partial + ((size_t)blockIdx.x * 2 + slot) * (size_t)g.RTp * 128;
          // Direct stores from registers: for accumulator column j the 128 lanes write 512
          // contiguous bytes ([column][row] blocks, the layout the summing CTA loads in bulk).
          // This keeps the SM's copy engine, busy with the next segment's loads, out of it.
          for (int b = 0; b < nblk; ++b) {
            float v[32];
            ld_acc(b, v);
            float* Pb = P + (size_t)b * 32 * 128 + m;
#pragma unroll
            for (int j = 0; j < 32; ++j) Pb[j * 128] = v[j];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) acc_release(acc);
          __threadfence();                        // this thread's partial stores are visible
          named_bar_sync(1, 128);
          if (et == 0) {
            asm volatile("fence.proxy.async;" ::: "memory");
            const unsigned prev = atomicAdd(&g.counters[ctile], 1u);
            const int is_last = (prev == nseg_u - 1) ? 1 : 0;
            if (is_last) g.counters[ctile] = 0u;  // ready for the next launch
            __threadfence();
            asm volatile("fence.proxy.async;" ::: "memory");
            *last_flag = is_last;
          }
          named_bar_sync(1, 128);
          do_epi = (*last_flag != 0);
        }
      }
      if (do_epi) {
        if (ep.kind == kEpiQKV) {
          for (int r = et; r < nvalid_rows; r += 128) {
            const int row = rbase + r;
            meta_pos[r] = ep.row_pos[row];
            meta_kv[r] = (long long)ep.row_seq[row] * ep.kv.seq_stride +
                         (long long)ep.row_slot[row] * ep.d_head;
          }
          named_bar_sync(1, 128);
        }
        const int nseg = (int)(g_last - g_first + 1);
        const int own_idx = (int)(gp - g_first);
        auto src = [&](int sidx, int b) {
          const long long gg = g_first + sidx;
          const int sl = (cta_start(gg, U, G) < tstart) ? 1 : 0;
          const size_t cta = (size_t)gg * kPair + rank;
          return g.partial + (cta * 2 + sl) * (size_t)g.RTp * 128 + (size_t)b * 32 * 128;
        };
        // Segments to fetch from memory (all but our own when it is still in TMEM).
        const int nfetch = (from_tmem) ? 0 : (own_in_tmem ? nseg - 1 : nseg);
        // When this was the CTA's final segment the pipeline stages are idle: use them as a
        // ring of 16 KB landing slots so that several blocks' partial loads are in flight.
        const int ring_cap = min(kRing, (g.nstages * g.stage_bytes) / 16384);
        const bool use_ring = !from_tmem && nfetch > 0 && (seg_end == u_end) && ring_cap >= nfetch;
        const int nload = use_ring ? nblk * nfetch : 0;
        int issued = 0;
        auto load_src = [&](int k) {    // k-th load: block k / nfetch, k % nfetch-th fetched segment
          const int b = k / nfetch, kf = k % nfetch;
          int c = -1, sidx = 0;
          for (; sidx < nseg; ++sidx) {
            if (own_in_tmem && sidx == own_idx) continue;
            if (++c == kf) break;
          }
          return src(sidx, b);
        };
        if (use_ring) {
          named_bar_sync(1, 128);
          if (et == 0) {
            for (; issued < min(ring_cap, nload); ++issued) {
              const int slot = issued % ring_cap;
              mbar_arrive_expect_tx(&ring_bar[slot], 16384);
              bulk_load(smem + (size_t)slot * 16384, load_src(issued), 16384, &ring_bar[slot]);
            }
          }
        }
        for (int b = 0; b < nblk; ++b) {
          float v[32];
          if (from_tmem) {
            ld_acc(b, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
            if (use_ring) {
              int kf = 0;
              for (int sidx = 0; sidx < nseg; ++sidx) {
                if (own_in_tmem && sidx == own_idx) {
                  float w[32];
                  ld_acc(b, w);
#pragma unroll
                  for (int j = 0; j < 32; ++j) v[j] += w[j];
                } else {
                  const int k = b * nfetch + kf;
                  const int slot = k % ring_cap;
                  mbar_wait(&ring_bar[slot], (uint32_t)((k / ring_cap) & 1), abort_flag, g.status);
                  const float* blkp = reinterpret_cast<const float*>(smem + (size_t)slot * 16384);
#pragma unroll
                  for (int j = 0; j < 32; ++j) v[j] += blkp[j * 128 + m];
                  ++kf;
                }
              }
            } else {
              // two staging buffers, two loads in flight
              named_bar_sync(1, 128);
              int order[2];
              int nf = 0;
              auto fetch_index = [&](int k) {   // k-th fetched segment index
                int c = -1;
                for (int sidx = 0; sidx < nseg; ++sidx) {
                  if (own_in_tmem && sidx == own_idx) continue;
                  if (++c == k) return sidx;
                }
                return -1;
              };
              if (et == 0) {
                bulk_wait_read<0>();   // output copies issued from these buffers are done reading
                for (int k = 0; k < min(2, nfetch); ++k) {
                  mbar_arrive_expect_tx(&io_bar[k], 16384);
                  bulk_load(&staging[k][0][0], src(fetch_index(k), b), 16384, &io_bar[k]);
                }
              }
              (void)order;
              (void)nf;
              int k = 0;
              for (int sidx = 0; sidx < nseg; ++sidx) {
                if (own_in_tmem && sidx == own_idx) {
                  float w[32];
                  ld_acc(b, w);
#pragma unroll
                  for (int j = 0; j < 32; ++j) v[j] += w[j];
                  continue;
                }
                const int bi = k & 1;
                mbar_wait(&io_bar[bi], io_phase[bi], abort_flag, g.status);
                io_phase[bi] ^= 1;
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] += staging[bi][j][m];
                named_bar_sync(1, 128);           // everyone done with this buffer
                if (et == 0 && k + 2 < nfetch) {
                  mbar_arrive_expect_tx(&io_bar[bi], 16384);
                  bulk_load(&staging[bi][0][0], src(fetch_index(k + 2), b), 16384, &io_bar[bi]);
                }
                ++k;
              }
            }
          }
          epilogue_block<T>(ep, &tmOut, v, reinterpret_cast<uint8_t*>(&staging[sbuf][0][0]),
                            at * 128, rbase + b * 32, m, et, min(32, nvalid_rows - b * 32),
                            meta_pos, meta_kv, rbase);
          sbuf ^= 1;
          // every thread passed the barrier inside the epilogue, so block b's slots are free
          if (use_ring && et == 0) {
            const int consumed = (b + 1) * nfetch;
            for (; issued < min(nload, consumed + ring_cap); ++issued) {
              const int slot = issued % ring_cap;
              mbar_arrive_expect_tx(&ring_bar[slot], 16384);
              bulk_load(smem + (size_t)slot * 16384, load_src(issued), 16384, &ring_bar[slot]);
            }
          }
        }
        if (et == 0) bulk_wait_read<0>();   // staging buffers are free once the copies read them
        named_bar_sync(1, 128);   // meta / staging / stages are reused afterwards
      }
      if (own_in_tmem || from_tmem) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) acc_release(acc);
      }
      if (g.n_acc == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      } else {
        acc_phase ^= 1;
      }
    }
    if (et == 0) bulk_wait_all();   // output copies complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair == 2) cluster_sync_all();   // the peer is done with our TMEM and barriers
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair == 2) tmem_dealloc_pair(tbase, g.tmem_cols);
    else tmem_dealloc(tbase, g.tmem_cols);
  }
}

// ------------------------------------------------------------------------------------------
// fp32 SIMT GEMM: CTA = 128 features x 16 rows, 128 threads, K in steps of 32.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    gemm_simt_kernel(const float* __restrict__ W, const float* __restrict__ W2,
                     const float* __restrict__ X, int ldx, int K, int n_rows_w, int rows,
                     int swiglu, EpiParams ep) {
  __shared__ float Ws[128][33];
  __shared__ float Xs[16][33];
  __shared__ float S[16][128];
  const int m = threadIdx.x;
  const int nt = blockIdx.x, r0 = blockIdx.y * 16;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    // load W tile rows (128) x 32
    for (int idx = m; idx < 128 * 32; idx += 128) {
      const int rr = idx / 32, kk = idx % 32;
      int wrow;
      const float* src;
      if (swiglu) {
        wrow = nt * 64 + (rr & 63);
        src = (rr < 64) ? W : W2;
      } else {
        wrow = nt * 128 + rr;
        src = W;
      }
      Ws[rr][kk] = (wrow < n_rows_w && k0 + kk < K) ? src[(size_t)wrow * K + k0 + kk] : 0.f;
    }
    for (int idx = m; idx < 16 * 32; idx += 128) {
      const int j = idx / 32, kk = idx % 32;
      Xs[j][kk] = (r0 + j < rows && k0 + kk < K) ? X[(size_t)(r0 + j) * ldx + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float w = Ws[m][kk];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = fmaf(w, Xs[j][kk], acc[j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) S[j][m] = acc[j];
  __syncthreads();
  epilogue_tile<float>(ep, S, nt * 128, r0, m, false);
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------

int gemm_tc_row_tile(int rows, int min_blocks) {
  if (min_blocks > 1) {   // at least min_blocks blocks of a multiple of 32 rows
    const int rt = ((rows + min_blocks - 1) / min_blocks + 31) & ~31;
    return rt > 256 ? 256 : rt;
  }
  // One row block of up to 512 rows keeps every weight tile streamed exactly once.
  const int R16 = (rows + 15) & ~15;
  if (R16 <= 256) return R16;
  if (R16 <= 512) return (rows + 31) & ~31;
  return 256;
}

int gemm_tc_box_rows(int rows, int pair, int min_blocks) {
  const int RT = gemm_tc_row_tile(rows, min_blocks);
  return (RT > 256 ? RT / 2 : RT) / pair;
}

int gemm_tc_min_row_blocks(int n_out, int rows, int epi_kind, int sms) {
  // The LM head's whole tiles (V / 128, 64 for V = 8192) leave most SMs idle while each CTA
  // runs the row-statistics epilogue over every decode row; two row blocks put twice the CTAs
  // on it, each with half the epilogue (the weight tile is then read twice, from L2).
  const int n_tiles = (n_out + 127) / 128;
  return (epi_kind == kEpiLMHead && rows >= 64 && 2 * n_tiles <= sms) ? 2 : 1;
}

// Whole tiles (one CTA per tile, no split-K fix-up) when the tile count is at least this
// percentage of the grid (measured on the 4096-token run: 40 puts the QKV GEMM (96 tiles) and
// the LM head (64 tiles) on whole tiles, the O / down GEMMs (32 tiles) on stream-K).
constexpr int kWholeTileMinPct = 40;

int gemm_tc_pair(int n_out, int swiglu, int rows, int epi_kind) {
  (void)rows;
  const int n_tiles = swiglu ? (n_out + 63) / 64 : (n_out + 127) / 128;
  // Measured on the 4096-token run: pairs help the QKV and gate/up GEMMs and cost the residual
  // (O, down) and LM-head GEMMs a little.  The pair covers two adjacent 128-row weight tiles, so
  // their count must be even.
  const bool wants = epi_kind == kEpiQKV || epi_kind == kEpiSwiGLU;
  return (wants && n_tiles % 2 == 0) ? 2 : 1;
}

static int pow2_ceil(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

cudaError_t gemm_tc_set_smem_attr() {
  const void* fns[4] = {(const void*)gemm_tc_kernel<__half, 1, 1>,
                        (const void*)gemm_tc_kernel<__half, 1, 2>,
                        (const void*)gemm_tc_kernel<__half, 2, 1>,
                        (const void*)gemm_tc_kernel<__half, 2, 2>};
  for (const void* f : fns) {
    const cudaError_t e =
        cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Co-resident 2-CTA clusters of the pair kernel on the current device (cached per device).
static int max_pair_clusters(int smem_bytes) {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<__half, 2, 1>, &cfg) !=
        cudaSuccess) {
      cudaGetLastError();
      n = -1;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t launch_gemm_tc(const GemmCall& c, cudaStream_t stream) {
  if (c.rows <= 0) return cudaSuccess;
  GemmDev g{};
  g.KC = c.K / 64;
  g.swiglu = c.swiglu;
  g.a_mode = c.swiglu ? (c.swiglu_il ? 4 : 1) : c.a_interleave == 128 ? 2 : c.a_interleave == 64 ? 3 : 0;
  g.n_tiles = c.swiglu ? (c.n_out + 63) / 64 : (c.n_out + 127) / 128;
  g.RT = gemm_tc_row_tile(c.rows, c.min_row_blocks);
  g.row_blocks = (c.rows + g.RT - 1) / g.RT;
  g.rows = c.rows;
  g.row0 = c.row0;
  const int pair = (c.pair == 2) ? 2 : 1;
  if (pair == 2 && (g.n_tiles & 1)) return cudaErrorInvalidValue;
  const int pair_tiles = g.n_tiles / pair;     // tiles of pair * 128 weight rows
  g.units = (long long)pair_tiles * g.row_blocks * g.KC;
  const SmemLayout L = gemm_smem_layout(g.RT / pair, c.max_stages > 0 ? c.max_stages : 8);
  g.RTp = (g.RT + 31) & ~31;
  g.nstages = L.nstages;
  g.stage_bytes = L.stage_bytes;
  g.staging_off = L.staging_off;
  g.meta_off = L.meta_off;
  g.bar_off = L.bar_off;
  g.np = (c.producers == 1) ? 1 : 2;
  g.n_acc = (g.RT <= 256) ? 2 : 1;   // double-buffered accumulators where TMEM allows
  g.tmem_cols = pow2_ceil(g.n_acc * g.RT);
  g.partial = c.partial;
  g.counters = c.counters;
  g.status = c.status;
  // Grid: one CTA per SM, units split stream-K style.  When the tile count is close to the SM
  // count, one whole tile per CTA (no split-K fixups, tight tail) beats splitting.
  // G counts work groups: CTAs, or CTA pairs in pair mode (no more pairs than can be resident
  // at once: some GPCs have an odd number of usable SMs).
  long long G = c.num_ctas / pair;
  if (pair == 2) {
    const int mc = max_pair_clusters(L.total);
    if (mc > 0 && G > mc) G = mc;
  }
  const long long tiles_total = (long long)pair_tiles * g.row_blocks;
  const int whole_pct = kWholeTileMinPct;
  if (c.sched == 1 ? tiles_total <= G
                   : c.sched == 0 && tiles_total <= G && tiles_total * 100 >= G * whole_pct)
    G = tiles_total;
  if (G > g.units) G = g.units;
  if (G < 1) G = 1;
  if (g.n_tiles * g.row_blocks > c.max_tiles) return cudaErrorInvalidValue;
  // 32-row output blocks of a row tile must not reach into the next row tile
  if (g.row_blocks > 1 && (g.RT & 31)) return cudaErrorInvalidValue;
  if (!c.tmOut) return cudaErrorInvalidValue;
  if ((long long)g.RTp * 128 * 2 * G * pair * 4 > (long long)c.partial_bytes)
    return cudaErrorInvalidValue;  // split-K scratch too small for this row tile
  // (kEpiQKV requires a rotary-interleaved A map: a_interleave == d_head)
  const CUtensorMap& tA2 = (c.swiglu && !c.swiglu_il) ? *c.tmA2 : *c.tmA;
  const bool two_parts = g.RT > 256;
  if (pair == 1) {
    if (two_parts)
      return launch_pdl(gemm_tc_kernel<__half, 1, 2>, dim3((unsigned)G), dim3(kGemmThreads),
                        L.total, stream, 1, *c.tmA, tA2, *c.tmB, *c.tmOut, g, c.epi);
    return launch_pdl(gemm_tc_kernel<__half, 1, 1>, dim3((unsigned)G), dim3(kGemmThreads),
                      L.total, stream, 1, *c.tmA, tA2, *c.tmB, *c.tmOut, g, c.epi);
  }
  if (two_parts)
    return launch_pdl(gemm_tc_kernel<__half, 2, 2>, dim3((unsigned)(G * 2)),
                      dim3(kGemmThreads), L.total, stream, 2, *c.tmA, tA2, *c.tmB, *c.tmOut, g,
                      c.epi);
  return launch_pdl(gemm_tc_kernel<__half, 2, 1>, dim3((unsigned)(G * 2)),
                    dim3(kGemmThreads), L.total, stream, 2, *c.tmA, tA2, *c.tmB, *c.tmOut, g,
                    c.epi);
}

cudaError_t launch_gemm_simt(const float* W, const float* W2, const float* X, int ldx, int K,
                             int n_out, int rows, int swiglu, const EpiParams& ep,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int n_tiles = swiglu ? (n_out + 63) / 64 : (n_out + 127) / 128;
  dim3 grid(n_tiles, (rows + 15) / 16);
  gemm_simt_kernel<<<grid, 128, 0, stream>>>(W, W2, X, ldx, K, n_out, rows, swiglu, ep);
  return cudaGetLastError();
}


}  // namespace smdm
