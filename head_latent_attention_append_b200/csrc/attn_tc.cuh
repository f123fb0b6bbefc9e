// Absorbed latent attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// one 2-CTA cluster per worker.
//
// What it computes is the same as attn_simt.cuh ("ai-decoupled-rope-mla",
// absorbed score and output equations): for one query token, all of its heads
// form the M = 128 rows (heads beyond n_h are zero rows), and for each 64-key
// cache page
//   S  = Q_abs [128 x d_cr] * page^T [d_cr x 64]      (content + position
//        score in one contraction: the cache row is [c | k_R] and the query
//        row is [q~ | q_R], both pre-scaled by s*log2(e))
//   P  = exp2(S - m)  (online softmax, running max m, running sum l)
//   O += P [128 x 64] * page[:, latent] [64 x d_c]
// Both products are dense because every head shares the cache ("Latent
// Attention Meets RoPE": one shared position key; the latent is shared by
// construction).
//
// B200 layout.  TMEM (128 lanes x 512 fp32 columns per SM) cannot hold the
// 128 x 512 fp32 latent accumulator of one token next to anything else, so
// the two CTAs of a cluster split the columns of the cache row:
//   rank 0: latent columns [0, d_c/2) and the first ra RoPE-key columns
//   rank 1: latent columns [d_c/2, d_c) and the other rb = d_r - ra,
// with ra = 16 * (d_r / 32) so that both score shares are whole 16-column MMA
// steps and, for d_r = 32 or 64, equal.  Each CTA streams only its own
// columns of every page (no byte is read twice from HBM) and computes the
// partial score over them into TMEM.  The partial goes to the peer as fp16
// (saturated at +-65504, log2 units) through distributed shared memory; each
// CTA's softmax threads add the peer's partial to their own exact fp32 one.
// So the two CTAs' scores differ by the rounding of one fp16 partial and each
// runs its own softmax state (m, l) for its half of the latent columns: each
// half is normalised by its own state, and split row blocks leave one
// (m, l) per half.  fp16's 11-bit significand keeps this well below the
// rounding the bf16 cache rows put into every score (a bf16 exchange doubled
// the error against the fp64 oracle once logits reach ~30).
//
// TMEM columns: O [0, d_c/2), two score buffers S0 [256, 320) and
// S1 [320, 384), the latent part of this CTA's Q slice from 384 (at most 128
// columns).  A score buffer is free again as soon as the sender and the
// finishers have read it (the peer's partial is not waited for first), so the
// DSMEM latency of the exchange stays out of the score pipeline.
//
// Shared memory (1024-byte aligned pieces):
//   three 16 KB exchange buffers, filled by the peer with bulk copies (one
//     4 KB copy per sender warp per page) that complete on this CTA's
//     mbarrier; each goes back to the peer with a tcgen05.commit multicast
//     onto the peer's credit barrier after the page's P*V, which is issued
//     only once the finishers have read the buffer (a remote arrive from the
//     finishers themselves is a cluster-scope release that stalls the warp);
//   a 16 KB staging block for this CTA's outgoing partial;
//   score ring, 2 slots: this CTA's columns of a page (its latent chunks and
//     its RoPE share, loaded with a 16- or 32-column box swizzled to 32 or 64
//     bytes), freed as soon as the page's score MMA completes;
//   latent ring, 2 slots: the page's latent columns again (4 chunks) for
//     P*V, freed by P*V.  The second read is an L2 hit (the first was a few
//     microseconds earlier), so HBM still sees every byte once;
//   the RoPE part of the Q slice (SS MMA operand, swizzled like the page's
//     RoPE share) and the 16 KB P tile (SS P*V operand);
//   two 1 KB slots of half-row maxima for the finishers' pair exchange
//     (a segment's row sums borrow the idle one).
// Segment metadata and page ids are loaded a step ahead so no global load
// sits on a page's critical path.
//
// Warp roles (512 threads): warp 0 = score-ring TMA producer, warp 2 = TMEM
// allocator and latent-ring TMA producer, warp 1 = score-MMA issuer, warp 3 =
// P*V-MMA issuer (all warp-uniform; one elected lane issues), warps 4-7 =
// sender (reads each page's own partial score from TMEM, ships it to the
// peer, loads each segment's Q slice), warps 8-11 and 12-15 = the two
// finisher halves (keys 0-31 and 32-63 of every row: score, softmax, P, and
// half of O in the epilogue); thread r of any of these owns row r = TMEM
// lane r.  Two score buffers let the score MMA of page t+1 run while the
// finishers work on page t.  Every wait is bounded (sm100::mbar_wait).
#pragma once
#include "attn_simt.cuh"
#include "sm100.cuh"

namespace mla {
namespace attn_tc {
using namespace sm100;

constexpr int THREADS = 512;
constexpr int KT = 64;                        // keys per tile (one page)
constexpr int CHUNK_BYTES = 64 * 64 * 2;      // 64 keys x 64 bf16 columns
constexpr int MAX_PV = 4;                     // latent chunks per CTA per page (d_c <= 512)
constexpr int MAX_ROPE = 32;                  // RoPE-key columns per CTA (d_r <= 64)
constexpr int SGROUPS = 2;                    // score ring: a page's own columns, freed by its score MMA
constexpr int VGROUPS = 2;                    // latent ring: the page's latent columns again, freed by P*V
constexpr int XBUF = 3;                       // exchange buffers per CTA (credit-controlled)
constexpr int ROPE_OFF = MAX_PV * CHUNK_BYTES;  // a score slot: latent chunks, then the RoPE share
constexpr int SG_BYTES = ROPE_OFF + KT * MAX_ROPE * 2;
constexpr int VG_BYTES = MAX_PV * CHUNK_BYTES;
constexpr int X_BYTES = 128 * KT * 2;         // one fp16 partial-score tile
constexpr int QR_BYTES = 128 * MAX_ROPE * 2;  // the RoPE part of the Q slice
constexpr int P_BYTES = 128 * KT * 2;         // P tile: 128 rows x 64 keys bf16
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384, TM_COLS = 512;

// The exchange buffers and the credit barriers sit at the same offsets in
// both CTAs (the peer addresses them through mapa).
constexpr int OFF_X = 0;
constexpr int OFF_XS = OFF_X + XBUF * X_BYTES;    // outgoing partial, staged for the bulk copy
constexpr int OFF_SG = OFF_XS + X_BYTES;
constexpr int OFF_VG = OFF_SG + SGROUPS * SG_BYTES;
constexpr int OFF_QR = OFF_VG + VGROUPS * VG_BYTES;
constexpr int OFF_P = OFF_QR + QR_BYTES;
constexpr int OFF_MH = OFF_P + P_BYTES;           // half-row maxima [2][2][128] fp32 (sums reuse a slot)
constexpr int OFF_BAR = OFF_MH + 2 * 2 * 128 * 4;
constexpr int NUM_BARS = 2 * XBUF + 2 * SGROUPS + 2 * VGROUPS + 2 + 2 + 1 + 1 + 3 + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
static_assert(OFF_SG % 1024 == 0 && OFF_VG % 1024 == 0 && OFF_QR % 1024 == 0 && OFF_P % 1024 == 0 &&
                  SG_BYTES % 1024 == 0,
              "swizzled operands need 1024-byte aligned tiles");
// No slack for aligning the base: the kernel has no static shared memory, so
// its dynamic block starts on a 1024-byte boundary (the kernel checks this
// and reports MLA_ERR_UNSUPPORTED otherwise).
constexpr size_t SMEM_BYTES = SMEM_USED;
static_assert(SMEM_BYTES <= 232448, "over the 227 KB of shared memory a CTA can have");

struct Params {
  AttnArgs a;
  int npv;     // latent chunks per CTA (d_c / 128)
  int ra, rb;  // RoPE-key columns scored by rank 0 and rank 1 (multiples of 16, ra + rb = d_r)
};

// 2^x with the MUFU ex2 instruction (flush-to-zero; ~2 ulp), used for the
// softmax weights, which are rounded to bf16 right after.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b, float& sum) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  sum += __low2float(v) + __high2float(v);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Bulk copy of `bytes` (a multiple of 16) from this CTA's shared memory into
// a peer CTA's, completing as transaction bytes on the peer's mbarrier
// `bar_cluster_addr`.  One copy carries what would otherwise be many small
// remote stores, each with its own transaction-count update at the peer.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster_addr, uint32_t src_smem, uint32_t bytes,
                                                  uint32_t bar_cluster_addr) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster_addr),
      "r"(src_smem), "r"(bytes), "r"(bar_cluster_addr)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the sources of this thread's committed bulk copies have been read.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Arrives once on the mbarrier at the same shared-memory offset in every CTA
// of `cta_mask` when every tcgen05 operation this thread issued has completed.
__device__ __forceinline__ void tc_commit_to(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
// Asks L2 to fetch `bytes` (a multiple of 16) from global memory ahead of use.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// Partial scores travel between the CTAs as fp16 pairs, saturated at
// +-65504 (one conversion per pair).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t u;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
  return u;
}
// Exact fp16 pair -> two floats with integer work and one multiply per value
// (no conversion-pipe work): the 15 bits below a half's sign, moved to an
// fp32's exponent and significand positions, are its value times 2^-112
// (subnormal halves included, as fp32 subnormals); the sign moves over.
__device__ __forceinline__ float2 unpack_f16x2(uint32_t u) {
  const float lo = __uint_as_float((u << 13) & 0x0fffe000u) * 0x1p112f;
  const float hi = __uint_as_float((u >> 3) & 0x0fffe000u) * 0x1p112f;
  return make_float2(__uint_as_float(__float_as_uint(lo) | ((u << 16) & 0x80000000u)),
                     __uint_as_float(__float_as_uint(hi) | (u & 0x80000000u)));
}

// Byte offset, in an exchange tile and in the P tile, of 16-byte piece u
// (0..7) of row r's 64 16-bit values: row r at r * 128, piece u at
// (u ^ (r & 7)) * 16.  This is the 128-byte-swizzled K-major operand layout
// (8-row groups of 1 KB) the P*V MMA reads P in; each warp's 32 rows are one
// contiguous 4 KB block (one bulk copy), and the eight rows a quarter-warp
// touches at once fall in eight bank groups.
constexpr int X_WARP_BYTES = 32 * KT * 2;
__device__ __forceinline__ uint32_t x_off(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }
// Byte offset of 16-byte piece u of row r in the RoPE part of the Q slice,
// rows of rw * 2 bytes swizzled to that width (64-byte rows: piece ^ row
// bits 1-2; 32-byte rows: piece ^ row bit 2), matching sdesc_swz.
__device__ __forceinline__ uint32_t qr_off(int r, int u, int rw) {
  return rw == 32 ? (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4)) : (uint32_t)(r * 32 + ((u ^ ((r >> 2) & 1)) << 4));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap rmap16,
                   const __grid_constant__ CUtensorMap rmap32, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_trigger();
  pdl_wait();  // the schedule and Q_abs come from earlier kernels
  if (smem_u32(smem) & 1023u) {  // the same in every CTA: all leave before any barrier
    if (threadIdx.x == 0) flag_error(p.a.err, kErrLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* x_full = bars;               // [XBUF] the peer's partial has landed here
  uint64_t* x_free = x_full + XBUF;      // [XBUF] the peer has consumed what this CTA sent
  uint64_t* sg_full = x_free + XBUF;     // [SGROUPS]
  uint64_t* sg_empty = sg_full + SGROUPS;
  uint64_t* vg_full = sg_empty + SGROUPS;  // [VGROUPS]
  uint64_t* vg_empty = vg_full + VGROUPS;
  uint64_t* s_full = vg_empty + VGROUPS;   // [2] own partial score in buffer b
  uint64_t* s_free = s_full + 2;           // [2] the sender and the finishers have read buffer b
  uint64_t* p_ready = s_free + 2;          // P of the current page is in the P tile
  uint64_t* pv_done = p_ready + 1;         // P*V of the current page has completed
  uint64_t* q_ready = pv_done + 1;
  uint64_t* o_free = q_ready + 1;
  uint64_t* final_bar = q_ready + 2;
  uint64_t* pair_bars = q_ready + 3;       // [4]: the two finisher warps of a lane quarter
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const AttnArgs& a = p.a;
  const int npv = p.npv, dh = npv * 64;
  const int c_lo = (int)rank * npv;                // first latent chunk of this CTA
  const int rw = rank ? p.rb : p.ra;               // RoPE-key columns this CTA scores (0, 16 or 32)
  const int rx = a.d_c + (rank ? p.ra : 0);        // and the first of them
  const CUtensorMap* rmap = rw == 32 ? &rmap32 : &rmap16;
  const uint64_t rswz = rw == 32 ? kSwizzle64 : kSwizzle32;
  const Seg* segs = a.sched.segs;
  const int seg_lo = a.sched.worker_seg[w], seg_hi = a.sched.worker_seg[w + 1];

  if (tid == 32) {
    for (int i = 0; i < XBUF; ++i) {
      mbar_init(&x_full[i], 1);  // own expect_tx + the peer's bytes
      mbar_init(&x_free[i], 1);  // the peer's P*V commit
    }
    for (int i = 0; i < SGROUPS; ++i) {
      mbar_init(&sg_full[i], 1);
      mbar_init(&sg_empty[i], 1);
    }
    for (int i = 0; i < VGROUPS; ++i) {
      mbar_init(&vg_full[i], 1);
      mbar_init(&vg_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 384);  // sender + finishers
    }
    mbar_init(p_ready, 256);  // finishers
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 128);  // sender
    mbar_init(o_free, 256);   // finishers
    mbar_init(final_bar, 2);  // one commit per issuer warp
    for (int i = 0; i < 4; ++i) mbar_init(&pair_bars[i], 64);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    tma_prefetch_desc(&tmap);
    if (rw) tma_prefetch_desc(rmap);
  }
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0 || warp == 2) {
    // ---------------------------------------------------- TMA producers
    // Warp 0 fills the score ring with this CTA's columns of each page;
    // warp 2 fills the latent ring with the page's latent columns again
    // (an L2 hit: the score ring read them a few microseconds earlier).
    // Metadata loads run one step ahead: the next segment while this one
    // streams, the next page id while this page waits for its ring slot.
    const bool score_ring = warp == 0;
    const int nring = score_ring ? SGROUPS : VGROUPS;
    const int ring_bytes = score_ring ? SG_BYTES : VG_BYTES;
    const int rope_cols = score_ring ? rw : 0;
    uint8_t* ring = smem + (score_ring ? OFF_SG : OFF_VG);
    uint64_t* full = score_ring ? sg_full : vg_full;
    uint64_t* empty = score_ring ? sg_empty : vg_empty;
    uint32_t cnt = 0;
    if (seg_lo < seg_hi) {
      int si = seg_lo;
      Seg g = segs[si];
      Seg gn = si + 1 < seg_hi ? segs[si + 1] : g;
      int t = g.t_lo;
      int page_n = a.page_table[(long long)(g.rb / a.n_q) * a.max_pages + t];
      bool more = true;
      while (more) {
        int page = page_n;
        if (++t >= g.t_hi) {
          if (++si < seg_hi) {
            g = gn;
            if (si + 1 < seg_hi) gn = segs[si + 1];
            t = g.t_lo;
          } else {
            more = false;
          }
        }
        if (more) page_n = a.page_table[(long long)(g.rb / a.n_q) * a.max_pages + t];
        const uint32_t gs = cnt % nring;
        if (!mbar_wait_warp(&empty[gs], ((cnt / nring) & 1) ^ 1, abort_flag, a.err)) break;
        if (page < 0 || page >= a.num_pages) {
          if (rank == 0 && score_ring && elect_one()) flag_error(a.err, kErrBounds);
          page = 0;  // keep the pipeline's byte counts; outputs are flagged invalid
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[gs], npv * CHUNK_BYTES + rope_cols * KT * 2);
          for (int q = 0; q < npv; ++q)
            tma_load_2d(ring + gs * ring_bytes + q * CHUNK_BYTES, &tmap, (c_lo + q) * 64, page * KT, &full[gs]);
          if (rope_cols) tma_load_2d(ring + gs * ring_bytes + ROPE_OFF, rmap, rx, page * KT, &full[gs]);
        }
        __syncwarp();
        ++cnt;
      }
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit.
      for (uint32_t q = 0; q < (uint32_t)nring && q < cnt; ++q) {
        const uint32_t last = q + nring * ((cnt - 1 - q) / nring);
        mbar_wait_warp(&full[q], (last / nring) & 1, abort_flag, nullptr, 50000000ull, false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- score-MMA issuer
    // Page t's partial score goes into buffer t & 1, free once the sender and
    // the finishers have read page t - 2's scores from it.
    const uint32_t tS = tbase + TM_S, tQ = tbase + TM_Q;
    const uint32_t sSG = smem_u32(smem + OFF_SG), sQR = smem_u32(smem + OFF_QR);
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);
    uint32_t tg = 0, seg_k = 0;
    bool ok = true;
    Seg gn = seg_lo < seg_hi ? segs[seg_lo] : Seg{};
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = gn;
      if (si + 1 < seg_hi) gn = segs[si + 1];  // in flight while this segment runs
      const int n = g.t_hi - g.t_lo;
      if (!(ok = mbar_wait_warp(q_ready, seg_k & 1, abort_flag, a.err))) break;
      tc_fence_after();
      for (int i = 0; i < n; ++i, ++tg) {
        const uint32_t b = tg & 1;
        if (tg >= 2 && !(ok = mbar_wait_warp(&s_free[b], ((tg - 2) >> 1) & 1, abort_flag, a.err))) break;
        const uint32_t gs = tg % SGROUPS;
        if (!(ok = mbar_wait_warp(&sg_full[gs], (tg / SGROUPS) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t gb = sSG + gs * SG_BYTES, d = tS + b * KT;
          for (int q = 0; q < npv; ++q) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_ts(d, tQ + q * 32 + k * 8, sdesc_sw128(gb + q * CHUNK_BYTES + k * 32, 16, 1024), idS,
                     (q | k) ? 1u : 0u);
          }
          // The RoPE share: rows of rw * 2 bytes, swizzled to that width, both
          // operands in shared memory.
          for (int k = 0; k < rw / 16; ++k)
            mma_ss(d, sdesc_swz(sQR + k * 32, 8 * rw * 2, rswz), sdesc_swz(gb + ROPE_OFF + k * 32, 8 * rw * 2, rswz),
                   idS, 1u);
          tc_commit(&s_full[b]);
          tc_commit(&sg_empty[gs]);  // the score ring slot is free once its MMAs are done
        }
        __syncwarp();
      }
      ++seg_k;
    }
    if (elect_one()) tc_commit(final_bar);
    __syncwarp();
    mbar_wait_warp(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
  } else if (warp == 3) {
    // ------------------------------------------------------ P*V issuer
    const uint32_t tO = tbase + TM_O;
    const uint32_t sVG = smem_u32(smem + OFF_VG), sP = smem_u32(smem + OFF_P);
    const uint32_t idPV = idesc_bf16(128, dh, 0, 1);
    uint32_t tg = 0, seg_k = 0;
    bool ok = true;
    Seg gn = seg_lo < seg_hi ? segs[seg_lo] : Seg{};
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = gn;
      if (si + 1 < seg_hi) gn = segs[si + 1];
      const int n = g.t_hi - g.t_lo;
      for (int i = 0; i < n; ++i, ++tg) {
        if (!(ok = mbar_wait_warp(p_ready, tg & 1, abort_flag, a.err))) break;
        if (i == 0 && seg_k > 0 && !(ok = mbar_wait_warp(o_free, (seg_k - 1) & 1, abort_flag, a.err))) break;
        const uint32_t vs = tg % VGROUPS;
        if (!(ok = mbar_wait_warp(&vg_full[vs], (tg / VGROUPS) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk)
            mma_ss(tO, sdesc_sw128(sP + kk * 32, 16, 1024),
                   sdesc_sw128(sVG + vs * VG_BYTES + kk * 2048, CHUNK_BYTES, 1024), idPV,
                   (i == 0 && kk == 0) ? 0u : 1u);
          tc_commit(pv_done);
          tc_commit(&vg_empty[vs]);
          // The finishers read exchange buffer tg % XBUF before P_tg was
          // ready: hand it back to the peer's sender.
          tc_commit_to(&x_free[tg % XBUF], (uint16_t)(1u << peer));
        }
        __syncwarp();
      }
      ++seg_k;
    }
    if (elect_one()) tc_commit(final_bar);
    __syncwarp();
    mbar_wait_warp(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
  } else if (warp >= 4) {
    // ------------------------------------------- sender and finisher warpgroups
    // Thread r of either warpgroup owns row r (= TMEM lane r) of the page.
    const bool sender = warp < 8;
    const int h = warp >= 12 ? 1 : 0;  // finisher half: keys [32h, 32h + 32)
    const int r = tid - (sender ? 128 : 256 + 128 * h);
    const int lane = tid & 31;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + TM_S, tO = tbase + lane_off + TM_O, tQ = tbase + lane_off + TM_Q;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool r_ok = mbar_wait(bar, parity, abort_flag, a.err);
      return __all_sync(0xffffffffu, r_ok);
    };

    if (sender) {
      // Reads each page's own partial score (all 64 keys of its row) from
      // TMEM, packs it to fp16, stages it and ships it to the peer with one
      // bulk copy per warp; also loads each segment's Q slice.
      uint8_t* sQR = smem + OFF_QR;
      uint8_t* sXS = smem + OFF_XS;
      const uint32_t peer_x = map_peer(smem_u32(smem + OFF_X), peer);
      const uint32_t peer_xbar = map_peer(smem_u32(&x_full[0]), peer);
      const __nv_bfloat16* qabs = static_cast<const __nv_bfloat16*>(a.qabs);
      // Row r of this CTA's Q slice: the latent chunks c_lo .. c_lo + npv - 1
      // into TMEM, the RoPE share into shared memory.
      auto load_q = [&](int rb) {
        const uint4* src =
            (r < a.n_h) ? reinterpret_cast<const uint4*>(qabs + ((long long)rb * a.qrows + r) * a.d_cr) : nullptr;
        for (int q = 0; q < npv; ++q) {
          uint32_t wv[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 v = src ? __ldg(src + ((c_lo + q) * 64 + u * 8) / 8) : make_uint4(0, 0, 0, 0);
            wv[4 * u + 0] = v.x;
            wv[4 * u + 1] = v.y;
            wv[4 * u + 2] = v.z;
            wv[4 * u + 3] = v.w;
          }
          tmem_st32(tQ + q * 32, wv);
        }
        for (int u = 0; u < rw / 8; ++u) {
          const uint4 v = src ? __ldg(src + (rx + u * 8) / 8) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(sQR + qr_off(r, u, rw)) = v;
        }
        fence_proxy_async_smem();  // the MMA (async proxy) reads what the threads wrote
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(q_ready);
      };
      // Segment metadata stays in registers, the next segment's loaded a
      // segment ahead.
      Seg g_cur = seg_lo < seg_hi ? segs[seg_lo] : Seg{};
      Seg g_nxt = seg_lo + 1 < seg_hi ? segs[seg_lo + 1] : Seg{};
      if (seg_lo < seg_hi) load_q(g_cur.rb);
      // The next segment's query rows are pulled into L2 while this segment
      // streams, so loading them at the segment boundary reads L2, not HBM.
      const uint32_t q_half = (uint32_t)((a.n_h + 1) / 2) * a.d_cr * 2;
      auto prefetch_q = [&](int rb) {
        if (tid == 128) {
          const uint8_t* base = reinterpret_cast<const uint8_t*>(qabs + (long long)rb * a.qrows * a.d_cr);
          const uint32_t lo = rank ? q_half : 0, hi = rank ? (uint32_t)a.n_h * a.d_cr * 2 : q_half;
          if (hi > lo) prefetch_l2(base + lo, hi - lo);
        }
      };
      uint32_t tg = 0;
      for (int si = seg_lo; si < seg_hi && ok; ++si) {
        const Seg g = g_cur;
        const int n = g.t_hi - g.t_lo;
        if (si + 1 < seg_hi) prefetch_q(g_nxt.rb);
        for (int i = 0; i < n; ++i, ++tg) {
          const uint32_t b = tg & 1, xb = tg % XBUF;
          if (!(ok = wait_all(&s_full[b], (tg >> 1) & 1))) break;
          tc_fence_after();
          uint32_t cur[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
            tmem_ld32(tS + b * KT + 32 * half, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              cur[16 * half + j] = pack_f16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          }
          // Keys past the row block's end (the tail of its last page) may hold
          // anything, NaN included; the peer's exchange MMA multiplies every
          // key of a row by the identity's zeros too, so they travel as 0.
          const int valid_all = min(KT, g.nkeys - (g.t_lo + i) * KT);
          if (valid_all < KT) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              if (2 * x >= valid_all) cur[x] = 0u;
              else if (2 * x + 1 >= valid_all) cur[x] &= 0x0000ffffu;
            }
          }
          tc_fence_before();
          mbar_arrive(&s_free[b]);
          // The segment's scores are all read after its last page, so the next
          // segment's Q may replace this one's.
          if (i + 1 == n && si + 1 < seg_hi) load_q(g_nxt.rb);
          // The staging block is reused once the copy engine has read it.
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(sXS + x_off(r, u)) =
                make_uint4(cur[4 * u], cur[4 * u + 1], cur[4 * u + 2], cur[4 * u + 3]);
          fence_proxy_async_smem();  // the copy engine reads what the threads wrote
          // The peer's partial of this page will land in exchange buffer xb.
          if (r == 0) mbar_arrive_expect_tx(&x_full[xb], X_BYTES);
          // Buffer xb of the peer is free once its finishers have read page
          // tg - XBUF from it.
          if (tg >= XBUF && !(ok = wait_all(&x_free[xb], ((tg / XBUF) - 1) & 1))) break;
          __syncwarp();
          if (lane == 0) {
            const uint32_t blk = (uint32_t)((warp & 3) * X_WARP_BYTES);
            bulk_copy_to_peer(peer_x + xb * X_BYTES + blk, smem_u32(sXS) + blk, X_WARP_BYTES, peer_xbar + xb * 8);
            bulk_commit();
          }
        }
        g_cur = g_nxt;
        if (si + 2 < seg_hi) g_nxt = segs[si + 2];
      }
      // Every credit the peer returns lands before this CTA may exit: wait for
      // its consumption of the last pages shipped (page p is the (p / XBUF)-th
      // use of buffer p % XBUF).
      if (ok)
        for (uint32_t pg = tg > (uint32_t)XBUF ? tg - XBUF : 0; pg < tg; ++pg)
          if (!wait_all(&x_free[pg % XBUF], (pg / XBUF) & 1)) break;
      if (lane == 0) bulk_wait_read_all();  // no copy may still read the staging block at exit
    } else {
      // Two finisher warpgroups: half h owns keys [32h, 32h + 32) of every
      // row and half of O's columns; the two threads of a row (their warps
      // share a lane quarter) agree on the row max through a bounded
      // 64-arrival mbarrier.
      uint64_t* pair_bar = &pair_bars[warp & 3];
      uint32_t pair_phase = 0;
      auto pair_sync = [&]() -> bool {
        mbar_arrive(pair_bar);
        bool r_ok = mbar_wait(pair_bar, pair_phase & 1, abort_flag, a.err);
        ++pair_phase;
        return __all_sync(0xffffffffu, r_ok);
      };
      float* mh = reinterpret_cast<float*>(smem + OFF_MH);
      const int hc0 = h * (dh / 64), hc1 = hc0 + dh / 64;  // this half's 32-column chunks of O
      Seg g_cur = seg_lo < seg_hi ? segs[seg_lo] : Seg{};
      Seg g_nxt = seg_lo + 1 < seg_hi ? segs[seg_lo + 1] : g_cur;
      uint8_t* sV = smem + OFF_VG;
      uint8_t* sPt = smem + OFF_P;
      const uint8_t* sX = smem + OFF_X;
      float m_used = -INFINITY, l = 0.f;
      uint32_t tg = 0;
      for (int si = seg_lo; si < seg_hi && ok; ++si) {
        const Seg g = g_cur;
        const int n = g.t_hi - g.t_lo;
        for (int i = 0; i < n; ++i, ++tg) {
          const int t = g.t_lo + i;
          const uint32_t b = tg & 1;
          // This CTA's exact partial from TMEM (the buffer is released at
          // once), then the peer's fp16 partial from the exchange buffer.
          if (!(ok = wait_all(&s_full[b], (tg >> 1) & 1))) break;
          tc_fence_after();
          float s[32];
          {
            uint32_t v[32];
            tmem_ld32(tS + b * KT + 32 * h, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(v[j]);
          }
          tc_fence_before();
          mbar_arrive(&s_free[b]);  // the score MMA of page tg + 2 may overwrite it
          const uint32_t xb = tg % XBUF;
          if (!(ok = wait_all(&x_full[xb], (tg / XBUF) & 1))) break;
          {
            uint4 pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              pv[u] = *reinterpret_cast<const uint4*>(sX + xb * X_BYTES + x_off(r, 4 * h + u));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t pw[4] = {pv[u].x, pv[u].y, pv[u].z, pv[u].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 y = unpack_f16x2(pw[e]);
                s[8 * u + 2 * e] += y.x;
                s[8 * u + 2 * e + 1] += y.y;
              }
            }
          }
          const int valid_all = min(KT, g.nkeys - t * KT);  // >= 1: every tile holds a key
          const int valid = valid_all - 32 * h;             // valid keys among this half's 32
          if (valid < 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j >= valid) s[j] = -INFINITY;
          }
          float mt;
          {
            float mx[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) mx[j] = fmaxf(s[j], s[j + 16]);
#pragma unroll
            for (int w2 = 8; w2 >= 1; w2 >>= 1)
#pragma unroll
              for (int j = 0; j < w2; ++j) mx[j] = fmaxf(mx[j], mx[j + w2]);
            float* slot = mh + (tg & 1) * 256;
            slot[h * 128 + r] = mx[0];
            if (!(ok = pair_sync())) break;
            mt = fmaxf(slot[r], slot[128 + r]);
          }
          // Running max with lazy rescaling: O and l stay relative to m_used
          // until a page's max exceeds it by more than 2^8.  Both halves take
          // the same decision from the same two numbers.
          bool resc = false;
          float scale = 1.f;
          if (i == 0) {
            m_used = mt;
            l = 0.f;
          } else if (mt > m_used + 8.f) {
            scale = fast_exp2(m_used - mt);
            m_used = mt;
            resc = true;
          }
          uint32_t pk[16];
          float psum;
          {
            float ps[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) ps[u] = 0.f;
            // The row sum adds the fp32 weights (not their bf16 roundings: the
            // difference is random, 2^-9 relative per key, and unpacking the
            // rounded pairs would cost two more instructions per pair).
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float e0 = fast_exp2(s[2 * u] - m_used), e1 = fast_exp2(s[2 * u + 1] - m_used);
              ps[u & 7] += e0 + e1;
              __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
              pk[u] = *reinterpret_cast<uint32_t*>(&v2);
            }
#pragma unroll
            for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
              for (int j = 0; j < w2; ++j) ps[j] += ps[j + w2];
            psum = ps[0];
          }
          // The previous page's P*V must be done before P is overwritten or O
          // rescaled.
          if (tg > 0) {
            if (!(ok = wait_all(pv_done, (tg - 1) & 1))) break;
            tc_fence_after();
          }
          if (__any_sync(0xffffffffu, resc)) {
            for (int cc = hc0; cc < hc1; ++cc) {
              uint32_t v[32];
              tmem_ld32(tO + cc * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * scale);
              tmem_st32(tO + cc * 32, v);
            }
            l *= scale;
          }
          // P row r, keys 32h .. 32h + 31: pieces 4h .. 4h + 3 of the
          // 128-byte-swizzled K-major tile (the SS P*V MMA's A operand).
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(sPt + x_off(r, 4 * h + u)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          l += psum;
          if (valid_all < KT) {
            // Keys past the end: P is 0 there, but 0 * NaN would still poison
            // O, so clear those rows of this page's latent chunks (once they
            // have landed).
            if (!(ok = wait_all(&vg_full[tg % VGROUPS], (tg / VGROUPS) & 1))) break;
            uint8_t* gb = sV + (tg % VGROUPS) * VG_BYTES;
            const int rows = KT - valid_all, units = rows * 8 * npv;
            for (int x = r + 128 * h; x < units; x += 256) {
              const int q = x / (rows * 8), rem = x - q * rows * 8;
              *reinterpret_cast<uint4*>(gb + q * CHUNK_BYTES + (valid_all + rem / 8) * 128 + (rem % 8) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();  // the MMA (async proxy) reads P and the cleared rows
          tc_fence_before();
          mbar_arrive(p_ready);
          if (i + 1 < n) continue;

          // ---- epilogue of the segment ----
          if (!(ok = wait_all(pv_done, tg & 1))) break;
          tc_fence_after();
          // Row sum: both halves add the two partial sums in the same order.
          // The sums borrow the max slot of the previous page: the partner
          // read that page's maxima before the last pair sync, and the next
          // page's maxima go there only after the second sync below.
          float* ls = mh + ((tg + 1) & 1) * 256;
          ls[h * 128 + r] = l;
          if (!(ok = pair_sync())) break;
          const float lrow = ls[r] + ls[128 + r];
          if (!(ok = pair_sync())) break;
          // A whole row block is normalised into obar (bf16); a piece of a
          // split row block is normalised by its own sum into its partial
          // slot (bf16) and leaves this CTA's (m, l) beside it.
          const bool whole = g.slot < 0;
          const float inv = 1.f / lrow;
          __nv_bfloat16* const dst_row =
              whole ? static_cast<__nv_bfloat16*>(a.obar) + ((long long)g.rb * a.n_h + r) * a.d_c
                    : static_cast<__nv_bfloat16*>(a.part_o) + ((long long)g.slot * a.n_h + r) * a.d_c;
          for (int cc = hc0; cc < hc1; ++cc) {
            uint32_t v[32];
            tmem_ld32(tO + cc * 32, v);
            tmem_ld_wait();
            if (r < a.n_h) {
              uint4* dst = reinterpret_cast<uint4*>(dst_row + (int)rank * dh + cc * 32);
              float dummy = 0.f;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 o;
                o.x = pack_bf16(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv, dummy);
                o.y = pack_bf16(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv, dummy);
                o.z = pack_bf16(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv, dummy);
                o.w = pack_bf16(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv, dummy);
                dst[q] = o;
              }
            }
          }
          if (!whole && h == 0 && r < a.n_h) {
            float* ml = a.part_ml + ml_index(g.slot, (int)rank, a.n_h, r);
            ml[0] = m_used;
            ml[1] = lrow;
          }
          tc_fence_before();
          mbar_arrive(o_free);
        }
        g_cur = g_nxt;
        if (si + 2 < seg_hi) g_nxt = segs[si + 2];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still write into it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
}

}  // namespace attn_tc
}  // namespace mla
