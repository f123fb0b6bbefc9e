// Absorbed latent attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// one 2-CTA cluster per worker, the two CTAs working as one MMA pair.
//
// What it computes is the same as attn_simt.cuh ("ai-decoupled-rope-mla",
// absorbed score and output equations): for one query token, its heads form
// the M = 128 rows (heads beyond n_h are zero rows), and for each 64-key cache
// page
//   S  = Q_abs [128 x d_cr] * page^T [d_cr x 64]      (content + position
//        score in one contraction: the cache row is [c | k_R] and the query
//        row is [q~ | q_R], both pre-scaled by s*log2(e))
//   P  = exp2(S - m)  (online softmax, running max m, running sum l)
//   O += P [128 x 64] * page[:, latent] [64 x d_c]
// Both products are dense because every head shares the cache ("Latent
// Attention Meets RoPE": one shared position key; the latent is shared by
// construction).
//
// B200 layout.  The 128 x d_c fp32 accumulator of one token fills a whole
// SM's TMEM, so the work is spread over a CTA pair with cta_group::2 MMAs:
// each CTA owns 64 of the heads (64 rows of A) and keeps the complete score
// and softmax state for them, and half of B's columns come from each CTA:
//   score:  B = the page rows; CTA r supplies keys [32r, 32r + 32) of all
//           d_cr columns, and holds S for its heads over all 64 keys;
//   output: B = the page's latent columns; CTA r supplies columns
//           [r d_c/2, (r + 1) d_c/2) of all 64 keys, and holds O for its heads
//           over all d_c columns (lanes 0-63: the first half, 64-127: the
//           second, d_c/2 TMEM columns).
// No partial score crosses between the CTAs and each CTA's softmax covers
// only its own 64 heads.  The RoPE key is read as one more 64-column chunk of
// the row (columns past d_cr read as zero; the query's RoPE part is padded
// with zeros to match).
//
// TMEM columns: O [0, d_c/2), two score buffers S0 [256, 288) and
// S1 [288, 320) (64 keys of 64 heads: 32 columns each), the first (up to six)
// 64-column chunks of the CTA's Q rows from 320 (an A operand in TMEM holds
// the CTA's rows twice, 32 columns per chunk).  The rest of Q (at most three
// chunks) sits in shared memory.
//
// Shared memory (1024-byte aligned pieces):
//   score ring, 3 slots: the CTA's 32 keys of every 64-column chunk of a page
//     (128-byte swizzled, 4 KB per chunk), freed when the page's score MMA
//     completes;
//   latent ring, 2 slots: all 64 keys of the CTA's d_c/128 latent chunks
//     (8 KB each), freed by P*V.  The page went through L2 for the score
//     ring a few microseconds earlier, so HBM sees its bytes once;
//   the shared-memory part of Q, two P tiles (64 heads x 64 keys bf16, the
//   A operand of P*V), a staging tile through which the TMEM part of Q
//   passes (loaded coalesced, read back one row per thread), and the
//   row-max / row-sum exchange slots.
// The page loads of both CTAs complete on the even CTA's barriers (the MMA
// issuer's).  The last page of a row block, whose tail rows may hold
// anything (NaN included), lands on a barrier of the CTA's own instead, so
// that its softmax threads can clear those rows before P*V multiplies them
// by zero.
//
// Warp roles (384 threads): warp 0 = score-ring TMA producer, warp 2 = TMEM
// allocator and latent-ring producer, warp 1 of the even CTA = MMA issuer
// (order: S(t), then P*V(t-1), so each page's softmax overlaps the next
// page's score MMA), warps 4-11 = softmax.  Softmax thread (lane quarter q,
// column half c) owns TMEM lane L = 32q + lane: head L mod 64, keys
// [32 (L div 64) + 16c, +16) of each page, and O columns
// [(L div 64) d_c/2 + c d_c/4, +d_c/4); the four threads of a head agree on
// its row max through shared memory and a 128-thread named barrier, and each
// keeps a partial row sum (the same rescalings), added at the end.  Every
// wait is bounded (sm100::mbar_wait).
//
// A worker walks its schedule segments (sched.cuh).  At a segment's end the
// softmax warps load the next segment's Q rows, then write this segment's O:
// normalised into obar for a whole row block, or for a piece of a split row
// block into its partial slot with its (m, l).  When the launch passes
// arrival counters (AttnArgs::arrive), each piece then counts in, and the
// last piece of a row block to do so merges every piece's slot into obar
// (otherwise combine_kernel does it after the launch).
#pragma once
#include "attn_simt.cuh"
#include "sm100.cuh"

namespace mla {
namespace attn_tc {
using namespace sm100;

constexpr int THREADS = 384;
constexpr int KT = 64;                    // keys per page
constexpr int HEADS = 64;                 // query rows per CTA
constexpr int CH_S = 32 * 128;            // 32 keys x 64 bf16 columns (4 KB)
constexpr int CH_V = KT * 128;            // 64 keys x 64 bf16 columns (8 KB)
constexpr int MAX_NK = 9;                 // 64-column chunks of a cache row (d_c <= 512, d_r <= 64)
constexpr int MAX_NPV = 4;                // latent chunks per CTA (d_c / 128)
constexpr int MAX_TS = 6;                 // chunks of Q held in TMEM
constexpr int MAX_PIECES = 80;            // pieces of a split row block merged in the kernel (<= workers)
constexpr int SGS = 3, VGS = 2;           // ring slots
constexpr int SG_BYTES = MAX_NK * CH_S;   // 36 KB
constexpr int VG_BYTES = MAX_NPV * CH_V;  // 32 KB
constexpr int QS_BYTES = 3 * CH_V;        // the chunks of Q beyond the first MAX_TS (64 rows each)
constexpr int P_BYTES = HEADS * KT * 2;   // 8 KB
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 320, TM_COLS = 512;

constexpr int OFF_SG = 0;
constexpr int OFF_VG = OFF_SG + SGS * SG_BYTES;
constexpr int OFF_QS = OFF_VG + VGS * VG_BYTES;
constexpr int OFF_P = OFF_QS + QS_BYTES;
constexpr int OFF_STG = OFF_P + 2 * P_BYTES;       // staging tile for the TMEM part of Q (64 rows x 128 B)
constexpr int OFF_MX = OFF_STG + CH_V;             // [2][64] float4: the four partial maxima of a head
constexpr int OFF_LS = OFF_MX + 2 * HEADS * 16;    // [64] float4: the four partial sums
constexpr int OFF_BAR = OFF_LS + HEADS * 16;
constexpr int NUM_BARS = 2 * SGS + 3 * VGS + 2 + 2 + 2 + 3;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
static_assert(OFF_VG % 1024 == 0 && OFF_QS % 1024 == 0 && OFF_P % 1024 == 0 && OFF_STG % 1024 == 0 &&
                  SG_BYTES % 1024 == 0 &&
                  VG_BYTES % 1024 == 0,
              "swizzled operands need 1024-byte aligned tiles");
// No slack for aligning the base: the kernel has no static shared memory, so
// its dynamic block starts on a 1024-byte boundary (the kernel checks this
// and reports MLA_ERR_UNSUPPORTED otherwise).
constexpr size_t SMEM_BYTES = SMEM_USED;
static_assert(SMEM_BYTES <= 232448, "over the 227 KB of shared memory a CTA can have");

// 2^x with the MUFU ex2 instruction (flush-to-zero; ~2 ulp), used for the
// softmax weights, which are rounded to bf16 right after.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

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
// Asks L2 to fetch `bytes` (a multiple of 16) from global memory ahead of use.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// A shared-memory descriptor advanced by `bytes` (its address field counts
// 16-byte units; every operand here stays below 256 KB, so no carry leaves it).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// Walks a worker's segments page by page: (segment, tile) and the cache page
// id, with the next page's id loaded one step ahead.
struct PageWalk {
  const Seg* segs;
  const int32_t* page_table;
  int max_pages, n_q;
  int si, seg_hi, t;
  Seg g, gn;
  bool more;
  int page_next;
  __device__ void start(int seg_lo) {
    si = seg_lo;
    more = si < seg_hi;
    if (!more) return;
    g = segs[si];
    gn = si + 1 < seg_hi ? segs[si + 1] : g;
    t = g.t_lo;
    page_next = page_table[(long long)(g.rb / n_q) * max_pages + t];
  }
  // The current page's id; steps to the next page.
  __device__ int next(Seg& cur, int& tile) {
    cur = g;
    tile = t;
    const int page = page_next;
    if (++t >= g.t_hi) {
      if (++si < seg_hi) {
        g = gn;
        if (si + 1 < seg_hi) gn = segs[si + 1];
        t = g.t_lo;
      } else {
        more = false;
      }
    }
    if (more) page_next = page_table[(long long)(g.rb / n_q) * max_pages + t];
    return page;
  }
};

template <int NPV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap mapS, const __grid_constant__ CUtensorMap mapV,
                   const AttnArgs a) {
  constexpr int NCH = 2 * NPV;                       // latent chunks of a row
  constexpr int NK = NCH + 1;                        // + the RoPE chunk
  constexpr int NTS = NK < MAX_TS ? NK : MAX_TS;     // chunks of Q in TMEM
  constexpr int NSS = NK - NTS;                      // chunks of Q in shared memory
  static_assert(NPV >= 1 && NPV <= MAX_NPV && NSS * CH_V <= QS_BYTES, "latent width");
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the same in every CTA: all leave before any barrier
    if (threadIdx.x == 0) flag_error(a.err, kErrLayout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* sg_full = bars;                // [SGS] both CTAs' score chunks landed (even CTA's)
  uint64_t* sg_empty = sg_full + SGS;      // [SGS] the page's score MMA is done (both CTAs)
  uint64_t* vg_full = sg_empty + SGS;      // [VGS] both CTAs' latent chunks landed (even CTA's)
  uint64_t* vg_empty = vg_full + VGS;      // [VGS] the page's P*V is done (both CTAs)
  uint64_t* vg_part = vg_empty + VGS;      // [VGS] this CTA's chunks of a row block's last page landed
  uint64_t* s_full = vg_part + VGS;        // [2] S of the page in buffer b is complete (both CTAs)
  uint64_t* p_ready = s_full + 2;          // [2] both CTAs' P of the page are in their P tiles (even CTA's)
  uint64_t* pv_done = p_ready + 2;         // [2] P*V of the page has completed (both CTAs)
  uint64_t* q_ready = pv_done + 2;         // a segment's Q rows are in place in both CTAs (even CTA's)
  uint64_t* o_free = q_ready + 1;          // both CTAs have read a segment's O (even CTA's)
  uint64_t* final_bar = o_free + 1;        // the MMA issuer's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int w = blockIdx.x >> 1;

  if (tid == 32) {
    for (int i = 0; i < SGS; ++i) {
      mbar_init(&sg_full[i], 1);   // the even CTA's arrive.expect_tx + both CTAs' bytes
      mbar_init(&sg_empty[i], 1);  // commit of the score MMA
    }
    for (int i = 0; i < VGS; ++i) {
      mbar_init(&vg_full[i], 1);
      mbar_init(&vg_empty[i], 1);
      mbar_init(&vg_part[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 16);  // one arrive per softmax warp of both CTAs
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(q_ready, 16);
    mbar_init(o_free, 16);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, TM_COLS);
    tmem_relinquish_pair();
  }
  if (tid == 0) {
    tma_prefetch_desc(&mapS);
    tma_prefetch_desc(&mapV);
  }
  __syncthreads();
  cluster_sync_all();  // the peer's barriers and TMEM exist before anyone signals them
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // Everything above overlaps the previous kernel's tail; the schedule and
  // Q_abs come from earlier kernels.
  pdl_wait();
  pdl_trigger();  // only now: a successor may read its weights before its own wait
  const Seg* segs = a.sched.segs;
  const int seg_lo = a.sched.worker_seg[w], seg_hi = a.sched.worker_seg[w + 1];

  if (warp == 0 || warp == 2) {
    // ---------------------------------------------------- TMA producers
    // Warp 0 fills the score ring (this CTA's 32 keys of every chunk), warp
    // 2 the latent ring (all 64 keys of this CTA's latent chunks); both
    // complete on the even CTA's barriers, except a row block's last page in
    // the latent ring (see above).
    const bool score_ring = warp == 0;
    const int nslots = score_ring ? SGS : VGS;
    uint64_t* full = score_ring ? sg_full : vg_full;
    uint64_t* empty = score_ring ? sg_empty : vg_empty;
    uint8_t* ring = smem + (score_ring ? OFF_SG : OFF_VG);
    const int slot_bytes = score_ring ? SG_BYTES : VG_BYTES;
    const uint32_t full_even = map_peer(smem_u32(full), 0);
    PageWalk pw{segs, a.page_table, a.max_pages, a.n_q, 0, seg_hi, 0, Seg{}, Seg{}, false, 0};
    pw.start(seg_lo);
    static_assert(VGS == 2, "two latent slots");
    uint32_t cnt = 0, part_cnt0 = 0, part_cnt1 = 0;  // tail loads per latent slot
    while (pw.more) {
      Seg g;
      int t;
      int page = pw.next(g, t);
      const uint32_t s = cnt % nslots;
      if (!mbar_wait_warp(&empty[s], ((cnt / nslots) & 1) ^ 1, abort_flag, a.err)) break;
      if (page < 0 || page >= a.num_pages) {
        if (rank == 0 && score_ring && elect_one()) flag_error(a.err, kErrBounds);
        page = 0;  // keep the pipeline's byte counts; outputs are flagged invalid
      }
      const bool tail = (t + 1) * KT > g.nkeys;  // keys past the row block's end in this page
      uint8_t* dst = ring + s * slot_bytes;
      if (elect_one()) {
        if (score_ring) {
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * NK * CH_S);
          for (int c = 0; c < NK; ++c)
            tma_load_2d_pair(dst + c * CH_S, &mapS, 64 * c, page * KT + (int)rank * 32, full_even + 8 * s);
        } else if (!tail) {
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * NPV * CH_V);
          for (int q = 0; q < NPV; ++q)
            tma_load_2d_pair(dst + q * CH_V, &mapV, ((int)rank * NPV + q) * 64, page * KT, full_even + 8 * s);
        } else {
          mbar_arrive_expect_tx(&vg_part[s], NPV * CH_V);
          for (int q = 0; q < NPV; ++q)
            tma_load_2d(dst + q * CH_V, &mapV, ((int)rank * NPV + q) * 64, page * KT, &vg_part[s]);
          if (rank == 0) mbar_arrive(&full[s]);  // the phase still advances; p_ready covers the bytes
        }
      }
      __syncwarp();
      if (!score_ring && tail) {
        if (s == 0) ++part_cnt0;
        else ++part_cnt1;
      }
      ++cnt;
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit (the even
      // CTA's barriers count the odd CTA's bytes too).
      if (rank == 0)
        for (uint32_t q = 0; q < (uint32_t)nslots && q < cnt; ++q) {
          const uint32_t last = q + nslots * ((cnt - 1 - q) / nslots);
          mbar_wait_warp(&full[q], (last / nslots) & 1, abort_flag, nullptr, 50000000ull, false);
        }
      if (!score_ring)
        for (int q = 0; q < VGS; ++q) {
          const uint32_t n_q = q == 0 ? part_cnt0 : part_cnt1;
          if (n_q) mbar_wait_warp(&vg_part[q], (n_q - 1) & 1, abort_flag, nullptr, 50000000ull, false);
        }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t tS = tbase + TM_S, tO = tbase + TM_O, tQ = tbase + TM_Q;
    const uint64_t dS0 = sdesc_sw128(smem_u32(smem + OFF_SG), 16, 1024);
    const uint64_t dQ0 = sdesc_sw128(smem_u32(smem + OFF_QS), 16, 1024);
    const uint64_t dP0 = sdesc_sw128(smem_u32(smem + OFF_P), 16, 1024);
    const uint64_t dV0 = sdesc_sw128(smem_u32(smem + OFF_VG), CH_V, 1024);  // MN-major: LBO = chunk stride
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);
    const uint32_t idV2 = idesc_bf16(128, 256, 0, 1), idV1 = idesc_bf16(128, 128, 0, 1);
    bool ok = true;
    // P*V of page pj: waits for both CTAs' P (and, at a segment's first page,
    // for both CTAs to have read the previous segment's O).
    auto issue_pv = [&](uint32_t pj, bool first, uint32_t sk) -> bool {
      const uint32_t vs = pj % VGS;
      bool r_ok = mbar_wait(&vg_full[vs], (pj / VGS) & 1, abort_flag, a.err);
      if (r_ok && first && sk > 0) r_ok = mbar_wait(o_free, (sk - 1) & 1, abort_flag, a.err);
      if (r_ok) r_ok = mbar_wait(&p_ready[pj & 1], (pj >> 1) & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, r_ok)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t a0 = desc_add(dP0, (pj & 1) * P_BYTES);
        const uint64_t b0 = desc_add(dV0, vs * VG_BYTES);
#pragma unroll
        for (int k = 0; k < KT / 16; ++k) {
#pragma unroll
          for (int m = 0; m < (NPV + 1) / 2; ++m)
            mma_pair_ss(tO + m * 128, desc_add(a0, k * 32), desc_add(b0, m * 2 * CH_V + k * 2048),
                        (2 * m + 1 < NPV) ? idV2 : idV1, (first && k == 0) ? 0u : 1u);
        }
        tc_commit_pair(&pv_done[pj & 1], 3);
        tc_commit_pair(&vg_empty[vs], 3);
      }
      __syncwarp();
      return true;
    };
    uint32_t j = 0, seg_k = 0, prev_j = 0, prev_sk = 0;
    bool have_prev = false, prev_first = false;
    for (int si = seg_lo; si < seg_hi && ok; ++si, ++seg_k) {
      const Seg g = segs[si];
      const int n = g.t_hi - g.t_lo;
      for (int i = 0; i < n; ++i, ++j) {
        if (i == 0) {
          // The previous segment's last P*V first, then this segment's Q.
          if (have_prev && !(ok = issue_pv(prev_j, prev_first, prev_sk))) break;
          have_prev = false;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_ready, seg_k & 1, abort_flag, a.err)))) break;
        }
        const uint32_t gs = j % SGS;
        if (!(ok = mbar_wait_warp(&sg_full[gs], (j / SGS) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t d = tS + (j & 1) * 32;
          const uint64_t b0 = desc_add(dS0, gs * SG_BYTES);
#pragma unroll
          for (int c = 0; c < NK; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t b = desc_add(b0, c * CH_S + k * 32);
              if (c < NTS)
                mma_pair_ts(d, tQ + c * 32 + k * 8, b, idS, (c | k) ? 1u : 0u);
              else
                mma_pair_ss(d, desc_add(dQ0, (c - NTS) * CH_V + k * 32), b, idS, (c | k) ? 1u : 0u);
            }
          }
          tc_commit_pair(&s_full[j & 1], 3);
          tc_commit_pair(&sg_empty[gs], 3);
        }
        __syncwarp();
        if (have_prev && !(ok = issue_pv(prev_j, prev_first, prev_sk))) break;
        have_prev = true;
        prev_j = j;
        prev_first = i == 0;
        prev_sk = seg_k;
      }
    }
    if (ok && have_prev) issue_pv(prev_j, prev_first, prev_sk);
    if (elect_one()) tc_commit_pair(final_bar, 1);
    __syncwarp();
    mbar_wait_warp(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax
    const int q4 = warp & 3, ch = (warp - 4) >> 2, grp = warp & 1;
    const int L = q4 * 32 + lane, hl = L & 63, kh = L >> 6, part = kh * 2 + ch;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + lane_off + TM_S, tO = tbase + lane_off + TM_O, tQ = tbase + lane_off + TM_Q;
    const int head = (int)rank * HEADS + hl;
    const bool live = head < a.n_h;
    float* mx = reinterpret_cast<float*>(smem + OFF_MX);  // [2][64][4]
    float* lsum = reinterpret_cast<float*>(smem + OFF_LS);  // [64][4]
    const uint32_t p_ready_even = map_peer(smem_u32(p_ready), 0);
    const uint32_t q_ready_even = map_peer(smem_u32(q_ready), 0);
    const uint32_t o_free_even = map_peer(smem_u32(o_free), 0);
    const __nv_bfloat16* qabs = static_cast<const __nv_bfloat16*>(a.qabs);
    // A failed wait clears `ok` (warp-uniform) and the rest of the work is
    // skipped, but every thread still walks every page and every Q load so
    // that the named barriers always see all of their threads.
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool r_ok = mbar_wait(bar, parity, abort_flag, a.err);
      return __all_sync(0xffffffffu, r_ok);
    };
    auto signal_even = [&](uint32_t bar_even) {
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(bar_even);
    };
    // This CTA's Q rows of row block rb: chunks [0, NTS) into TMEM (lane L
    // holds head hl; both lane halves take the row), the rest into shared
    // memory (one thread per row and chunk).
    // A segment's Q rows: q_issue() issues every global load into registers
    // before any store (coalesced: softmax thread tau = 0..255 takes 16-byte
    // pieces tau and tau + 256 of each 64-row x 128-byte chunk, eight threads
    // per row segment); q_store() writes them.  The next segment's rows are
    // loaded once the current segment's last score MMA is complete, from L2
    // (prefetched a few pages earlier).
    uint4 pv[NK][2];
    auto q_issue = [&](int rb) {
      const int tau = tid - 128;
#pragma unroll
      for (int c = 0; c < NK; ++c)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int pc = tau + 256 * h, r = pc >> 3, e0 = 64 * c + 8 * (pc & 7), hd = (int)rank * HEADS + r;
          pv[c][h] = (ok && hd < a.n_h && e0 < a.q_row)
                         ? __ldg(reinterpret_cast<const uint4*>(qabs + ((long long)rb * a.qrows + hd) * a.q_row + e0))
                         : make_uint4(0, 0, 0, 0);
        }
    };
    auto q_store = [&]() {
      const int tau = tid - 128;
      // Chunks [NTS, NK) go straight to their shared-memory tiles.
#pragma unroll
      for (int s2 = 0; s2 < NSS; ++s2)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int pc = tau + 256 * h, r = pc >> 3, u = pc & 7;
          *reinterpret_cast<uint4*>(smem + OFF_QS + s2 * CH_V + r * 128 + ((u ^ (r & 7)) << 4)) = pv[NTS + s2][h];
        }
      // Chunks [0, NTS) pass through the staging tile, one at a time: thread
      // (L, ch) then stores columns [16 ch, 16 ch + 16) of the chunk for
      // TMEM lane L (both lane halves hold row L mod 64).
#pragma unroll
      for (int c = 0; c < NTS; ++c) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int pc = tau + 256 * h, r = pc >> 3, u = pc & 7;
          *reinterpret_cast<uint4*>(smem + OFF_STG + r * 128 + ((u ^ (r & 7)) << 4)) = pv[c][h];
        }
        named_bar_sync(3, 256);
        uint32_t wv[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = *reinterpret_cast<const uint4*>(smem + OFF_STG + hl * 128 + (((4 * ch + v) ^ (hl & 7)) << 4));
          wv[4 * v + 0] = x.x;
          wv[4 * v + 1] = x.y;
          wv[4 * v + 2] = x.z;
          wv[4 * v + 3] = x.w;
        }
        if (ok) tmem_st16(tQ + 32 * c + 16 * ch, wv);
        named_bar_sync(3, 256);
      }
      if (ok) {
        fence_proxy_async_smem();  // the MMA (async proxy) reads what the threads wrote
        tmem_st_wait();
        tc_fence_before();
        signal_even(q_ready_even);
      }
    };
    // The next segment's Q rows are pulled into L2 a few pages before they
    // are loaded (an earlier prefetch would be evicted by the page stream).
    auto prefetch_q = [&](int rb) {
      if (tid == 128) {
        const int h0 = (int)rank * HEADS, h1 = min(a.n_h, h0 + HEADS);
        if (h1 > h0)
          prefetch_l2(qabs + ((long long)rb * a.qrows + h0) * a.q_row, (uint32_t)((h1 - h0) * a.q_row * 2));
      }
    };

    uint32_t j = 0, part_par = 0;  // bit s: parity of the next tail load in latent slot s
    Seg g_cur = seg_lo < seg_hi ? segs[seg_lo] : Seg{};
    Seg g_nxt = seg_lo + 1 < seg_hi ? segs[seg_lo + 1] : g_cur;
    if (seg_lo < seg_hi) {  // every softmax thread: q_store holds named barriers
      q_issue(g_cur.rb);
      q_store();
    }
    for (int si = seg_lo; si < seg_hi; ++si) {
      const Seg g = g_cur;
      const int n = g.t_hi - g.t_lo;
      float m_used = -INFINITY, lt = 0.f;
      for (int i = 0; i < n; ++i, ++j) {
        const int t = g.t_lo + i;
        const uint32_t b = j & 1;
        const int valid_all = min(KT, g.nkeys - t * KT);  // >= 1: every tile holds a key
        const bool q_next = i + 1 == n && si + 1 < seg_hi;
        if (si + 1 < seg_hi && i == max(0, n - 6)) prefetch_q(g_nxt.rb);
        // S of page j is complete, and with it every earlier MMA: P*V of page
        // j - 2 (issued before S(j)) has released P tile b.
        ok = ok && wait_all(&s_full[b], (j >> 1) & 1);
        float s[16];
        if (ok) {
          tc_fence_after();
          uint32_t v[16];
          tmem_ld16(tS + b * 32 + ch * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 16; ++x) s[x] = __uint_as_float(v[x]);
        } else {
#pragma unroll
          for (int x = 0; x < 16; ++x) s[x] = 0.f;
        }
        const int k0 = kh * 32 + ch * 16;  // this thread's first key of the page
        if (valid_all < KT) {
#pragma unroll
          for (int x = 0; x < 16; ++x)
            if (k0 + x >= valid_all) s[x] = -INFINITY;
        }
        float mt;
        {
          float m8[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) m8[x] = fmaxf(s[x], s[x + 8]);
#pragma unroll
          for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
            for (int x = 0; x < w2; ++x) m8[x] = fmaxf(m8[x], m8[x + w2]);
          mx[(b * HEADS + hl) * 4 + part] = m8[0];
          named_bar_sync(1 + grp, 128);
          const float4 m4 = reinterpret_cast<const float4*>(mx)[b * HEADS + hl];
          mt = fmaxf(fmaxf(m4.x, m4.y), fmaxf(m4.z, m4.w));
        }
        // Running max with lazy rescaling: O and the sums stay relative to
        // m_used until a page's max exceeds it by more than 2^8.  The four
        // threads of a head take the same decision from the same numbers.
        bool resc = false;
        float scale = 1.f;
        if (i == 0) {
          m_used = mt;
          lt = 0.f;
        } else if (mt > m_used + 8.f) {
          scale = fast_exp2(m_used - mt);
          m_used = mt;
          resc = true;
        }
        uint32_t pk[8];
        {
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
          // The row sum adds the fp32 weights (not their bf16 roundings: the
          // difference is random, 2^-9 relative per key).
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float e0 = fast_exp2(s[2 * u] - m_used), e1 = fast_exp2(s[2 * u + 1] - m_used);
            ps[u & 3] += e0 + e1;
            pk[u] = pack_bf16x2(e0, e1);
          }
          lt = lt * scale + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        }
        // O is rescaled only after P*V of page j - 1 has completed.
        if (ok && __any_sync(0xffffffffu, resc)) {
          ok = wait_all(&pv_done[b ^ 1], ((j - 1) >> 1) & 1);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < NPV; ++cc) {
              uint32_t v[32];
              tmem_ld32(tO + ch * (NPV * 32) + cc * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * scale);
              tmem_st32(tO + ch * (NPV * 32) + cc * 32, v);
            }
            tmem_st_wait();
          }
        }
        // P row hl, keys k0 .. k0 + 15: 16-byte pieces k0/8 and k0/8 + 1 of
        // the 128-byte-swizzled K-major tile.
        if (ok) {
          uint8_t* prow = smem + OFF_P + b * P_BYTES + hl * 128;
          const int u0 = k0 >> 3;
          *reinterpret_cast<uint4*>(prow + ((u0 ^ (hl & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(prow + (((u0 + 1) ^ (hl & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        if (ok && (t + 1) * KT > g.nkeys) {
          // The row block's last page: P is 0 past its end, but 0 * NaN would
          // still poison O, so clear those rows of this CTA's latent chunks
          // once they have landed.
          const uint32_t vs = j % VGS;
          ok = wait_all(&vg_part[vs], (part_par >> vs) & 1);
          part_par ^= 1u << vs;
          if (ok) {
            uint8_t* vb = smem + OFF_VG + vs * VG_BYTES;
            const int rows = KT - valid_all, units = rows * 8 * NPV;
            for (int x = tid - 128; x < units; x += 256) {
              const int qq = x / (rows * 8), rem = x - qq * rows * 8;
              *reinterpret_cast<uint4*>(vb + qq * CH_V + (valid_all + rem / 8) * 128 + (rem % 8) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (ok) {
          fence_proxy_async_smem();  // the MMA (async proxy) reads P and the cleared rows
          tc_fence_before();
          signal_even(p_ready_even + 8 * b);
        }
        if (i + 1 < n) continue;

        // ---- end of the segment ----
        // The next segment's Q replaces this one's (its last score MMA is
        // complete); then O of this segment, once its last P*V is done.
        if (q_next) {  // every softmax thread: q_store holds named barriers
          q_issue(g_nxt.rb);
          q_store();
        }
        ok = ok && wait_all(&pv_done[b], (j >> 1) & 1);
        lsum[hl * 4 + part] = lt;
        named_bar_sync(1 + grp, 128);
        if (ok) tc_fence_after();
        const float4 l4 = reinterpret_cast<const float4*>(lsum)[hl];
        const float lrow = (l4.x + l4.y) + (l4.z + l4.w);
        // A whole row block is normalised into obar (bf16); a piece of a
        // split row block is normalised by its own sum into its partial slot
        // and leaves its (m, l) beside it (the same for both column halves).
        // The rows go out through shared memory (the P tiles and the staging
        // tile, free now) so that the global stores are coalesced: in round
        // rho the threads with part == rho write their d_c/4 columns of O,
        // normalised and rounded, into padded rows, then all softmax threads
        // store the 64 rows x d_c/4 columns, eight threads per 128 bytes.
        const bool whole = g.slot < 0;
        const float inv = 1.f / lrow;
        constexpr int PPR = 4 * NPV;          // 16-byte pieces per staged row
        constexpr int SROW = 16 * PPR + 16;   // padded row: consecutive rows start in different banks
        static_assert(64 * SROW <= 2 * P_BYTES + CH_V, "staged output fits the P and staging tiles");
        static_assert((HEADS + 1) * MAX_PIECES * 4 <= 2 * P_BYTES + CH_V, "merge weights fit the P and staging tiles");
        uint8_t* const so = smem + OFF_P;
        __nv_bfloat16* const obase = whole ? static_cast<__nv_bfloat16*>(a.obar) + (long long)g.rb * a.n_h * a.d_c
                                           : static_cast<__nv_bfloat16*>(a.part_o) + (long long)g.slot * a.n_h * a.d_c;
#pragma unroll 1
        for (int rho = 0; rho < 4; ++rho) {
          if (ok && part == rho) {
#pragma unroll
            for (int cc = 0; cc < NPV; ++cc) {
              uint32_t v[32];
              tmem_ld32(tO + ch * (NPV * 32) + cc * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 o;
                o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
                o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
                o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
                o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
                *reinterpret_cast<uint4*>(so + hl * SROW + (4 * cc + q) * 16) = o;
              }
            }
          }
          named_bar_sync(3, 256);
#pragma unroll
          for (int m = 0; m < NPV; ++m) {
            const int pc = (tid - 128) + 256 * m, r = pc / PPR, pp = pc - r * PPR;
            const int hd = (int)rank * HEADS + r;
            if (ok && hd < a.n_h)
              *reinterpret_cast<uint4*>(obase + (long long)hd * a.d_c + rho * (NPV * 32) + 8 * pp) =
                  *reinterpret_cast<const uint4*>(so + r * SROW + 16 * pp);
          }
          named_bar_sync(3, 256);
        }
        if (ok && !whole && part == 0 && live) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float* ml = a.part_ml + ml_index(g.slot, half, a.n_h, head);
            ml[0] = m_used;
            ml[1] = lrow;
          }
        }
        if (a.arrive && !whole) {
          // A piece of a split row block counts in; the last piece of this
          // CTA rank to do so merges all of them, read back from their slots
          // in segment order, so the result does not depend on which piece
          // came last:
          //   w_k = 2^(m_k - max_j m_j) l_k,  obar = sum_k w_k N_k / sum_k w_k
          // (N_k the piece's normalised rows).  One thread publishes the
          // CTA's slot writes (barrier, fence, atomic) and, if last, fences
          // again before the others read the other pieces' slots.
          volatile int* const merge_info = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);  // np or 0, sb
          named_bar_sync(3, 256);
          if (tid == 128) {
            const int sb = a.sched.rb_seg_first[g.rb], se = a.sched.rb_seg_first[g.rb + 1];
            __threadfence();
            const int old = ok ? atomicAdd(a.arrive + 2 * g.rb + (int)rank, 1) : -1;
            const bool last = old == se - sb - 1;
            if (last) __threadfence();
            merge_info[0] = last ? se - sb : 0;
            merge_info[1] = sb;
          }
          named_bar_sync(3, 256);
          const int np = merge_info[0];
          if (np > 0) {
            const int sb = merge_info[1];
            float* const coef = reinterpret_cast<float*>(smem + OFF_P);  // [HEADS][MAX_PIECES] w_k / sum w
            int* const slot_of = reinterpret_cast<int*>(coef + HEADS * MAX_PIECES);
            const int u = tid - 128;
            for (int k = u; k < np; k += 256) slot_of[k] = __ldg(&segs[sb + k].slot);
            if (u < HEADS && (int)rank * HEADS + u < a.n_h) {
              // One pass over the pieces' (m_k, l_k), four in flight:
              // e_k = m_k + log2 l_k (l_k >= 1: a piece holds its own
              // maximum), then w_k = 2^(e_k - m) from shared memory.
              const int hd = (int)rank * HEADS + u;
              float m = -INFINITY;
              for (int k0 = 0; k0 < np; k0 += 4) {
                int sl[4];
                float2 mlk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) sl[i] = k0 + i < np ? __ldg(&segs[sb + k0 + i].slot) : -1;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  mlk[i] = sl[i] >= 0 ? __ldcg(reinterpret_cast<const float2*>(a.part_ml + ml_index(sl[i], 0, a.n_h, hd)))
                                      : make_float2(-INFINITY, 1.f);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  m = fmaxf(m, mlk[i].x);
                  if (k0 + i < np) coef[u * MAX_PIECES + k0 + i] = mlk[i].x + __log2f(mlk[i].y);
                }
              }
              float l = 0.f;
              for (int k = 0; k < np; ++k) l += exp2f(coef[u * MAX_PIECES + k] - m);
              const float il = 1.f / l;
              for (int k = 0; k < np; ++k) coef[u * MAX_PIECES + k] = exp2f(coef[u * MAX_PIECES + k] - m) * il;
            }
            named_bar_sync(3, 256);
            // GM sixteen-byte pieces of output per thread at a time, the GM
            // loads of one partial slot in flight together.
            constexpr int PPR = 16 * NPV;  // 16-byte pieces per row
            constexpr int GM = 4 * NPV % 8 == 0 ? 8 : (4 * NPV < 8 ? 4 * NPV : 2 * NPV);
            static_assert(HEADS * PPR % (256 * GM) == 0, "whole groups of pieces per thread");
            __nv_bfloat16* const orow = static_cast<__nv_bfloat16*>(a.obar) + (long long)g.rb * a.n_h * a.d_c;
            const __nv_bfloat16* const pbase = static_cast<const __nv_bfloat16*>(a.part_o);
            const long long slot_elems = (long long)a.n_h * a.d_c;
#pragma unroll 1
            for (int gi = 0; gi < HEADS * PPR / 256; gi += GM) {
              int off[GM], cr[GM];
              float acc[GM][8];
#pragma unroll
              for (int i = 0; i < GM; ++i) {
                const int x = u + 256 * (gi + i), r = x / PPR, hd = (int)rank * HEADS + r;
                off[i] = hd < a.n_h ? hd * a.d_c + 8 * (x - r * PPR) : -1;
                cr[i] = r * MAX_PIECES;
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;
              }
#pragma unroll 1
              for (int k = 0; k < np; ++k) {
                const __nv_bfloat16* const src = pbase + slot_of[k] * slot_elems;
                uint4 v[GM];
#pragma unroll
                for (int i = 0; i < GM; ++i)
                  v[i] = off[i] >= 0 ? __ldcg(reinterpret_cast<const uint4*>(src + off[i])) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < GM; ++i) {
                  const float c = coef[cr[i] + k];
                  const uint32_t vw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vw[q]));
                    acc[i][2 * q] = __fmaf_rn(c, f.x, acc[i][2 * q]);
                    acc[i][2 * q + 1] = __fmaf_rn(c, f.y, acc[i][2 * q + 1]);
                  }
                }
              }
#pragma unroll
              for (int i = 0; i < GM; ++i)
                if (ok && off[i] >= 0)
                  *reinterpret_cast<uint4*>(orow + off[i]) =
                      make_uint4(pack_bf16x2(acc[i][0], acc[i][1]), pack_bf16x2(acc[i][2], acc[i][3]),
                                 pack_bf16x2(acc[i][4], acc[i][5]), pack_bf16x2(acc[i][6], acc[i][7]));
            }
            named_bar_sync(3, 256);  // shared memory is the next segment's again
          }
        }
        if (ok) {
          tc_fence_before();
          signal_even(o_free_even);
        }
      }
      g_cur = g_nxt;
      if (si + 2 < seg_hi) g_nxt = segs[si + 2];
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still use its shared memory or TMEM
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, TM_COLS);
  }
}

}  // namespace attn_tc
}  // namespace mla
