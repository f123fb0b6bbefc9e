// Absorbed latent attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes is the same as attn_simt.cuh ("ai-decoupled-rope-mla",
// absorbed score and output equations): for one query token, all of its heads
// form the M = 128 rows (heads beyond n_h are zero rows), and for each 64-key
// cache page
//   S  = Q_abs [128 x d_cr] * page^T [d_cr x 64]      (content + position
//        score in one contraction, because the cache row is [c | k_R] and the
//        query row is [q~ | q_R], both pre-scaled by s*log2(e))
//   P  = exp2(S - m)  (online softmax, running max m, running sum l)
//   O += P [128 x 64] * page[:, latent half] [64 x d_c/2]
// Only the cache tile is streamed; both products are dense because every
// head shares the cache ("Latent Attention Meets RoPE": one shared position
// key; the latent is shared by construction).
//
// Layout decisions (B200): TMEM holds 512 columns x 128 lanes of fp32.  The
// full latent accumulator of 128 heads x 512 would fill it, so each CTA of a
// pair owns half of the latent output columns (blockIdx.y) and computes the
// full score tile itself.  TMEM columns: O half [0, d_c/2), S [256, 320),
// the first six 64-column chunks of Q [320, 512) (bf16 pairs packed in 32-bit
// columns, the A operand of the score MMA); the remaining Q chunks are in
// shared memory.  The cache is streamed by TMA in 64-key x 64-column chunks
// (8 KB, 128-byte swizzle) through two rings: chunks only the score needs
// (the other half of the latent and the RoPE key) are released as soon as
// the score MMA has read them; the chunks of this CTA's own half stay until
// the P*V MMA is done.  The two CTAs of a pair read the same pages at about
// the same time, so the second read is served by L2.
//
// Warp roles (256 threads): warps 0 and 3 = TMA producers (one per ring),
// warp 1 = MMA issuer (each runs warp-uniformly; one elected lane issues),
// warp 2 = TMEM allocator,
// warps 4-7 = softmax / epilogue (thread r owns row r = TMEM lane r).  Every
// wait is bounded (sm100::mbar_wait).
#pragma once
#include "attn_simt.cuh"
#include "sm100.cuh"

namespace mla {
namespace attn_tc {
using namespace sm100;

constexpr int THREADS = 256;
constexpr int KT = 64;                       // keys per tile (one page)
constexpr int CHUNK_BYTES = 64 * 64 * 2;     // 64 keys x 64 bf16 columns
constexpr int A_SLOTS = 8;
constexpr int B_GROUPS = 3;
constexpr int B_GROUP_BYTES = 4 * CHUNK_BYTES;
constexpr int Q_TMEM_CHUNKS = 6;
constexpr int Q_SMEM_CHUNKS = 3;
constexpr int Q_CHUNK_BYTES = 128 * 128;
constexpr int P_BYTES = 128 * 128;
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 320, TM_COLS = 512;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + A_SLOTS * CHUNK_BYTES;
constexpr int OFF_Q = OFF_B + B_GROUPS * B_GROUP_BYTES;
constexpr int OFF_P = OFF_Q + Q_SMEM_CHUNKS * Q_CHUNK_BYTES;
constexpr int OFF_BAR = OFF_P + P_BYTES;
constexpr int NUM_BARS = 2 * A_SLOTS + 2 * B_GROUPS + 7;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // + slack to align the base to 1024

struct Params {
  AttnArgs a;
  int nkc;  // 64-column chunks per cache row (ceil(d_cr / 64))
  int dh;   // latent columns per CTA (d_c / 2)
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b, float& sum) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  sum += __low2float(v) + __high2float(v);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(THREADS, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + A_SLOTS;
  uint64_t* b_full = bars + 2 * A_SLOTS;
  uint64_t* b_empty = b_full + B_GROUPS;
  uint64_t* s_full = b_empty + B_GROUPS;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_ready = s_full + 2;
  uint64_t* pv_done = s_full + 3;
  uint64_t* q_ready = s_full + 4;
  uint64_t* o_free = s_full + 5;
  uint64_t* final_bar = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int w = blockIdx.x, half = blockIdx.y;
  const AttnArgs& a = p.a;
  const int nkc = p.nkc, dh = p.dh, npv = dh / 64;
  const int own0 = half * npv;  // first chunk of this CTA's latent half
  const Seg* segs = a.sched.segs;
  const int seg_lo = a.sched.worker_seg[w], seg_hi = a.sched.worker_seg[w + 1];

  if (tid == 32) {
    for (int i = 0; i < A_SLOTS; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < B_GROUPS; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_ready, 128);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 128);
    mbar_init(o_free, 128);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) tma_prefetch_desc(&tmap);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0 || warp == 3) {
    // ----------------------------------------------------- TMA producers
    // Warp 0 feeds the score-only ring, warp 3 the own-half ring; each walks
    // every tile of the worker on its own, so neither ring waits for the
    // other's slots.  The warp runs uniformly; one elected lane issues.
    const bool ring_b = (warp == 3);
    uint32_t cnt = 0;  // chunks (score-only ring) or tile groups (own-half ring) issued
    bool ok = true;
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = segs[si];
      const int seq = g.rb / a.n_q;
      for (int t = g.t_lo; t < g.t_hi && ok; ++t) {
        int page = a.page_table[(long long)seq * a.max_pages + t];
        if (page < 0 || page >= a.num_pages) {
          if (!ring_b && elect_one()) flag_error(a.err, kErrBounds);
          page = 0;  // keep the pipeline's byte counts; outputs are flagged invalid
        }
        const int y = page * KT;
        if (ring_b) {
          const uint32_t gs = cnt % B_GROUPS;
          if (!(ok = mbar_wait_warp(&b_empty[gs], ((cnt / B_GROUPS) & 1) ^ 1, abort_flag, a.err))) break;
          if (elect_one()) {
            mbar_arrive_expect_tx(&b_full[gs], npv * CHUNK_BYTES);
            for (int q = 0; q < npv; ++q)
              tma_load_2d(smem + OFF_B + gs * B_GROUP_BYTES + q * CHUNK_BYTES, &tmap, (own0 + q) * 64, y,
                          &b_full[gs]);
          }
          __syncwarp();
          ++cnt;
        } else {
          for (int c = 0; c < nkc; ++c) {
            if (c >= own0 && c < own0 + npv) continue;
            const uint32_t slot = cnt % A_SLOTS;
            if (!(ok = mbar_wait_warp(&a_empty[slot], ((cnt / A_SLOTS) & 1) ^ 1, abort_flag, a.err))) break;
            if (elect_one()) {
              mbar_arrive_expect_tx(&a_full[slot], CHUNK_BYTES);
              tma_load_2d(smem + OFF_A + slot * CHUNK_BYTES, &tmap, c * 64, y, &a_full[slot]);
            }
            __syncwarp();
            ++cnt;
          }
        }
      }
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit.
      const uint32_t n = ring_b ? B_GROUPS : A_SLOTS;
      uint64_t* full = ring_b ? b_full : a_full;
      for (uint32_t q = 0; q < n && q < cnt; ++q) {
        const uint32_t last = q + n * ((cnt - 1 - q) / n);
        mbar_wait_warp(&full[q], (last / n) & 1, abort_flag, nullptr, 50000000ull, false);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // Issue order per tile: the score MMA of tile t (own-half chunks first,
    // they were prefetched furthest ahead), and the P*V MMA of tile t-1 as
    // soon as its P is ready -- polled while waiting for score data, so a
    // late chunk never holds back the release of the own-half ring.  The
    // whole warp runs this loop with uniform values; one elected lane issues
    // each tcgen05 instruction.
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);
    const uint32_t idPV = idesc_bf16(128, dh, 0, 1);
    const uint32_t tS = tbase + TM_S, tO = tbase + TM_O, tQ = tbase + TM_Q;
    const uint32_t sA = smem_u32(smem + OFF_A), sB = smem_u32(smem + OFF_B);
    const uint32_t sQ = smem_u32(smem + OFF_Q), sP = smem_u32(smem + OFF_P);
    uint32_t a_cnt = 0, b_cnt = 0, tg = 0, seg_k = 0;
    bool ok = true;
    bool pv_pending = false, pv_first = false;
    uint32_t pv_gs = 0, pv_tg = 0, pv_seg = 0;
    // Issues the pending P*V MMA if its inputs are ready; never blocks.
    auto try_pv = [&]() {
      if (!pv_pending || !mbar_try_wait_warp(p_ready, pv_tg & 1)) return;
      if (pv_first && pv_seg > 0 && !mbar_try_wait_warp(o_free, (pv_seg - 1) & 1)) return;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sP + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sB + pv_gs * B_GROUP_BYTES + kk * 2048, CHUNK_BYTES, 1024);
          mma_ss(tO, ad, bd, idPV, (pv_first && kk == 0) ? 0u : 1u);
        }
        tc_commit(pv_done);
        tc_commit(&b_empty[pv_gs]);
      }
      __syncwarp();
      pv_pending = false;
    };
    // Bounded wait on `bar` that keeps issuing the pending P*V meanwhile.
    auto wait_polling = [&](uint64_t* bar, uint32_t parity) -> bool {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_warp(bar, parity)) {
        try_pv();
        int stop = 0;
        if (*abort_flag) stop = 1;
        else if (globaltimer_ns() - t0 > 2000000000ull) stop = 2;
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (stop) {
          if (stop == 2 && elect_one()) {
            *abort_flag = 1;
            flag_error(a.err, kErrTimeout);
          }
          __syncwarp();
          return false;
        }
      }
      return true;
    };
    auto flush_pv = [&]() -> bool {
      const uint64_t t0 = globaltimer_ns();
      while (pv_pending) {
        try_pv();
        if (!pv_pending) break;
        int stop = 0;
        if (*abort_flag) stop = 1;
        else if (globaltimer_ns() - t0 > 2000000000ull) stop = 2;
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (stop) {
          if (stop == 2 && elect_one()) {
            *abort_flag = 1;
            flag_error(a.err, kErrTimeout);
          }
          __syncwarp();
          return false;
        }
      }
      return true;
    };
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = segs[si];
      const int n = g.t_hi - g.t_lo;
      if (!(ok = wait_polling(q_ready, seg_k & 1))) break;
      tc_fence_after();
      for (int i = 0; i < n && ok; ++i) {
        if (tg > 0 && !(ok = wait_polling(s_free, (tg - 1) & 1))) break;
        tc_fence_after();
        const uint32_t gs = b_cnt % B_GROUPS;
        uint32_t acc = 0;
        for (int k2 = 0; k2 < nkc; ++k2) {
          // own-half chunks first, then the rest in column order
          int c;
          if (k2 < npv) c = own0 + k2;
          else {
            const int j = k2 - npv;
            c = (j < own0) ? j : j + npv;
          }
          const bool own = k2 < npv;
          uint32_t bsrc, slot = 0;
          if (own) {
            if (k2 == 0 && !(ok = wait_polling(&b_full[gs], (b_cnt / B_GROUPS) & 1))) break;
            bsrc = sB + gs * B_GROUP_BYTES + k2 * CHUNK_BYTES;
          } else {
            slot = a_cnt % A_SLOTS;
            if (!(ok = wait_polling(&a_full[slot], (a_cnt / A_SLOTS) & 1))) break;
            bsrc = sA + slot * CHUNK_BYTES;
          }
          tc_fence_after();
          if (elect_one()) {
            if (c < Q_TMEM_CHUNKS) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_ts(tS, tQ + c * 32 + k * 8, sdesc_sw128(bsrc + k * 32, 16, 1024), idS, (acc | k) ? 1u : 0u);
            } else {
              const uint32_t qa = sQ + (c - Q_TMEM_CHUNKS) * Q_CHUNK_BYTES;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_ss(tS, sdesc_sw128(qa + k * 32, 16, 1024), sdesc_sw128(bsrc + k * 32, 16, 1024), idS,
                       (acc | k) ? 1u : 0u);
            }
            if (!own) tc_commit(&a_empty[slot]);
          }
          __syncwarp();
          acc = 1;
          if (!own) ++a_cnt;
        }
        if (!ok) break;
        if (elect_one()) tc_commit(s_full);
        __syncwarp();
        ++b_cnt;
        // The previous tile's P*V must be out before this tile's is queued.
        if (!(ok = flush_pv())) break;
        pv_pending = true;
        pv_first = (i == 0);
        pv_gs = gs;
        pv_tg = tg;
        pv_seg = seg_k;
        ++tg;
      }
      ++seg_k;
    }
    if (ok) flush_pv();
    if (elect_one()) tc_commit(final_bar);
    __syncwarp();
    mbar_wait_warp(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
  } else if (warp >= 4) {
    // ------------------------------------------- softmax and epilogue (WG 1)
    const int r = tid - 128;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + TM_S, tO = tbase + lane_off + TM_O, tQ = tbase + lane_off + TM_Q;
    uint8_t* sP = smem + OFF_P;
    uint8_t* sQ = smem + OFF_Q;
    uint8_t* sB = smem + OFF_B;
    const __nv_bfloat16* qabs = static_cast<const __nv_bfloat16*>(a.qabs);
    const int nq_tmem = min(nkc, Q_TMEM_CHUNKS);
    uint32_t tg = 0, b_cnt = 0;
    bool ok = true;

    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool r_ok = mbar_wait(bar, parity, abort_flag, a.err);
      return __all_sync(0xffffffffu, r_ok);
    };
    // Q row r of token rb into TMEM (chunks < 6) and swizzled smem (the rest).
    auto load_q = [&](int rb) {
      const uint4* src =
          (r < a.n_h) ? reinterpret_cast<const uint4*>(qabs + ((long long)rb * a.qrows + r) * a.d_cr) : nullptr;
      for (int c = 0; c < nq_tmem; ++c) {
        uint32_t wv[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int col = c * 64 + u * 8;
          uint4 v = (src && col < a.d_cr) ? __ldg(src + col / 8) : make_uint4(0, 0, 0, 0);
          wv[4 * u + 0] = v.x;
          wv[4 * u + 1] = v.y;
          wv[4 * u + 2] = v.z;
          wv[4 * u + 3] = v.w;
        }
        tmem_st32(tQ + c * 32, wv);
      }
      tmem_st_wait();
      for (int c = nq_tmem; c < nkc; ++c) {
        uint8_t* chunk = sQ + (c - Q_TMEM_CHUNKS) * Q_CHUNK_BYTES + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int col = c * 64 + u * 8;
          uint4 v = (src && col < a.d_cr) ? __ldg(src + col / 8) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(chunk + ((u ^ (r & 7)) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(q_ready);
    };

    if (seg_lo < seg_hi) load_q(segs[seg_lo].rb);
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = segs[si];
      const int rb = g.rb;
      const int nkeys = rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, nullptr);
      const int n = g.t_hi - g.t_lo;
      float m_used = -INFINITY, l = 0.f;
      for (int i = 0; i < n; ++i) {
        const int t = g.t_lo + i;
        if (!(ok = wait_all(s_full, tg & 1))) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(tS, v0);
          tmem_ld32(tS + 32, v1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            s[j] = __uint_as_float(v0[j]);
            s[32 + j] = __uint_as_float(v1[j]);
          }
        }
        tc_fence_before();
        mbar_arrive(s_free);
        const int valid = min(KT, nkeys - t * KT);
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j >= valid) s[j] = -INFINITY;
          mt = fmaxf(mt, s[j]);
        }
        // Running max with lazy rescaling: O and l stay relative to m_used
        // until a tile's max exceeds it by more than 2^8.
        bool resc = false;
        float scale = 1.f;
        if (i == 0) {
          m_used = mt;
          l = 0.f;
        } else if (mt > m_used + 8.f) {
          scale = exp2f(m_used - mt);
          m_used = mt;
          resc = true;
        }
        float psum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) pk[u] = pack_bf16(exp2f(s[2 * u] - m_used), exp2f(s[2 * u + 1] - m_used), psum);
        if (i > 0) {
          if (!(ok = wait_all(pv_done, (tg - 1) & 1))) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, resc)) {
          for (int cc = 0; cc < dh / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tO + cc * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * scale);
            tmem_st32(tO + cc * 32, v);
          }
          tmem_st_wait();
          l *= scale;
        }
        uint8_t* prow = sP + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(prow + ((u ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        l += psum;
        if (valid < KT) {
          // Keys past the end: P is 0 there, but 0 * NaN would still poison O,
          // so clear those rows of this tile's own-half chunks.
          uint8_t* gb = sB + (b_cnt % B_GROUPS) * B_GROUP_BYTES;
          const int rows = KT - valid, units = rows * 8 * npv;
          for (int x = r; x < units; x += 128) {
            const int q = x / (rows * 8), rem = x - q * rows * 8;
            *reinterpret_cast<uint4*>(gb + q * CHUNK_BYTES + (valid + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
        ++tg;
        ++b_cnt;
      }
      if (!ok) break;
      if (si + 1 < seg_hi) load_q(segs[si + 1].rb);
      if (!(ok = wait_all(pv_done, (tg - 1) & 1))) break;
      tc_fence_after();
      // Epilogue: a whole row block is normalised into obar (bf16); a piece of
      // a split row block leaves its unnormalised sum and (m, l) in its slot.
      const bool whole = g.slot < 0;
      const float inv = 1.f / l;
      for (int cc = 0; cc < dh / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tO + cc * 32, v);
        tmem_ld_wait();
        if (r < a.n_h) {
          const int col = half * dh + cc * 32;
          if (whole) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.obar) +
                                                  ((long long)rb * a.n_h + r) * a.d_c + col);
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
          } else {
            uint4* dst = reinterpret_cast<uint4*>(a.part_o + ((long long)g.slot * a.n_h + r) * a.d_c + col);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
      if (!whole && half == 0 && r < a.n_h) {
        a.part_ml[((long long)g.slot * a.n_h + r) * 2 + 0] = m_used;
        a.part_ml[((long long)g.slot * a.n_h + r) * 2 + 1] = l;
      }
      tc_fence_before();
      mbar_arrive(o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
}

}  // namespace attn_tc
}  // namespace mla
