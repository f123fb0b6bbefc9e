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
// Warp roles (256 threads): warp 0 lane 0 = TMA producer, warp 1 lane 0 =
// MMA issuer, warp 2 = TMEM allocator, warps 4-7 = softmax / epilogue (thread
// r owns row r = TMEM lane r).  Every wait is bounded (sm100::mbar_wait).
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

__global__ void __launch_bounds__(THREADS, 1) kernel(const __grid_constant__ CUtensorMap tmap, const Params p) {
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

  if (tid == 0) {
    // ------------------------------------------------------ TMA producer
    uint32_t a_cnt = 0, b_cnt = 0;
    bool ok = true;
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = segs[si];
      const int seq = g.rb / a.n_q;
      for (int t = g.t_lo; t < g.t_hi && ok; ++t) {
        int page = a.page_table[(long long)seq * a.max_pages + t];
        if (page < 0 || page >= a.num_pages) {
          flag_error(a.err, kErrBounds);
          page = 0;  // keep the pipeline's byte counts; outputs are flagged invalid
        }
        const int y = page * KT;
        const uint32_t gs = b_cnt % B_GROUPS;
        for (int c = 0; c < nkc; ++c) {
          if (c >= own0 && c < own0 + npv) {
            if (c == own0) {
              if (!(ok = mbar_wait(&b_empty[gs], ((b_cnt / B_GROUPS) & 1) ^ 1, abort_flag, a.err))) break;
              mbar_arrive_expect_tx(&b_full[gs], npv * CHUNK_BYTES);
            }
            tma_load_2d(smem + OFF_B + gs * B_GROUP_BYTES + (c - own0) * CHUNK_BYTES, &tmap, c * 64, y,
                        &b_full[gs]);
          } else {
            const uint32_t slot = a_cnt % A_SLOTS;
            if (!(ok = mbar_wait(&a_empty[slot], ((a_cnt / A_SLOTS) & 1) ^ 1, abort_flag, a.err))) break;
            mbar_arrive_expect_tx(&a_full[slot], CHUNK_BYTES);
            tma_load_2d(smem + OFF_A + slot * CHUNK_BYTES, &tmap, c * 64, y, &a_full[slot]);
            ++a_cnt;
          }
        }
        ++b_cnt;
      }
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit.
      for (uint32_t s = 0; s < A_SLOTS && s < a_cnt; ++s) {
        uint32_t last = ((a_cnt - 1 - s) / A_SLOTS) * A_SLOTS + s;
        mbar_wait(&a_full[s], (last / A_SLOTS) & 1, abort_flag, nullptr, 50000000ull, false);
      }
      for (uint32_t s = 0; s < B_GROUPS && s < b_cnt; ++s) {
        uint32_t last = ((b_cnt - 1 - s) / B_GROUPS) * B_GROUPS + s;
        mbar_wait(&b_full[s], (last / B_GROUPS) & 1, abort_flag, nullptr, 50000000ull, false);
      }
    }
  } else if (tid == 32) {
    // --------------------------------------------------------- MMA issuer
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);
    const uint32_t idPV = idesc_bf16(128, dh, 0, 1);
    const uint32_t tS = tbase + TM_S, tO = tbase + TM_O, tQ = tbase + TM_Q;
    const uint32_t sA = smem_u32(smem + OFF_A), sB = smem_u32(smem + OFF_B);
    const uint32_t sQ = smem_u32(smem + OFF_Q), sP = smem_u32(smem + OFF_P);
    uint32_t a_cnt = 0, b_cnt = 0, tg = 0, seg_k = 0;
    bool ok = true;
    auto issue_pv = [&](uint32_t gs, uint32_t tile_tg, bool first) -> bool {
      if (!mbar_wait(p_ready, tile_tg & 1, abort_flag, a.err)) return false;
      if (first && seg_k > 0 && !mbar_wait(o_free, (seg_k - 1) & 1, abort_flag, a.err)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(sP + kk * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sB + gs * B_GROUP_BYTES + kk * 2048, CHUNK_BYTES, 1024);
        mma_ss(tO, ad, bd, idPV, (first && kk == 0) ? 0u : 1u);
      }
      tc_commit(pv_done);
      tc_commit(&b_empty[gs]);
      return true;
    };
    for (int si = seg_lo; si < seg_hi && ok; ++si) {
      const Seg g = segs[si];
      const int n = g.t_hi - g.t_lo;
      if (!(ok = mbar_wait(q_ready, seg_k & 1, abort_flag, a.err))) break;
      tc_fence_after();
      uint32_t prev_gs = 0, prev_tg = 0;
      for (int i = 0; i < n && ok; ++i) {
        if (tg > 0 && !(ok = mbar_wait(s_free, (tg - 1) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t gs = b_cnt % B_GROUPS;
        uint32_t acc = 0;
        for (int c = 0; c < nkc; ++c) {
          const bool own = (c >= own0 && c < own0 + npv);
          uint32_t bsrc, slot = 0;
          if (own) {
            if (c == own0 && !(ok = mbar_wait(&b_full[gs], (b_cnt / B_GROUPS) & 1, abort_flag, a.err))) break;
            bsrc = sB + gs * B_GROUP_BYTES + (c - own0) * CHUNK_BYTES;
          } else {
            slot = a_cnt % A_SLOTS;
            if (!(ok = mbar_wait(&a_full[slot], (a_cnt / A_SLOTS) & 1, abort_flag, a.err))) break;
            bsrc = sA + slot * CHUNK_BYTES;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bd = sdesc_sw128(bsrc + k * 32, 16, 1024);
            if (c < Q_TMEM_CHUNKS) {
              mma_ts(tS, tQ + c * 32 + k * 8, bd, idS, acc);
            } else {
              const uint64_t ad = sdesc_sw128(sQ + (c - Q_TMEM_CHUNKS) * Q_CHUNK_BYTES + k * 32, 16, 1024);
              mma_ss(tS, ad, bd, idS, acc);
            }
            acc = 1;
          }
          if (!own) {
            tc_commit(&a_empty[slot]);
            ++a_cnt;
          }
        }
        if (!ok) break;
        tc_commit(s_full);
        ++b_cnt;
        if (i > 0 && !(ok = issue_pv(prev_gs, prev_tg, i == 1))) break;
        prev_gs = gs;
        prev_tg = tg;
        ++tg;
      }
      if (ok && n > 0) ok = issue_pv(prev_gs, prev_tg, n == 1);
      ++seg_k;
    }
    tc_commit(final_bar);
    mbar_wait(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
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
        float psum = 0.f;
        uint8_t* prow = sP + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 pk;
          pk.x = pack_bf16(exp2f(s[8 * u + 0] - m_used), exp2f(s[8 * u + 1] - m_used), psum);
          pk.y = pack_bf16(exp2f(s[8 * u + 2] - m_used), exp2f(s[8 * u + 3] - m_used), psum);
          pk.z = pack_bf16(exp2f(s[8 * u + 4] - m_used), exp2f(s[8 * u + 5] - m_used), psum);
          pk.w = pack_bf16(exp2f(s[8 * u + 6] - m_used), exp2f(s[8 * u + 7] - m_used), psum);
          *reinterpret_cast<uint4*>(prow + ((u ^ (r & 7)) << 4)) = pk;
        }
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
