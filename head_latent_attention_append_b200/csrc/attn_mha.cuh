// Causal prefill in the materialised form, on the sm_100a tensor cores.
//
// "Multi-Head Latent Attention" (talalahmed), "Compress first, expand later"
// and its closing flow diagram: the per-head keys and values are expanded
// from the latent, K_C = W_UK,h c_t and V = W_UV,h c_t, and ordinary
// multi-head attention runs on them.  With the decoupled RoPE key of
// "ai-decoupled-rope-mla" (one k_R,t shared by every head), head h's key row
// is [K_C,h,t | k_R,t] and its query row [q_C,h | RoPE_m(q_R,h)], so the score
// is the same content + position sum as the absorbed path, over
// d_qk = d_h + d_r columns instead of d_c + d_r; the output is sum_t alpha_t
// V_h,t directly (no W_UV after the sum).  Per causal (query, key) pair and
// head that is 2 (d_h + d_r) + 2 d_v flops against 2 (d_c + d_r) + 2 d_c on
// the absorbed path (640 vs 2176 at d_h = d_v = 128, d_c = 512, d_r = 64).
//
// One CTA per (128-query tile, head, sequence), heaviest query tiles first.
// For each 128-key tile j <= i of the causal prefix:
//   S_j  = Q [128 x d_qk] * K_j^T [d_qk x 128]   (SS tcgen05.mma, fp32 in TMEM)
//   P_j  = exp2(S_j - m)   (online softmax, running max m with lazy rescale)
//   O   += P_j [128 x 128] * V_j [128 x d_v]      (TS tcgen05.mma, P in TMEM)
// The queries arrive pre-scaled by s * log2(e), so S is in log2 units.
// Operands: Q and K tiles are K-major 64-column chunks with 128-byte swizzle
// (the last chunk of a key tile is the RoPE key, two 64-row boxes from two
// cache pages); V chunks are MN-major for the P*V product.  TMEM columns:
// S double-buffered [0, 256), O [256, 256 + d_v), P [384, 448).
//
// Warp roles (256 threads): warp 0 = TMA producer, warp 1 = MMA issuer
// (S_{j+1} is issued before P_j*V_j so the next score overlaps this softmax),
// warp 2 = TMEM allocator, warp 3 idle, warps 4-7 = softmax: thread r owns
// query row r (TMEM lane r), keeps its running max and sum, rescales its O
// row when the max grows by more than 2^8, and writes its normalised output
// row at the end.  Every wait is bounded (sm100::mbar_wait).
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace attn_mha {
using namespace sm100;

constexpr int THREADS = 256;
constexpr int BQ = 128, BKV = 128;         // query rows and keys per tile
constexpr int DR = 64;                     // RoPE-key width this kernel takes
constexpr int CH = 128 * 64 * 2;           // one 128-row x 64-column bf16 chunk (16 KB)
constexpr int MAX_QK = 3;                  // chunks of d_h + d_r (d_h <= 128)
constexpr int MAX_V = 2;                   // chunks of d_v (d_v <= 128)
constexpr int STAGES = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + MAX_QK * CH;
constexpr int OFF_V = OFF_K + STAGES * MAX_QK * CH;
constexpr int OFF_BAR = OFF_V + STAGES * MAX_V * CH;
constexpr int NUM_BARS = 1 + 4 * STAGES + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // slack to align the block to 1024 bytes
static_assert(SMEM_BYTES <= 232448, "over the 227 KB of shared memory a CTA can have");
constexpr uint32_t TM_S = 0, TM_O = 256, TM_P = 384, TM_COLS = 512;

struct Params {
  int B, S, n_h, d_h, d_v, d_c;  // the RoPE key is DR wide
  int nqk, nv;                   // chunks: (d_h + DR) / 64 and d_v / 64
  const int32_t* page_table;     // [B][max_pages]
  int max_pages, num_pages;
  float* out;                    // [B*S][n_h][d_v]
  int* err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// mapQ: [T][n_h][d_h + DR] bf16; mapK: [T][n_h][d_h]; mapV: [T][n_h][d_v]
// (boxes of 64 columns x 1 head x 128 tokens); mapR: the cache as
// [num_pages * 64][d_c + DR] (boxes of 64 columns x 64 rows).
__global__ void __launch_bounds__(THREADS, 1)
    attn_mha_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapR,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                // [STAGES]
  uint64_t* k_empty = k_full + STAGES;
  uint64_t* v_full = k_empty + STAGES;
  uint64_t* v_empty = v_full + STAGES;
  uint64_t* s_full = v_empty + STAGES;        // [2]
  uint64_t* p_ready = s_full + 2;
  uint64_t* pv_done = p_ready + 1;
  uint64_t* final_bar = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int nqt = (p.S + BQ - 1) / BQ;
  const int i = nqt - 1 - (int)blockIdx.x;     // query tile: the longest causal prefixes first
  const int h = blockIdx.y, b = blockIdx.z;
  const int tok0 = b * p.S;                    // first token of the sequence
  const int n = i + 1;                         // key tiles 0 .. i

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_ready, 128);
    mbar_init(pv_done, 1);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  if (tid == 32) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    tma_prefetch_desc(&mapR);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    uint32_t kc = 0, vc = 0;  // loads issued (for the drain on abort)
    if (elect_one()) {
      mbar_arrive_expect_tx(q_full, p.nqk * CH);
      for (int c = 0; c < p.nqk; ++c) tma_load_3d(smem + OFF_Q + c * CH, &mapQ, c * 64, h, tok0 + BQ * i, q_full);
    }
    __syncwarp();
    for (int j = 0; j < n; ++j) {
      const int st = j % STAGES;
      const uint32_t ph = ((j / STAGES) & 1) ^ 1;
      if (!mbar_wait_warp(&k_empty[st], ph, abort_flag, p.err)) break;
      // The two cache pages that hold this key tile's RoPE keys.  Pages past
      // the sequence's end only feed keys the causal mask removes.
      int pg[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pi = 2 * j + u;
        int g = 0;
        if (pi * 64 < p.S && pi < p.max_pages) {
          g = p.page_table[(long long)b * p.max_pages + pi];
          if (g < 0 || g >= p.num_pages) {
            if (h == 0 && elect_one()) flag_error(p.err, kErrBounds);
            g = 0;
          }
        }
        pg[u] = g;
      }
      if (elect_one()) {
        uint8_t* kb = smem + OFF_K + st * (MAX_QK * CH);
        mbar_arrive_expect_tx(&k_full[st], p.nqk * CH);
        for (int c = 0; c + 1 < p.nqk; ++c) tma_load_3d(kb + c * CH, &mapK, c * 64, h, tok0 + BKV * j, &k_full[st]);
        tma_load_2d(kb + (p.nqk - 1) * CH, &mapR, p.d_c, pg[0] * 64, &k_full[st]);
        tma_load_2d(kb + (p.nqk - 1) * CH + CH / 2, &mapR, p.d_c, pg[1] * 64, &k_full[st]);
      }
      __syncwarp();
      ++kc;
      if (!mbar_wait_warp(&v_empty[st], ph, abort_flag, p.err)) break;
      if (elect_one()) {
        uint8_t* vb = smem + OFF_V + st * (MAX_V * CH);
        mbar_arrive_expect_tx(&v_full[st], p.nv * CH);
        for (int c = 0; c < p.nv; ++c) tma_load_3d(vb + c * CH, &mapV, c * 64, h, tok0 + BKV * j, &v_full[st]);
      }
      __syncwarp();
      ++vc;
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit.
      mbar_wait_warp(q_full, 0, abort_flag, nullptr, 50000000ull, false);
      for (uint32_t q = 0; q < (uint32_t)STAGES; ++q) {
        if (q < kc) mbar_wait_warp(&k_full[q], ((q + STAGES * ((kc - 1 - q) / STAGES)) / STAGES) & 1, abort_flag,
                                   nullptr, 50000000ull, false);
        if (q < vc) mbar_wait_warp(&v_full[q], ((q + STAGES * ((vc - 1 - q) / STAGES)) / STAGES) & 1, abort_flag,
                                   nullptr, 50000000ull, false);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    const uint32_t idS = idesc_bf16(128, BKV, 0, 0);
    const uint32_t idPV = idesc_bf16(128, p.d_v, 0, 1);
    const uint32_t sQ = smem_u32(smem + OFF_Q), sK = smem_u32(smem + OFF_K), sV = smem_u32(smem + OFF_V);
    const uint32_t tS = tbase + TM_S, tO = tbase + TM_O, tP = tbase + TM_P;
    bool ok = mbar_wait_warp(q_full, 0, abort_flag, p.err);
    tc_fence_after();
    for (int j = 0; j <= n && ok; ++j) {
      if (j < n) {
        // S_j into buffer j & 1: free, since the softmax read S_{j-2} before
        // it signalled P_{j-2}, which this warp waited for one step ago.
        const int st = j % STAGES;
        if (!(ok = mbar_wait_warp(&k_full[st], (j / STAGES) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t kb = sK + st * (MAX_QK * CH);
          for (int c = 0; c < p.nqk; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_ss(tS + (j & 1) * BKV, sdesc_sw128(sQ + c * CH + k * 32, 16, 1024),
                     sdesc_sw128(kb + c * CH + k * 32, 16, 1024), idS, (c | k) ? 1u : 0u);
          tc_commit(&s_full[j & 1]);
          tc_commit(&k_empty[st]);
        }
        __syncwarp();
      }
      if (j >= 1) {
        const int jj = j - 1, st = jj % STAGES;
        if (!(ok = mbar_wait_warp(p_ready, jj & 1, abort_flag, p.err))) break;
        if (!(ok = mbar_wait_warp(&v_full[st], (jj / STAGES) & 1, abort_flag, p.err))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t vb = sV + st * (MAX_V * CH);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            mma_ts(tO, tP + kk * 8, sdesc_sw128(vb + kk * 2048, CH, 1024), idPV, (jj | kk) ? 1u : 0u);
          tc_commit(pv_done);
          tc_commit(&v_empty[st]);
        }
        __syncwarp();
      }
    }
    // TMEM is freed only after the last MMA, even on an abandoned run.
    if (elect_one()) tc_commit(final_bar);
    __syncwarp();
    mbar_wait_warp(final_bar, 0, abort_flag, nullptr, 50000000ull, false);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int r = tid - 128;                          // query row = TMEM lane
    const int qpos = BQ * i + r;                      // its position in the sequence
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + TM_S, tO = tbase + lane_off + TM_O, tP = tbase + lane_off + TM_P;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool r_ok = mbar_wait(bar, parity, abort_flag, p.err);
      return __all_sync(0xffffffffu, r_ok);
    };
    for (int j = 0; j < n; ++j) {
      if (!(ok = wait_all(&s_full[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      float s[BKV];
      {
        uint32_t u[BKV];
#pragma unroll
        for (int q = 0; q < BKV / 32; ++q)
          tmem_ld32(tS + (j & 1) * BKV + q * 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * q));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < BKV; ++c) s[c] = __uint_as_float(u[c]);
      }
      if (j == i) {
        // The diagonal tile: key BKV*j + c is visible to query BQ*i + r iff c <= r.
#pragma unroll
        for (int c = 0; c < BKV; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      float mt;
      {
        float mx[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) mx[c] = fmaxf(fmaxf(s[c], s[c + 32]), fmaxf(s[c + 64], s[c + 96]));
#pragma unroll
        for (int w2 = 16; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int c = 0; c < w2; ++c) mx[c] = fmaxf(mx[c], mx[c + w2]);
        mt = mx[0];
      }
      bool resc = false;
      float scale = 1.f;
      if (j == 0) {
        m_used = mt;   // key 0 is visible to every query: finite
      } else if (mt > m_used + 8.f) {
        scale = ex2(m_used - mt);
        m_used = mt;
        resc = true;
      }
      uint32_t pk[BKV / 2];
      float ps[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
      for (int u = 0; u < BKV / 2; ++u) {
        __nv_bfloat162 v2 = __floats2bfloat162_rn(ex2(s[2 * u] - m_used), ex2(s[2 * u + 1] - m_used));
        ps[u & 7] += __low2float(v2) + __high2float(v2);
        pk[u] = *reinterpret_cast<uint32_t*>(&v2);
      }
#pragma unroll
      for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int u = 0; u < w2; ++u) ps[u] += ps[u + w2];
      // P_{j-1} * V_{j-1} must be done before P is overwritten or O rescaled.
      if (j > 0) {
        if (!(ok = wait_all(pv_done, (j - 1) & 1))) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
        for (int cc = 0; cc < p.d_v / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tO + cc * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * scale);
          tmem_st32(tO + cc * 32, v);
        }
        l *= scale;
      }
      tmem_st32(tP, *reinterpret_cast<const uint32_t(*)[32]>(pk));
      tmem_st32(tP + 32, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32));
      tmem_st_wait();
      l += ps[0];
      tc_fence_before();
      mbar_arrive(p_ready);
    }
    if (ok && (ok = wait_all(pv_done, (n - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.f / l;
      for (int cc = 0; cc < p.d_v / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tO + cc * 32, v);
        tmem_ld_wait();
        if (qpos < p.S) {
          float4* dst = reinterpret_cast<float4*>(p.out + (((long long)tok0 + qpos) * p.n_h + h) * p.d_v + cc * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv, __uint_as_float(v[4 * q + 1]) * inv,
                                 __uint_as_float(v[4 * q + 2]) * inv, __uint_as_float(v[4 * q + 3]) * inv);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
}

}  // namespace attn_mha
}  // namespace mla
