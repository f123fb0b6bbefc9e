// Batched "NT" GEMM with fused epilogues for the projection steps:
//   C[b][m][n] = sum_k A[b][m][k] * B[b][n][k]        (fp32 accumulation)
// A rows are tokens (K-major), B rows are weight rows (K-major), so C = A B^T
// is exactly y = W x applied to every token.  The epilogue functor receives
// adjacent column pairs (n even) and places, rotates and rounds them.
//
// Two main loops share the split-K bookkeeping and the epilogue:
//   * bf16: mma.sync m16n8k16 tensor-core tiles fed by a 3-stage cp.async
//     pipeline (used for the weight-streaming projections);
//   * fp32: FFMA tiles (the fp32 path must stay within 1e-4, which excludes
//     single-pass TF32).
// Split-K: every split writes its fp32 tile to scratch and bumps a per-tile
// counter; the last split to arrive sums all splits in split order (so the
// result is deterministic) and runs the epilogue, then re-arms the counter.
#pragma once
#include "common.cuh"

namespace mla {

struct GemmArgs {
  const void* A;
  long long lda, strideA;  // elements
  const void* B;
  long long ldb, strideB;
  int M, N, K, batch;
  int splits;              // split-K factor (>= 1)
  int kchunk;              // K elements per split (multiple of 32)
  float* partial;          // split-K scratch: [batch][tiles][splits][BM*BN]
  int* counters;           // [batch][tiles], zero between calls
};

// ---------------------------------------------------------------- epilogues
// Plain store with a scale: C + b*strideC + m*ldc + n.
template <typename OutT>
struct EpiStore {
  OutT* C;
  long long ldc, strideC;
  float alpha;
  __device__ void operator()(int b, int m, int n, float v0, float v1) const {
    store_pair(C + b * strideC + (long long)m * ldc + n, alpha * v0, alpha * v1);
  }
};

// Append: columns [0, d_c) are the latent, [d_c, d_c + d_r) the position key,
// rotated by the token's position, then the row goes to its cache slot.
// Without seq_idx/pos (prefill), row m is token m % prefill_S of sequence
// m / prefill_S.
template <typename OutT>
struct EpiAppend {
  OutT* cache;
  const int32_t* seq_idx;
  const int32_t* pos;
  int prefill_S;
  const int32_t* page_table;
  double theta[32];        // RoPE frequencies
  int max_pages, num_pages, page_size, d_c, d_cr, n_seq;
  int* err;
  __device__ void operator()(int, int m, int n, float v0, float v1) const {
    int s, p;
    if (seq_idx) {
      s = seq_idx[m];
      p = pos[m];
    } else {
      s = m / prefill_S;
      p = m - s * prefill_S;
    }
    if (s < 0 || s >= n_seq || p < 0 || p >= max_pages * page_size) {
      flag_error(err, kErrBounds);
      return;
    }
    int page = page_table[(long long)s * max_pages + p / page_size];
    if (page < 0 || page >= num_pages) {
      flag_error(err, kErrBounds);
      return;
    }
    if (n >= d_c) rope_rotate_pair(v0, v1, p, theta[(n - d_c) >> 1]);
    store_pair(cache + ((long long)page * page_size + p % page_size) * d_cr + n, v0, v1);
  }
};

// Query projection: columns [0, n_h*d_h) are q_C (stored unscaled for the
// absorption GEMM); the rest are q_R, head h at n_h*d_h + h*d_r, rotated by
// the query's position, scaled, and written into Q_abs[t][h][d_c + j].
template <typename OutT>
struct EpiQProj {
  OutT* qc;                // [T, n_h*d_h]
  OutT* qabs;              // [T, qabs_rows, d_cr]
  const int32_t* kv_len;   // decode: position = kv_len[t / n_q] - n_q + t % n_q
  int uniform_kv_len;      // used when kv_len is null
  double theta[32];
  int n_h, d_h, d_r, d_c, d_cr, qabs_rows, n_q, prefill_S;
  float qr_scale;
  __device__ void operator()(int, int m, int n, float v0, float v1) const {
    const int nc = n_h * d_h;
    if (n < nc) {
      store_pair(qc + (long long)m * nc + n, v0, v1);
      return;
    }
    int j = n - nc, h = j / d_r, jj = j - h * d_r;
    int p;
    if (prefill_S > 0) p = m % prefill_S;
    else p = (kv_len ? kv_len[m / n_q] : uniform_kv_len) - n_q + m % n_q;
    rope_rotate_pair(v0, v1, p, theta[jj >> 1]);
    store_pair(qabs + ((long long)m * qabs_rows + h) * d_cr + d_c + jj, qr_scale * v0, qr_scale * v1);
  }
};

// -------------------------------------------------------- split-K finishing
// Each thread owns NP column pairs; map(p, r, c) gives a pair's local row and
// (even) local column inside the BM x BN tile.
template <int BM, int BN, int NP, class Epi, class Map>
__device__ __forceinline__ void gemm_finish(const GemmArgs& a, int bz, int tile, int split, int m0,
                                            int n0, float (&acc)[NP][2], Map map, const Epi& epi) {
  if (a.splits == 1) {
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      int r, c;
      map(p, r, c);
      int m = m0 + r, n = n0 + c;
      if (m < a.M && n < a.N) epi(bz, m, n, acc[p][0], acc[p][1]);
    }
    return;
  }
  const int tiles = gridDim.x * gridDim.y;
  float* base = a.partial + ((long long)bz * tiles + tile) * a.splits * (BM * BN);
  float* mine = base + (long long)split * (BM * BN);
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    int r, c;
    map(p, r, c);
    __stcg(reinterpret_cast<float2*>(mine + r * BN + c), make_float2(acc[p][0], acc[p][1]));
  }
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  int* ctr = a.counters + (long long)bz * tiles + tile;
  if (threadIdx.x == 0) is_last = (atomicAdd(ctr, 1) == a.splits - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // The last split sums all splits in split order.  Each thread owns whole
  // float4 groups of the tile and keeps eight loads in flight per group.
  for (int q = threadIdx.x; q < BM * BN / 4; q += blockDim.x) {
    const int r = q / (BN / 4), c = (q % (BN / 4)) * 4;
    const float4* src = reinterpret_cast<const float4*>(base + r * BN + c);
    float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 8 <= a.splits; s += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (long long)(s + u) * (BM * BN / 4));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc4.x += v[u].x;
        acc4.y += v[u].y;
        acc4.z += v[u].z;
        acc4.w += v[u].w;
      }
    }
    for (; s < a.splits; ++s) {
      float4 v = __ldcg(src + (long long)s * (BM * BN / 4));
      acc4.x += v.x;
      acc4.y += v.y;
      acc4.z += v.z;
      acc4.w += v.w;
    }
    const int m = m0 + r, n = n0 + c;
    if (m < a.M) {
      if (n < a.N) epi(bz, m, n, acc4.x, acc4.y);
      if (n + 2 < a.N) epi(bz, m, n + 2, acc4.z, acc4.w);
    }
  }
  if (threadIdx.x == 0) *ctr = 0;
}

// ------------------------------------------------------------ bf16 kernel
namespace gemm_bf16 {
constexpr int BM = 64, BN = 64, BK = 32, STAGES = 3, PITCH = BK + 8, THREADS = 128;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int bytes) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldmatrix_x4(unsigned (&r)[4], const void* p) {
  unsigned s = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const unsigned (&a)[4], unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <class Epi>
__global__ void __launch_bounds__(THREADS) gemm_bf16_kernel(GemmArgs a, Epi epi) {
  __shared__ __align__(128) __nv_bfloat16 As[STAGES][BM][PITCH];
  __shared__ __align__(128) __nv_bfloat16 Bs[STAGES][BN][PITCH];
  const int bz = blockIdx.z / a.splits, split = blockIdx.z % a.splits;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tile = blockIdx.y * gridDim.x + blockIdx.x;
  const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A) + bz * a.strideA;
  const __nv_bfloat16* B = static_cast<const __nv_bfloat16*>(a.B) + bz * a.strideB;
  const int k_begin = split * a.kchunk;
  const int k_end = min(a.K, k_begin + a.kchunk);
  const int nk = k_end > k_begin ? ceil_div(k_end - k_begin, BK) : 0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 1, wn = warp & 1;

  auto load = [&](int stage, int k0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      int idx = tid + i * THREADS;  // 256 chunks of 16 B per operand tile
      int r = idx >> 2, ck = (idx & 3) * 8;
      int gk = k0 + ck;
      {
        int gm = m0 + r;
        bool ok = gm < a.M && gk < k_end;
        const void* src = ok ? (const void*)(A + (long long)gm * a.lda + gk) : (const void*)A;
        cp_async16(&As[stage][r][ck], src, ok ? 16 : 0);
      }
      {
        int gn = n0 + r;
        bool ok = gn < a.N && gk < k_end;
        const void* src = ok ? (const void*)(B + (long long)gn * a.ldb + gk) : (const void*)B;
        cp_async16(&Bs[stage][r][ck], src, ok ? 16 : 0);
      }
    }
  };

  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nk) load(s, k_begin + s * BK);
    cp_async_commit();
  }
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    int nxt = kt + STAGES - 1;
    if (nxt < nk) load(nxt % STAGES, k_begin + nxt * BK);
    cp_async_commit();
    const int st = kt % STAGES;
#pragma unroll
    for (int kk = 0; kk < BK; kk += 16) {
      unsigned af[2][4], bfr[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
        ldmatrix_x4(af[i], &As[st][wm * 32 + i * 16 + (lane & 15)][kk + (lane >> 4) * 8]);
#pragma unroll
      for (int j = 0; j < 2; ++j)
        ldmatrix_x4(bfr[j], &Bs[st][wn * 32 + j * 16 + (lane & 7) + (lane >> 4) * 8][kk + ((lane >> 3) & 1) * 8]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          mma16816(acc[i][2 * j], af[i], bfr[j][0], bfr[j][1]);
          mma16816(acc[i][2 * j + 1], af[i], bfr[j][2], bfr[j][3]);
        }
    }
  }
  cp_async_wait<0>();

  // Pair p = (i, j, half): rows wm*32 + i*16 + g (+8), cols wn*32 + j*8 + 2t.
  float pairs[16][2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        pairs[(i * 4 + j) * 2 + h][0] = acc[i][j][2 * h];
        pairs[(i * 4 + j) * 2 + h][1] = acc[i][j][2 * h + 1];
      }
  const int g = lane >> 2, t4 = lane & 3;
  auto map = [&](int p, int& r, int& c) {
    int h = p & 1, j = (p >> 1) & 3, i = p >> 3;
    r = wm * 32 + i * 16 + g + h * 8;
    c = wn * 32 + j * 8 + 2 * t4;
  };
  gemm_finish<BM, BN, 16>(a, bz, tile, split, m0, n0, pairs, map, epi);
}
}  // namespace gemm_bf16

// ------------------------------------------------------------ fp32 kernel
namespace gemm_f32 {
constexpr int BM = 64, BN = 64, BK = 16, THREADS = 256;

template <class Epi>
__global__ void __launch_bounds__(THREADS) gemm_f32_kernel(GemmArgs a, Epi epi) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int bz = blockIdx.z / a.splits, split = blockIdx.z % a.splits;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tile = blockIdx.y * gridDim.x + blockIdx.x;
  const float* A = static_cast<const float*>(a.A) + bz * a.strideA;
  const float* B = static_cast<const float*>(a.B) + bz * a.strideB;
  const int k_begin = split * a.kchunk;
  const int k_end = min(a.K, k_begin + a.kchunk);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += BK) {
    for (int idx = tid; idx < BM * BK; idx += THREADS) {
      int r = idx / BK, kk = idx % BK;
      int gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < a.M && gk < k_end) ? A[(long long)gm * a.lda + gk] : 0.f;
      int gn = n0 + r;
      Bs[kk][r] = (gn < a.N && gk < k_end) ? B[(long long)gn * a.ldb + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float pairs[8][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      pairs[i * 2 + h][0] = acc[i][2 * h];
      pairs[i * 2 + h][1] = acc[i][2 * h + 1];
    }
  auto map = [&](int p, int& r, int& c) {
    r = ty * 4 + (p >> 1);
    c = tx * 4 + (p & 1) * 2;
  };
  gemm_finish<BM, BN, 8>(a, bz, tile, split, m0, n0, pairs, map, epi);
}
}  // namespace gemm_f32

}  // namespace mla
