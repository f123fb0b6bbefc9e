// Batched "NT" GEMM with fused epilogues for the projection steps:
//   C[b][m][n] = sum_k A[b][m][k] * B[b][n][k]        (fp32 accumulation)
// A rows are tokens (K-major), B rows are weight rows (K-major), so C = A B^T
// is exactly y = W x applied to every token.  The epilogue functor receives
// adjacent column pairs (n even) and places, rotates and rounds them.
//
// This file holds the epilogue functors shared with the tensor-core GEMM
// (gemm_tc.cuh) and the fp32 CUDA-core main loop (the fp32 path must stay
// within 1e-4, which excludes single-pass TF32).
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
  // Columns n0 .. n0 + 7 (n0 a multiple of 8) of row m.
  __device__ void store8(int b, int m, int n0, const float (&v)[8]) const {
    float w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = alpha * v[i];
    mla::store8(C + b * strideC + (long long)m * ldc + n0, w);
  }
};

// Append: columns [0, d_c) are the latent, [d_c, d_cr) the position key (one
// shared key of d_r, or one per head), every d_r-wide key rotated by the
// token's position, then the row goes to its cache slot.
// Without seq_idx/pos, row m is either token m % prefill_S of sequence
// m / prefill_S (prefill) or, with kv_len, new token q = m % n_q of sequence
// b = m / n_q at position kv_len[b] - n_q + q (a decode step).
template <typename OutT>
struct EpiAppend {
  OutT* cache;
  const int32_t* seq_idx;
  const int32_t* pos;
  int prefill_S;
  const int32_t* page_table;
  double theta[32];        // RoPE frequencies
  int max_pages, num_pages, page_size, d_c, d_cr, n_seq;
  int d_r;                 // RoPE-key width: columns [d_c, d_cr) are one key or n_h keys of d_r each
  int* err;
  OutT* dense;             // optional: every row also at dense[m * d_cr] (token order), else null
  const int32_t* kv_len;   // decode step: lengths after the append, and
  int n_q;                 // new tokens per sequence
  __device__ void locate(int m, int& s, int& p) const {
    if (seq_idx) {
      s = seq_idx[m];
      p = pos[m];
    } else if (kv_len) {
      s = m / n_q;
      p = kv_len[s] - n_q + (m - s * n_q);
    } else {
      s = m / prefill_S;
      p = m - s * prefill_S;
    }
  }
  __device__ void operator()(int, int m, int n, float v0, float v1) const {
    int s, p;
    locate(m, s, p);
    if (s < 0 || s >= n_seq || p < 0 || p >= max_pages * page_size) {
      flag_error(err, kErrBounds);
      return;
    }
    int page = page_table[(long long)s * max_pages + p / page_size];
    if (page < 0 || page >= num_pages) {
      flag_error(err, kErrBounds);
      return;
    }
    if (n >= d_c) rope_rotate_pair(v0, v1, p, theta[((n - d_c) % d_r) >> 1]);
    store_pair(cache + ((long long)page * page_size + p % page_size) * d_cr + n, v0, v1);
    if (dense) store_pair(dense + (long long)m * d_cr + n, v0, v1);
  }
  // Columns n0 .. n0 + 7 of token m (n0 a multiple of 8; d_c is one too, so
  // the eight are all latent or all position key).
  __device__ void store8(int, int m, int n0, const float (&v)[8]) const {
    int s, p;
    locate(m, s, p);
    if (s < 0 || s >= n_seq || p < 0 || p >= max_pages * page_size) {
      flag_error(err, kErrBounds);
      return;
    }
    int page = page_table[(long long)s * max_pages + p / page_size];
    if (page < 0 || page >= num_pages) {
      flag_error(err, kErrBounds);
      return;
    }
    float w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = v[i];
    if (n0 >= d_c) {
#pragma unroll
      for (int i = 0; i < 4; ++i) rope_rotate_pair(w[2 * i], w[2 * i + 1], p, theta[(((n0 - d_c) % d_r) >> 1) + i]);
    }
    mla::store8(cache + ((long long)page * page_size + p % page_size) * d_cr + n0, w);
    if (dense) mla::store8(dense + (long long)m * d_cr + n0, w);
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
  // Columns n0 .. n0 + 7 of token m (n0 a multiple of 8; n_h*d_h and d_r are
  // too, so the eight are all q_C or all one head's q_R).
  __device__ void store8(int, int m, int n0, const float (&v)[8]) const {
    const int nc = n_h * d_h;
    if (n0 < nc) {
      mla::store8(qc + (long long)m * nc + n0, v);
      return;
    }
    const int j = n0 - nc, h = j / d_r, jj = j - h * d_r;
    int p;
    if (prefill_S > 0) p = m % prefill_S;
    else p = (kv_len ? kv_len[m / n_q] : uniform_kv_len) - n_q + m % n_q;
    float w[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x0 = v[2 * i], x1 = v[2 * i + 1];
      rope_rotate_pair(x0, x1, p, theta[(jj >> 1) + i]);
      w[2 * i] = qr_scale * x0;
      w[2 * i + 1] = qr_scale * x1;
    }
    mla::store8(qabs + ((long long)m * qabs_rows + h) * d_cr + d_c + jj, w);
  }
};

// Query projection for the materialised form: q = [q_C | RoPE_m(q_R)] per
// head, both parts multiplied by qscale (the softmax scale times log2 e),
// written to q[t][h][0 .. d_h + d_r).  Columns [0, n_h*d_h) are q_C (head h
// at h*d_h), the rest q_R (head h at n_h*d_h + h*d_r).  Token m of a prefill
// is position m % prefill_S.
template <typename OutT>
struct EpiQProjM {
  OutT* q;                 // [T, n_h, d_h + d_r]
  double theta[32];
  int n_h, d_h, d_r, prefill_S;
  float qscale;
  __device__ void operator()(int, int m, int n, float v0, float v1) const {
    const int nc = n_h * d_h, dq = d_h + d_r;
    if (n < nc) {
      const int h = n / d_h, i = n - h * d_h;
      store_pair(q + ((long long)m * n_h + h) * dq + i, qscale * v0, qscale * v1);
      return;
    }
    const int j = n - nc, h = j / d_r, jj = j - h * d_r;
    rope_rotate_pair(v0, v1, m % prefill_S, theta[jj >> 1]);
    store_pair(q + ((long long)m * n_h + h) * dq + d_h + jj, qscale * v0, qscale * v1);
  }
  // Columns n0 .. n0 + 7 (n0 a multiple of 8; d_h and d_r are too, so the
  // eight belong to one head's q_C or one head's q_R).
  __device__ void store8(int, int m, int n0, const float (&v)[8]) const {
    const int nc = n_h * d_h, dq = d_h + d_r;
    float w[8];
    if (n0 < nc) {
      const int h = n0 / d_h, i = n0 - h * d_h;
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = qscale * v[k];
      mla::store8(q + ((long long)m * n_h + h) * dq + i, w);
      return;
    }
    const int j = n0 - nc, h = j / d_r, jj = j - h * d_r;
    const int p = m % prefill_S;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float x0 = v[2 * k], x1 = v[2 * k + 1];
      rope_rotate_pair(x0, x1, p, theta[(jj >> 1) + k]);
      w[2 * k] = qscale * x0;
      w[2 * k + 1] = qscale * x1;
    }
    mla::store8(q + ((long long)m * n_h + h) * dq + d_h + jj, w);
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
