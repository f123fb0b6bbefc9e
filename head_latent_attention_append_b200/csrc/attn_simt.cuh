// Absorbed latent attention on CUDA cores (fp32 FFMA), split-KV.
//
// This is the fp32 path (the fp32 workload's 1e-4 bound rules out single-pass
// TF32 on the tensor cores).  Per query token and head it computes
//   a_t   = Q_abs[h] . cache[t]          over the d_c latent columns and
//           the d_r columns of the RoPE key (the shared one, or head h's own
//           in the per-head layout of "Multi-Head Latent Attention",
//           "A concrete size comparison")
//           (Q_abs = [s*log2(e)*W_UK,h^T q_C,h | s*log2(e)*RoPE_m(q_R,h)], so
//           a_t is the pages' score in log2 units)
//   alpha = softmax over the visible keys (exp2, online, running max)
//   obar  = sum_t alpha_t c_t            over the d_c latent columns
// ("ai-decoupled-rope-mla": absorbed score and output equations).
//
// Grid: (worker, head group).  A CTA walks its worker's segments (sched.cuh)
// for HG heads; 32 keys at a time are staged in shared memory as fp32.
#pragma once
#include "common.cuh"
#include "sched.cuh"

namespace mla {

struct AttnArgs {
  const void* qabs;          // [R][qrows][q_row]
  int qrows;
  const void* cache;         // [num_pages][page_size][d_cr]: a row is [c | k_R] (one shared key or n_h keys)
  const int32_t* page_table; // [n_seq][max_pages]
  int max_pages, num_pages, page_size;
  int n_h, d_c, d_r, d_cr;
  int q_row;                 // Q_abs row: d_c + d_r ([q~ | q_R])
  int rope_per_head;         // 0: one shared RoPE key per row; 1: head h's key at d_c + h*d_r
  const int32_t* kv_len;
  int uniform_kv_len, n_q, max_kv_len;
  Sched sched;
  void* part_o;              // [2W][n_h][d_c], type of the path: a split segment's latent sum over
                             // its keys, normalised by its own l (so bf16 keeps it as well as obar)
  float* part_ml;            // [2W][2][n_h][2]: (m, l) per latent-column half (ml_index)
  void* obar;                // [R][n_h][d_c] (type of the path)
  int* err;
  // Arrival counters [R][2] (zero at the start of a call), or null.  With
  // them the tensor-core kernel merges a split row block itself: each piece
  // counts in after writing its partial slot, and the last of a CTA rank's
  // pieces merges all of them (in segment order) into obar; no combine
  // kernel runs.
  int* arrive;
};

// Index into part_ml of the (m, l) pair of partial slot `slot`, latent-column
// half `half` ([0, d_c/2) or [d_c/2, d_c)) and head h.  The tensor-core
// kernel's two CTAs each keep their own softmax state for their half; the
// CUDA-core kernel writes the same pair to both halves.
__host__ __device__ __forceinline__ long long ml_index(int slot, int half, int n_h, int h) {
  return (((long long)slot * 2 + half) * n_h + h) * 2;
}

namespace attn_simt {
constexpr int THREADS = 256, KC = 32, MAX_CPT = 32;

// Staged rows (cache rows and Q rows, fp32) are padded to 4 mod 32 floats:
// 16-byte aligned, and the 32 rows of a warp's score loads start in eight
// different 4-bank groups (conflict-free 16-byte loads).
__host__ __device__ constexpr int row_pitch(int d_cr) { return (d_cr + 31) / 32 * 32 + 4; }

// The eight bf16 (or four fp32) values of a 16-byte load, as floats.
template <typename T> __device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
    f[2 * q] = v.x;
    f[2 * q + 1] = v.y;
  }
}
template <> __device__ __forceinline__ void unpack16<float>(const uint4& u, float* f) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}

template <typename T>
__global__ void __launch_bounds__(THREADS) attn_simt_kernel(AttnArgs a, int HG) {
  extern __shared__ float smem[];
  const int pitch = row_pitch(a.d_cr);  // cache rows; a Q row uses the first q_row of its pitch
  float* Qs = smem;                    // [HG][pitch]
  float* Cs = Qs + HG * pitch;         // [KC][pitch]
  float* Ps = Cs + KC * pitch;         // [HG][KC]
  float* st = Ps + HG * KC;            // [HG][3]: m, l, corr
  const int w = blockIdx.x, h0 = blockIdx.y * HG;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int TPH = THREADS / HG;        // threads per head in the output update
  const int oh = tid / TPH, oj = tid % TPH;
  const int cpt = ceil_div(a.d_c, TPH);  // <= MAX_CPT (d_c <= 512, TPH >= 16)
  // d_c % 4 == 0: the latent columns are read four at a time (16-byte
  // shared-memory loads), and an output thread owns groups of four columns.
  const bool vec_c = (a.d_c & 3) == 0;
  const int cpt4 = ceil_div(a.d_c / 4, TPH);  // <= MAX_CPT / 4
  const T* qabs = static_cast<const T*>(a.qabs);
  const T* cache = static_cast<const T*>(a.cache);
  const Sched& S = a.sched;
  const bool vec_rows = ((a.d_cr * (int)sizeof(T)) & 15) == 0 && (reinterpret_cast<uintptr_t>(cache) & 15) == 0;

  for (int si = S.worker_seg[w]; si < S.worker_seg[w + 1]; ++si) {
    const Seg g = S.segs[si];
    const int rb = g.rb, seq = rb / a.n_q;
    const int nkeys = rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, nullptr);
    __syncthreads();
    for (int i = tid; i < HG * a.q_row; i += THREADS) {
      int h = i / a.q_row, j = i % a.q_row;
      Qs[h * pitch + j] = (h0 + h < a.n_h) ? to_f32(qabs[((long long)rb * a.qrows + h0 + h) * a.q_row + j]) : 0.f;
    }
    if (tid < HG) {
      st[tid * 3 + 0] = -INFINITY;
      st[tid * 3 + 1] = 0.f;
    }
    float o[MAX_CPT];
#pragma unroll
    for (int r = 0; r < MAX_CPT; ++r) o[r] = 0.f;

    const int k_begin = g.t_lo * a.page_size;
    const int k_end = min(nkeys, g.t_hi * a.page_size);
    for (int k0 = k_begin; k0 < k_end; k0 += KC) {
      __syncthreads();
      // Stage KC cache rows (positions k0 .. k0+KC-1) through the page table:
      // each warp takes RPW rows, looks up their pages first (one load per
      // row for the whole warp), then reads the rows with 16-byte loads when
      // every row starts on a 16-byte boundary, element by element if not.
      {
        constexpr int RPW = KC / (THREADS / 32);
        constexpr int EPV = 16 / (int)sizeof(T);  // elements per 16-byte load
        const T* src[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const int p = k0 + warp * RPW + r;
          src[r] = nullptr;
          if (p < k_end) {
            const int page = a.page_table[(long long)seq * a.max_pages + p / a.page_size];
            if (page >= 0 && page < a.num_pages)
              src[r] = cache + ((long long)page * a.page_size + p % a.page_size) * a.d_cr;
            else if (lane == 0)
              flag_error(a.err, kErrBounds);
          }
        }
        if (vec_rows) {
          const int nv = a.d_cr / EPV;
          for (int v0 = 0; v0 < nv; v0 += 32) {
            const int v = v0 + lane;
            uint4 u[RPW];
#pragma unroll
            for (int r = 0; r < RPW; ++r)
              u[r] = (src[r] && v < nv) ? __ldg(reinterpret_cast<const uint4*>(src[r]) + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
              if (v >= nv) continue;
              float f[EPV];
              unpack16<T>(u[r], f);
              float* crow = Cs + (warp * RPW + r) * pitch + v * EPV;
#pragma unroll
              for (int e = 0; e < EPV; ++e) crow[e] = f[e];
            }
          }
        } else {
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            float* crow = Cs + (warp * RPW + r) * pitch;
            for (int j = lane; j < a.d_cr; j += 32) crow[j] = src[r] ? to_f32(src[r][j]) : 0.f;
          }
        }
      }
      __syncthreads();
      // Scores for HG x KC (head, key) pairs.
      for (int i = tid; i < HG * KC; i += THREADS) {
        int h = i / KC, k = i % KC;
        const float* q = Qs + h * pitch;
        const float* c = Cs + k * pitch;
        const float* kr = c + a.d_c + (a.rope_per_head ? (h0 + h) * a.d_r : 0);
        float acc = 0.f;
        if (vec_c) {
          float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int j = 0; j < a.d_c; j += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(q + j);
            const float4 cv = *reinterpret_cast<const float4*>(c + j);
            s4.x = fmaf(qv.x, cv.x, s4.x);
            s4.y = fmaf(qv.y, cv.y, s4.y);
            s4.z = fmaf(qv.z, cv.z, s4.z);
            s4.w = fmaf(qv.w, cv.w, s4.w);
          }
          acc = (s4.x + s4.y) + (s4.z + s4.w);
        } else {
          for (int j = 0; j < a.d_c; ++j) acc = fmaf(q[j], c[j], acc);
        }
        for (int j = 0; j < a.d_r; ++j) acc = fmaf(q[a.d_c + j], kr[j], acc);
        Ps[h * KC + k] = (k0 + k < k_end) ? acc : -INFINITY;
      }
      __syncthreads();
      // Online softmax: one warp per head, one lane per key.
      for (int h = warp; h < HG; h += THREADS / 32) {
        float s = Ps[h * KC + lane];
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float m_old = st[h * 3 + 0];
        float m_new = fmaxf(m_old, mx);
        float p = exp2f(s - m_new);
        float sum = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        Ps[h * KC + lane] = p;
        __syncwarp();
        if (lane == 0) {
          float corr = exp2f(m_old - m_new);
          st[h * 3 + 0] = m_new;
          st[h * 3 + 1] = st[h * 3 + 1] * corr + sum;
          st[h * 3 + 2] = corr;
        }
      }
      __syncthreads();
      // obar[h][j] = obar*corr + sum_k P[h][k] * c[k][j].
      if (oh < HG) {
        const float corr = st[oh * 3 + 2];
        const float* P = Ps + oh * KC;
        if (vec_c) {
#pragma unroll
          for (int r = 0; r < MAX_CPT / 4; ++r) {
            const int g4 = oj + r * TPH;
            if (r < cpt4 && 4 * g4 < a.d_c) {
              float4 acc = make_float4(o[4 * r] * corr, o[4 * r + 1] * corr, o[4 * r + 2] * corr, o[4 * r + 3] * corr);
#pragma unroll 8
              for (int k = 0; k < KC; ++k) {
                const float pk = P[k];
                const float4 cv = *reinterpret_cast<const float4*>(Cs + k * pitch + 4 * g4);
                acc.x = fmaf(pk, cv.x, acc.x);
                acc.y = fmaf(pk, cv.y, acc.y);
                acc.z = fmaf(pk, cv.z, acc.z);
                acc.w = fmaf(pk, cv.w, acc.w);
              }
              o[4 * r] = acc.x;
              o[4 * r + 1] = acc.y;
              o[4 * r + 2] = acc.z;
              o[4 * r + 3] = acc.w;
            }
          }
        } else {
#pragma unroll
          for (int r = 0; r < MAX_CPT; ++r) {
            if (r < cpt && oj + r * TPH < a.d_c) {
              int j = oj + r * TPH;
              float acc = o[r] * corr;
#pragma unroll 8
              for (int k = 0; k < KC; ++k) acc = fmaf(P[k], Cs[k * pitch + j], acc);
              o[r] = acc;
            }
          }
        }
      }
    }
    __syncthreads();
    // Finish: a whole row block is normalised straight into obar; a piece of
    // a split row block leaves (m, l, unnormalised sum) in its partial slot.
    if (oh < HG && h0 + oh < a.n_h) {
      const int h = h0 + oh;
      const float m = st[oh * 3 + 0], l = st[oh * 3 + 1];
      // Column of o[r]: groups of four (4 (oj + (r / 4) TPH) + r % 4) when
      // vec_c, else oj + r TPH.
      T* dst = g.slot < 0 ? static_cast<T*>(a.obar) + ((long long)rb * a.n_h + h) * a.d_c
                          : static_cast<T*>(a.part_o) + ((long long)g.slot * a.n_h + h) * a.d_c;
      const float inv = 1.f / l;
#pragma unroll
      for (int r = 0; r < MAX_CPT; ++r) {
        const int col = vec_c ? 4 * (oj + (r / 4) * TPH) + (r % 4) : oj + r * TPH;
        const bool mine = vec_c ? (r / 4 < cpt4 && col < a.d_c) : (r < cpt && col < a.d_c);
        if (mine) dst[col] = from_f32<T>(o[r] * inv);
      }
      if (g.slot >= 0) {
        if (oj == 0) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            a.part_ml[ml_index(g.slot, half, a.n_h, h) + 0] = m;
            a.part_ml[ml_index(g.slot, half, a.n_h, h) + 1] = l;
          }
        }
      }
    }
  }
}

inline size_t smem_bytes(int HG, int d_cr) {
  return sizeof(float) * ((size_t)(HG + KC) * row_pitch(d_cr) + HG * KC + HG * 3);
}
}  // namespace attn_simt

// ------------------------------------------------------------ combine -----
// Merges the partial slots of each split row block (log-sum-exp in base 2);
// slot s holds its normalised sum N_s = O_s / l_s and (m_s, l_s):
//   m = max_s m_s,  l = sum_s 2^(m_s - m) l_s,  obar = sum_s 2^(m_s - m) l_s N_s / l.
// Block = (split row block, 8 heads), one warp per head.  Lane k gathers the
// (slot, m, l) of segments k, k + 32, ...; the warp reduces them with
// shuffles, then each lane accumulates four consecutive latent columns of
// each 128-column chunk (d_c <= 512), two slots' loads in flight at a time.
// Slots are added in segment order, so the result is deterministic.
__device__ __forceinline__ float4 load4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = __ldcg(reinterpret_cast<const uint2*>(p));
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ void store4(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
}

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(AttnArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partial slots come from the attention kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const Sched& S = a.sched;
  const int idx = blockIdx.x;
  const int W = gridDim.x >> 1;
  if (idx >= S.split_rbs[0]) return;
  const int s0 = S.split_rbs[1 + idx];  // the row block's first segment; the others follow it
  const int nall = S.worker_seg[W];
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= a.n_h) return;
  // Lane k reads segment s0 + k; the row block's segments are the leading
  // lanes with its row block id.
  Seg gk;
  gk.rb = -1;
  gk.slot = 0;
  if (s0 + lane < nall) gk = S.segs[s0 + lane];
  const int rb = __shfl_sync(0xffffffffu, gk.rb, 0);
  const uint32_t same = __ballot_sync(0xffffffffu, gk.rb == rb);
  const int lead = __ffs(~same) - 1;  // -1: all 32 lanes belong to rb
  const int s1 = lead < 0 ? S.rb_seg_first[rb + 1] : s0 + lead;
  const int half_cols = a.d_c / 2;
  T* out = static_cast<T*>(a.obar) + ((long long)rb * a.n_h + h) * a.d_c;
  float4 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  // Adds the rows of slots sa and sb (if has_b) with weights (w0, w1) for
  // the two column halves; both slots' loads are in flight together.
  auto add2 = [&](int sa, float wa0, float wa1, bool has_b, int sb, float wb0, float wb1) {
    const T* pa = static_cast<const T*>(a.part_o) + ((long long)sa * a.n_h + h) * a.d_c;
    const T* pb = static_cast<const T*>(a.part_o) + ((long long)sb * a.n_h + h) * a.d_c;
    float4 va[4], vb[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = c * 128 + 4 * lane;
      va[c] = j < a.d_c ? load4(pa + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      vb[c] = (has_b && j < a.d_c) ? load4(pb + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const bool lo = (c * 128 + 4 * lane) < half_cols;
      const float x = lo ? wa0 : wa1, y = lo ? wb0 : wb1;
      acc[c].x += x * va[c].x + y * vb[c].x;
      acc[c].y += x * va[c].y + y * vb[c].y;
      acc[c].z += x * va[c].z + y * vb[c].z;
      acc[c].w += x * va[c].w + y * vb[c].w;
    }
  };
  float inv[2] = {1.f, 1.f};
  if (s1 - s0 <= 32) {
    // One round trip for the segments (above), one for the (m, l) pairs and
    // the rows, which do not depend on each other.
    const int nseg = s1 - s0;
    const int slot = gk.slot;
    float mk[2] = {-INFINITY, -INFINITY}, lk[2] = {0.f, 0.f};
    if (lane < nseg) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + ml_index(slot, hf, a.n_h, h));
        mk[hf] = ml.x;
        lk[hf] = ml.y;
      }
    }
    float w[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float m = mk[hf];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      w[hf] = lane < nseg ? exp2f(mk[hf] - m) * lk[hf] : 0.f;
      float l = w[hf];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      inv[hf] = 1.f / l;
    }
    for (int k = 0; k < nseg; k += 2) {
      const bool has_b = k + 1 < nseg;
      const int kb = has_b ? k + 1 : k;
      add2(__shfl_sync(0xffffffffu, slot, k), __shfl_sync(0xffffffffu, w[0], k), __shfl_sync(0xffffffffu, w[1], k),
           has_b, __shfl_sync(0xffffffffu, slot, kb), __shfl_sync(0xffffffffu, w[0], kb),
           __shfl_sync(0xffffffffu, w[1], kb));
    }
  } else {
    // More than 32 segments: the same in batches of 32.
    float m[2] = {-INFINITY, -INFINITY};
    for (int s = s0 + lane; s < s1; s += 32)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) m[hf] = fmaxf(m[hf], a.part_ml[ml_index(S.segs[s].slot, hf, a.n_h, h)]);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m[hf] = fmaxf(m[hf], __shfl_xor_sync(0xffffffffu, m[hf], o));
    float l[2] = {0.f, 0.f};
    for (int sb = s0; sb < s1; sb += 32) {
      int slot = 0;
      float w0 = 0.f, w1 = 0.f;
      if (sb + lane < s1) {
        slot = S.segs[sb + lane].slot;
        const float* ml0 = a.part_ml + ml_index(slot, 0, a.n_h, h);
        const float* ml1 = a.part_ml + ml_index(slot, 1, a.n_h, h);
        w0 = exp2f(ml0[0] - m[0]) * ml0[1];
        w1 = exp2f(ml1[0] - m[1]) * ml1[1];
      }
      l[0] += w0;
      l[1] += w1;
      const int cnt = min(32, s1 - sb);
      for (int k = 0; k < cnt; k += 2) {
        const bool has_b = k + 1 < cnt;
        const int kb = has_b ? k + 1 : k;
        add2(__shfl_sync(0xffffffffu, slot, k), __shfl_sync(0xffffffffu, w0, k), __shfl_sync(0xffffffffu, w1, k),
             has_b, __shfl_sync(0xffffffffu, slot, kb), __shfl_sync(0xffffffffu, w0, kb),
             __shfl_sync(0xffffffffu, w1, kb));
      }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) l[hf] += __shfl_xor_sync(0xffffffffu, l[hf], o);
      inv[hf] = 1.f / l[hf];
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = c * 128 + 4 * lane;
    const float iv = j < half_cols ? inv[0] : inv[1];
    if (j < a.d_c) store4(out + j, acc[c].x * iv, acc[c].y * iv, acc[c].z * iv, acc[c].w * iv);
  }
}

}  // namespace mla
