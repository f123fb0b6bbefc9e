// Context-parallel decode: one sequence's keys spread over ranks.
//
// A rank holds one page-aligned window of each sequence, positions
// [start, start + count), in its own page pool: local page i of the window
// holds positions start + i*page .. start + (i+1)*page - 1.  For every new
// token and head the rank computes the attention over the keys of its window
// that the token may see (causal range clipped to the window): the normalised
// latent sum obar_r and lse_r = log2 of the sum of 2^(score) over those keys
// (scores are kept in base 2, pre-multiplied by log2 e).  The ranks exchange
// (obar_r, lse_r) and merge
//     L = log2 sum_r 2^lse_r,   obar = sum_r 2^(lse_r - L) obar_r,
// which is the attention over the union of the windows, because the softmax
// denominators of disjoint key sets add up.  A rank that sees no key of a row
// has lse_r = -inf and weight 0.
//
// The attention kernel itself is the decode kernel, unchanged: the schedule
// below gives every segment its own partial slot, so every row block leaves
// (m, l, unnormalised sum) and cp_combine_kernel turns them into (obar_r,
// lse_r).
#pragma once
#include "attn_simt.cuh"  // AttnArgs
#include "common.cuh"
#include "sched.cuh"

namespace mla {

struct CpWindow {
  const int32_t* start;  // [B] first position held, a multiple of the page size
  const int32_t* count;  // [B] positions held from there
  int max_count;         // capacity of the local page table in positions
};

// Keys of row block rb inside the window.  A window that is negative, not
// page-aligned or larger than the local page table sets the bounds flag and
// counts as empty.
__device__ __forceinline__ int cp_local_keys(const SchedArgs& a, const CpWindow& win, int rb, int* err) {
  const int causal = rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, err);
  const int seq = rb / a.n_q;
  const int s0 = win.start[seq], cnt = win.count[seq];
  if (s0 < 0 || cnt < 0 || s0 % a.tile != 0 || cnt > win.max_count) {
    flag_error(err, kErrBounds);
    return 0;
  }
  return min(max(causal - s0, 0), cnt);
}

// Schedule of a window.  The cut is the decode schedule's (the tiles of all
// row blocks, in row-block order, split into W equal contiguous ranges, one
// per worker); here a row block without a key in the window has no tile and
// gets no segment, and segment s writes partial slot s.  rb_seg_first[rb] ..
// rb_seg_first[rb + 1] lists the segments of row block rb (empty for a row
// block without a tile).  One block of 1024 threads; arrays in global memory.
__global__ void __launch_bounds__(1024) cp_sched_kernel(SchedArgs a, CpWindow win) {
  const int tid = threadIdx.x, T = blockDim.x;
  const int R = a.R, W = a.W;
  int* ts = a.s.tile_start;
  for (int rb = tid; rb < R; rb += T) ts[rb] = ceil_div(cp_local_keys(a, win, rb, a.err), a.tile);
  __syncthreads();
  const int total = block_exclusive_scan(ts, R);
  if (tid == 0) ts[R] = total;
  __syncthreads();

  // Segments per worker.  find_le returns the last of equal offsets, so the
  // row blocks holding a worker's first and last tile have tiles; one in
  // between may have none.
  int* ws = a.s.worker_seg;
  for (int w = tid; w < W; w += T) {
    const long long lo = (long long)w * total / W, hi = (long long)(w + 1) * total / W;
    int cnt = 0;
    if (hi > lo) {
      const int r0 = find_le(ts, R, (int)lo), r1 = find_le(ts, R, (int)(hi - 1));
      for (int rb = r0; rb <= r1; ++rb) cnt += ts[rb + 1] > ts[rb];
    }
    ws[w] = cnt;
  }
  __syncthreads();
  const int nseg = block_exclusive_scan(ws, W);
  if (tid == 0) ws[W] = nseg;
  __syncthreads();

  for (int w = tid; w < W; w += T) {
    const long long lo = (long long)w * total / W, hi = (long long)(w + 1) * total / W;
    if (hi <= lo) continue;
    const int r0 = find_le(ts, R, (int)lo), r1 = find_le(ts, R, (int)(hi - 1));
    int s = ws[w];
    for (int rb = r0; rb <= r1; ++rb) {
      if (ts[rb + 1] == ts[rb]) continue;
      Seg g;
      g.rb = rb;
      g.t_lo = max((int)lo, ts[rb]) - ts[rb];
      g.t_hi = min((int)hi, ts[rb + 1]) - ts[rb];
      g.slot = s;
      g.nkeys = cp_local_keys(a, win, rb, nullptr);
      g.pad[0] = g.pad[1] = g.pad[2] = 0;
      a.s.segs[s] = g;
      if (g.t_lo == 0) a.s.rb_seg_first[rb] = s;
      ++s;
    }
  }
  if (tid == 0) a.s.rb_seg_first[R] = nseg;
  __syncthreads();
  // A row block without a tile starts where the next row block with tiles
  // does (or at nseg), which also ends the list of the row block before it.
  for (int rb = tid; rb < R; rb += T)
    if (ts[rb + 1] == ts[rb]) {
      int n = rb + 1;
      while (n < R && ts[n + 1] == ts[n]) ++n;
      a.s.rb_seg_first[rb] = n < R ? a.s.rb_seg_first[n] : nseg;
    }
}


// Per (row block, head): merges the row block's segment slots into the
// normalised latent sum obar_r (type T) and lse_r = m + log2 l.  A row block
// without a segment gets lse_r = -inf and its obar_r row is left unwritten.
// Block = (row block, 8 heads), one warp per head; lane j holds latent
// columns 4j .. 4j+3 of each 128-column chunk (the bf16 path has d_c <= 512,
// d_c % 128 == 0).
template <typename T>
__global__ void __launch_bounds__(256) cp_combine_kernel(AttnArgs a, T* obar_out, float* lse_out) {
  const Sched& S = a.sched;
  const int rb = blockIdx.x;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= a.n_h) return;
  const long long row = (long long)rb * a.n_h + h;
  const int s0 = S.rb_seg_first[rb], s1 = S.rb_seg_first[rb + 1];
  if (s0 >= s1) {
    if (lane == 0) lse_out[row] = -INFINITY;
    return;
  }
  // Max and sum over the segments, for each latent-column half (the two CTAs
  // of the tensor-core kernel keep their own softmax state, equal to within
  // the fp16 rounding of the exchanged partial scores).
  float m[2] = {-INFINITY, -INFINITY};
  for (int s = s0 + lane; s < s1; s += 32)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) m[hf] = fmaxf(m[hf], a.part_ml[ml_index(S.segs[s].slot, hf, a.n_h, h)]);
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m[hf] = fmaxf(m[hf], __shfl_xor_sync(0xffffffffu, m[hf], o));
  float l[2] = {0.f, 0.f};
  for (int s = s0 + lane; s < s1; s += 32)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const float* ml = a.part_ml + ml_index(S.segs[s].slot, hf, a.n_h, h);
      l[hf] += exp2f(ml[0] - m[hf]) * ml[1];
    }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l[hf] += __shfl_xor_sync(0xffffffffu, l[hf], o);
  const int half_cols = a.d_c / 2;
  float4 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = s0; s < s1; ++s) {
    const int slot = S.segs[s].slot;
    const float* ml0 = a.part_ml + ml_index(slot, 0, a.n_h, h);
    const float* ml1 = a.part_ml + ml_index(slot, 1, a.n_h, h);
    const float w0 = exp2f(ml0[0] - m[0]) * ml0[1];  // the slots hold normalised sums
    const float w1 = exp2f(ml1[0] - m[1]) * ml1[1];
    const T* src = static_cast<const T*>(a.part_o) + ((long long)slot * a.n_h + h) * a.d_c;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = c * 128 + 4 * lane;
      if (j < a.d_c) {
        const float4 v = load4(src + j);
        const float wgt = j < half_cols ? w0 : w1;
        acc[c].x += wgt * v.x;
        acc[c].y += wgt * v.y;
        acc[c].z += wgt * v.z;
        acc[c].w += wgt * v.w;
      }
    }
  }
  const float inv[2] = {1.f / l[0], 1.f / l[1]};
  T* out = obar_out + row * a.d_c;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = c * 128 + 4 * lane;
    const float iv = j < half_cols ? inv[0] : inv[1];
    if (j < a.d_c) store4(out + j, acc[c].x * iv, acc[c].y * iv, acc[c].z * iv, acc[c].w * iv);
  }
  // One log-sum-exp per row: the first half's (the second half's differs by
  // the rounding of the exchanged scores).
  if (lane == 0) lse_out[row] = m[0] + log2f(l[0]);
}

// Merges the ranks' partials of every (row, head) into obar (type T):
// obar = sum_r 2^(lse_r - L) obar_r with L = log2 sum_r 2^lse_r.  A rank
// with lse_r = -inf is skipped (its obar_r row may be unwritten).  A row that
// no rank saw sets the bounds flag and is written as zeros.
// parts: obar_parts [n_ranks][R][n_h][d_c], lse_parts [n_ranks][R][n_h].
template <typename T>
__global__ void __launch_bounds__(256) cp_merge_kernel(int n_ranks, const T* __restrict__ obar_parts,
                                                      const float* __restrict__ lse_parts, T* __restrict__ obar,
                                                      int R, int n_h, int d_c, int* err) {
  const int rb = blockIdx.x;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= n_h) return;
  const long long row = (long long)rb * n_h + h, lse_stride = (long long)R * n_h;
  float m = -INFINITY;
  for (int r = lane; r < n_ranks; r += 32) m = fmaxf(m, lse_parts[r * lse_stride + row]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  T* out = obar + row * d_c;
  if (m == -INFINITY) {
    if (lane == 0) flag_error(err, kErrBounds);
    for (int j = 4 * lane; j < d_c; j += 128) store4(out + j, 0.f, 0.f, 0.f, 0.f);
    return;
  }
  float l = 0.f;
  for (int r = lane; r < n_ranks; r += 32) l += exp2f(lse_parts[r * lse_stride + row] - m);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  const float inv = 1.f / l;
  float4 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < n_ranks; ++r) {
    const float lr = lse_parts[r * lse_stride + row];
    if (lr == -INFINITY) continue;  // the same for the whole warp
    const float wgt = exp2f(lr - m) * inv;
    const T* src = obar_parts + (r * lse_stride + row) * d_c;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = c * 128 + 4 * lane;
      if (j < d_c) {
        const float4 v = load4(src + j);
        acc[c].x += wgt * v.x;
        acc[c].y += wgt * v.y;
        acc[c].z += wgt * v.z;
        acc[c].w += wgt * v.w;
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int j = c * 128 + 4 * lane;
    if (j < d_c) store4(out + j, acc[c].x, acc[c].y, acc[c].z, acc[c].w);
  }
}

}  // namespace mla
