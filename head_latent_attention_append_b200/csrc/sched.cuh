// Ragged split-KV scheduling.
//
// A "row block" rb is one query token: all n_h heads of token rb (decode:
// sequence rb / n_q, new token rb % n_q).  Its keys are the cache positions
// 0 .. nkeys(rb)-1 with nkeys = kv_len[seq] - n_q + 1 + q, cut into tiles of
// one page.  The tiles of all row blocks, in row-block order, are split into
// W contiguous, equal ranges, one per worker, so every worker streams the
// same number of cache tiles whatever the length mix.  A worker's range
// crosses row blocks as "segments".  A segment that covers a whole row block
// is finished by the worker itself; only the first and the last segment of a
// worker can be part of a split row block, and those write a partial result
// (running max, running sum, unnormalised latent sum) into partial slot
// 2w or 2w+1, which the combine step merges.
//
// When there are about as many row blocks as workers and they are of about
// the same length (uniform decode), each worker takes one whole row block
// instead, and nothing is split (see sched_kernel).
//
// Everything is integer arithmetic and deterministic: the split points depend
// only on the lengths, never on the physical page order.
#pragma once
#include "common.cuh"

namespace mla {

// 32 bytes, read with two vector loads: a worker needs everything about a
// segment (its row block's key count too) from one round trip to memory.
struct __align__(16) Seg {
  int rb;      // row block
  int t_lo;    // first tile (inclusive), relative to the row block
  int t_hi;    // last tile (exclusive)
  int slot;    // partial slot, or -1 when the segment covers the whole row block
  int nkeys;   // keys of the row block (its causal length)
  int pad[3];
};

struct Sched {
  int* tile_start;    // [R+1]  exclusive prefix of tiles per row block
  int* worker_seg;    // [W+1]  first segment of each worker
  Seg* segs;          // [W+R]
  int* rb_seg_first;  // [R+1]  first segment of each row block
  int* split_rbs;     // [2W+1] first segment of each row block with more than one segment; [0] = count
};

struct SchedArgs {
  const int32_t* kv_len;  // [B] or null (then uniform_kv_len)
  int uniform_kv_len;
  int n_q, R, W, tile, max_kv_len;
  Sched s;
  int* err;
};

__device__ __forceinline__ int rb_nkeys(const int32_t* kv_len, int uniform, int n_q, int max_kv_len,
                                        int rb, int* err) {
  int seq = rb / n_q, q = rb - seq * n_q;
  int L = kv_len ? kv_len[seq] : uniform;
  if (L < n_q || L > max_kv_len) {
    flag_error(err, kErrBounds);
    L = min(max(L, n_q), max_kv_len);
  }
  return L - n_q + 1 + q;
}

// Exclusive scan of one int per thread across the block (warp shuffles).
__device__ int block_scan_excl(int v, int* total_out) {
  __shared__ int warp_tot[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int before = wid > 0 ? warp_tot[wid - 1] : 0;
  *total_out = warp_tot[nw - 1];
  __syncthreads();
  return before + x - v;
}

// In-place exclusive scan of data[0..n) by one block; returns the total.
__device__ int block_exclusive_scan(int* data, int n) {
  const int T = blockDim.x, tid = threadIdx.x;
  const int chunk = (n + T - 1) / T;
  const int lo = min(n, tid * chunk), hi = min(n, lo + chunk);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += data[i];
  int total;
  int run = block_scan_excl(s, &total);
  for (int i = lo; i < hi; ++i) {
    int v = data[i];
    data[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

// Largest i in [0, n) with a[i] <= x (a non-decreasing, a[0] <= x).
__device__ __forceinline__ int find_le(const int* a, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Row blocks whose tile offsets the schedule keeps in shared memory (the
// binary searches below then cost no global round trips); beyond this they
// stay in global memory.
constexpr int kSchedSmemRb = 49152;

__global__ void __launch_bounds__(1024) sched_kernel(SchedArgs a) {
  extern __shared__ int sched_smem[];
  const int tid = threadIdx.x, T = blockDim.x;
  const int R = a.R, W = a.W;
  const bool in_smem = R + 1 <= kSchedSmemRb;
  int* ts = in_smem ? sched_smem : a.s.tile_start;
  __shared__ int longest;
  if (tid == 0) longest = 0;
  __syncthreads();
  int my_longest = 0;
  for (int rb = tid; rb < R; rb += T) {
    ts[rb] = ceil_div(rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, a.err), a.tile);
    my_longest = max(my_longest, ts[rb]);
  }
  atomicMax(&longest, my_longest);
  __syncthreads();
  const int total = block_exclusive_scan(ts, R);
  if (tid == 0) ts[R] = total;
  __syncthreads();

  // One whole row block per worker when there are nearly as many row blocks
  // as workers (at least 7/8 of them) and none is more than 10% longer than
  // the mean: nothing is split, so there are no partial results to combine
  // and no worker changes query rows in mid-stream, which outweighs the at
  // most 1/7 more pages per busy worker.  Workers past R get nothing.
  if (R <= W && 8LL * R >= 7LL * W && 10LL * longest * R <= 11LL * total) {
    int* wseg = a.s.worker_seg;
    for (int w = tid; w <= W; w += T) wseg[w] = min(w, R);
    for (int rb = tid; rb < R; rb += T) {
      Seg g;
      g.rb = rb;
      g.t_lo = 0;
      g.t_hi = ts[rb + 1] - ts[rb];
      g.slot = -1;
      g.nkeys = rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, nullptr);
      g.pad[0] = g.pad[1] = g.pad[2] = 0;
      a.s.segs[rb] = g;
      a.s.rb_seg_first[rb] = rb;
    }
    if (tid == 0) {
      a.s.rb_seg_first[R] = R;
      a.s.split_rbs[0] = 0;
    }
    if (in_smem)
      for (int i = tid; i <= R; i += T) a.s.tile_start[i] = ts[i];
    return;
  }

  // Segment counts per worker.
  int* ws = a.s.worker_seg;
  for (int w = tid; w < W; w += T) {
    long long lo = (long long)w * total / W, hi = (long long)(w + 1) * total / W;
    int cnt = 0;
    if (hi > lo) cnt = find_le(ts, R, (int)(hi - 1)) - find_le(ts, R, (int)lo) + 1;
    ws[w] = cnt;
  }
  __syncthreads();
  const int nseg = block_exclusive_scan(ws, W);
  if (tid == 0) ws[W] = nseg;
  __syncthreads();

  for (int w = tid; w < W; w += T) {
    long long lo = (long long)w * total / W, hi = (long long)(w + 1) * total / W;
    if (hi <= lo) continue;
    int r0 = find_le(ts, R, (int)lo), r1 = find_le(ts, R, (int)(hi - 1));
    int s = ws[w];
    for (int rb = r0; rb <= r1; ++rb, ++s) {
      int a0 = max((int)lo, ts[rb]) - ts[rb];
      int a1 = min((int)hi, ts[rb + 1]) - ts[rb];
      bool whole = (a0 == 0 && a1 == ts[rb + 1] - ts[rb]);
      Seg g;
      g.rb = rb;
      g.t_lo = a0;
      g.t_hi = a1;
      g.slot = whole ? -1 : (rb == r0 ? 2 * w : 2 * w + 1);
      g.nkeys = rb_nkeys(a.kv_len, a.uniform_kv_len, a.n_q, a.max_kv_len, rb, nullptr);
      g.pad[0] = g.pad[1] = g.pad[2] = 0;
      a.s.segs[s] = g;
      if (a0 == 0) a.s.rb_seg_first[rb] = s;
    }
  }
  if (tid == 0) a.s.rb_seg_first[R] = nseg;
  if (in_smem)
    for (int i = tid; i <= R; i += T) a.s.tile_start[i] = ts[i];
  __syncthreads();

  // Row blocks with more than one segment, by their first segment (their
  // segments are consecutive in segs).  Such a row block starts with a
  // partial segment, which is the last segment of its worker; that worker
  // lists it (the order of the list does not affect any result).
  if (tid == 0) a.s.split_rbs[0] = 0;
  __syncthreads();
  for (int w = tid; w < W; w += T) {
    int s0 = ws[w], s1 = ws[w + 1];
    if (s1 > s0) {
      Seg g = a.s.segs[s1 - 1];
      if (g.slot >= 0 && g.t_lo == 0) a.s.split_rbs[1 + atomicAdd(&a.s.split_rbs[0], 1)] = s1 - 1;
    }
  }
}

}  // namespace mla
