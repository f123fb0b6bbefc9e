// Projection GEMMs on the sm_100a tensor cores, "weights as M":
//   D[col][tok] = sum_k W[col][k] * X[tok][k]        (fp32 in TMEM)
// i.e. y = W x for every token, with the weight rows filling the 128 rows of
// the MMA and the tokens (64 per tile in decode, 128 in prefill) as N.  Both
// operands are K-major and arrive by TMA with 128-byte swizzle; one elected
// lane issues tcgen05.mma (kind::f16, bf16 inputs).  The epilogue reads
// TMEM (thread r = weight row r) and hands adjacent column pairs, taken from
// neighbouring lanes, to the same functors as the CUDA-core GEMM (gemm.cuh).
// Split-K tiles write fp32 partials that a separate kernel sums in split
// order (deterministic) before the epilogue.
#pragma once
#include "gemm.cuh"
#include "sm100.cuh"

namespace mla {
namespace gemm_tc {
using namespace sm100;

constexpr int BM = 128;      // weight rows per tile
constexpr int BK = 64;       // K per stage (one 128-byte swizzle row)
constexpr int EPI_WARPS = 16;  // four per TMEM lane quarter, each draining a quarter of the tile's columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;  // warp 0: TMA producer; warp 1: TMEM + MMA issue; then the epilogue

struct Args {
  int Mw;                    // weight rows per batch entry (output columns)
  int Nt;                    // tokens
  int K;
  int splits, kchunk;        // kchunk is a multiple of BK
  int a_batch_rows;          // row offset of batch entry b in A = b * a_batch_rows
  int b_is_3d;               // B map has a per-batch (head) dimension
  float* partial;            // [batch][tiles_m][tiles_n][splits][BN][BM] when splits > 1
  int tiles_m, tiles_n, batch;
  // The weights (A) were not written by the kernel before this one, nor by
  // anything still running: the first STAGES stages' weight tiles are
  // requested before the programmatic wait.
  int pre_a;
};

template <int BN>
__host__ __device__ constexpr int stages() {
  return BN == 64 ? 8 : (BN == 128 ? 6 : 4);
}
// Per epilogue warp: 8 tokens x 32 rows of fp32, each token's row padded to
// 36 floats so that the transposed reads fall in different bank groups.
constexpr int EPI_PITCH = 36;
constexpr int EPI_STAGE_BYTES = EPI_WARPS * 8 * EPI_PITCH * 4;
template <int BN>
constexpr size_t smem_bytes() {
  return (size_t)stages<BN>() * (BM + BN) * BK * 2 + EPI_STAGE_BYTES + 1024 + 256;
}

// Persistent and warp-specialised: each CTA walks work items (weight tile,
// token tile, batch entry, K split) item = blockIdx.x, += gridDim.x.  The
// producer streams every item's K steps through an stages<BN>()-deep ring
// without stopping between items; the MMA warp accumulates item i into one
// of two TMEM accumulators while the epilogue warps drain the other, so a
// tile's epilogue overlaps the next tile's loads and MMAs.
template <int BN, class Epi>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const Args g, const Epi epi) {
  constexpr int STAGES = stages<BN>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE = A_BYTES + B_BYTES;
  float* epi_stage = reinterpret_cast<float*>(smem + STAGES * STAGE);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE + EPI_STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* drained = acc_empty + 2;     // every MMA this CTA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int per_z = g.tiles_m * g.tiles_n;
  const int items = per_z * g.batch * g.splits;
  // Weight tiles are walked from the last: when items outnumber CTAs, the
  // first round takes the high rows, which is where a projection keeps the
  // columns with the costlier epilogue (the rotated q_R of the query
  // projection), so that epilogue overlaps the CTA's next main loop.
  auto decode = [&](int item, int& bz, int& split, int& tm, int& tn) {
    const int z = item / per_z, rem = item - z * per_z;
    bz = z / g.splits;
    split = z - bz * g.splits;
    tm = g.tiles_m - 1 - rem % g.tiles_m;
    tn = rem / g.tiles_m;
  };
  auto ksteps = [&](int split) {
    const int k_begin = split * g.kchunk, k_end = min(g.K, k_begin + g.kchunk);
    return k_end > k_begin ? (k_end - k_begin + BK - 1) / BK : 0;
  };

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 32 * EPI_WARPS);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // The weight halves of the first stages go out while the previous kernel
  // finishes (every kernel here lets its successor launch only once it has
  // passed its own wait, so nothing older than the previous kernel is still
  // running, and that one does not write weights); the activation halves
  // follow the wait, completing the same barriers.
  uint32_t pre = 0;
  if (g.pre_a && warp == 0) {
    for (int item = blockIdx.x; item < items && pre < (uint32_t)STAGES; item += gridDim.x) {
      int bz, split, tm, tn;
      decode(item, bz, split, tm, tn);
      const int nk = ksteps(split);
      for (int kt = 0; kt < nk && pre < (uint32_t)STAGES; ++kt, ++pre) {
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[pre], STAGE);
          tma_load_2d(smem + pre * STAGE, &mapA, split * g.kchunk + kt * BK, bz * g.a_batch_rows + tm * BM,
                      &full[pre]);
        }
        __syncwarp();
      }
    }
  }
  pdl_wait();  // the activations (and the split-K scratch) come from the previous kernel
  pdl_trigger();

  if (warp == 0) {
    // TMA producer: runs ahead across items as far as the ring allows.
    uint32_t cnt = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
      int bz, split, tm, tn;
      decode(item, bz, split, tm, tn);
      const int nk = ksteps(split);
      for (int kt = 0; kt < nk; ++kt, ++cnt) {
        const int s = cnt % STAGES;
        const bool a_done = cnt < pre;  // weight half already requested before the wait
        if (!a_done && !(ok = mbar_wait_warp(&empty[s], ((cnt / STAGES) & 1) ^ 1, abort_flag, nullptr))) break;
        if (elect_one()) {
          const int k = split * g.kchunk + kt * BK;
          if (!a_done) {
            mbar_arrive_expect_tx(&full[s], STAGE);
            tma_load_2d(smem + s * STAGE, &mapA, k, bz * g.a_batch_rows + tm * BM, &full[s]);
          }
          if (g.b_is_3d) tma_load_3d(smem + s * STAGE + A_BYTES, &mapB, k, bz, tn * BN, &full[s]);
          else tma_load_2d(smem + s * STAGE + A_BYTES, &mapB, k, tn * BN, &full[s]);
        }
        __syncwarp();
      }
    }
    if (*abort_flag) {
      // Let every copy already issued land before the CTA can exit.
      for (uint32_t q = 0; q < (uint32_t)STAGES && q < cnt; ++q) {
        const uint32_t last = q + STAGES * ((cnt - 1 - q) / STAGES);
        mbar_wait_warp(&full[q], (last / STAGES) & 1, abort_flag, nullptr, 50000000ull, false);
      }
    }
  } else if (warp == 1) {
    // MMA issuer.
    const uint32_t idesc = idesc_bf16(BM, BN, 0, 0);
    const uint32_t s0 = smem_u32(smem);
    uint32_t cnt = 0, li = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++li) {
      int bz, split, tm, tn;
      decode(item, bz, split, tm, tn);
      const int nk = ksteps(split);
      const uint32_t acc = li & 1;
      if (!(ok = mbar_wait_warp(&acc_empty[acc], ((li >> 1) & 1) ^ 1, abort_flag, nullptr))) break;
      tc_fence_after();
      for (int kt = 0; kt < nk; ++kt, ++cnt) {
        const int s = cnt % STAGES;
        if (!(ok = mbar_wait_warp(&full[s], (cnt / STAGES) & 1, abort_flag, nullptr))) break;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a = s0 + s * STAGE, b = a + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_ss(tbase + acc * BN, sdesc_sw128(a + k * 32, 16, 1024), sdesc_sw128(b + k * 32, 16, 1024), idesc,
                   (kt | k) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&acc_full[acc]);
      __syncwarp();
    }
    // TMEM is freed only after the last MMA, even on an abandoned run.
    if (elect_one()) tc_commit(drained);
    __syncwarp();
    mbar_wait_warp(drained, 0, abort_flag, nullptr, 50000000ull, false);
  } else {
    // Epilogue (warps 2 .. 2 + EPI_WARPS - 1): thread r holds weight row
    // tm * BM + r of the item; a warp reaches the TMEM lanes of its quarter
    // and drains one quarter of the item's BN token columns, 8 at a time.
    // Each 32-row x 8-token block goes through shared memory so that lane l
    // ends up with 8 consecutive weight rows (output columns) of one token:
    // the functor then writes them as one 16-byte (bf16) or 32-byte (fp32)
    // vector.
    const int q = warp & 3, lane = tid & 31;
    const int part = (warp - 2) / 4, c_lo = part * (BN / 4), c_hi = c_lo + BN / 4;
    float* stg = epi_stage + (warp - 2) * (8 * EPI_PITCH);
    const int tj = lane >> 2, rg = (lane & 3) * 8;  // token and first row this lane stores
    uint32_t li = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++li) {
      int bz, split, tm, tn;
      decode(item, bz, split, tm, tn);
      const int nk = ksteps(split);
      const uint32_t acc = li & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (li >> 1) & 1, abort_flag, nullptr))) break;
      tc_fence_after();
      const uint32_t taddr = tbase + acc * BN + ((uint32_t)(q * 32) << 16);
      float* pdst = nullptr;
      if (g.splits > 1)
        pdst = g.partial + (((long long)bz * per_z + tm * g.tiles_n + tn) * g.splits + split) * (long long)(BN * BM);
      const int col0 = tm * BM + q * 32 + rg;  // first output column of this lane's 8
#pragma unroll 1
      for (int c0 = c_lo; c0 < c_hi; c0 += 8) {
        uint32_t v[8];
        if (nk > 0) {
          tmem_ld8(taddr + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) stg[j * EPI_PITCH + lane] = __uint_as_float(v[j]);
        __syncwarp();
        float o[8];
        {
          const float4 a0 = *reinterpret_cast<const float4*>(stg + tj * EPI_PITCH + rg);
          const float4 a1 = *reinterpret_cast<const float4*>(stg + tj * EPI_PITCH + rg + 4);
          o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
          o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
        }
        __syncwarp();  // the block is read before the next chunk overwrites it
        const int tok = tn * BN + c0 + tj;
        if (pdst) {
          float* d = pdst + (c0 + tj) * BM + q * 32 + rg;
          reinterpret_cast<float4*>(d)[0] = make_float4(o[0], o[1], o[2], o[3]);
          reinterpret_cast<float4*>(d)[1] = make_float4(o[4], o[5], o[6], o[7]);
        } else if (col0 < g.Mw && tok < g.Nt) {
          epi.store8(bz, tok, col0, o);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 2 * BN);
  }
}

// Sums the split-K partials of every tile in split order and runs the
// epilogue.  Grid: (2 * tiles_m, tiles_n * BN / 8, batch); block 256 = 8
// tokens x 32 lanes covering 64 weight rows, each lane one column pair of one
// token, with all of its split loads in flight.
constexpr int MAX_SPLITS = 32;
template <int BN, class Epi>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const Args g, const Epi epi) {
  pdl_wait();
  pdl_trigger();
  const int bz = blockIdx.z, slices = BN / 8;
  const int tile_m = blockIdx.x >> 1, half = blockIdx.x & 1;
  const int tile_n = blockIdx.y / slices, slice = blockIdx.y % slices;
  const int m0 = tile_m * BM, n0 = tile_n * BN;
  const float* base = g.partial + ((long long)bz * g.tiles_m * g.tiles_n + tile_m * g.tiles_n + tile_n) * g.splits *
                                      (long long)(BN * BM);
  const int tok_l = slice * 8 + threadIdx.x / 32;
  const int cp = (half * 32 + (threadIdx.x % 32)) * 2;
  float2 v[MAX_SPLITS];
#pragma unroll
  for (int s = 0; s < MAX_SPLITS; ++s)
    if (s < g.splits)
      v[s] = __ldcg(reinterpret_cast<const float2*>(base + (long long)s * (BN * BM) + tok_l * BM + cp));
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int s = 0; s < MAX_SPLITS; ++s)
    if (s < g.splits) {
      s0 += v[s].x;
      s1 += v[s].y;
    }
  const int tok = n0 + tok_l, col = m0 + cp;
  if (tok < g.Nt && col < g.Mw) epi(bz, tok, col, s0, s1);
}

}  // namespace gemm_tc
}  // namespace mla
