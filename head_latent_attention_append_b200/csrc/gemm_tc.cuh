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
constexpr int STAGES = 4;
constexpr int THREADS = 128;

struct Args {
  int Mw;                    // weight rows per batch entry (output columns)
  int Nt;                    // tokens
  int K;
  int splits, kchunk;        // kchunk is a multiple of BK
  int a_batch_rows;          // row offset of batch entry b in A = b * a_batch_rows
  int b_is_3d;               // B map has a per-batch (head) dimension
  float* partial;            // [batch][tiles_m][tiles_n][splits][BN][BM] when splits > 1
};

template <int BN>
constexpr size_t smem_bytes() {
  return (size_t)STAGES * (BM + BN) * BK * 2 + 1024 + 256;
}

template <int BN, class Epi>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const Args g, const Epi epi) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE = A_BYTES + B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int tiles_n = gridDim.y;
  const int bz = blockIdx.z / g.splits, split = blockIdx.z % g.splits;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  const int k_begin = split * g.kchunk;
  const int k_end = min(g.K, k_begin + g.kchunk);
  const int nk = k_end > k_begin ? (k_end - k_begin + BK - 1) / BK : 0;

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN < 32 ? 32 : BN);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // TMA producer.
    for (int kt = 0; kt < nk; ++kt) {
      const int s = kt % STAGES;
      if (!mbar_wait_warp(&empty[s], ((kt / STAGES) & 1) ^ 1, abort_flag, nullptr)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&full[s], STAGE);
        const int k = k_begin + kt * BK;
        tma_load_2d(smem + s * STAGE, &mapA, k, bz * g.a_batch_rows + m0, &full[s]);
        if (g.b_is_3d) tma_load_3d(smem + s * STAGE + A_BYTES, &mapB, k, bz, n0, &full[s]);
        else tma_load_2d(smem + s * STAGE + A_BYTES, &mapB, k, n0, &full[s]);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // MMA issuer.
    const uint32_t idesc = idesc_bf16(BM, BN, 0, 0);
    const uint32_t s0 = smem_u32(smem);
    for (int kt = 0; kt < nk; ++kt) {
      const int s = kt % STAGES;
      if (!mbar_wait_warp(&full[s], (kt / STAGES) & 1, abort_flag, nullptr)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t a = s0 + s * STAGE, b = a + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_ss(tbase, sdesc_sw128(a + k * 32, 16, 1024), sdesc_sw128(b + k * 32, 16, 1024), idesc,
                 (kt | k) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (elect_one()) tc_commit(done);
    __syncwarp();
  }

  // Epilogue (all four warps): thread r holds weight row m0 + r for the BN
  // tokens of the tile.
  mbar_wait(done, 0, abort_flag, nullptr, 2000000000ull, false);
  __syncwarp();
  tc_fence_after();
  const int r = tid;
  const uint32_t taddr = tbase + ((uint32_t)(warp * 32) << 16);
  const int col = m0 + r;
  const int ntiles = gridDim.x * tiles_n;
  float* part = nullptr;
  if (g.splits > 1)
    part = g.partial + (((long long)bz * ntiles + blockIdx.x * tiles_n + blockIdx.y) * g.splits + split) *
                           (long long)(BN * BM);
  // Eight token columns at a time (a short body keeps the functor's code
  // small enough for the instruction cache).
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 8) {
    uint32_t v[8];
    if (nk > 0) {
      tmem_ld8(taddr + c0, v);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0u;
    }
    if (part) {
#pragma unroll
      for (int j = 0; j < 8; ++j) __stcg(part + (c0 + j) * BM + r, __uint_as_float(v[j]));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float mine = __uint_as_float(v[j]);
        const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
        const int tok = n0 + c0 + j;
        if ((r & 1) == 0 && col < g.Mw && tok < g.Nt) epi(bz, tok, col, mine, other);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, BN < 32 ? 32 : BN);
  }
}

// Sums the split-K partials of every tile in split order and runs the
// epilogue.  Grid: (tiles_m, tiles_n * BN / 8, batch); block 256 = 8 tokens x
// 32 lanes; each thread owns two column pairs of one token and keeps all of
// their split loads in flight.
constexpr int MAX_SPLITS = 8;
template <int BN, class Epi>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const Args g, const Epi epi) {
  const int bz = blockIdx.z, slices = BN / 8;
  const int tile_n = blockIdx.y / slices, slice = blockIdx.y % slices;
  const int tiles_n = gridDim.y / slices, ntiles = gridDim.x * tiles_n;
  const int m0 = blockIdx.x * BM, n0 = tile_n * BN;
  const float* base =
      g.partial + ((long long)bz * ntiles + blockIdx.x * tiles_n + tile_n) * g.splits * (long long)(BN * BM);
  const int tok_l = slice * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int cp = (half * 32 + lane) * 2;
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
}

}  // namespace gemm_tc
}  // namespace mla
