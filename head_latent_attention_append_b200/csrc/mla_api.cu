// libmla C ABI: argument checks, workspace layout and launch sequencing.
// Every step of the path runs in this library's kernels; the host code only
// validates, carves the caller's workspace and launches on the caller's
// stream.
#include "../../include/mla.h"

#include <limits.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <cstring>
#include <mutex>
#include <utility>

#include <cudaTypedefs.h>

#include "attn_mha.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "cp.cuh"
#include "gemm.cuh"
#include "gemm_tc.cuh"
#include "prep.cuh"
#include "sched.cuh"

using namespace mla;

struct mla_weights {
  mla_dims d;
  float scale;         // softmax scale actually used
  size_t esz;          // element size of the path (4 or 2)
  void* dkr;           // [d_cr][d_model]: W_DKV then W_KR (d_r rows, or n_h * d_r per head)
  void* dq;            // [d_cq][d_model] or null
  void* uqr;           // [n_h*(d_h + d_r)][d_in]
  void* ukt;           // [n_h][d_c][d_h]
  void* uk;            // [n_h*d_h][d_c] (as given: the materialised prefill expands K_C with it)
  void* uv;            // [n_h*d_v][d_c]
  double theta[32];    // RoPE frequencies, theta_i = base^(-2i/d_r)
};

namespace {

thread_local int g_launches = 0;

// Event pairs bracketing the attention kernel while profiling is on.
struct Profiler {
  bool on = false;
  int cap = 0, used = 0;
  cudaEvent_t* ev = nullptr;  // 2 * cap
};
thread_local Profiler g_prof;

void prof_mark(cudaStream_t st, bool start) {
  if (!g_prof.on || g_prof.used >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.used + (start ? 0 : 1)], st);
  if (!start) ++g_prof.used;
}

constexpr int kWorkerSlots = 296;        // partial-slot capacity: 2 * kWorkerSlots
constexpr int kSplitKTileSplits = 1024;  // split-K scratch: tiles * splits <= this
constexpr int kCounterCap = 1024;
constexpr int kSideTileSplits = 1024;    // split-K scratch of the side-stream append (tiles * splits): as the main one's
constexpr int kSideAppendCtas = 32;      // CTAs of the side-stream append GEMM
constexpr double kLog2e = 1.4426950408889634074;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms() {
  static thread_local int cached_dev = -1, cached_n = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cached_n;
  if (dev != cached_dev) {
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached_n = n > 0 ? n : 148;
    cached_dev = dev;
  }
  return cached_n;
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device), so
// later calls, including ones made during CUDA graph capture, skip it.
template <class F>
cudaError_t set_smem_once(F* fn, size_t bytes) {
  struct Entry {
    const void* fn;
    unsigned long long devices;
  };
  static std::mutex mu;
  static Entry table[64];
  static int used = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  std::lock_guard<std::mutex> lock(mu);
  Entry* ent = nullptr;
  for (int i = 0; i < used; ++i)
    if (table[i].fn == reinterpret_cast<const void*>(fn)) ent = &table[i];
  if (ent && (ent->devices & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (!ent && used < 64) ent = &table[used++];
  if (ent) {
    ent->fn = reinterpret_cast<const void*>(fn);
    ent->devices |= bit;
  }
  return cudaSuccess;
}

// Cache row width: the latent, then one shared RoPE key or one per head.
int cache_row(const mla_dims& d) { return d.d_c + (d.rope_key_per_head ? d.n_h : 1) * d.d_r; }

// Rows of a cache row that the CUDA-core attention kernel stages per key
// (shared memory: 32 keys plus up to 16 heads' queries, fp32).
constexpr int kSimtMaxRow = 1024;

// A second stream of the library's own for work that depends only on the
// call's inputs and can run beside the main chain (the attention schedule,
// which needs only the lengths, runs beside the query projections).  One
// non-blocking stream and two timing-free events per host thread and device,
// created on first use and kept until the thread exits.  The fork/join
// through the events is ordinary stream ordering, so it also holds inside a
// CUDA graph capture of the caller's stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
cudaError_t side_stream(SideStream** out) {
  static thread_local SideStream table[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  SideStream& t = table[dev];
  if (!t.s) {
    if ((e = cudaStreamCreateWithFlags(&t.s, cudaStreamNonBlocking))) return e;
    if ((e = cudaEventCreateWithFlags(&t.fork, cudaEventDisableTiming))) return e;
    if ((e = cudaEventCreateWithFlags(&t.join, cudaEventDisableTiming))) return e;
  }
  *out = &t;
  return cudaSuccess;
}

mla_status check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->rope_key_per_head != 0 && d->rope_key_per_head != 1) return MLA_ERR_INVALID_ARG;
  if (d->n_h <= 0 || d->d_h <= 0 || d->d_v <= 0 || d->d_c <= 0 || d->d_r <= 0 || d->d_model <= 0 ||
      d->d_cq < 0 || d->page_size <= 0 || !(d->rope_base > 0.f) || d->softmax_scale < 0.f)
    return MLA_ERR_INVALID_ARG;
  if (d->dtype != MLA_F32 && d->dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  if (d->d_r % 2 != 0 || d->d_r > 64) return MLA_ERR_UNSUPPORTED;
  if (d->page_size != 64) return MLA_ERR_UNSUPPORTED;
  if (d->n_h > 128) return MLA_ERR_UNSUPPORTED;
  if (d->dtype == MLA_BF16) {
    // 16-byte row alignment for the tensor-core loads; the latent splits into
    // two halves of whole 64-column chunks; a cache row is at most nine chunks.
    if (d->d_h % 8 || d->d_v % 8 || d->d_c % 128 || d->d_r % 16 || d->d_model % 8 || d->d_cq % 8)
      return MLA_ERR_UNSUPPORTED;
    if (d->d_c > 512 || (!d->rope_key_per_head && d->d_c + d->d_r > 576)) return MLA_ERR_UNSUPPORTED;
  } else {
    if (d->d_c > 512) return MLA_ERR_UNSUPPORTED;
  }
  // Per-head RoPE keys run on the CUDA-core attention kernel, which stages
  // whole cache rows.
  if (d->rope_key_per_head && cache_row(*d) > kSimtMaxRow) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

size_t esize(const mla_dims& d) { return d.dtype == MLA_BF16 ? 2 : 4; }
int d_in(const mla_dims& d) { return d.d_cq > 0 ? d.d_cq : d.d_model; }

struct WeightLayout {
  size_t dkr, dq, uqr, ukt, uk, uv, total;
};
WeightLayout weight_layout(const mla_dims& d) {
  const size_t e = esize(d);
  WeightLayout L{};
  size_t o = 0;
  L.dkr = o; o = align_up(o + e * (size_t)cache_row(d) * d.d_model, 256);
  L.dq = o;  o = align_up(o + e * (size_t)d.d_cq * d.d_model, 256);
  L.uqr = o; o = align_up(o + e * (size_t)d.n_h * (d.d_h + d.d_r) * d_in(d), 256);
  L.ukt = o; o = align_up(o + e * (size_t)d.n_h * d.d_c * d.d_h, 256);
  L.uk = o;  o = align_up(o + e * (size_t)d.n_h * d.d_h * d.d_c, 256);
  L.uv = o;  o = align_up(o + e * (size_t)d.n_h * d.d_v * d.d_c, 256);
  L.total = o;
  return L;
}

// Workspace layout shared by the size queries and the calls.
struct Plan {
  size_t hdr, counters, arrive, partial, cq, qc, qabs, tile_start, worker_seg, segs, rb_first, split_rbs,
      part_o, part_ml, obar, side_partial, total;
  int R, qrows;
};
// cp: context-parallel partials, where every segment (at most W + R) has its
// own partial slot.
// side_append: the split-K scratch of an append GEMM that runs on the side
// stream beside the query projections (a decode step).
Plan make_plan(const mla_dims& d, int R, bool attention, bool cp = false, bool side_append = false) {
  const size_t e = esize(d);
  Plan P{};
  P.R = R;
  P.qrows = (d.dtype == MLA_BF16) ? 128 : d.n_h;
  const int W = kWorkerSlots;
  const size_t slots = cp ? std::max<size_t>(2 * (size_t)W, (size_t)W + R) : 2 * (size_t)W;
  size_t o = 0;
  P.hdr = o;        o = align_up(o + 256, 256);
  P.counters = o;   o = align_up(o + sizeof(int) * kCounterCap, 256);
  // Arrival counters of split row blocks per CTA rank, zeroed with the
  // header and the split-K counters at the start of every call.
  P.arrive = o;     o = align_up(o + sizeof(int) * (attention ? 2 * (size_t)R : 0), 256);
  P.partial = o;    o = align_up(o + sizeof(float) * (size_t)kSplitKTileSplits * 64 * 64, 256);
  if (attention) {
    P.cq = o;         o = align_up(o + e * (size_t)R * d.d_cq, 256);
    P.qc = o;         o = align_up(o + e * (size_t)R * d.n_h * d.d_h, 256);
    P.qabs = o;       o = align_up(o + e * (size_t)R * P.qrows * (d.d_c + d.d_r), 256);
    P.tile_start = o; o = align_up(o + sizeof(int) * (size_t)(R + 1), 256);
    P.worker_seg = o; o = align_up(o + sizeof(int) * (size_t)(W + 1), 256);
    P.segs = o;       o = align_up(o + sizeof(Seg) * (size_t)(W + R), 256);
    P.rb_first = o;   o = align_up(o + sizeof(int) * (size_t)(R + 1), 256);
    P.split_rbs = o;  o = align_up(o + sizeof(int) * (size_t)(2 * W + 1), 256);
    P.part_o = o;     o = align_up(o + e * slots * d.n_h * d.d_c, 256);
    P.part_ml = o;    o = align_up(o + sizeof(float) * slots * 2 * d.n_h * 2, 256);
    P.obar = o;       o = align_up(o + e * (size_t)R * d.n_h * d.d_c, 256);
  }
  if (side_append) {
    P.side_partial = o; o = align_up(o + sizeof(float) * (size_t)kSideTileSplits * 64 * 64, 256);
  }
  P.total = o;
  return P;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

mla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Launches `kernel` with programmatic stream serialization: it may begin
// while the previous kernel in the stream is finishing, and waits for it
// (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}


// The tensor-core attention kernel for a latent width of 128 * NPV.
template <int NPV>
cudaError_t launch_attn_tc(const CUtensorMap& mapS, const CUtensorMap& mapV, const AttnArgs& aa, int W,
                           cudaStream_t st) {
  auto kfn = attn_tc::attn_tc_kernel<NPV>;
  cudaError_t e = set_smem_once(kfn, attn_tc::SMEM_BYTES);
  if (e) return e;
  return launch_pdl(kfn, dim3(2 * W), dim3(attn_tc::THREADS), attn_tc::SMEM_BYTES, st, mapS, mapV, aa);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda at build time).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Every map here is a bf16 tensor of rank 2 or 3, 128-byte swizzle, no
// interleave, 256-byte L2 promotion, zero fill; it is a pure function of
// (base, dims, byte strides, box).  The last kMapCache encodings of this host
// thread are kept, so a steady stream of calls on the same buffers does not
// re-encode its dozen maps every step.
constexpr int kMapCache = 32;
struct MapKey {
  const void* base;
  int rank;
  cuuint64_t dim[3], stride[2];
  cuuint32_t box[3];
  bool operator==(const MapKey& o) const {
    return base == o.base && rank == o.rank && std::memcmp(dim, o.dim, sizeof dim) == 0 &&
           std::memcmp(stride, o.stride, sizeof stride) == 0 && std::memcmp(box, o.box, sizeof box) == 0;
  }
};
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  int used = 0, next = 0;
};
thread_local MapCache g_maps;

bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dim, const cuuint64_t* stride,
                 const cuuint32_t* box) {
  MapKey k{};
  k.base = base;
  k.rank = rank;
  for (int i = 0; i < rank; ++i) {
    k.dim[i] = dim[i];
    k.box[i] = box[i];
    if (i + 1 < rank) k.stride[i] = stride[i];
  }
  for (int i = 0; i < g_maps.used; ++i)
    if (g_maps.key[i] == k) {
      *map = g_maps.map[i];
      return true;
    }
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  if (fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), k.dim, k.stride, k.box,
         es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = g_maps.next;
  g_maps.key[slot] = k;
  g_maps.map[slot] = *map;
  g_maps.next = (slot + 1) % kMapCache;
  if (g_maps.used < kMapCache) ++g_maps.used;
  return true;
}

// The cache as a 2-D tensor [rows = num_pages * 64][d_cr] bf16, read in boxes
// of 64 columns x `box_rows` rows with 128-byte swizzle.  Columns past d_cr
// read as zero (the RoPE chunk of a row narrower than 64 columns).
bool encode_cache_map(CUtensorMap* map, const void* cache, int d_cr, long long rows, int box_rows) {
  cuuint64_t gdim[2] = {(cuuint64_t)d_cr, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)d_cr * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  return encode_bf16(map, cache, 2, gdim, gstride, box);
}

// bf16 tensor maps with 128-byte swizzle for the projection GEMMs.
bool encode_bf16_2d(CUtensorMap* map, const void* base, long long dim0, long long dim1, long long stride1_elems,
                    int box0, int box1) {
  cuuint64_t gdim[2] = {(cuuint64_t)dim0, (cuuint64_t)dim1};
  cuuint64_t gstride[1] = {(cuuint64_t)stride1_elems * 2};
  cuuint32_t box[2] = {(cuuint32_t)box0, (cuuint32_t)box1};
  return encode_bf16(map, base, 2, gdim, gstride, box);
}
bool encode_bf16_3d(CUtensorMap* map, const void* base, long long dim0, long long dim1, long long dim2,
                    long long stride1_elems, long long stride2_elems, int box0, int box1, int box2) {
  cuuint64_t gdim[3] = {(cuuint64_t)dim0, (cuuint64_t)dim1, (cuuint64_t)dim2};
  cuuint64_t gstride[2] = {(cuuint64_t)stride1_elems * 2, (cuuint64_t)stride2_elems * 2};
  cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)box1, (cuuint32_t)box2};
  return encode_bf16(map, base, 3, gdim, gstride, box);
}

// tcgen05 projection GEMM: C[b][m][n] = sum_k A[b][m][k] * B[b][n][k] with A
// the activations (m = token) and B the weights (n = output column); the
// kernel runs it as D = W X^T (weights as the MMA's M).  `partial_floats`
// bounds the split-K scratch.
template <int BN, class Epi>
cudaError_t gemm_tc_launch(const void* A, long long lda, long long sA, const void* B, long long ldb, long long sB,
                           int M, int N, int K, int batch, const Epi& epi, float* partial, long long partial_floats,
                           cudaStream_t st, int max_ctas, bool pre_a) {
  CUtensorMap mapW, mapX;
  // Weights: batches are contiguous row blocks of N rows.
  if (batch > 1 && sB != (long long)N * ldb) return cudaErrorInvalidValue;
  if (!encode_bf16_2d(&mapW, B, K, (long long)batch * N, ldb, gemm_tc::BK, gemm_tc::BM)) return cudaErrorInvalidValue;
  const bool x3d = batch > 1;
  if (x3d) {
    if (!encode_bf16_3d(&mapX, A, K, batch, M, sA, lda, gemm_tc::BK, 1, BN)) return cudaErrorInvalidValue;
  } else if (!encode_bf16_2d(&mapX, A, K, M, lda, gemm_tc::BK, BN)) {
    return cudaErrorInvalidValue;
  }
  const int tm = ceil_div(N, gemm_tc::BM), tn = ceil_div(M, BN), tiles = tm * tn * batch;
  const int nk = ceil_div(K, gemm_tc::BK);
  // Few output tiles (decode): split K so that every SM streams weights in a
  // single round (one work item per SM; two per SM measured 1-2 us slower
  // on the decode step); the reduce kernel sums the splits in order and runs
  // the epilogue.
  int splits = 1;
  // The split count depends on the GPU, not on `max_ctas`, so a GEMM capped
  // to a few CTAs (the side-stream append) sums its partials exactly as the
  // uncapped one does: the same cache rows, bit for bit.
  const int sms = std::min(num_sms(), max_ctas);
  if (2 * tiles < num_sms())
    splits = std::min(std::min(gemm_tc::MAX_SPLITS, nk), std::max(1, num_sms() / tiles));
  while (splits > 1 && (long long)tiles * splits * BN * gemm_tc::BM > partial_floats) --splits;
  const int kchunk = ceil_div(nk, splits) * gemm_tc::BK;
  splits = ceil_div(K, kchunk);
  gemm_tc::Args g{N, M, K, splits, kchunk, N, x3d ? 1 : 0, partial, tm, tn, batch, pre_a ? 1 : 0};
  const size_t smem = gemm_tc::smem_bytes<BN>();
  auto kfn = gemm_tc::gemm_tc_kernel<BN, Epi>;
  cudaError_t e = set_smem_once(kfn, smem);
  if (e != cudaSuccess) return e;
  ++g_launches;
  const int items = tiles * splits;
  if ((e = launch_pdl(kfn, dim3(std::min(items, sms)), dim3(gemm_tc::THREADS), smem, st, mapW, mapX, g, epi)))
    return e;
  if (splits > 1) {
    ++g_launches;
    e = launch_pdl(gemm_tc::splitk_reduce_kernel<BN, Epi>, dim3(2 * tm, tn * (BN / 8), batch), dim3(256), 0, st,
                   g, epi);
  }
  return e;
}

// ----------------------------------------------------------- GEMM launcher
template <class Epi>
cudaError_t gemm_simt(const void* A, long long lda, long long sA, const void* B, long long ldb, long long sB, int M,
                      int N, int K, int batch, const Epi& epi, void* ws, const Plan& P, cudaStream_t st,
                      int tile_split_cap);

// `max_ctas` caps the CTAs of the tensor-core GEMM (a GEMM sharing the GPU
// with another stream's).  `pre_a`: the kernel before this one in the stream
// is one of this call's own (which writes no weights), so the GEMM may
// request its first weight tiles before its programmatic wait.
template <typename T, class Epi>
cudaError_t gemm(const void* A, long long lda, long long sA, const void* B, long long ldb, long long sB,
                 int M, int N, int K, int batch, const Epi& epi, void* ws, const Plan& P,
                 cudaStream_t st, int tile_split_cap = kSplitKTileSplits, int max_ctas = INT_MAX,
                 bool pre_a = false) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if constexpr (sizeof(T) == 2) {
    const long long cap = (long long)tile_split_cap * 64 * 64;
    if (M <= 512)
      return gemm_tc_launch<64>(A, lda, sA, B, ldb, sB, M, N, K, batch, epi, at<float>(ws, P.partial), cap, st,
                                max_ctas, pre_a);
    if (M < 4096)
      return gemm_tc_launch<128>(A, lda, sA, B, ldb, sB, M, N, K, batch, epi, at<float>(ws, P.partial), cap, st,
                                 max_ctas, pre_a);
    // Many tokens (prefill): 256-token tiles, so each 48 KB stage (weights
    // 16 KB, tokens 32 KB) feeds twice the tensor work of a 128-token one.
    return gemm_tc_launch<256>(A, lda, sA, B, ldb, sB, M, N, K, batch, epi, at<float>(ws, P.partial), cap, st,
                               max_ctas, pre_a);
  } else {
    return gemm_simt(A, lda, sA, B, ldb, sB, M, N, K, batch, epi, ws, P, st, tile_split_cap);
  }
}

// fp32 CUDA-core GEMM (the fp32 path).
template <class Epi>
cudaError_t gemm_simt(const void* A, long long lda, long long sA, const void* B, long long ldb, long long sB, int M,
                      int N, int K, int batch, const Epi& epi, void* ws, const Plan& P, cudaStream_t st,
                      int tile_split_cap) {
  GemmArgs a{};
  a.A = A; a.lda = lda; a.strideA = sA;
  a.B = B; a.ldb = ldb; a.strideB = sB;
  a.M = M; a.N = N; a.K = K; a.batch = batch;
  const int tm = ceil_div(M, 64), tn = ceil_div(N, 64), tiles = tm * tn * batch;
  int splits = 1;
  const int want = num_sms();
  if (tiles < want && tiles <= kCounterCap) {
    splits = ceil_div(want, tiles);
    splits = std::min(splits, std::max(1, K / 256));
    splits = std::min(splits, tile_split_cap / tiles);
    splits = std::max(splits, 1);
  }
  int kchunk = ceil_div(ceil_div(K, splits), 32) * 32;
  splits = ceil_div(K, kchunk);
  a.splits = splits;
  a.kchunk = kchunk;
  a.partial = at<float>(ws, P.partial);
  a.counters = at<int>(ws, P.counters);
  dim3 grid(tn, tm, batch * splits);
  ++g_launches;
  gemm_f32::gemm_f32_kernel<Epi><<<grid, gemm_f32::THREADS, 0, st>>>(a, epi);
  return cudaGetLastError();
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------- pipelines
// kv_len (decode step): token m is new token m % n_q of sequence m / n_q, at
// position kv_len[b] - n_q + q.
template <typename T>
mla_status append_impl(const mla_weights* w, const void* h, const int32_t* seq_idx, const int32_t* pos,
                       int prefill_S, int n_seq, const int32_t* page_table, int max_pages, int num_pages,
                       void* cache, int T_, void* ws, const Plan& P, cudaStream_t st,
                       const int32_t* kv_len = nullptr, int n_q = 0, int tile_split_cap = kSplitKTileSplits,
                       int max_ctas = INT_MAX) {
  const mla_dims& d = w->d;
  EpiAppend<T> epi{};
  epi.cache = static_cast<T*>(cache);
  epi.seq_idx = seq_idx;
  epi.pos = pos;
  epi.prefill_S = prefill_S;
  epi.kv_len = kv_len;
  epi.n_q = n_q;
  epi.page_table = page_table;
  for (int i = 0; i < d.d_r / 2; ++i) epi.theta[i] = w->theta[i];
  epi.max_pages = max_pages;
  epi.num_pages = num_pages;
  epi.page_size = d.page_size;
  epi.d_c = d.d_c;
  epi.d_cr = cache_row(d);
  epi.d_r = d.d_r;
  epi.n_seq = n_seq;
  epi.err = at<int>(ws, P.hdr);
  return cuda_status(gemm<T>(h, d.d_model, 0, w->dkr, d.d_model, 0, T_, cache_row(d), d.d_model, 1, epi,
                             ws, P, st, tile_split_cap, max_ctas));
}

// Context-parallel partial: the rank's window and where its (obar_r, lse_r)
// go instead of the W_UV projection.
struct CpOut {
  CpWindow win;
  void* obar;  // [R][n_h][d_c], type of the path
  float* lse;  // [R][n_h]
};

// A decode step's append, run on the side stream beside the query
// projections: the new tokens' rows (h, one per row block) into `cache`.
struct SideAppend {
  void* cache;
  int n_seq;
};

template <typename T>
mla_status attend_impl(const mla_weights* w, const void* hq, const int32_t* kv_len, int uniform_kv_len,
                       int n_q, int prefill_S, const int32_t* page_table, int max_pages, int num_pages,
                       const void* cache, float* out, int R, int max_kv_len, void* ws, const Plan& P,
                       cudaStream_t st, const CpOut* cp = nullptr, const SideAppend* side_append = nullptr) {
  const mla_dims& d = w->d;
  const int q_row = d.d_c + d.d_r;  // a Q_abs row: [q~ | q_R]
  const int d_cr = cache_row(d);    // a cache row: [c | k_R] (one key or n_h)
  const int din = d_in(d);
  int* err = at<int>(ws, P.hdr);
  cudaError_t e;
  // (0) the attention schedule, on the side stream: it depends only on the
  // lengths, so it runs while the query projections below stream weights
  // (one 512-thread CTA, small enough to sit on an SM beside a GEMM CTA).
  SideStream* side = nullptr;
  if ((e = side_stream(&side))) return cuda_status(e);
  Sched S{at<int>(ws, P.tile_start), at<int>(ws, P.worker_seg), at<Seg>(ws, P.segs), at<int>(ws, P.rb_first),
          at<int>(ws, P.split_rbs)};
  AttnArgs aa{};
  aa.qabs = at<T>(ws, P.qabs);
  aa.qrows = P.qrows;
  aa.cache = cache;
  aa.page_table = page_table;
  aa.max_pages = max_pages;
  aa.num_pages = num_pages;
  aa.page_size = d.page_size;
  aa.n_h = d.n_h; aa.d_c = d.d_c; aa.d_r = d.d_r; aa.d_cr = d_cr;
  aa.q_row = q_row;
  aa.rope_per_head = d.rope_key_per_head;
  aa.kv_len = kv_len; aa.uniform_kv_len = uniform_kv_len; aa.n_q = n_q; aa.max_kv_len = max_kv_len;
  aa.sched = S;
  aa.part_o = at<T>(ws, P.part_o);
  aa.part_ml = at<float>(ws, P.part_ml);
  aa.obar = at<T>(ws, P.obar);
  aa.err = err;

  // bf16 with one shared RoPE key runs on the tensor cores; per-head RoPE
  // keys (whose position term is a per-head contraction, not one dense
  // product over the shared row) and fp32 run on the CUDA cores.
  const bool kTensorCores = sizeof(T) == 2 && !d.rope_key_per_head;
  // fp32: heads per CTA a power of two so that 256 threads split evenly.
  int HG = 16;
  while (HG > d.n_h) HG >>= 1;
  const int G = kTensorCores ? 2 : ceil_div(d.n_h, HG);
  // bf16: one CTA pair per two SMs (one CTA per SM; all of TMEM each).
  // CUDA-core kernel: one CTA per SM and head group (its registers and the
  // staged rows fill an SM), so every worker runs in a single round.
  int W = kTensorCores ? std::max(1, std::min(kWorkerSlots, num_sms() / 2))
                       : std::max(1, std::min(kWorkerSlots, num_sms() / G));
  // bf16 without context parallelism, with at least half as many row blocks
  // as workers (so a split row block has two or three pieces): the attention
  // kernel merges split row blocks itself (a row block has at most one piece
  // per worker), and no combine kernel runs.  With fewer row blocks each has
  // many pieces, all ending together, and the combine kernel spreads their
  // merge over every SM instead.
  const bool self_merge = kTensorCores && !cp && W <= attn_tc::MAX_PIECES && 2 * R >= W;
  if (self_merge) aa.arrive = at<int>(ws, P.arrive);
  {
    SchedArgs sa{kv_len, uniform_kv_len, n_q, R, W, d.page_size, max_kv_len, S, err};
    ++g_launches;
    if ((e = cudaEventRecord(side->fork, st)) || (e = cudaStreamWaitEvent(side->s, side->fork, 0)))
      return cuda_status(e);
    if (cp) {
      cp_sched_kernel<<<1, 512, 0, side->s>>>(sa, cp->win);
    } else {
      const size_t sched_smem = R + 1 <= kSchedSmemRb ? sizeof(int) * (size_t)(R + 1) : 0;
      if ((e = set_smem_once(sched_kernel, sizeof(int) * (size_t)kSchedSmemRb))) return cuda_status(e);
      sched_kernel<<<1, 512, sched_smem, side->s>>>(sa);
    }
    if ((e = cudaGetLastError())) return cuda_status(e);
    if (side_append) {
      // The append GEMM on a share of the SMs, with its own split-K scratch
      // (the query projections' splits use P.partial at the same time).
      Plan Ps = P;
      Ps.partial = P.side_partial;
      const mla_status s = append_impl<T>(w, hq, nullptr, nullptr, 0, side_append->n_seq, page_table, max_pages,
                                          num_pages, side_append->cache, R, ws, Ps, side->s, kv_len, n_q,
                                          kSideTileSplits, kSideAppendCtas);
      if (s != MLA_OK) return s;
    }
    if ((e = cudaEventRecord(side->join, side->s))) return cuda_status(e);
  }
  // (1) query latent.
  const void* src = hq;
  if (d.d_cq > 0) {
    EpiStore<T> epi{at<T>(ws, P.cq), d.d_cq, 0, 1.f};
    if ((e = gemm<T>(hq, d.d_model, 0, w->dq, d.d_model, 0, R, d.d_cq, d.d_model, 1, epi, ws, P, st)))
      return cuda_status(e);
    src = at<T>(ws, P.cq);
  }
  // (2) q_C and rotated, scaled q_R.
  const float qscale = (float)((double)w->scale * kLog2e);
  {
    EpiQProj<T> epi{};
    epi.qc = at<T>(ws, P.qc);
    epi.qabs = at<T>(ws, P.qabs);
    epi.kv_len = kv_len;
    epi.uniform_kv_len = uniform_kv_len;
    for (int i = 0; i < d.d_r / 2; ++i) epi.theta[i] = w->theta[i];
    epi.n_h = d.n_h; epi.d_h = d.d_h; epi.d_r = d.d_r; epi.d_c = d.d_c; epi.d_cr = q_row;
    epi.qabs_rows = P.qrows; epi.n_q = n_q; epi.prefill_S = prefill_S;
    epi.qr_scale = qscale;
    if ((e = gemm<T>(src, din, 0, w->uqr, din, 0, R, d.n_h * (d.d_h + d.d_r), din, 1, epi, ws, P, st,
                     kSplitKTileSplits, INT_MAX, d.d_cq > 0)))
      return cuda_status(e);
  }
  // (3) absorption q~_h = W_UK,h^T q_C,h, scaled.
  {
    EpiStore<T> epi{at<T>(ws, P.qabs), (long long)P.qrows * q_row, q_row, qscale};
    if ((e = gemm<T>(at<T>(ws, P.qc), (long long)d.n_h * d.d_h, d.d_h, w->ukt, d.d_h, (long long)d.d_c * d.d_h,
                     R, d.d_c, d.d_h, d.n_h, epi, ws, P, st, kSplitKTileSplits, INT_MAX, true)))
      return cuda_status(e);
  }
  // The schedule has run on the side stream beside steps (1) - (3).
  if ((e = cudaStreamWaitEvent(st, side->join, 0))) return cuda_status(e);
  // (5) attention on the latent cache, (6) combine of split row blocks.
  if (kTensorCores) {
    // Score ring: 32-row boxes (one CTA's keys of a page); latent ring:
    // 64-row boxes.
    CUtensorMap mapS, mapV;
    const long long rows = (long long)num_pages * d.page_size;
    if (!encode_cache_map(&mapS, cache, d_cr, rows, 32) || !encode_cache_map(&mapV, cache, d_cr, rows, 64))
      return MLA_ERR_CUDA;
    ++g_launches;
    prof_mark(st, true);
    switch (d.d_c / 128) {
      case 1: e = launch_attn_tc<1>(mapS, mapV, aa, W, st); break;
      case 2: e = launch_attn_tc<2>(mapS, mapV, aa, W, st); break;
      case 3: e = launch_attn_tc<3>(mapS, mapV, aa, W, st); break;
      default: e = launch_attn_tc<4>(mapS, mapV, aa, W, st); break;
    }
    if (e) return cuda_status(e);
    prof_mark(st, false);
    if ((e = cudaGetLastError())) return cuda_status(e);
  } else {
    size_t sm = attn_simt::smem_bytes(HG, d_cr);
    auto kfn = attn_simt::attn_simt_kernel<T>;
    if ((e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)))
      return cuda_status(e);  // fp32 path: size depends on the head group
    ++g_launches;
    prof_mark(st, true);
    kfn<<<dim3(W, G), attn_simt::THREADS, sm, st>>>(aa, HG);
    prof_mark(st, false);
    if ((e = cudaGetLastError())) return cuda_status(e);
  }
  if (cp) {
    ++g_launches;
    cp_combine_kernel<T><<<dim3(R, ceil_div(d.n_h, 8)), 256, 0, st>>>(aa, static_cast<T*>(cp->obar), cp->lse);
    return cuda_status(cudaGetLastError());
  }
  if (!self_merge) {
    ++g_launches;
    if ((e = launch_pdl(combine_kernel<T>, dim3(2 * W, ceil_div(d.n_h, 8)), dim3(256), 0, st, aa)))
      return cuda_status(e);
    if ((e = cudaGetLastError())) return cuda_status(e);
  }
  // (7) o_h = W_UV,h obar_h.
  {
    EpiStore<float> epi{out, (long long)d.n_h * d.d_v, d.d_v, 1.f};
    if ((e = gemm<T>(at<T>(ws, P.obar), (long long)d.n_h * d.d_c, d.d_c, w->uv, d.d_c, (long long)d.d_v * d.d_c,
                     R, d.d_v, d.d_c, d.n_h, epi, ws, P, st, kSplitKTileSplits, INT_MAX, true)))
      return cuda_status(e);
  }
  return MLA_OK;
}

// ------------------------------------------------ materialised causal prefill
// Workspace: the split-K scratch of the projections, then the token-ordered
// cache rows, c_Q, the queries [T][n_h][d_h + d_r], K_C [T][n_h][d_h] and
// V [T][n_h][d_v].
struct MatPlan {
  Plan base;   // hdr, counters, partial
  size_t dense, cq, q, kc, v, total;
};
MatPlan make_mat_plan(const mla_dims& d, int T) {
  MatPlan M{};
  M.base = make_plan(d, T, false);
  size_t o = M.base.total;
  M.dense = o; o = align_up(o + 2 * (size_t)T * (d.d_c + d.d_r), 256);
  M.cq = o;    o = align_up(o + 2 * (size_t)T * d.d_cq, 256);
  M.q = o;     o = align_up(o + 2 * (size_t)T * d.n_h * (d.d_h + d.d_r), 256);
  M.kc = o;    o = align_up(o + 2 * (size_t)T * d.n_h * d.d_h, 256);
  M.v = o;     o = align_up(o + 2 * (size_t)T * d.n_h * d.d_v, 256);
  M.total = o;
  return M;
}

// Dimensions the materialised kernel takes: bf16, a 64-wide RoPE key, and
// head widths that are whole 64-column chunks of at most 128.
bool mat_supported(const mla_dims& d) {
  return d.dtype == MLA_BF16 && !d.rope_key_per_head && d.d_r == attn_mha::DR && (d.d_h == 64 || d.d_h == 128) &&
         (d.d_v == 64 || d.d_v == 128);
}

mla_status prefill_mat_impl(const mla_weights* w, const void* h, const int32_t* page_table, int max_pages,
                            int num_pages, void* cache, float* out, int B, int S, void* ws, const MatPlan& M,
                            cudaStream_t st) {
  using T = __nv_bfloat16;
  const mla_dims& d = w->d;
  const int T_ = B * S, d_cr = d.d_c + d.d_r, din = d_in(d), dq = d.d_h + d.d_r;
  const Plan& P = M.base;
  cudaError_t e;
  // (1) append every token, keeping a token-ordered copy of the rows.
  {
    EpiAppend<T> epi{};
    epi.cache = static_cast<T*>(cache);
    epi.prefill_S = S;
    epi.page_table = page_table;
    for (int i = 0; i < d.d_r / 2; ++i) epi.theta[i] = w->theta[i];
    epi.max_pages = max_pages;
    epi.num_pages = num_pages;
    epi.page_size = d.page_size;
    epi.d_c = d.d_c;
    epi.d_cr = d_cr;
    epi.d_r = d.d_r;
    epi.n_seq = B;
    epi.err = at<int>(ws, P.hdr);
    epi.dense = at<T>(ws, M.dense);
    if ((e = gemm<T>(h, d.d_model, 0, w->dkr, d.d_model, 0, T_, d_cr, d.d_model, 1, epi, ws, P, st)))
      return cuda_status(e);
  }
  // (2) query latent, (3) [q_C | RoPE(q_R)] per head, scaled by s * log2 e.
  const void* src = h;
  if (d.d_cq > 0) {
    EpiStore<T> epi{at<T>(ws, M.cq), d.d_cq, 0, 1.f};
    if ((e = gemm<T>(h, d.d_model, 0, w->dq, d.d_model, 0, T_, d.d_cq, d.d_model, 1, epi, ws, P, st)))
      return cuda_status(e);
    src = at<T>(ws, M.cq);
  }
  {
    EpiQProjM<T> epi{};
    epi.q = at<T>(ws, M.q);
    for (int i = 0; i < d.d_r / 2; ++i) epi.theta[i] = w->theta[i];
    epi.n_h = d.n_h; epi.d_h = d.d_h; epi.d_r = d.d_r; epi.prefill_S = S;
    epi.qscale = (float)((double)w->scale * kLog2e);
    if ((e = gemm<T>(src, din, 0, w->uqr, din, 0, T_, d.n_h * (d.d_h + d.d_r), din, 1, epi, ws, P, st)))
      return cuda_status(e);
  }
  // (4) expansion: K_C = W_UK c and V = W_UV c for every token and head.
  {
    EpiStore<T> ek{at<T>(ws, M.kc), (long long)d.n_h * d.d_h, 0, 1.f};
    if ((e = gemm<T>(at<T>(ws, M.dense), d_cr, 0, w->uk, d.d_c, 0, T_, d.n_h * d.d_h, d.d_c, 1, ek, ws, P, st)))
      return cuda_status(e);
    EpiStore<T> ev{at<T>(ws, M.v), (long long)d.n_h * d.d_v, 0, 1.f};
    if ((e = gemm<T>(at<T>(ws, M.dense), d_cr, 0, w->uv, d.d_c, 0, T_, d.n_h * d.d_v, d.d_c, 1, ev, ws, P, st)))
      return cuda_status(e);
  }
  // (5) causal multi-head attention on the expanded keys and values.
  CUtensorMap mq, mk, mv, mr;
  if (!encode_bf16_3d(&mq, at<T>(ws, M.q), dq, d.n_h, T_, dq, (long long)d.n_h * dq, 64, 1, attn_mha::BQ) ||
      !encode_bf16_3d(&mk, at<T>(ws, M.kc), d.d_h, d.n_h, T_, d.d_h, (long long)d.n_h * d.d_h, 64, 1,
                      attn_mha::BKV) ||
      !encode_bf16_3d(&mv, at<T>(ws, M.v), d.d_v, d.n_h, T_, d.d_v, (long long)d.n_h * d.d_v, 64, 1,
                      attn_mha::BKV) ||
      !encode_cache_map(&mr, cache, d_cr, (long long)num_pages * d.page_size, 64))
    return MLA_ERR_CUDA;
  attn_mha::Params pp{B, S, d.n_h, d.d_h, d.d_v, d.d_c, dq / 64, d.d_v / 64, page_table, max_pages, num_pages,
                      out, at<int>(ws, P.hdr)};
  if ((e = set_smem_once(attn_mha::attn_mha_kernel, attn_mha::SMEM_BYTES))) return cuda_status(e);
  ++g_launches;
  prof_mark(st, true);
  attn_mha::attn_mha_kernel<<<dim3(ceil_div(S, attn_mha::BQ), d.n_h, B), attn_mha::THREADS, attn_mha::SMEM_BYTES,
                              st>>>(mq, mk, mv, mr, pp);
  prof_mark(st, false);
  return cuda_status(cudaGetLastError());
}

// One warp waits on an mbarrier nobody arrives at; the bounded wait gives up
// after limit_ns, records kErrTimeout in *err and the kernel returns.
__global__ void wait_timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::mbar_fence_init();
  }
  __syncwarp();
  sm100::mbar_wait_warp(&bar, 0, &abort_flag, err, limit_ns);
}

mla_status begin_call(void* ws, cudaStream_t st, const Plan& P) {
  g_launches = 0;
  return cuda_status(cudaMemsetAsync(ws, 0, P.partial, st));  // header, split-K and arrival counters
}

}  // namespace

// =============================================================== C ABI ====
extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_BOUNDS: return "MLA_ERR_DEVICE_BOUNDS";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
  }
  return "MLA_ERR_UNKNOWN";
}

int mla_last_launch_count(void) { return g_launches; }

mla_status mla_profile_begin(int max_launches) {
  if (max_launches <= 0 || g_prof.on) return MLA_ERR_INVALID_ARG;
  g_prof.ev = static_cast<cudaEvent_t*>(calloc(2 * (size_t)max_launches, sizeof(cudaEvent_t)));
  if (!g_prof.ev) return MLA_ERR_INVALID_ARG;
  for (int i = 0; i < 2 * max_launches; ++i)
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
      free(g_prof.ev);
      g_prof.ev = nullptr;
      return MLA_ERR_CUDA;
    }
  g_prof.cap = max_launches;
  g_prof.used = 0;
  g_prof.on = true;
  return MLA_OK;
}

mla_status mla_profile_end(double* total_ms, int* launches) {
  if (!g_prof.on || !total_ms || !launches) return MLA_ERR_INVALID_ARG;
  mla_status st = MLA_OK;
  double sum = 0.0;
  for (int i = 0; i < g_prof.used; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) {
      st = MLA_ERR_CUDA;
      break;
    }
    sum += ms;
  }
  *total_ms = sum;
  *launches = g_prof.used;
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  free(g_prof.ev);
  g_prof = Profiler{};
  return st;
}

size_t mla_absorbed_weights_bytes(const mla_dims* dims) {
  if (check_dims(dims) != MLA_OK) return 0;
  return weight_layout(*dims).total;
}

mla_status mla_absorb_weights(const mla_dims* dims, const void* W_DKV, const void* W_KR, const void* W_DQ,
                              const void* W_UQ, const void* W_QR, const void* W_UK, const void* W_UV,
                              void* absorbed, size_t absorbed_bytes, mla_weights** out, cudaStream_t stream) {
  mla_status s = check_dims(dims);
  if (s != MLA_OK) return s;
  if (!out || !W_DKV || !W_KR || !W_UQ || !W_QR || !W_UK || !W_UV || !absorbed) return MLA_ERR_INVALID_ARG;
  if ((dims->d_cq > 0) != (W_DQ != nullptr)) return MLA_ERR_INVALID_ARG;
  if (!aligned(absorbed, 256)) return MLA_ERR_INVALID_ARG;
  const mla_dims& d = *dims;
  const WeightLayout L = weight_layout(d);
  if (absorbed_bytes < L.total) return MLA_ERR_WORKSPACE;
  const size_t e = esize(d);
  char* base = static_cast<char*>(absorbed);
  g_launches = 0;
  cudaError_t err;
  // Stacked [W_DKV; W_KR] and [W_UQ; W_QR]: plain contiguous copies.
  size_t n1 = e * (size_t)d.d_c * d.d_model, n2 = e * (size_t)(cache_row(d) - d.d_c) * d.d_model;
  if ((err = cudaMemcpyAsync(base + L.dkr, W_DKV, n1, cudaMemcpyDeviceToDevice, stream))) return cuda_status(err);
  if ((err = cudaMemcpyAsync(base + L.dkr + n1, W_KR, n2, cudaMemcpyDeviceToDevice, stream))) return cuda_status(err);
  if (d.d_cq > 0 &&
      (err = cudaMemcpyAsync(base + L.dq, W_DQ, e * (size_t)d.d_cq * d.d_model, cudaMemcpyDeviceToDevice, stream)))
    return cuda_status(err);
  size_t q1 = e * (size_t)d.n_h * d.d_h * d_in(d), q2 = e * (size_t)d.n_h * d.d_r * d_in(d);
  if ((err = cudaMemcpyAsync(base + L.uqr, W_UQ, q1, cudaMemcpyDeviceToDevice, stream))) return cuda_status(err);
  if ((err = cudaMemcpyAsync(base + L.uqr + q1, W_QR, q2, cudaMemcpyDeviceToDevice, stream))) return cuda_status(err);
  if ((err = cudaMemcpyAsync(base + L.uv, W_UV, e * (size_t)d.n_h * d.d_v * d.d_c, cudaMemcpyDeviceToDevice,
                             stream)))
    return cuda_status(err);
  if ((err = cudaMemcpyAsync(base + L.uk, W_UK, e * (size_t)d.n_h * d.d_h * d.d_c, cudaMemcpyDeviceToDevice,
                             stream)))
    return cuda_status(err);
  // Per-head transpose of W_UK: [n_h][d_h][d_c] -> [n_h][d_c][d_h].
  {
    dim3 grid(ceil_div(d.d_c, 32), ceil_div(d.d_h, 32), d.n_h);
    ++g_launches;
    if (d.dtype == MLA_BF16)
      transpose_heads_kernel<__nv_bfloat16><<<grid, dim3(32, 8), 0, stream>>>(
          static_cast<const __nv_bfloat16*>(W_UK), reinterpret_cast<__nv_bfloat16*>(base + L.ukt), d.d_h, d.d_c);
    else
      transpose_heads_kernel<float><<<grid, dim3(32, 8), 0, stream>>>(
          static_cast<const float*>(W_UK), reinterpret_cast<float*>(base + L.ukt), d.d_h, d.d_c);
    if ((err = cudaGetLastError())) return cuda_status(err);
  }
  mla_weights* w = static_cast<mla_weights*>(calloc(1, sizeof(mla_weights)));
  if (!w) return MLA_ERR_INVALID_ARG;
  w->d = d;
  w->scale = d.softmax_scale > 0.f ? d.softmax_scale : (float)(1.0 / sqrt((double)(d.d_h + d.d_r)));
  w->esz = e;
  w->dkr = base + L.dkr;
  w->dq = d.d_cq > 0 ? base + L.dq : nullptr;
  w->uqr = base + L.uqr;
  w->ukt = base + L.ukt;
  w->uk = base + L.uk;
  w->uv = base + L.uv;
  for (int i = 0; i < d.d_r / 2; ++i) w->theta[i] = pow((double)d.rope_base, -2.0 * i / d.d_r);
  *out = w;
  return MLA_OK;
}

void mla_release_weights(mla_weights* w) { free(w); }

mla_status mla_weights_dims(const mla_weights* w, mla_dims* dims) {
  if (!w || !dims) return MLA_ERR_INVALID_ARG;
  *dims = w->d;
  return MLA_OK;
}

size_t mla_append_workspace_bytes(const mla_dims* dims, int T) {
  if (check_dims(dims) != MLA_OK || T < 0) return 0;
  return make_plan(*dims, T, false).total;
}

mla_status mla_append_latent(const mla_weights* w, const void* h, const int32_t* seq_idx, const int32_t* pos,
                             const int32_t* page_table, int num_seqs, int max_pages, int num_pages, void* cache,
                             int T, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!w || T < 0 || num_seqs <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!h || !seq_idx || !pos || !page_table || !cache || !workspace) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h, 16) || !aligned(cache, 16)) return MLA_ERR_INVALID_ARG;
  const Plan P = make_plan(w->d, T, false);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  const int n_seq = num_seqs;
  if (w->d.dtype == MLA_BF16)
    return append_impl<__nv_bfloat16>(w, h, seq_idx, pos, 0, n_seq, page_table, max_pages, num_pages, cache, T,
                                      workspace, P, stream);
  return append_impl<float>(w, h, seq_idx, pos, 0, n_seq, page_table, max_pages, num_pages, cache, T, workspace,
                            P, stream);
}

size_t mla_decode_workspace_bytes(const mla_dims* dims, int B, int n_q, int max_kv_len) {
  if (check_dims(dims) != MLA_OK || B <= 0 || n_q <= 0 || max_kv_len < n_q) return 0;
  return make_plan(*dims, B * n_q, true).total;
}

mla_status mla_decode(const mla_weights* w, const void* h_q, const int32_t* kv_len, const int32_t* page_table,
                      int max_pages, int num_pages, const void* cache, float* out, int B, int n_q, int max_kv_len,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!w || B <= 0 || n_q <= 0 || max_kv_len < n_q || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!h_q || !kv_len || !page_table || !cache || !out || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)max_pages * w->d.page_size < max_kv_len) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h_q, 16) || !aligned(cache, 16) || !aligned(out, 16))
    return MLA_ERR_INVALID_ARG;
  const Plan P = make_plan(w->d, B * n_q, true);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  if (w->d.dtype == MLA_BF16)
    return attend_impl<__nv_bfloat16>(w, h_q, kv_len, 0, n_q, 0, page_table, max_pages, num_pages, cache, out,
                                      B * n_q, max_kv_len, workspace, P, stream);
  return attend_impl<float>(w, h_q, kv_len, 0, n_q, 0, page_table, max_pages, num_pages, cache, out, B * n_q,
                            max_kv_len, workspace, P, stream);
}

size_t mla_decode_step_workspace_bytes(const mla_dims* dims, int B, int n_q, int max_kv_len) {
  if (check_dims(dims) != MLA_OK || B <= 0 || n_q <= 0 || max_kv_len < n_q) return 0;
  return make_plan(*dims, B * n_q, true, false, true).total;
}

mla_status mla_decode_step(const mla_weights* w, const void* h, const int32_t* kv_len, const int32_t* page_table,
                           int max_pages, int num_pages, void* cache, float* out, int B, int n_q, int max_kv_len,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!w || B <= 0 || n_q <= 0 || max_kv_len < n_q || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if (!h || !kv_len || !page_table || !cache || !out || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)max_pages * w->d.page_size < max_kv_len) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h, 16) || !aligned(cache, 16) || !aligned(out, 16))
    return MLA_ERR_INVALID_ARG;
  const Plan P = make_plan(w->d, B * n_q, true, false, true);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  if (w->d.dtype == MLA_BF16) {
    const SideAppend sa{cache, B};
    return attend_impl<__nv_bfloat16>(w, h, kv_len, 0, n_q, 0, page_table, max_pages, num_pages, cache, out,
                                      B * n_q, max_kv_len, workspace, P, stream, nullptr, &sa);
  }
  // fp32: the CUDA-core GEMMs share one arrival-counter array, so the append
  // runs first on the caller's stream.
  s = append_impl<float>(w, h, nullptr, nullptr, 0, B, page_table, max_pages, num_pages, cache, B * n_q, workspace,
                         P, stream, kv_len, n_q);
  if (s != MLA_OK) return s;
  return attend_impl<float>(w, h, kv_len, 0, n_q, 0, page_table, max_pages, num_pages, cache, out, B * n_q,
                            max_kv_len, workspace, P, stream);
}

size_t mla_decode_cp_workspace_bytes(const mla_dims* dims, int B, int n_q) {
  if (check_dims(dims) != MLA_OK || dims->dtype != MLA_BF16 || dims->rope_key_per_head || B <= 0 || n_q <= 0)
    return 0;
  return make_plan(*dims, B * n_q, true, true).total;
}

mla_status mla_decode_cp_partial(const mla_weights* w, const void* h_q, const int32_t* kv_len,
                                 const int32_t* window_start, const int32_t* window_count,
                                 const int32_t* page_table, int max_pages, int num_pages, const void* cache,
                                 void* obar_out, float* lse_out, int B, int n_q, int max_kv_len, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  if (!w || B <= 0 || n_q <= 0 || max_kv_len < n_q || max_pages <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if (w->d.dtype != MLA_BF16 || w->d.rope_key_per_head) return MLA_ERR_UNSUPPORTED;
  if (!h_q || !kv_len || !window_start || !window_count || !page_table || !cache || !obar_out || !lse_out ||
      !workspace)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h_q, 16) || !aligned(cache, 16) || !aligned(obar_out, 16) ||
      !aligned(lse_out, 4))
    return MLA_ERR_INVALID_ARG;
  const Plan P = make_plan(w->d, B * n_q, true, true);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  const int max_count = (int)std::min<long long>((long long)max_pages * w->d.page_size, INT_MAX);
  CpOut cp{CpWindow{window_start, window_count, max_count}, obar_out, lse_out};
  return attend_impl<__nv_bfloat16>(w, h_q, kv_len, 0, n_q, 0, page_table, max_pages, num_pages, cache, nullptr,
                                    B * n_q, max_kv_len, workspace, P, stream, &cp);
}

mla_status mla_decode_cp_combine(const mla_weights* w, int n_ranks, const void* obar_parts,
                                 const float* lse_parts, float* out, int B, int n_q, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  if (!w || n_ranks <= 0 || B <= 0 || n_q <= 0) return MLA_ERR_INVALID_ARG;
  if (w->d.dtype != MLA_BF16 || w->d.rope_key_per_head) return MLA_ERR_UNSUPPORTED;
  if (!obar_parts || !lse_parts || !out || !workspace) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(obar_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16))
    return MLA_ERR_INVALID_ARG;
  const mla_dims& d = w->d;
  const int R = B * n_q;
  const Plan P = make_plan(d, R, true, true);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  using T = __nv_bfloat16;
  ++g_launches;
  cp_merge_kernel<T><<<dim3(R, ceil_div(d.n_h, 8)), 256, 0, stream>>>(
      n_ranks, static_cast<const T*>(obar_parts), lse_parts, at<T>(workspace, P.obar), R, d.n_h, d.d_c,
      at<int>(workspace, P.hdr));
  cudaError_t e = cudaGetLastError();
  if (e) return cuda_status(e);
  EpiStore<float> epi{out, (long long)d.n_h * d.d_v, d.d_v, 1.f};
  return cuda_status(gemm<T>(at<T>(workspace, P.obar), (long long)d.n_h * d.d_c, d.d_c, w->uv, d.d_c,
                             (long long)d.d_v * d.d_c, R, d.d_v, d.d_c, d.n_h, epi, workspace, P, stream));
}

size_t mla_prefill_workspace_bytes(const mla_dims* dims, int B, int S) {
  if (check_dims(dims) != MLA_OK || B <= 0 || S <= 0) return 0;
  return make_plan(*dims, B * S, true).total;
}

mla_status mla_prefill(const mla_weights* w, const void* h, const int32_t* page_table, int max_pages,
                       int num_pages, void* cache, float* out, int B, int S, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  if (!w || B <= 0 || S <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!h || !page_table || !cache || !out || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)max_pages * w->d.page_size < S) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h, 16) || !aligned(cache, 16) || !aligned(out, 16))
    return MLA_ERR_INVALID_ARG;
  const Plan P = make_plan(w->d, B * S, true);
  if (workspace_bytes < P.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, P);
  if (s != MLA_OK) return s;
  if (w->d.dtype == MLA_BF16) {
    s = append_impl<__nv_bfloat16>(w, h, nullptr, nullptr, S, B, page_table, max_pages, num_pages, cache, B * S,
                                   workspace, P, stream);
    if (s != MLA_OK) return s;
    return attend_impl<__nv_bfloat16>(w, h, nullptr, S, S, S, page_table, max_pages, num_pages, cache, out, B * S,
                                      S, workspace, P, stream);
  }
  s = append_impl<float>(w, h, nullptr, nullptr, S, B, page_table, max_pages, num_pages, cache, B * S, workspace,
                         P, stream);
  if (s != MLA_OK) return s;
  return attend_impl<float>(w, h, nullptr, S, S, S, page_table, max_pages, num_pages, cache, out, B * S, S,
                            workspace, P, stream);
}

size_t mla_prefill_materialised_workspace_bytes(const mla_dims* dims, int B, int S) {
  if (check_dims(dims) != MLA_OK || !mat_supported(*dims) || B <= 0 || S <= 0) return 0;
  return make_mat_plan(*dims, B * S).total;
}

mla_status mla_prefill_materialised(const mla_weights* w, const void* h, const int32_t* page_table, int max_pages,
                                    int num_pages, void* cache, float* out, int B, int S, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
  if (!w || B <= 0 || S <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!mat_supported(w->d)) return MLA_ERR_UNSUPPORTED;
  if (!h || !page_table || !cache || !out || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)max_pages * w->d.page_size < S || (long long)B * S > INT_MAX / 2) return MLA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(h, 16) || !aligned(cache, 16) || !aligned(out, 16))
    return MLA_ERR_INVALID_ARG;
  const MatPlan M = make_mat_plan(w->d, B * S);
  if (workspace_bytes < M.total) return MLA_ERR_WORKSPACE;
  mla_status s = begin_call(workspace, stream, M.base);
  if (s != MLA_OK) return s;
  return prefill_mat_impl(w, h, page_table, max_pages, num_pages, cache, out, B, S, workspace, M, stream);
}

mla_status mla_get_error(const void* workspace, cudaStream_t stream) {
  if (!workspace) return MLA_ERR_INVALID_ARG;
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (word & kErrLayout) return MLA_ERR_UNSUPPORTED;
  if (word & kErrTimeout) return MLA_ERR_TIMEOUT;
  if (word & kErrBounds) return MLA_ERR_DEVICE_BOUNDS;
  return MLA_OK;
}

mla_status mla_selftest_wait_timeout(void* workspace, int limit_us, cudaStream_t stream) {
  if (!workspace || !aligned(workspace, 256) || limit_us < 1 || limit_us > 1000000) return MLA_ERR_INVALID_ARG;
  g_launches = 0;
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), stream);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  ++g_launches;
  wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<int*>(workspace), 1000ull * (unsigned long long)limit_us);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ===================================================================
// Append without a caller workspace.
//
// Some callers cannot hand this library a workspace because they cannot
// allocate device memory at the point where they append: an inference engine
// that owns every byte of HBM through its own fixed pool and forbids other
// allocations, code running while a CUDA graph is being captured (where
// cudaMalloc is not permitted), or a host thread that must not take the
// implicit device synchronisation cudaMalloc/cudaFree can cause.  For them,
// mla_append_latent_noalloc keeps the append's scratch (the split-K partial
// tiles and their arrival counters) in one fixed array in this library's own
// device memory instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads
// libmla holds it (kNoAllocScratchBytes, about 2 MiB) until the process exits.
// Host code must not pass the symbol itself to a kernel (on the host it is
// only a stand-in, not a device address); its device address is looked up
// once per device with cudaGetSymbolAddress and cached.
// ===================================================================
namespace {

constexpr int kNoAllocMaxT = 256;                 // tokens per call
constexpr int kNoAllocTileSplits = 128;           // split-K tiles x splits
constexpr size_t kNoAllocHdr = 256;               // error word: takes device errors when device_error is NULL (then discarded)
constexpr size_t kNoAllocCounters = sizeof(int) * kCounterCap;
constexpr size_t kNoAllocScratchBytes =
    kNoAllocHdr + kNoAllocCounters + sizeof(float) * (size_t)kNoAllocTileSplits * 64 * 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};
std::once_flag g_noalloc_once[kMaxDevices];
cudaError_t g_noalloc_err[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on
// the first call made with that device current).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_noalloc_once[dev], [dev] {
    void* p = nullptr;
    g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_noalloc_ptr[dev] = (g_noalloc_err[dev] == cudaSuccess) ? p : nullptr;
  });
  if (g_noalloc_err[dev] != cudaSuccess) return g_noalloc_err[dev];
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

template <typename T>
mla_status append_noalloc_impl(const mla_weights* w, const void* h, const int32_t* seq_idx, const int32_t* pos,
                               const int32_t* page_table, int num_seqs, int max_pages, int num_pages, void* cache,
                               int T_, int32_t* device_error, void* scratch, cudaStream_t st) {
  const mla_dims& d = w->d;
  Plan P{};
  P.hdr = 0;
  P.counters = kNoAllocHdr;
  P.partial = kNoAllocHdr + kNoAllocCounters;
  P.total = kNoAllocScratchBytes;
  EpiAppend<T> epi{};
  epi.cache = static_cast<T*>(cache);
  epi.seq_idx = seq_idx;
  epi.pos = pos;
  epi.prefill_S = 0;
  epi.page_table = page_table;
  for (int i = 0; i < d.d_r / 2; ++i) epi.theta[i] = w->theta[i];
  epi.max_pages = max_pages;
  epi.num_pages = num_pages;
  epi.page_size = d.page_size;
  epi.d_c = d.d_c;
  epi.d_cr = cache_row(d);
  epi.d_r = d.d_r;
  epi.n_seq = num_seqs;
  epi.err = device_error ? reinterpret_cast<int*>(device_error) : at<int>(scratch, P.hdr);
  return cuda_status(gemm<T>(h, d.d_model, 0, w->dkr, d.d_model, 0, T_, cache_row(d), d.d_model, 1, epi, scratch,
                             P, st, kNoAllocTileSplits));
}

}  // namespace

extern "C" mla_status mla_append_latent_noalloc(const mla_weights* w, const void* h, const int32_t* seq_idx,
                                                const int32_t* pos, const int32_t* page_table, int num_seqs,
                                                int max_pages, int num_pages, void* cache, int T,
                                                int32_t* device_error, cudaStream_t stream) {
  if (!w || T < 0 || num_seqs <= 0 || max_pages <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (T > kNoAllocMaxT) return MLA_ERR_WORKSPACE;
  if (T == 0) return MLA_OK;
  if (!h || !seq_idx || !pos || !page_table || !cache) return MLA_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(cache, 16) || (device_error && !aligned(device_error, 4)))
    return MLA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return MLA_ERR_CUDA;
  g_launches = 0;
  // The arrival counters must start at zero; the array keeps whatever the
  // previous call left in it.
  if (cudaMemsetAsync(scratch, 0, kNoAllocHdr + kNoAllocCounters, stream) != cudaSuccess) return MLA_ERR_CUDA;
  if (w->d.dtype == MLA_BF16)
    return append_noalloc_impl<__nv_bfloat16>(w, h, seq_idx, pos, page_table, num_seqs, max_pages, num_pages,
                                              cache, T, device_error, scratch, stream);
  return append_noalloc_impl<float>(w, h, seq_idx, pos, page_table, num_seqs, max_pages, num_pages, cache, T,
                                    device_error, scratch, stream);
}
