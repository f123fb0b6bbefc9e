// Shared device helpers for libmla kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace mla {

// Bits OR-ed into the workspace error word by device-side checks.
enum DeviceErr : int { kErrBounds = 1, kErrTimeout = 2, kErrLayout = 4 };

__device__ __forceinline__ void flag_error(int* err_word, int bit) {
  if (err_word) atomicOr(err_word, bit);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Stores two adjacent elements (index n even, 8- or 4-byte aligned pair).
__device__ __forceinline__ void store_pair(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
__device__ __forceinline__ void store_pair(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// Stores eight consecutive elements: one or two 16-byte stores when the
// address allows, else pairs.
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) store_pair(p + 2 * i, v[2 * i], v[2 * i + 1]);
  }
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) store_pair(p + 2 * i, v[2 * i], v[2 * i + 1]);
  }
}

// RoPE on one interleaved pair (x0, x1) = components (2i, 2i+1), rotated by
// angle pos * theta_i.  The angle is formed and reduced to [-pi, pi] in fp64
// (positions reach 2^15, where an fp32 angle would be off by ~4e-3 rad); the
// sine and cosine of the reduced angle come from the fp32 hardware
// approximation (absolute error ~1e-6 on [-pi, pi]).
__device__ __forceinline__ void rope_rotate_pair(float& x0, float& x1, int pos, double theta) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  double ang = (double)pos * theta;
  double r = ang - two_pi * rint(ang * inv_two_pi);
  float s, c;
  __sincosf((float)r, &s, &c);  // |r| <= pi: the fast path is accurate to ~1e-6
  float y0 = x0 * c - x1 * s;
  float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace mla
