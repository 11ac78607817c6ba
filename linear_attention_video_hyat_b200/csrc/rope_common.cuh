// Pieces of the capped temporal rotary embedding shared by its standalone kernel (rope.cu) and
// the fused streaming prep kernel (stream_prep.cu), so that both turn a value the same way:
// the same angles (sin / cos formed in double from the same per-pair frequencies) and the same
// rounding of the rotation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace hyat {

constexpr int kRopeMaxPairs = 64;     // d <= 128

// A 16-byte vector of T as fp32 lanes, and back (round to nearest even for bf16).
template <typename T>
struct RopeLanes;
template <>
struct RopeLanes<float> {
  static constexpr int kElems = 4;
  __device__ static void to_f32(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 from_f32(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};
template <>
struct RopeLanes<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ static void to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      f[2 * e] = t.x;
      f[2 * e + 1] = t.y;
    }
  }
  __device__ static uint4 from_f32(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      w[e] = *reinterpret_cast<const uint32_t*>(&t);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// cos and sin of the angle p * theta (theta = base^(-2i / t_dims), formed on the host in
// double), rounded to fp32.
__device__ __forceinline__ void rope_cos_sin(int p, double theta, float* c, float* s) {
  double sd, cd;
  sincos(static_cast<double>(p) * theta, &sd, &cd);
  *c = static_cast<float>(cd);
  *s = static_cast<float>(sd);
}

// (x0, x1) turned by the angle whose cos and sin are c and s, with fixed rounding steps.
__device__ __forceinline__ void rope_turn(float& x0, float& x1, float c, float s) {
  const float y0 = fmaf(x0, c, -(x1 * s));
  const float y1 = fmaf(x0, s, x1 * c);
  x0 = y0;
  x1 = y1;
}

}  // namespace hyat
