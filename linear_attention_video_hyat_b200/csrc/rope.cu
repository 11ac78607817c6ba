// Temporal rotary embedding with a capped relative index: the step before attention that
// keeps the temporal positions of a streaming window inside the range a pretrained video model
// has seen (Long-Horizon Streaming Video Generation via Hybrid Attention with Decoupled
// Distillation, Section 2.C, the relative RoPE constraint).
//
// Pair i < t_dims / 2 of the head dimension, (x[2i], x[2i + 1]), turns by p * theta_i with
// theta_i = base^(-2i / t_dims) and p = min(frame - ref_frame, cap - 1); the other dimensions
// pass through unchanged. The op streams each row once (HBM-bound): a block owns 128 tokens of
// one (b, h), each thread one 16-byte column of the head dimension, and a thread recomputes
// its cos / sin (in double, from angles built on the host in double) only when its row enters
// a new frame, which is once per frame.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "hyat.h"

namespace hyat {
namespace {

constexpr int kRopeRows = 128;    // tokens of one (b, h) per block
constexpr int kRopeThreads = 256;
constexpr int kMaxPairs = 64;     // d <= 128
constexpr int kBatch = 4;         // rows a thread loads before it stores (memory parallelism)

struct RopeArgs {
  const void* x;
  void* y;
  int32_t n_tokens, d, tokens_per_frame, first_frame, ref_frame, cap, half_t;
  double theta[kMaxPairs];        // base^(-2i / t_dims), i < half_t
};

template <typename T>
struct Lanes;
template <>
struct Lanes<float> {
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
struct Lanes<__nv_bfloat16> {
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

template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_temporal_kernel(const RopeArgs a) {
  constexpr int E = Lanes<T>::kElems, P = E / 2;
  const int cols = a.d / E;                        // 16-byte columns per row
  const int tx = threadIdx.x % cols, ty = threadIdx.x / cols, ny = kRopeThreads / cols;
  const int pair0 = tx * P;                        // first pair of this thread's column
  const int r0 = blockIdx.x * kRopeRows;
  const int r1 = min(r0 + kRopeRows, a.n_tokens);
  const int64_t base_row = static_cast<int64_t>(blockIdx.y) * a.n_tokens;
  const uint4* src = static_cast<const uint4*>(a.x);
  uint4* dst = static_cast<uint4*>(a.y);
  bool band = false;                               // does this column touch the rotated band?
#pragma unroll
  for (int k = 0; k < P; ++k) band |= pair0 + k < a.half_t;
  if (!band && a.x == a.y) return;                 // in place: columns outside the band stay
  int cur_p = -1;
  float c[P], s[P];
#pragma unroll
  for (int k = 0; k < P; ++k) { c[k] = 1.0f; s[k] = 0.0f; }
  for (int rb = r0 + ty; rb < r1; rb += kBatch * ny) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int r = rb + b * ny;
      if (r < r1) v[b] = src[(base_row + r) * cols + tx];
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int r = rb + b * ny;
      if (r >= r1) break;
      if (band) {
        const int p = min(a.first_frame + r / a.tokens_per_frame - a.ref_frame, a.cap - 1);
        if (p != cur_p) {
          cur_p = p;
#pragma unroll
          for (int k = 0; k < P; ++k) {
            if (pair0 + k < a.half_t) {
              double sd, cd;
              sincos(static_cast<double>(p) * a.theta[pair0 + k], &sd, &cd);
              c[k] = static_cast<float>(cd);
              s[k] = static_cast<float>(sd);
            }
          }
        }
        float f[E];
        Lanes<T>::to_f32(v[b], f);
#pragma unroll
        for (int k = 0; k < P; ++k) {
          if (pair0 + k < a.half_t) {
            const float x0 = f[2 * k], x1 = f[2 * k + 1];
            f[2 * k] = x0 * c[k] - x1 * s[k];
            f[2 * k + 1] = x0 * s[k] + x1 * c[k];
          }
        }
        v[b] = Lanes<T>::from_f32(f);
      }
      dst[(base_row + r) * cols + tx] = v[b];
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace hyat

extern "C" HYAT_API hyat_status hyat_rope_temporal(const void* x, void* y, int32_t BH, int32_t n_tokens, int32_t d,
                                                  int32_t dtype, int32_t tokens_per_frame, int32_t first_frame,
                                                  int32_t ref_frame, int32_t cap, int32_t t_dims, float base,
                                                  void* stream) {
  using namespace hyat;
  if (BH < 0 || n_tokens < 0 || (d != 64 && d != 128) || (dtype != HYAT_F32 && dtype != HYAT_BF16) ||
      tokens_per_frame < 1 || cap < 1 || t_dims < 0 || t_dims > d || (t_dims & 1) || !(base > 0.0f) ||
      !std::isfinite(base) || first_frame < ref_frame || BH > 65535)
    return HYAT_ERR_INVALID_ARG;
  if (BH == 0 || n_tokens == 0) return HYAT_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return HYAT_ERR_INVALID_ARG;
  RopeArgs a{};
  a.x = x;
  a.y = y;
  a.n_tokens = n_tokens;
  a.d = d;
  a.tokens_per_frame = tokens_per_frame;
  a.first_frame = first_frame;
  a.ref_frame = ref_frame;
  a.cap = cap;
  a.half_t = t_dims / 2;
  for (int i = 0; i < a.half_t; ++i) a.theta[i] = std::pow(static_cast<double>(base), -2.0 * i / t_dims);
  const dim3 grid((n_tokens + kRopeRows - 1) / kRopeRows, BH);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == HYAT_BF16)
    rope_temporal_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, s>>>(a);
  else
    rope_temporal_kernel<float><<<grid, kRopeThreads, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? HYAT_OK : HYAT_ERR_CUDA;
}
