// Temporal rotary embedding with a capped relative index: the step before attention that
// keeps the temporal positions of a streaming window inside the range a pretrained video model
// has seen (Long-Horizon Streaming Video Generation via Hybrid Attention with Decoupled
// Distillation, Section 2.C, the relative RoPE constraint).
//
// Pair i < t_dims / 2 of the head dimension, (x[2i], x[2i + 1]), turns by p * theta_i with
// theta_i = base^(-2i / t_dims) and p = min(frame - ref_frame, cap - 1); the other dimensions
// pass through unchanged. The op streams each row once (HBM-bound); the cos / sin of each
// (frame, pair) are formed once per block (in double, from angles built on the host in double).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "hyat.h"
#include "rope_common.cuh"

namespace hyat {
namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeBatch = 8;          // rows a thread loads before it stores (memory parallelism)
constexpr int kRopeMaxFrames = 64;     // frames one block's rows may span (table rows)

struct RopeArgs {
  const void* x;
  void* y;
  int32_t n_tokens, d, tokens_per_frame, first_frame, ref_frame, cap, half_t;
  int32_t rows_per_block;              // a multiple of the rows one pass of the block covers
  double theta[kRopeMaxPairs];         // base^(-2i / t_dims), i < half_t
};

// A block owns rows_per_block tokens of one (b, h); each thread one 16-byte column of the head
// dimension in kRopeBatch rows at a time. The block first issues its loads, then forms the
// (cos, sin) table of the frames its rows span (one sincos per frame and pair, in double, into
// shared memory) while they are in flight, then turns and stores.
template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_temporal_kernel(const RopeArgs a) {
  constexpr int E = RopeLanes<T>::kElems, P = E / 2;
  __shared__ float2 cs[kRopeMaxFrames * kRopeMaxPairs];
  const int cols = a.d / E;                        // 16-byte columns per row
  const int tx = threadIdx.x % cols, ty = threadIdx.x / cols, ny = kRopeThreads / cols;
  const int pair0 = tx * P;                        // first pair of this thread's column
  const int r0 = blockIdx.x * a.rows_per_block;
  const int r1 = min(r0 + a.rows_per_block, a.n_tokens);
  const int f_lo = r0 / a.tokens_per_frame;
  const int n_f = (r1 - 1) / a.tokens_per_frame - f_lo + 1;
  const int64_t base_row = static_cast<int64_t>(blockIdx.y) * a.n_tokens;
  const uint4* src = static_cast<const uint4*>(a.x);
  uint4* dst = static_cast<uint4*>(a.y);
  const bool band = pair0 < a.half_t;              // does this column touch the rotated band?
  const bool active = band || a.x != a.y;          // in place: columns outside the band stay
  uint4 v[kRopeBatch];
  auto load = [&](int rb) {
#pragma unroll
    for (int b = 0; b < kRopeBatch; ++b) {
      const int r = rb + b * ny;
      if (active && r < r1) v[b] = src[(base_row + r) * cols + tx];
    }
  };
  load(r0 + ty);                                   // the first batch is in flight while ...
  for (int e = threadIdx.x; e < n_f * a.half_t; e += kRopeThreads) {   // ... the table forms
    const int f = e / a.half_t, pr = e % a.half_t;
    const int p = min(a.first_frame + f_lo + f - a.ref_frame, a.cap - 1);
    float c, sn;
    rope_cos_sin(p, a.theta[pr], &c, &sn);
    cs[f * kRopeMaxPairs + pr] = make_float2(c, sn);
  }
  __syncthreads();
  for (int rb = r0 + ty; rb < r1; rb += kRopeBatch * ny) {
    if (rb != r0 + ty) load(rb);
    if (!active) continue;
#pragma unroll
    for (int b = 0; b < kRopeBatch; ++b) {
      const int r = rb + b * ny;
      if (r >= r1) break;
      if (band) {
        const float2* t = cs + (r / a.tokens_per_frame - f_lo) * kRopeMaxPairs;
        float f[E];
        RopeLanes<T>::to_f32(v[b], f);
#pragma unroll
        for (int k = 0; k < P; ++k)
          if (pair0 + k < a.half_t) rope_turn(f[2 * k], f[2 * k + 1], t[pair0 + k].x, t[pair0 + k].y);
        v[b] = RopeLanes<T>::from_f32(f);
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
  // 128 rows per block (one batch per thread at d = 128 bf16), fewer when frames are so short
  // that the rows would span more than kRopeMaxFrames frames
  const int ny = kRopeThreads / (d / (dtype == HYAT_BF16 ? 8 : 4));
  const int64_t by_frames = (static_cast<int64_t>(kRopeMaxFrames - 2) * tokens_per_frame + 1) / ny * ny;
  a.rows_per_block = static_cast<int32_t>(std::max<int64_t>(ny, std::min<int64_t>(128, by_frames)));
  const dim3 grid((n_tokens + a.rows_per_block - 1) / a.rows_per_block, BH);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == HYAT_BF16)
    rope_temporal_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, s>>>(a);
  else
    rope_temporal_kernel<float><<<grid, kRopeThreads, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? HYAT_OK : HYAT_ERR_CUDA;
}
