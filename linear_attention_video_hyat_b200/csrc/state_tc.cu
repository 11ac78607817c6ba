// Tensor-core linear-state kernel for bf16, d = 128, on sm_100a.
//
// For every key segment g (a frame, a 128-key tile, or an evicted chunk) of every (b, h):
//     S_g = sum_{j in g} phi(k_j) v_j^T   (d x d),     z_g = sum_{j in g} phi(k_j)   (d)
// the linear-attention state of Hybrid Forcing, Section 2.A (key/value states of frames
// outside the window aggregated into a compact state) and of ReHyAt's chunk-wise form.
//
// As a contraction over tokens, S_g = A B^T with A = phi(K_g)^T (M = 128 features, K = tokens)
// and B = V_g^T (N = 128 features, K = tokens). Both tiles arrive from HBM by TMA as
// [128 tokens x 128 features] with 128-byte swizzle, which is exactly the MN-major operand
// layout, so no transpose is needed:
//   * warp 8 streams 64-token K and V tiles through a 6-stage ring (about 160 KB in
//     flight per SM, enough to cover loaded-HBM latency);
//   * warps 0-3 and 10-13 apply phi in place in shared memory, 32 rows of a stage each
//     (zeroing rows past the segment end); loads, arithmetic and stores are batched so
//     the chunks of a thread overlap;
//   * warp 9 issues tcgen05.mma into a double-buffered TMEM accumulator; z comes from a
//     second MMA against an all-ones 16-column operand (N = 16), so it costs no CUDA-core work;
//   * warps 4-7 drain the accumulator of a finished segment to HBM while the next segment
//     accumulates in the other buffer.
// The kernel is bound by HBM: it reads K and V once (4d bytes per key) and writes d^2 + d
// floats per segment.
#include "hyat_internal.h"
#include "tc_common.cuh"

namespace hyat {
namespace {

using namespace tc;

constexpr int TOK = 64;                          // tokens per stage
constexpr int NST = 6;
constexpr int KT_BYTES = TOK * D * 2;            // one [64 tokens x 128 features] bf16 tile
constexpr int KT_HALF = KT_BYTES / 2;            // 64 features (128-byte rows)
constexpr int STAGE_BYTES = 2 * KT_BYTES;        // K tile, then V tile
constexpr int ST_THREADS = 448;                  // warps 0-3, 10-13 phi; 4-7 drain; 8 TMA; 9 MMA
constexpr int PHI_THREADS = 256;                 // two phi warpgroups, 32 rows of a stage each
constexpr int ST_TMA_WARP = 8, ST_MMA_WARP = 9;

// D f32, A and B bf16 MN-major, M = 128, N = 128
constexpr uint32_t kIdescState =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
// D f32, A bf16 MN-major, B bf16 K-major (all ones), M = 128, N = 16
constexpr uint32_t kIdescOnes = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

struct __align__(1024) StateSmem {
  uint8_t stage[NST][STAGE_BYTES];
  uint8_t ones[2048];                            // 16 rows x 64 bf16 ones
  uint64_t full[NST], phi_done[NST], empty[NST];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct StateParams {
  int32_t nseg, n_units, seg_base, seg_stride, seg_len;
  int32_t parts, part_len;   // each segment is split into `parts` token ranges of part_len
  float* partial;            // if set: unit u's state -> partial[u] (fp32, plain store)
  int64_t rows;
  float* out;
  int32_t accumulate;
  uint32_t* status;
  uint16_t* out_hi;          // if set: bf16 hi/lo parts instead of fp32 `out`
  uint16_t* out_lo;
  int32_t phi;               // feature map (hyat_phi)
};

// Bounded wait. After one plain probe the thread lets the hardware suspend it until the phase
// completes (at most 1 ms per try), so waiting warps do not poll shared memory while the
// TMA engine fills it.
__device__ __forceinline__ bool swait(uint64_t* b, uint32_t parity, StateSmem* sm, uint32_t* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_suspend(b, parity, 1000000u)) return true;
    if (*reinterpret_cast<volatile int32_t*>(&sm->abort_flag)) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      atomicOr(status, kStatusTimeout);
      *reinterpret_cast<volatile int32_t*>(&sm->abort_flag) = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool swait_warp(uint64_t* b, uint32_t parity, StateSmem* sm, uint32_t* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(b, parity))) return true;
  return __all_sync(0xffffffffu, swait(b, parity, sm, status));
}

struct Unit {
  int bh, g, start, len, ntiles;
};

// Unit u covers part (u mod parts) of segment (u / parts): tokens
// [start, start + len) of (b, h) row block bh.
__device__ __forceinline__ Unit unit_of(const StateParams& p, int u) {
  Unit x;
  const int su = u / p.parts, part = u - su * p.parts;
  x.bh = su / p.nseg;
  x.g = su % p.nseg;
  const int off = part * p.part_len;
  x.start = p.seg_base + x.g * p.seg_stride + off;
  int len = p.seg_len - off;
  if (len > p.part_len) len = p.part_len;
  if (len < 0) len = 0;
  const int64_t rem = p.rows - x.start;
  x.len = static_cast<int>(rem < len ? (rem > 0 ? rem : 0) : len);
  x.ntiles = x.len > 0 ? (x.len + TOK - 1) / TOK : 1;
  return x;
}

// Warps 0-3: apply phi in place to the K half of each stage (rows past the unit's end become
// zero), then hand the stage to the MMA warp.
template <int kKind>
__device__ __forceinline__ void phi_role(StateSmem* sm, const StateParams& p) {
  // phi in place: thread t of warpgroup g owns column chunk t % 16 of rows 32 g + t / 16 + 8 k
  const int g = threadIdx.x >= 128 ? 1 : 0;                  // warps 0-3: g = 0; warps 10-13: g = 1
  const int t = threadIdx.x - (g ? 320 : 0);
  const int cc = t & 15, half = cc >> 3, c8 = cc & 7;
  const int row0 = 32 * g + (t >> 4);
  int st = 0;
  uint32_t ph = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const Unit x = unit_of(p, u);
    for (int i = 0; i < x.ntiles; ++i) {
      if (!(ok = swait_warp(&sm->full[st], ph, sm, p.status))) break;
      const int valid = x.len - TOK * i;
      uint8_t* kt = sm->stage[st] + half * KT_HALF;
      // all loads first, then the arithmetic, then all stores: the chunks are independent, and
      // without this order every store would wait for the next load's address check
      uint4 raw[TOK / 16];
#pragma unroll
      for (int k = 0; k < TOK / 16; ++k) {
        const int r = row0 + 8 * k;
        raw[k] = *reinterpret_cast<const uint4*>(kt + r * 128 + ((c8 ^ (r & 7)) << 4));
      }
#pragma unroll
      for (int k = 0; k < TOK / 16; ++k) {
        const int r = row0 + 8 * k;
        const uint32_t in[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[e]));
          o4[e] = pack_bf16(phi_of<kKind>(f.x), phi_of<kKind>(f.y));
        }
        raw[k] = r < valid ? make_uint4(o4[0], o4[1], o4[2], o4[3]) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < TOK / 16; ++k) {
        const int r = row0 + 8 * k;
        *reinterpret_cast<uint4*>(kt + r * 128 + ((c8 ^ (r & 7)) << 4)) = raw[k];
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&sm->phi_done[st]);
      if (++st == NST) { st = 0; ph ^= 1u; }
    }
  }
}

// Warps 4-7: drain a finished accumulator (S_g and z_g) to global memory while the next unit
// accumulates in the other TMEM buffer.
__device__ __forceinline__ void drain_role(StateSmem* sm, const StateParams& p, uint32_t tmem, int warp, int lane) {
  // drain: row a of S_g (TMEM lane a) and z_g[a]
  const int a = (warp & 3) * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  int c = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++c) {
    const Unit x = unit_of(p, u);
    const int buf = c & 1;
    if (!swait_warp(&sm->acc_full[buf], (c >> 1) & 1, sm, p.status)) break;
    tc_fence_after();
    const uint32_t tacc = tmem + buf * 256 + lane_off;
    const int64_t obase = (static_cast<int64_t>(x.bh) * p.nseg + x.g) * (D * D + D);
    float* out = p.partial ? p.partial + static_cast<int64_t>(u) * (D * D + D) : p.out + obase;
    const bool acc_out = p.accumulate && !p.partial;
    uint32_t zr[1];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(zr[0]) : "r"(tacc + 128));
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      uint32_t r[64];
      tmem_ld32p(tacc + 64 * h, r);
      tmem_ld32p(tacc + 64 * h + 32, r + 32);
      tmem_wait_ld();
      if (h == 1) {
        tc_fence_before();
        mbar_arrive(&sm->acc_empty[buf]);
      }
      if (p.out_hi) {
        // hi = bf16(x), lo = bf16(x - hi): 16-byte stores of 8 values each
        uint4* dhi = reinterpret_cast<uint4*>(p.out_hi + obase + a * D + 64 * h);
        uint4* dlo = reinterpret_cast<uint4*>(p.out_lo + obase + a * D + 64 * h);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float x0 = u2f(r[8 * v + 2 * t]), x1 = u2f(r[8 * v + 2 * t + 1]);
            hw[t] = pack_bf16(x0, x1);
            const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[t]));
            lw[t] = pack_bf16(x0 - hf.x, x1 - hf.y);
          }
          dhi[v] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          dlo[v] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(out + a * D + 64 * h);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          float4 val = make_float4(u2f(r[4 * v]), u2f(r[4 * v + 1]), u2f(r[4 * v + 2]), u2f(r[4 * v + 3]));
          if (acc_out) {
            const float4 o = dst[v];
            val.x += o.x; val.y += o.y; val.z += o.z; val.w += o.w;
          }
          dst[v] = val;
        }
      }
    }
    const float zv = u2f(zr[0]);
    if (p.out_hi) {
      const __nv_bfloat16 zh = __float2bfloat16_rn(zv);
      const __nv_bfloat16 zl = __float2bfloat16_rn(zv - __bfloat162float(zh));
      p.out_hi[obase + D * D + a] = *reinterpret_cast<const uint16_t*>(&zh);
      p.out_lo[obase + D * D + a] = *reinterpret_cast<const uint16_t*>(&zl);
    } else {
      float* zp = out + D * D + a;
      *zp = acc_out ? *zp + zv : zv;
    }
  }
}

__global__ void __launch_bounds__(ST_THREADS, 1)
    state_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const StateParams p) {
  extern __shared__ uint8_t smem_raw[];
  StateSmem* sm = reinterpret_cast<StateSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < 128) {
    reinterpret_cast<uint32_t*>(sm->ones)[threadIdx.x] = 0x3F803F80u;          // bf16 1.0 pairs
    reinterpret_cast<uint32_t*>(sm->ones)[threadIdx.x + 128] = 0x3F803F80u;
    reinterpret_cast<uint32_t*>(sm->ones)[threadIdx.x + 256] = 0x3F803F80u;
    reinterpret_cast<uint32_t*>(sm->ones)[threadIdx.x + 384] = 0x3F803F80u;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&sm->full[i], 1);
      mbar_init(&sm->phi_done[i], PHI_THREADS);
      mbar_init(&sm->empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->acc_full[b], 1);
      mbar_init(&sm->acc_empty[b], 128);
    }
    mbar_init(&sm->drain, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == ST_MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  // Launched programmatically: the set-up above overlaps the end of the kernel before this one;
  // K, V (and the ring slot a fold reads) are read, and any output written, only after its wait.
  pdl_wait();
  pdl_launch_dependents();   // the complement kernel may begin launching; it waits for our results

  if (warp == ST_TMA_WARP) {
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, pending = 0, pending_ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const Unit x = unit_of(p, u);
        for (int i = 0; i < x.ntiles && ok; ++i) {
          if (!(ok = swait(&sm->empty[st], ph ^ 1u, sm, p.status))) break;
          mbar_expect_tx(&sm->full[st], STAGE_BYTES);
          const int row = x.start + TOK * i;
          uint8_t* dst = sm->stage[st];
          tma_load_3d(smem_u32(dst), &tmK, 0, row, x.bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + KT_HALF), &tmK, 64, row, x.bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + KT_BYTES), &tmV, 0, row, x.bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + KT_BYTES + KT_HALF), &tmV, 64, row, x.bh, &sm->full[st]);
          pending |= 1u << st;
          pending_ph = (pending_ph & ~(1u << st)) | (ph << st);
          if (++st == NST) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        for (int i = 0; i < NST; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->full[i], (pending_ph >> i) & 1u) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == ST_MMA_WARP) {
    if (lane == 0) {
      int st = 0, c = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint64_t ones = sdesc(smem_u32(sm->ones), 16, 1024);
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++c) {
        const Unit x = unit_of(p, u);
        const int buf = c & 1;
        const uint32_t tacc = tmem + buf * 256, tz = tacc + 128;
        if (!(ok = swait(&sm->acc_empty[buf], ((c >> 1) & 1) ^ 1u, sm, p.status))) break;
        tc_fence_after();
        for (int i = 0; i < x.ntiles && ok; ++i) {
          if (!(ok = swait(&sm->phi_done[st], ph, sm, p.status))) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(sm->stage[st]), vb = kb + KT_BYTES;
#pragma unroll
          for (int kk = 0; kk < TOK / 16; ++kk) {
            // MN-major, 64-feature halves KT_HALF apart, 16 tokens (2 x 8-row groups) per step
            const uint64_t a = sdesc(kb + kk * 2048, KT_HALF, 1024);
            mma_ss(tacc, a, sdesc(vb + kk * 2048, KT_HALF, 1024), kIdescState, (i | kk) != 0);
            mma_ss(tz, a, ones, kIdescOnes, (i | kk) != 0);
          }
          mma_commit(&sm->empty[st]);
          if (++st == NST) { st = 0; ph ^= 1u; }
        }
        if (ok) mma_commit(&sm->acc_full[buf]);
      }
      mma_commit(&sm->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
  } else if (warp < 4 || warp >= 10) {
    if (p.phi == 1) phi_role<1>(sm, p);
    else if (p.phi == 2) phi_role<2>(sm, p);
    else phi_role<0>(sm, p);
  } else {
    drain_role(sm, p, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == ST_MMA_WARP) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}
constexpr size_t kStateSmemBytes = sizeof(StateSmem) + 1024;

}  // namespace

cudaError_t launch_seg_state_tc(const SegStateArgs& a, int num_sms, cudaStream_t s) {
  if (a.nseg == 0 || a.BH == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  // boxes of TOK rows: 4 loads of 64 x TOK bf16 = STAGE_BYTES per stage
  static_assert(4 * 64 * TOK * 2 == STAGE_BYTES, "stage bytes must match the four TMA boxes");
  if (!tc::make_map(&mk, a.k, a.rows_per_bh, a.BH, TOK) || !tc::make_map(&mv, a.v, a.rows_per_bh, a.BH, TOK))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[tc::kMaxDevices];
  cudaError_t attr_e = tc::set_smem_attr_once(reinterpret_cast<const void*>(state_tc_kernel), kStateSmemBytes, attr_set);
  if (attr_e != cudaSuccess) return attr_e;
  const int parts = a.parts > 1 ? a.parts : 1;
  if (parts > 1 && (a.partial == nullptr || a.out_hi != nullptr || a.part_len <= 0)) return cudaErrorInvalidValue;
  StateParams p{};
  p.nseg = a.nseg;
  p.parts = parts;
  p.part_len = parts > 1 ? a.part_len : a.seg_len;
  p.partial = parts > 1 ? a.partial : nullptr;
  p.n_units = a.nseg * a.BH * parts;
  p.seg_base = a.seg_base;
  p.seg_stride = a.seg_stride;
  p.seg_len = a.seg_len;
  p.rows = a.rows_per_bh;
  p.out = a.out;
  p.accumulate = a.accumulate;
  p.status = a.status;
  p.out_hi = a.out_hi;
  p.out_lo = a.out_lo;
  p.phi = a.phi;
  const int grid = p.n_units < num_sms ? p.n_units : num_sms;
  return launch_pdl(state_tc_kernel, dim3(grid), dim3(ST_THREADS), kStateSmemBytes, s, mk, mv, p);
}

}  // namespace hyat
