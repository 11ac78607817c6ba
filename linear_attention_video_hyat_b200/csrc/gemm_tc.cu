// Tensor-core complement reduction for block-sparse masks (d = 128):
//     S_rest[g] = sum_s Mbar[g][s] * S_seg[s]        for every (b, h)
// where Mbar is the 0/1 matrix of the tiles a query tile does NOT keep (they reach it through
// the linear state: Radial Attention's static mask, or a caller's block mask) and S_seg[s] is
// the linear state of key tile s (S flattened, then z: d*d + d values). With 1024 query tiles
// and 1024 key tiles per head this is a dense GEMM (M = K = 1024, N = 16512 per head), the
// one step of the block-mask path that is a real contraction outside the attention itself.
//
// Layout: Mbar is bf16 (exact 0/1), [mask heads][groups][segments padded to 64], K-major.
// S_seg arrives as two bf16 parts, hi = bf16(S) and lo = bf16(S - hi), [B*H][segments][d*d+d]
// (the MN-major operand layout), so hi*Mbar + lo*Mbar keeps about 16 mantissa bits. One TMEM
// accumulator tile (128 groups x 128 state entries) gets both products; a drain warpgroup
// writes S_rest as bf16 in its natural [a][b] layout (the MN-major operand of the attention
// kernel's linear term) and z_rest as fp32.
//   warp 0: TMA producer (2-stage ring of A, B_hi, B_lo tiles); warp 1: MMA issuer;
//   warps 4-7: drain (TMEM lanes = groups). Units are (b*h, entry tile, group tile) with the
//   group tile fastest, so the 8 group tiles that share a state tile run side by side in L2.
#include "hyat_internal.h"
#include "tc_common.cuh"

namespace hyat {
namespace {

using namespace tc;

constexpr int G_NST = 2;
constexpr int G_STAGE = 3 * TILE_BYTES;          // A, B_hi, B_lo
constexpr int G_THREADS = 256;
constexpr uint32_t kIdescGemm = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct __align__(1024) GemmSmem {
  uint8_t stage[G_NST][G_STAGE];
  uint64_t full[G_NST], empty[G_NST];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct GemmParams {
  int32_t BH, H, mask_heads, nqg, nseg, E, n_gt, n_et, n_kt;
  float* srest;
  uint16_t* srest_bf16;
  int32_t write_f32_s;
  uint32_t* status;
};

// Bounded wait; after one plain probe the hardware may suspend the thread until the phase
// completes (at most 1 ms per try), so waiting warps do not poll shared memory.
__device__ __forceinline__ bool gwait(uint64_t* b, uint32_t parity, GemmSmem* sm, uint32_t* status) {
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

__global__ void __launch_bounds__(G_THREADS, 1)
    gemm_complement_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmHi,
                           const __grid_constant__ CUtensorMap tmLo, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem* sm = reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < G_NST; ++i) {
      mbar_init(&sm->full[i], 1);
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  pdl_wait();                // the segment states come from the kernel launched before this one

  const int per_bh = p.n_et * p.n_gt;
  const int n_units = p.BH * per_bh;
  if (warp == 0) {
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, pending = 0, pending_ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int bh = u / per_bh, et = (u % per_bh) / p.n_gt, gt = u % p.n_gt;
        const int hm = p.mask_heads == 1 ? 0 : bh % p.H;
        for (int kt = 0; kt < p.n_kt && ok; ++kt) {
          if (!(ok = gwait(&sm->empty[st], ph ^ 1u, sm, p.status))) break;
          uint8_t* dst = sm->stage[st];
          mbar_expect_tx(&sm->full[st], G_STAGE);
          tma_load_3d(smem_u32(dst), &tmA, kt * 128, gt * 128, hm, &sm->full[st]);
          tma_load_3d(smem_u32(dst + HALF_BYTES), &tmA, kt * 128 + 64, gt * 128, hm, &sm->full[st]);
          tma_load_3d(smem_u32(dst + TILE_BYTES), &tmHi, et * 128, kt * 128, bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + TILE_BYTES + HALF_BYTES), &tmHi, et * 128 + 64, kt * 128, bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + 2 * TILE_BYTES), &tmLo, et * 128, kt * 128, bh, &sm->full[st]);
          tma_load_3d(smem_u32(dst + 2 * TILE_BYTES + HALF_BYTES), &tmLo, et * 128 + 64, kt * 128, bh, &sm->full[st]);
          pending |= 1u << st;
          pending_ph = (pending_ph & ~(1u << st)) | (ph << st);
          if (++st == G_NST) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        for (int i = 0; i < G_NST; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->full[i], (pending_ph >> i) & 1u) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // the whole warp runs the MMA role (warp-uniform descriptors); one elected lane issues
    {
      int st = 0, c = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint64_t dA0 = sdesc(smem_u32(sm->stage[0]), 16, 1024);
      const uint64_t dB0 = sdesc(smem_u32(sm->stage[0] + TILE_BYTES), HALF_BYTES, 1024);
      constexpr uint64_t kStage = G_STAGE >> 4, kPart = TILE_BYTES >> 4;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++c) {
        const int buf = c & 1;
        const uint32_t tacc = tmem + buf * 128;
        if (!(ok = __all_sync(0xffffffffu, gwait(&sm->acc_empty[buf], ((c >> 1) & 1) ^ 1u, sm, p.status)))) break;
        tc_fence_after();
        for (int kt = 0; kt < p.n_kt && ok; ++kt) {
          if (!(ok = __all_sync(0xffffffffu, gwait(&sm->full[st], ph, sm, p.status)))) break;
          tc_fence_after();
          const uint64_t da = dA0 + static_cast<uint64_t>(st) * kStage;
          const uint64_t dhi = dB0 + static_cast<uint64_t>(st) * kStage, dlo = dhi + kPart;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = da + static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
            const uint64_t bo = static_cast<uint64_t>(kk * (2048 >> 4));
            mma_ss_elect(tacc, a, dhi + bo, kIdescGemm, (kt | kk) != 0);
            mma_ss_elect(tacc, a, dlo + bo, kIdescGemm, 1);
          }
          mma_commit_elect(&sm->empty[st]);
          if (++st == G_NST) { st = 0; ph ^= 1u; }
        }
        if (ok) mma_commit_elect(&sm->acc_full[buf]);
      }
      mma_commit_elect(&sm->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    const int rowl = (warp & 3) * 32 + lane;          // TMEM lane = group within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int64_t dd = static_cast<int64_t>(D) * D;
    int c = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++c) {
      const int bh = u / per_bh, et = (u % per_bh) / p.n_gt, gt = u % p.n_gt;
      const int buf = c & 1;
      if (!__all_sync(0xffffffffu, gwait(&sm->acc_full[buf], (c >> 1) & 1, sm, p.status))) break;
      tc_fence_after();
      uint32_t r[128];
      tmem_ld32p(tmem + buf * 128 + lane_off, r);
      tmem_ld32p(tmem + buf * 128 + lane_off + 32, r + 32);
      tmem_ld32p(tmem + buf * 128 + lane_off + 64, r + 64);
      tmem_ld32p(tmem + buf * 128 + lane_off + 96, r + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm->acc_empty[buf]);
      const int g = gt * 128 + rowl;
      if (g >= p.nqg) continue;
      const int64_t grp = static_cast<int64_t>(bh) * p.nqg + g;
      const int64_t e0 = static_cast<int64_t>(et) * 128;
      if (e0 < dd) {
        uint4* dst = reinterpret_cast<uint4*>(p.srest_bf16 + grp * dd + e0);
#pragma unroll
        for (int v = 0; v < 16; ++v)
          dst[v] = make_uint4(pack_bf16(u2f(r[8 * v]), u2f(r[8 * v + 1])), pack_bf16(u2f(r[8 * v + 2]), u2f(r[8 * v + 3])),
                              pack_bf16(u2f(r[8 * v + 4]), u2f(r[8 * v + 5])), pack_bf16(u2f(r[8 * v + 6]), u2f(r[8 * v + 7])));
      }
      if (e0 >= dd || p.write_f32_s) {
        float4* dst = reinterpret_cast<float4*>(p.srest + grp * p.E + e0);
#pragma unroll
        for (int v = 0; v < 32; ++v)
          dst[v] = make_float4(u2f(r[4 * v]), u2f(r[4 * v + 1]), u2f(r[4 * v + 2]), u2f(r[4 * v + 3]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
  }
}

constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

// bf16 2-D-per-z tensor [z][rows][cols] with 64 x 128 boxes and 128-byte swizzle
bool make_map_cols(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t zdim) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(zdim)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(rows) * cols * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool complement_tc_supported(int d, int nqg) { return d == D && nqg > 8; }

cudaError_t launch_complement_tc(const ComplementTcArgs& a, int num_sms, cudaStream_t s) {
  if (a.BH == 0 || a.nqg == 0) return cudaSuccess;
  if (a.E % 128 != 0 || a.nseg_pad % 64 != 0) return cudaErrorInvalidValue;
  CUtensorMap ma, mhi, mlo;
  if (!make_map_cols(&ma, a.cm_bf16, a.nseg_pad, a.nqg, a.mask_heads) ||
      !make_map_cols(&mhi, a.seg_hi, a.E, a.nseg, a.BH) || !make_map_cols(&mlo, a.seg_lo, a.E, a.nseg, a.BH))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[tc::kMaxDevices];
  cudaError_t attr_e = tc::set_smem_attr_once(reinterpret_cast<const void*>(gemm_complement_kernel), kGemmSmemBytes, attr_set);
  if (attr_e != cudaSuccess) return attr_e;
  GemmParams p{};
  p.BH = a.BH;
  p.H = a.H;
  p.mask_heads = a.mask_heads;
  p.nqg = a.nqg;
  p.nseg = a.nseg;
  p.E = a.E;
  p.n_gt = (a.nqg + 127) / 128;
  p.n_et = a.E / 128;
  p.n_kt = (a.nseg + 127) / 128;
  p.srest = a.srest;
  p.srest_bf16 = a.srest_bf16;
  p.write_f32_s = a.write_f32_s;
  p.status = a.status;
  const int units = a.BH * p.n_gt * p.n_et;
  const int grid = units < num_sms ? units : num_sms;
  return launch_pdl(gemm_complement_kernel, dim3(grid), dim3(G_THREADS), kGemmSmemBytes, s, ma, mhi, mlo, p);
}

}  // namespace hyat
