// Tensor-core hybrid attention for bf16, d = 128, on sm_100a.
//
// The method (ReHyAt, Abstract; Hybrid Forcing, Section 2.A): every query tile
// takes exact softmax attention over the key tiles of its window and reaches
// all other keys through the linear state (S_rest, z_rest) of its group; the
// two branches share one normaliser. The kernel starts each query row's
// accumulator from the linear branch with running max 0,
//     O = phi(Q) S_rest,   l = phi(q) . z_rest,   m = 0,
// and lets the online softmax over the window tiles rescale it, which yields
//     o = (sum_win e^{s-M} v + e^{-M} phi(q)^T S) / (sum_win e^{s-M} + e^{-M} phi(q)^T z)
// with M = max(0, max_win s) -- the hybrid normaliser.
//
// Design for B200:
//   * one persistent CTA per SM; a CTA owns a pair of 128-row query tiles
//     ("slots"), so the softmax of one slot overlaps the MMAs of the other.
//     Pairs are dealt largest first, a row of the grid at a time, each row to the
//     CTAs least loaded so far (longest-processing-time first); when that
//     would leave few waves, a "split pair" runs one query tile on both slots,
//     each over half of its key tiles, and slot 0 merges the halves;
//   * warp 8 issues TMA loads (Q tiles, K/V tiles, bf16 S_rest) into 128B-swizzled
//     shared memory through a 5-stage ring; warp 9 issues tcgen05.mma (the
//     whole warp runs the role, one elected lane issues) with fp32 accumulators
//     in TMEM; warps 0-3 / 4-7 run the softmax
//     of slot 0 / 1, one query row per thread, reading S from TMEM and writing
//     P (bf16) back into TMEM, where it is the A operand of the P.V MMA;
//   * TMEM (512 columns): S0 | S1 | O0 | O1, each 128 columns; P and phi(Q)
//     alias the first 64 columns of S;
//   * no per-tile row max: exponents use the row's current reference m, and m
//     moves (with a rescale of O in TMEM) only when the running sum would leave
//     the safe fp32 range, which keeps the result exact and the rescale rare;
//   * every mbarrier wait is bounded (%globaltimer); a wait that gives up sets
//     the status word, and all roles drain and free TMEM before exiting. Waiting
//     threads let the hardware suspend them instead of polling shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "hyat_internal.h"
#include "tc_common.cuh"

namespace hyat {
namespace {

using namespace tc;
constexpr int NS = 5;                            // K/V stage ring
constexpr int NUM_THREADS = 384;                 // 3 warpgroups
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512); warpgroup 2
// (TMA, MMA, 2 idle warps) drops to 104, the two softmax warpgroups rise to 200:
// 8 warps x 32 x 200 + 4 warps x 32 x 104 = 64512. Per SM sub-partition: 2 softmax warps
// and 1 warp of group 2 = 2 x 32 x 200 + 32 x 104 = 16128 <= 16384.
constexpr int kRegsSoftmax = 200;
constexpr int kRegsLoadMma = 104;
// The reference max m of a row moves only when the running sum l would leave the safe fp32
// range: every exponent uses the same m as its row's accumulators, so the result is exact.
constexpr float kSafeSum = 1.2676506e30f;        // 2^100
constexpr float kTinySum = 7.8886091e-31f;        // 2^-100

// instruction descriptor, kind::f16: D f32, A/B bf16, M = 128, N = 128
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescKK = kIdescBase;              // B K-major
constexpr uint32_t kIdescKMN = kIdescBase | (1u << 16);  // B MN-major

struct __align__(1024) Smem {
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[NS][TILE_BYTES];
  uint64_t kv_full[NS], kv_empty[NS];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t xfull, o1_free;       // split pairs: slot 1's (l, m) handed over; O1 read out
  uint64_t drain;
  float2 xchg[128];              // split pairs: slot 1's (l, m) per row
  uint32_t tmem_base;
  int32_t abort_flag;
  uint64_t never;                // test hook: a barrier nothing arrives on
  unsigned long long timeout_ns; // limit of every bounded wait
  int32_t n_pairs;               // pairs of this launch (read on the device in redo mode)
};

struct TcParams {
  const WorkItem* work;
  const Entry* entries;
  const int4* pairs;       // {item0, item1 (-1 = none), shared key list, split}
  int32_t n_pairs;
  const float* srest;      // [groups][d*d + d] fp32; z at offset d*d
  void* o;
  int64_t q_rows;
  int32_t nqg;
  float scale_log2;
  uint32_t* status;
  int32_t test_timeout;    // test hook: wait once on a barrier nothing signals (20 ms limit)
  int32_t phi;             // feature map of the linear branch (hyat_phi)
  // Redo mode: the pair count is read on the device from *n_pairs_dev (written by the kernel
  // before this one), and the last CTA to finish resets it and *done_count to 0.
  int32_t* n_pairs_dev;
  uint32_t* done_count;
};

// Bounded wait on a phase parity. Returns false if the kernel is aborting. After the first
// probe the thread lets the hardware suspend it until the phase completes (at most
// kSuspendNs per try), so waiting warps do not poll shared memory.
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Smem* sm, uint32_t* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_suspend(b, parity, kSuspendNs)) return true;
    if (*reinterpret_cast<volatile int32_t*>(&sm->abort_flag)) return false;
    if (globaltimer() - t0 > sm->timeout_ns) {
      atomicOr(status, kStatusTimeout);
      *reinterpret_cast<volatile int32_t*>(&sm->abort_flag) = 1;
      return false;
    }
  }
}

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if all lanes saw
// the phase (the TMEM instructions that follow are .sync.aligned).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* b, uint32_t parity, Smem* sm, uint32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait(b, parity, sm, status));
}

// ------------------------------------------------------------------ softmax role
// Warp-uniform wait with an inline fast path.
__device__ __forceinline__ bool wait_warp(uint64_t* b, uint32_t parity, Smem* sm, uint32_t* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(b, parity))) return true;
  return mbar_wait_warp(b, parity, sm, status);
}

// p = 2^(s * sl + neg_m) for the 128 scores of this row; P (bf16 pairs) -> TMEM at tS.
// Returns the row sum of p (fp32, 8 partial sums).
__device__ __forceinline__ float exp_tile(const uint32_t (&r)[128], float sl, float neg_m, uint32_t tS) {
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float p0 = ex2(fmaf(u2f(r[h * 64 + 2 * i]), sl, neg_m));
      const float p1 = ex2(fmaf(u2f(r[h * 64 + 2 * i + 1]), sl, neg_m));
      acc[(2 * i) & 7] += p0;
      acc[(2 * i + 1) & 7] += p1;
      pk[i] = pack_bf16(p0, p1);
    }
    tmem_st32(tS + h * 32, pk);
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// What each slot does for a pair. A split pair {item, item, 0, 1} runs one query tile on both
// slots: slot 0 takes the first half of its key tiles (and the linear term), slot 1 the
// second half, and slot 0's warpgroup merges the two partial results. Split pairs keep a
// grid of few query tiles busy (a streaming chunk of 37 tiles per head gives 1.5 waves of
// ordinary pairs on 148 SMs, and 3 waves of split pairs).
struct PairView {
  int item[2];
  int eb[2];            // first entry of each slot's key tiles
  int n[2];             // number of key tiles of each slot
  bool has1, shared, split;
};

__device__ __forceinline__ PairView pair_view(const TcParams& p, int pi) {
  const int4 pr = p.pairs[pi];
  PairView v;
  const WorkItem w0 = p.work[pr.x];
  const int n = w0.entry_end - w0.entry_begin;
  v.item[0] = pr.x;
  v.eb[0] = w0.entry_begin;
  if (pr.w != 0) {
    const int n0 = (n + 1) / 2;
    v.item[1] = pr.x;
    v.eb[1] = w0.entry_begin + n0;
    v.n[0] = n0;
    v.n[1] = n - n0;
    v.has1 = n - n0 > 0;
    v.split = v.has1;
    v.shared = false;
  } else {
    v.item[1] = pr.y;
    v.has1 = pr.y >= 0;
    const WorkItem w1 = v.has1 ? p.work[pr.y] : w0;
    v.eb[1] = w1.entry_begin;
    v.n[0] = n;
    v.n[1] = v.has1 ? w1.entry_end - w1.entry_begin : 0;
    v.split = false;
    v.shared = pr.z != 0;
  }
  return v;
}

// One query row per thread (TMEM lane = row). Slot s = warpgroup index.
__device__ __forceinline__ void softmax_role(Smem* sm, const TcParams& p, uint32_t tmem, int warp) {
  const int s = warp >> 2;
  const int row = threadIdx.x & 127;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tS = tmem + s * 128 + lane_off;
  const uint32_t tO = tmem + 256 + s * 128 + lane_off;
  uint64_t* q_full = &sm->q_full[s];
  uint64_t* s_full = &sm->s_full[s];
  uint64_t* p_full = &sm->p_full[s];
  uint64_t* pv_done = &sm->pv_done[s];
  const float sl = p.scale_log2;
  uint32_t qph = 0, sph = 0, xph = 0;
  uint32_t pv_phase = 0;                            // pv_done phases completed before this pair
  bool o1_busy = false;                             // slot 1: O1 not yet read out by slot 0
  const int n_pairs = sm->n_pairs;
  for (int pi = blockIdx.x; pi < n_pairs; pi += gridDim.x) {
    const PairView pv = pair_view(p, pi);
    if (s == 1 && !pv.has1) continue;
    const WorkItem wi = p.work[s == 0 ? pv.item[0] : pv.item[1]];
    const int n = s == 0 ? pv.n[0] : pv.n[1];
    const Entry* ent = p.entries + (s == 0 ? pv.eb[0] : pv.eb[1]);
    // slot 1 of a split pair carries no linear term and starts O1 with its first P.V
    const bool lin = !(pv.split && s == 1);
    int klen_next = n > 0 ? ent[0].k_len : 128;
    if (!wait_warp(q_full, qph, sm, p.status)) return;
    qph ^= 1u;
    if (o1_busy) {
      // O1 is rewritten once this warpgroup hands over its next operand: wait until slot 0
      // has read out the previous split pair's O1
      if (!wait_warp(&sm->o1_free, xph ^ 1u, sm, p.status)) return;
      o1_busy = false;
    }
    float l = 0.0f, m = 0.0f;
    if (lin) {
      // phi(q) of this row -> TMEM (bf16 pairs), l = phi(q) . z
      // z_rest of this tile's group: each lane holds 4 values (one coalesced 512-byte load per
      // warp) and the phi loop broadcasts them with shuffles
      const float4 zq = __ldg(reinterpret_cast<const float4*>(
          p.srest + (static_cast<int64_t>(wi.bh) * p.nqg + wi.state_group) * (D * D + D) + D * D) + (row & 31));
      const float zreg[4] = {zq.x, zq.y, zq.z, zq.w};
      const uint8_t* qrow = sm->q[s] + row * 128;
      float lz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {            // 8 columns per step
        const uint4 raw = *reinterpret_cast<const uint4*>(qrow + (c >> 3) * HALF_BYTES + (((c & 7) ^ (row & 7)) << 4));
        float zz[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) zz[t] = __shfl_sync(0xffffffffu, zreg[t & 3], 2 * c + (t >> 2));
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
          const float f0 = phi_map(f.x, p.phi), f1 = phi_map(f.y, p.phi);
          lz[e] = fmaf(f0, zz[2 * e], lz[e]);
          lz[e] = fmaf(f1, zz[2 * e + 1], lz[e]);
          pk[e] = pack_bf16(f0, f1);
        }
        tmem_st4(tS + 4 * c, pk);
      }
      l = (lz[0] + lz[1]) + (lz[2] + lz[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(p_full);   // one arrival per warp
    }
    if (p.test_timeout && !wait_warp(&sm->never, 0, sm, p.status)) return;
    for (int j = 0; j < n; ++j) {
      const int klen = klen_next;
      if (j + 1 < n) klen_next = ent[j + 1].k_len;
      if (!wait_warp(s_full, sph, sm, p.status)) return;
      sph ^= 1u;
      tc_fence_after();
      uint32_t r[128];
      tmem_ld32p(tS, r);
      tmem_ld32p(tS + 32, r + 32);
      tmem_ld32p(tS + 64, r + 64);
      tmem_ld32p(tS + 96, r + 96);
      tmem_wait_ld();
      if (klen < 128) {
#pragma unroll
        for (int i = 0; i < 128; ++i) r[i] = i < klen ? r[i] : 0xff800000u;   // -inf
      }
      // Optimistic pass: p = 2^(s * scale_log2 - m) with the row's current reference m.
      float rs = exp_tile(r, sl, -m, tS);
      // Rare slow path: the sum left the safe range. A score far above m: move m up to the
      // row max. A sum far below 1 (no linear term, every score so far far below m, so the
      // exponentials approach the flush-to-zero range): move m down to the larger of the row
      // max and log2 of the sum so far. Then rescale O and l (after the previous P.V has
      // landed) and redo the tile.
      if (__any_sync(0xffffffffu, !(l + rs < kSafeSum && l + rs >= kTinySum))) {
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float a = fmax3(u2f(r[k]), u2f(r[k + 8]), u2f(r[k + 16]));
#pragma unroll
          for (int t = 3; t < 15; t += 2) a = fmax3(a, u2f(r[k + 8 * t]), u2f(r[k + 8 * t + 8]));
          mx[k] = fmaxf(a, u2f(r[k + 120]));
        }
        const float mrow = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
        const bool under = !(l + rs >= kTinySum);
        const float m_new = under ? fmaxf(mrow * sl, l > 0.0f ? m + __log2f(l) : -INFINITY) : fmaxf(m, mrow * sl);
        // l = 0: nothing has been added yet, so O holds no weight (a zero linear term, or the
        // split slot's accumulator before its first P.V, which starts it afresh)
        const float alpha = l > 0.0f ? ex2(m - m_new) : 0.0f;
        // Rescale O once its last product so far (commit j - 1 + lin of this pair) has
        // landed. On slot 1 of a split pair at j = 0 nothing has been committed yet: the wait
        // is for the previous pair's last phase (already complete), and the values scaled
        // are overwritten by the first P.V, which starts the accumulator.
        if (!wait_warp(pv_done, (pv_phase + j - 1 + (lin ? 1u : 0u)) & 1u, sm, p.status)) return;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
        tmem_wait_st();
        l *= alpha;
        m = m_new;
        rs = exp_tile(r, sl, -m, tS);
      }
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(p_full);   // one arrival per warp
    }
    const uint32_t n_commits = static_cast<uint32_t>(n) + (lin ? 1u : 0u);
    if (!wait_warp(pv_done, (pv_phase + n_commits - 1) & 1u, sm, p.status)) return;
    pv_phase += n_commits;
    tc_fence_after();
    if (pv.split && s == 1) {
      // hand (l, m) and O1 to slot 0's warpgroup, which merges and stores the tile
      sm->xchg[row] = make_float2(l, m);
      tc_fence_before();
      mbar_arrive(&sm->xfull);
      xph ^= 1u;
      o1_busy = true;
      continue;
    }
    // epilogue: o = O / l (merged with slot 1's half for split pairs), bf16, 16-byte stores
    float a0 = 1.0f, a1 = 0.0f, inv;
    if (pv.split) {
      if (!wait_warp(&sm->xfull, xph, sm, p.status)) return;
      xph ^= 1u;
      tc_fence_after();
      const float2 o1s = sm->xchg[row];
      const float mm = fmaxf(m, o1s.y);
      a0 = ex2(m - mm);
      a1 = ex2(o1s.y - mm);
      inv = 1.0f / (l * a0 + o1s.x * a1);
    } else {
      inv = 1.0f / l;
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                          (static_cast<int64_t>(wi.bh) * p.q_rows + wi.q_row + row) * D);
#pragma unroll 1
    for (int h = 0; h < 4; ++h) {               // 32 columns at a time
      uint32_t r[32];
      tmem_ld32p(tO + h * 32, r);
      if (pv.split) {
        uint32_t r1[32];
        tmem_ld32p(tO + 128 + h * 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(fmaf(u2f(r[i]), a0, u2f(r1[i]) * a1));
      } else {
        tmem_wait_ld();
      }
      if (row < wi.q_len) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          w.x = pack_bf16(u2f(r[8 * v + 0]) * inv, u2f(r[8 * v + 1]) * inv);
          w.y = pack_bf16(u2f(r[8 * v + 2]) * inv, u2f(r[8 * v + 3]) * inv);
          w.z = pack_bf16(u2f(r[8 * v + 4]) * inv, u2f(r[8 * v + 5]) * inv);
          w.w = pack_bf16(u2f(r[8 * v + 6]) * inv, u2f(r[8 * v + 7]) * inv);
          dst[h * 4 + v] = w;
        }
      }
    }
    tc_fence_before();
    if (pv.split) mbar_arrive(&sm->o1_free);
  }
}

// Redo mode: every CTA has read the pair count by the time it gets here; the last one to
// arrive resets the count and this counter for the next launch.
__device__ __forceinline__ void redo_finish(const TcParams& p) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done_count, 1u) == gridDim.x - 1) {
      *reinterpret_cast<volatile int32_t*>(p.n_pairs_dev) = 0;
      *reinterpret_cast<volatile uint32_t*>(p.done_count) = 0u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                   const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_pairs = p.n_pairs;
  if (p.n_pairs_dev) {
    // redo mode: the count comes from the kernel before this one; CTAs without work leave
    // before they allocate anything
    pdl_wait();
    n_pairs = *reinterpret_cast<volatile const int32_t*>(p.n_pairs_dev);
    if (static_cast<int>(blockIdx.x) >= n_pairs) {
      redo_finish(p);
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm->kv_full[i], 1);
      mbar_init(&sm->kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm->q_full[s], 1);
      mbar_init(&sm->q_empty[s], 1);
      mbar_init(&sm->s_full[s], 1);
      mbar_init(&sm->p_full[s], 4);             // one arrival per softmax warp of the slot
      mbar_init(&sm->pv_done[s], 1);
    }
    mbar_init(&sm->xfull, 128);
    mbar_init(&sm->o1_free, 128);
    mbar_init(&sm->drain, 1);
    mbar_init(&sm->never, 1);
    sm->abort_flag = 0;
    sm->timeout_ns = p.test_timeout ? 20000000ull : kTimeoutNs;
    sm->n_pairs = n_pairs;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  pdl_wait();                // the linear states come from the kernels launched before this one
  // No early trigger of dependents: the next streaming step's fold starts only once this
  // kernel has exited, and the prep kernel behind the fold rewrites the work, entry and pair
  // tables this kernel reads.

  if (warp >= 8) {
    // ------------------------------------------------------------ warpgroup 2: TMA + MMA
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLoadMma));
    if (warp == PRODUCER_WARP && lane == 0) {
      int st = 0;
      uint32_t ph = 0, qph0 = 0, qph1 = 0;
      uint32_t pending = 0, pending_ph = 0;   // stages with a load in flight, and its phase bit
      bool ok = true;
      auto take = [&](const CUtensorMap* tm, int row, int z) -> bool {
        if (!mbar_wait(&sm->kv_empty[st], ph ^ 1u, sm, p.status)) return false;
        tma_tile(sm->kv[st], tm, row, z, &sm->kv_full[st]);
        pending |= 1u << st;
        pending_ph = (pending_ph & ~(1u << st)) | (ph << st);
        if (++st == NS) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int pi = blockIdx.x; pi < sm->n_pairs && ok; pi += gridDim.x) {
        const PairView pv = pair_view(p, pi);
        const bool has1 = pv.has1, shared = pv.shared;
        const WorkItem w0 = p.work[pv.item[0]];
        const WorkItem w1 = has1 ? p.work[pv.item[1]] : w0;
        const int n0 = pv.n[0], n1 = pv.n[1];
        const Entry* e0 = p.entries + pv.eb[0];
        const Entry* e1 = p.entries + pv.eb[1];
        ok = mbar_wait(&sm->q_empty[0], qph0 ^ 1u, sm, p.status);
        if (!ok) break;
        qph0 ^= 1u;
        tma_tile(sm->q[0], &tmQ, w0.q_row, w0.bh, &sm->q_full[0]);
        if (has1) {
          ok = mbar_wait(&sm->q_empty[1], qph1 ^ 1u, sm, p.status);
          if (!ok) break;
          qph1 ^= 1u;
          tma_tile(sm->q[1], &tmQ, w1.q_row, w1.bh, &sm->q_full[1]);
        }
        ok = take(&tmS, 0, w0.bh * p.nqg + w0.state_group);
        if (ok && n0 > 0) ok = take(&tmK, e0[0].k_row, w0.bh);
        if (ok && has1) {
          if (!pv.split) ok = take(&tmS, 0, w1.bh * p.nqg + w1.state_group);   // no linear term on split slot 1
          if (ok && n1 > 0 && !shared) ok = take(&tmK, e1[0].k_row, w1.bh);
        }
        const int nmax = n0 > n1 ? n0 : n1;
        for (int j = 0; j < nmax && ok; ++j) {
          if (j < n0) {
            ok = take(&tmV, e0[j].k_row, w0.bh);
            if (ok && j + 1 < n0) ok = take(&tmK, e0[j + 1].k_row, w0.bh);
          }
          if (ok && has1 && !shared && j < n1) {
            ok = take(&tmV, e1[j].k_row, w1.bh);
            if (ok && j + 1 < n1) ok = take(&tmK, e1[j + 1].k_row, w1.bh);
          }
        }
      }
      if (!ok) {
        // drain: wait (bounded) for every load this thread issued
        for (int i = 0; i < NS; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->kv_full[i], (pending_ph >> i) & 1u) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    } else if (warp == MMA_WARP) {
      // the whole warp runs this role (warp-uniform descriptors); one elected lane issues
      int st = 0;
      uint32_t ph = 0, qph0 = 0, qph1 = 0, pph0 = 0, pph1 = 0;
      bool ok = true;
      auto next_stage = [&](int& out) -> bool {
        if (!mbar_wait_warp(&sm->kv_full[st], ph, sm, p.status)) return false;
        tc_fence_after();
        out = st;
        if (++st == NS) { st = 0; ph ^= 1u; }
        return true;
      };
      auto wait_p = [&](uint64_t* bar, uint32_t& phase) -> bool {
        if (!mbar_wait_warp(bar, phase, sm, p.status)) return false;
        phase ^= 1u;
        tc_fence_after();
        return true;
      };
      // Descriptors: start address (>> 4) sits in the low bits, so a K step is an add of a
      // constant; bases are computed once (issue slots on this sub-partition are shared with
      // two softmax warps, so each MMA is kept to an add and the instruction).
      const uint64_t dQ0 = sdesc(smem_u32(sm->q[0]), 16, 1024), dQ1 = sdesc(smem_u32(sm->q[1]), 16, 1024);
      const uint64_t dK0 = sdesc(smem_u32(sm->kv[0]), 16, 1024);
      const uint64_t dV0 = sdesc(smem_u32(sm->kv[0]), HALF_BYTES, 1024);
      constexpr uint64_t kStageStep = TILE_BYTES >> 4;
      auto koff = [](int kk) -> uint64_t { return static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4); };
      auto qk = [&](uint32_t tS, uint64_t dq, int stage, uint64_t* done) {
        const uint64_t dk = dK0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss_elect(tS, dq + koff(kk), dk + koff(kk), kIdescKK, kk > 0);
        mma_commit_elect(done);
      };
      // first = true starts the accumulator (slot 1 of a split pair has no linear term)
      auto pv = [&](uint32_t tO, uint32_t tS, int stage, uint64_t* done, bool first) {
        const uint64_t dv = dV0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_elect(tO, tS + kk * 8, dv + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescKMN, (first && kk == 0) ? 0 : 1);
        mma_commit_elect(done);
      };
      auto linear = [&](uint32_t tO, uint32_t tS, int stage, uint64_t* done) {
        const uint64_t dv = dV0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ts_elect(tO, tS + kk * 8, dv + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescKMN, kk > 0);
        mma_commit_elect(done);
      };
      const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
      for (int pi = blockIdx.x; pi < sm->n_pairs && ok; pi += gridDim.x) {
        const PairView pvw = pair_view(p, pi);
        const bool has1 = pvw.has1, shared = pvw.shared, split = pvw.split;
        const int n0 = pvw.n[0], n1 = pvw.n[1];
        int k0 = -1, k1 = -1, v0 = -1, v1 = -1, sst = -1;
        // slot 0: O0 = phi(Q0) S_rest (S_rest [a][b] is the MN-major B operand), then S0 = Q0 K^T
        ok = wait_p(&sm->p_full[0], pph0) && next_stage(sst);
        if (!ok) break;
        linear(tO0, tS0, sst, &sm->pv_done[0]);
        mma_commit_elect(&sm->kv_empty[sst]);
        ok = mbar_wait_warp(&sm->q_full[0], qph0, sm, p.status);
        if (!ok) break;
        qph0 ^= 1u;
        tc_fence_after();
        if (n0 > 0) {
          ok = next_stage(k0);
          if (!ok) break;
          qk(tS0, dQ0, k0, &sm->s_full[0]);
          if (!shared) mma_commit_elect(&sm->kv_empty[k0]);
        }
        if (n0 <= 1) mma_commit_elect(&sm->q_empty[0]);
        // slot 1
        if (has1) {
          if (!split) {
            ok = wait_p(&sm->p_full[1], pph1) && next_stage(sst);
            if (!ok) break;
            linear(tO1, tS1, sst, &sm->pv_done[1]);
            mma_commit_elect(&sm->kv_empty[sst]);
          }
          ok = mbar_wait_warp(&sm->q_full[1], qph1, sm, p.status);
          if (!ok) break;
          qph1 ^= 1u;
          tc_fence_after();
          if (n1 > 0) {
            if (shared) k1 = k0;
            else if (!(ok = next_stage(k1))) break;
            qk(tS1, dQ1, k1, &sm->s_full[1]);
            mma_commit_elect(&sm->kv_empty[k1]);
          }
          if (n1 <= 1) mma_commit_elect(&sm->q_empty[1]);
        }
        const int nmax = n0 > n1 ? n0 : n1;
        for (int j = 0; j < nmax && ok; ++j) {
          if (j < n0) {
            // the stage waits come first: they are usually satisfied while the softmax still
            // runs, so once P lands the block issues with no wait in between
            if (!(ok = next_stage(v0))) break;
            if (j + 1 < n0 && !(ok = next_stage(k0))) break;
            if (!(ok = wait_p(&sm->p_full[0], pph0))) break;
            pv(tO0, tS0, v0, &sm->pv_done[0], false);
            if (!shared) mma_commit_elect(&sm->kv_empty[v0]);
            if (j + 1 < n0) {
              qk(tS0, dQ0, k0, &sm->s_full[0]);
              if (!shared) mma_commit_elect(&sm->kv_empty[k0]);
              if (j + 2 == n0) mma_commit_elect(&sm->q_empty[0]);
            }
          }
          if (has1 && j < n1) {
            if (shared) {
              v1 = v0;
              k1 = k0;
            } else {
              if (!(ok = next_stage(v1))) break;
              if (j + 1 < n1 && !(ok = next_stage(k1))) break;
            }
            if (!(ok = wait_p(&sm->p_full[1], pph1))) break;
            pv(tO1, tS1, v1, &sm->pv_done[1], split && j == 0);
            mma_commit_elect(&sm->kv_empty[v1]);
            if (j + 1 < n1) {
              qk(tS1, dQ1, k1, &sm->s_full[1]);
              mma_commit_elect(&sm->kv_empty[k1]);
              if (j + 2 == n1) mma_commit_elect(&sm->q_empty[1]);
            }
          }
        }
      }
      // wait for every issued MMA before TMEM is released
      mma_commit_elect(&sm->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------------------------- softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    softmax_role(sm, p, tmem, warp);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (p.n_pairs_dev) redo_finish(p);
}

// ------------------------------------------------------------------ host side
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB a CTA can have");

}  // namespace

bool attn_tc_supported(int d, int dtype) { return d == D && dtype == HYAT_BF16; }

static cudaError_t launch_attn_tc_impl(const AttnArgs& a, int32_t* n_pairs_dev, uint32_t* done_count, int num_sms,
                               cudaStream_t s) {
  if (a.n_pairs == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ms;       // 128-row boxes: two loads of 64 x 128 bf16 = TILE_BYTES
  static_assert(2 * 64 * 128 * 2 == TILE_BYTES, "tile bytes must match the two TMA boxes");
  if (!make_map(&mq, a.q, a.q_rows, a.BH) || !make_map(&mk, a.k, a.k_rows, a.BH) ||
      !make_map(&mv, a.v, a.k_rows, a.BH) || !make_map(&ms, a.srest_bf16, D, int64_t(a.BH) * a.nqg))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[tc::kMaxDevices];
  cudaError_t attr_e = tc::set_smem_attr_once(reinterpret_cast<const void*>(attn_tc_kernel), kSmemBytes, attr_set);
  if (attr_e != cudaSuccess) return attr_e;
  TcParams p{};
  p.work = a.work;
  p.entries = a.entries;
  p.pairs = a.pairs;
  p.n_pairs = a.n_pairs;
  p.srest = a.srest;
  p.o = a.o;
  p.q_rows = a.q_rows;
  p.nqg = a.nqg;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.test_timeout = a.test_timeout;
  p.phi = a.phi;
  p.n_pairs_dev = n_pairs_dev;
  p.done_count = done_count;
  const int grid = a.n_pairs < num_sms ? a.n_pairs : num_sms;
  return launch_pdl(attn_tc_kernel, dim3(grid), dim3(NUM_THREADS), kSmemBytes, s, mq, mk, mv, ms, p);
}

cudaError_t launch_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t s) {
  return launch_attn_tc_impl(a, nullptr, nullptr, num_sms, s);
}

cudaError_t launch_attn_tc_redo(const AttnArgs& a, const int4* redo_items, int32_t* redo_count,
                                uint32_t* done_count, int num_sms, cudaStream_t s) {
  AttnArgs r = a;
  r.pairs = redo_items;
  r.n_pairs = a.n_pairs < num_sms ? a.n_pairs : num_sms;   // grid; the count is read on the device
  return launch_attn_tc_impl(r, redo_count, done_count, num_sms, s);
}

}  // namespace hyat
