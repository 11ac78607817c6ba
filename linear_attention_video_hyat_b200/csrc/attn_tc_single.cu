// Tensor-core hybrid attention for bf16, d = 128, on sm_100a: one query tile per CTA at a
// time, three S buffers.
//
// The method and the accumulator's start are those of attn_tc.cu (ReHyAt, Abstract;
// Hybrid Forcing, Section 2.A): O = phi(Q) S_rest, l = phi(q) . z_rest, then the softmax over
// the window tiles, with one normaliser. The schedule differs:
//   * TMEM holds S0 | S1 | S2 | O (128 columns each). Key tile j of a query tile uses S
//     buffer j mod 3, so Q K^T of tile j + 2 runs while the softmax works on tile j and the
//     P.V of tile j - 1 lands: the tensor pipe does not wait for one softmax at a time;
//   * the two softmax warpgroups take alternate key tiles of the same query tile (warpgroup
//     j mod 2), each with its own partial row sum; the epilogue adds the two sums and each
//     warpgroup normalises and stores 64 columns of O;
//   * exponents use the fixed reference m = 0 (p = 2^(s * scale * log2 e)). A query tile
//     whose row sum leaves the safe fp32 range (>= 2^100 or < 2^-100, inf, NaN) is appended to a redo
//     list, and attn_tc_kernel, which moves its reference max exactly, recomputes it after
//     this kernel. For unit-scale inputs the list stays empty;
//   * phi(Q) (the A operand of the linear-term MMA) sits in S2's first 64 columns until the
//     linear-term MMA has read it; Q K^T of key tile 2 is issued after that MMA.
// Roles: warp 8 TMA (one Q buffer, 6-stage K/V ring), warp 9 MMA (warp-wide, elect.sync
// issue), warps 0-3 and 4-7 the softmax of even and odd key tiles. Every wait is bounded, and
// each barrier is waited on at most one phase behind its arrivals (the argument is given at
// each barrier's first use).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyat_internal.h"
#include "tc_common.cuh"

namespace hyat {
namespace {

using namespace tc;
constexpr int NS1 = 6;                           // K/V stage ring
constexpr int NT1 = 384;                         // 3 warpgroups
// Register split (setmaxnreg): launched at 168 per thread; the softmax warpgroups rise to
// 184 and warpgroup 2 (TMA, MMA) drops to 136: 8 x 32 x 184 + 4 x 32 x 136 = 384 x 168. The
// MMA role's phase bookkeeping for three S buffers needs more than 104.
constexpr int kRegsSm1 = 184;
constexpr int kRegsLm1 = 136;
constexpr float kSafe1 = 1.2676506e30f;          // 2^100
constexpr float kTiny1 = 7.8886091e-31f;          // 2^-100

// instruction descriptor, kind::f16: D f32, A/B bf16, M = 128, N = 128
constexpr uint32_t kIdesc1 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdesc1KK = kIdesc1;               // B K-major
constexpr uint32_t kIdesc1KMN = kIdesc1 | (1u << 16);  // B MN-major

struct __align__(1024) Smem1 {
  uint8_t q[TILE_BYTES];           // one Q buffer: a sixth K/V stage buys more than Q prefetch
  uint8_t kv[NS1][TILE_BYTES];
  uint64_t kv_full[NS1], kv_empty[NS1];
  uint64_t q_full, q_empty;
  uint64_t s_full[3], p_full[3];
  uint64_t phi_full, o_full, o_free, stats;
  uint64_t drain;
  uint64_t never;                  // test hook: a barrier nothing arrives on
  float lsum[2][128];              // each warpgroup's row sums of the current query tile
  uint32_t tmem_base;
  int32_t abort_flag;
  unsigned long long timeout_ns;   // limit of every bounded wait
};

struct SingleParams {
  const WorkItem* work;
  const Entry* entries;
  const int4* items;       // {item, -1, 0, 0} in processing order
  int32_t n_items;
  const float* srest;      // [groups][d*d + d] fp32; z at offset d*d
  void* o;
  int64_t q_rows;
  int32_t nqg;
  float scale_log2;
  uint32_t* status;
  int32_t test_timeout;
  int32_t phi;
  int32_t* redo_count;     // query tiles for attn_tc_kernel to recompute: count, then entries
  int4* redo_items;
};

constexpr uint32_t kSuspend1 = 1000000;
__device__ __forceinline__ bool w1(uint64_t* b, uint32_t parity, Smem1* sm, uint32_t* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_suspend(b, parity, kSuspend1)) return true;
    if (*reinterpret_cast<volatile int32_t*>(&sm->abort_flag)) return false;
    if (globaltimer() - t0 > sm->timeout_ns) {
      atomicOr(status, kStatusTimeout);
      *reinterpret_cast<volatile int32_t*>(&sm->abort_flag) = 1;
      return false;
    }
  }
}
// warp-uniform: the warp proceeds only if every lane saw the phase
__device__ __forceinline__ bool w1warp(uint64_t* b, uint32_t parity, Smem1* sm, uint32_t* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(b, parity))) return true;
  return __all_sync(0xffffffffu, w1(b, parity, sm, status));
}

// p = 2^(s * sl) for this row's 128 scores; P (bf16 pairs) -> TMEM at tS; returns the sum.
__device__ __forceinline__ float exp_row(const uint32_t (&r)[128], float sl, uint32_t tS) {
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float p0 = ex2(u2f(r[h * 64 + 2 * i]) * sl);
      const float p1 = ex2(u2f(r[h * 64 + 2 * i + 1]) * sl);
      acc[(2 * i) & 7] += p0;
      acc[(2 * i + 1) & 7] += p1;
      pk[i] = pack_bf16(p0, p1);
    }
    tmem_st32(tS + h * 32, pk);
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// Fills of S buffer b by a query tile of n key tiles (tile j uses buffer j mod 3).
__device__ __forceinline__ uint32_t fills_of(int n, int b) {
  return n > b ? static_cast<uint32_t>((n - b + 2) / 3) : 0u;
}

// Warpgroup g (warps 4g .. 4g + 3): the softmax of key tiles g, g + 2, ...; warpgroup 1 also
// writes phi(Q) and starts its row sum with the linear term; both share the epilogue.
__device__ __forceinline__ void softmax_single(Smem1* sm, const SingleParams& p, uint32_t tmem, int warp) {
  const int g = warp >> 2;
  const int row = threadIdx.x & 127;
  const int lane = threadIdx.x & 31;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tO = tmem + 384 + lane_off;
  const float sl = p.scale_log2;
  uint32_t f0 = 0, f1 = 0, f2 = 0;   // fills of each S buffer by the query tiles before this one
  uint32_t qph = 0, oph = 0, stph = 0;
  for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
    const int item = p.items[it].x;
    const WorkItem wi = p.work[item];
    const int n = wi.entry_end - wi.entry_begin;
    const Entry* ent = p.entries + wi.entry_begin;
    float l = 0.0f;
    // q_full is waited at most one phase behind: its next phase needs the producer's next Q
    // load, after q_empty, which the MMA commits only after phi_full, which both warpgroups
    // arrive on after this wait.
    if (!w1warp(&sm->q_full, qph, sm, p.status)) return;
    qph ^= 1u;
    if (g == 1) {
      // phi(q) of this row -> S2 columns 0-63 (bf16 pairs); l = phi(q) . z_rest. S2 is free:
      // this warpgroup waited o_full of the previous query tile, after its last MMA.
      const float4 zq = __ldg(reinterpret_cast<const float4*>(
          p.srest + (static_cast<int64_t>(wi.bh) * p.nqg + wi.state_group) * (D * D + D) + D * D) + lane);
      const float zreg[4] = {zq.x, zq.y, zq.z, zq.w};
      const uint8_t* qrow = sm->q + row * 128;
      const uint32_t tPhi = tmem + 256 + lane_off;
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
          const float a0 = phi_map(f.x, p.phi), a1 = phi_map(f.y, p.phi);
          lz[e] = fmaf(a0, zz[2 * e], lz[e]);
          lz[e] = fmaf(a1, zz[2 * e + 1], lz[e]);
          pk[e] = pack_bf16(a0, a1);
        }
        tmem_st4(tPhi + 4 * c, pk);
      }
      l = (lz[0] + lz[1]) + (lz[2] + lz[3]);
      tmem_wait_st();
      tc_fence_before();
    }
    mbar_arrive(&sm->phi_full);
    if (g == 0 && p.test_timeout && !w1warp(&sm->never, 0, sm, p.status)) return;
    for (int j = g; j < n; j += 2) {
      const int b = j % 3;
      const uint32_t tS = tmem + b * 128 + lane_off;
      const int klen = ent[j].k_len;
      // s_full[b]: fill u of buffer b is read by one warpgroup; fill u + 1 (key tile j + 3)
      // needs the MMA to have issued P.V of tile j, after this warpgroup's p_full arrive.
      const uint32_t fb = b == 0 ? f0 : b == 1 ? f1 : f2;
      if (!w1warp(&sm->s_full[b], (fb + static_cast<uint32_t>(j / 3)) & 1u, sm, p.status)) return;
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
      l += exp_row(r, sl, tS);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm->p_full[b]);
    }
    f0 += fills_of(n, 0);
    f1 += fills_of(n, 1);
    f2 += fills_of(n, 2);
    // epilogue. o_full comes first: its next phase needs the linear-term MMA of the next query
    // tile, which waits for o_free, which both warpgroups arrive on after they have read
    // lsum below -- so lsum is never rewritten while the other warpgroup still reads it.
    if (!w1warp(&sm->o_full, oph, sm, p.status)) return;
    oph ^= 1u;
    tc_fence_after();
    sm->lsum[g][row] = l;
    mbar_arrive(&sm->stats);
    if (!w1warp(&sm->stats, stph, sm, p.status)) return;
    stph ^= 1u;
    const float lt = sm->lsum[0][row] + sm->lsum[1][row];
    if (warp == 0) {
      // a row sum out of the safe range: the tile goes to the redo list (once per tile)
      bool bad = false;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = lane + 32 * k;
        const float sum = sm->lsum[0][rr] + sm->lsum[1][rr];
        // too large (overflow ahead), or too small: with no linear term a row whose logits
        // all lie far below 0 flushes its exponentials to zero
        bad |= rr < wi.q_len && !(sum < kSafe1 && sum >= kTiny1);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) {
        const int k = atomicAdd(p.redo_count, 1);
        if (k < p.n_items) p.redo_items[k] = make_int4(item, -1, 0, 0);
        else atomicOr(p.status, kStatusBadTile);
      }
    }
    const float inv = 1.0f / lt;
    uint32_t o[64];
    tmem_ld32p(tO + g * 64, o);
    tmem_ld32p(tO + g * 64 + 32, o + 32);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&sm->o_free);          // O may be overwritten once both warpgroups are here
    if (row < wi.q_len) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                            (static_cast<int64_t>(wi.bh) * p.q_rows + wi.q_row + row) * D) + g * 8;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        uint4 w;
        w.x = pack_bf16(u2f(o[8 * v + 0]) * inv, u2f(o[8 * v + 1]) * inv);
        w.y = pack_bf16(u2f(o[8 * v + 2]) * inv, u2f(o[8 * v + 3]) * inv);
        w.z = pack_bf16(u2f(o[8 * v + 4]) * inv, u2f(o[8 * v + 5]) * inv);
        w.w = pack_bf16(u2f(o[8 * v + 6]) * inv, u2f(o[8 * v + 7]) * inv);
        dst[v] = w;
      }
    }
  }
}

__global__ void __launch_bounds__(NT1, 1)
    attn_single_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                       const SingleParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem1* sm = reinterpret_cast<Smem1*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS1; ++i) {
      mbar_init(&sm->kv_full[i], 1);
      mbar_init(&sm->kv_empty[i], 1);
    }
    mbar_init(&sm->q_full, 1);
    mbar_init(&sm->q_empty, 1);
    for (int b = 0; b < 3; ++b) {
      mbar_init(&sm->s_full[b], 1);
      mbar_init(&sm->p_full[b], 128);
    }
    mbar_init(&sm->phi_full, 256);
    mbar_init(&sm->o_full, 1);
    mbar_init(&sm->o_free, 256);
    mbar_init(&sm->stats, 256);
    mbar_init(&sm->drain, 1);
    mbar_init(&sm->never, 1);
    sm->abort_flag = 0;
    sm->timeout_ns = p.test_timeout ? 20000000ull : kTimeoutNs;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  pdl_wait();                // the linear states come from the kernels launched before this one

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLm1));
    if (warp == 8 && lane == 0) {
      // TMA producer. Stage order of a query tile: K0, K1, S_rest, K2, then V(j), K(j + 3)
      // for j = 0 .. n - 1 -- the order in which the MMA role consumes them.
      int st = 0;
      uint32_t ph = 0, pending = 0, pending_ph = 0;   // stages with a load in flight, and its phase
      uint32_t qeph = 0;
      bool ok = true;
      auto take = [&](const CUtensorMap* tm, int row, int z) -> bool {
        if (!w1(&sm->kv_empty[st], ph ^ 1u, sm, p.status)) return false;
        tma_tile(sm->kv[st], tm, row, z, &sm->kv_full[st]);
        pending |= 1u << st;
        pending_ph = (pending_ph & ~(1u << st)) | (ph << st);
        if (++st == NS1) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
        const WorkItem wi = p.work[p.items[it].x];
        const int n = wi.entry_end - wi.entry_begin;
        const Entry* e = p.entries + wi.entry_begin;
        // K0, K1 into the ring first: the single Q buffer frees only after the previous query
        // tile's last Q K^T
        if (n > 0) ok = take(&tmK, e[0].k_row, wi.bh);
        if (ok && n > 1) ok = take(&tmK, e[1].k_row, wi.bh);
        if (!ok || !(ok = w1(&sm->q_empty, qeph ^ 1u, sm, p.status))) break;
        qeph ^= 1u;
        tma_tile(sm->q, &tmQ, wi.q_row, wi.bh, &sm->q_full);
        if (ok) ok = take(&tmS, 0, wi.bh * p.nqg + wi.state_group);
        if (ok && n > 2) ok = take(&tmK, e[2].k_row, wi.bh);
        for (int j = 0; j < n && ok; ++j) {
          ok = take(&tmV, e[j].k_row, wi.bh);
          if (ok && j + 3 < n) ok = take(&tmK, e[j + 3].k_row, wi.bh);
        }
      }
      if (!ok) {
        // aborting: let the copies in flight land before the CTA exits (bounded)
        for (int i = 0; i < NS1; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->kv_full[i], (pending_ph >> i) & 1u) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    } else if (warp == 9) {
      // MMA role: the whole warp runs it, one elected lane issues
      int st = 0;
      uint32_t ph = 0, phph = 0, ofph = 0;
      uint32_t qph = 0;
      uint32_t pf0 = 0, pf1 = 0, pf2 = 0;  // fills of each S buffer by earlier query tiles
      bool ok = true;
      bool first = true;
      auto next_stage = [&](int& out) -> bool {
        if (!__all_sync(0xffffffffu, w1(&sm->kv_full[st], ph, sm, p.status))) return false;
        tc_fence_after();
        out = st;
        if (++st == NS1) { st = 0; ph ^= 1u; }
        return true;
      };
      const uint64_t dK0 = sdesc(smem_u32(sm->kv[0]), 16, 1024);
      const uint64_t dV0 = sdesc(smem_u32(sm->kv[0]), HALF_BYTES, 1024);
      constexpr uint64_t kStageStep = TILE_BYTES >> 4;
      auto koff = [](int kk) -> uint64_t { return static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4); };
      auto qk = [&](uint32_t tS, uint64_t dq, int stage) {
        const uint64_t dk = dK0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss_elect(tS, dq + koff(kk), dk + koff(kk), kIdesc1KK, kk > 0);
      };
      // O (+)= A . B, A = 64 TMEM columns of bf16 pairs (P or phi(Q)), B = the stage as MN-major
      auto pv = [&](uint32_t tD, uint32_t tA, int stage, bool init) {
        const uint64_t dv = dV0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_elect(tD, tA + kk * 8, dv + static_cast<uint64_t>(kk * (2048 >> 4)), kIdesc1KMN,
                       (init && kk == 0) ? 0 : 1);
      };
      const uint32_t tO = tmem + 384, tPhi = tmem + 256;
      for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
        const WorkItem wi = p.work[p.items[it].x];
        const int n = wi.entry_end - wi.entry_begin;
        const uint64_t dq = sdesc(smem_u32(sm->q), 16, 1024);
        if (!(ok = __all_sync(0xffffffffu, w1(&sm->q_full, qph, sm, p.status)))) break;
        qph ^= 1u;
        tc_fence_after();
        int k0 = -1, k1 = -1, k2 = -1, sst = -1;
        // Q K^T of key tiles 0 and 1 into S0 and S1. They are free: every MMA of the previous
        // query tile that reads them was issued before, and the pipe executes in order.
        if (n > 0) {
          if (!(ok = next_stage(k0))) break;
          qk(tmem + 0, dq, k0);
          mma_commit_elect(&sm->s_full[0]);
          mma_commit_elect(&sm->kv_empty[k0]);
        }
        if (n > 1) {
          if (!(ok = next_stage(k1))) break;
          qk(tmem + 128, dq, k1);
          mma_commit_elect(&sm->s_full[1]);
          mma_commit_elect(&sm->kv_empty[k1]);
        }
        // The linear term starts O: phi(Q) (in S2) times S_rest, once both warpgroups have
        // read out the previous O. phi_full and o_free are each waited at most one phase
        // behind: their next phases need o_full of this query tile, committed below.
        if (!(ok = next_stage(sst))) break;
        if (!(ok = __all_sync(0xffffffffu, w1(&sm->phi_full, phph, sm, p.status)))) break;
        phph ^= 1u;
        if (!first) {
          if (!(ok = __all_sync(0xffffffffu, w1(&sm->o_free, ofph, sm, p.status)))) break;
          ofph ^= 1u;
        }
        first = false;
        tc_fence_after();
        pv(tO, tPhi, sst, true);
        mma_commit_elect(&sm->kv_empty[sst]);
        if (n > 2) {
          if (!(ok = next_stage(k2))) break;
          qk(tmem + 256, dq, k2);
          mma_commit_elect(&sm->s_full[2]);
          mma_commit_elect(&sm->kv_empty[k2]);
        }
        if (n <= 3) mma_commit_elect(&sm->q_empty);
        for (int j = 0; j < n && ok; ++j) {
          const int b = j % 3;
          int v = -1, kn = -1;
          // V(j) and P(j), then P.V; only then wait for K(j + 3), so a late K load does not hold
          // back the P.V. p_full[b] is waited at most one phase behind: its next phase needs the
          // S of key tile j + 3, which this warp issues below.
          if (!(ok = next_stage(v))) break;
          const uint32_t fb = b == 0 ? pf0 : b == 1 ? pf1 : pf2;
          if (!(ok = __all_sync(0xffffffffu, w1(&sm->p_full[b], (fb + static_cast<uint32_t>(j / 3)) & 1u, sm, p.status))))
            break;
          tc_fence_after();
          pv(tO, tmem + b * 128, v, false);
          mma_commit_elect(&sm->kv_empty[v]);
          if (j + 3 < n) {
            if (!(ok = next_stage(kn))) break;
            qk(tmem + b * 128, dq, kn);
            mma_commit_elect(&sm->s_full[b]);
            mma_commit_elect(&sm->kv_empty[kn]);
            if (j + 4 == n) mma_commit_elect(&sm->q_empty);
          }
        }
        if (!ok) break;
        mma_commit_elect(&sm->o_full);
        pf0 += fills_of(n, 0);
        pf1 += fills_of(n, 1);
        pf2 += fills_of(n, 2);
      }
      mma_commit_elect(&sm->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
      }
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSm1));
    softmax_single(sm, p, tmem, warp);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

constexpr size_t kSmem1Bytes = sizeof(Smem1) + 1024;
static_assert(kSmem1Bytes <= 232448, "shared memory above the 227 KB a CTA can have");

}  // namespace

cudaError_t launch_attn_single(const AttnArgs& a, int32_t* redo_count, int4* redo_items, int num_sms,
                               cudaStream_t s) {
  if (a.n_pairs == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ms;
  if (!make_map(&mq, a.q, a.q_rows, a.BH) || !make_map(&mk, a.k, a.k_rows, a.BH) ||
      !make_map(&mv, a.v, a.k_rows, a.BH) || !make_map(&ms, a.srest_bf16, D, int64_t(a.BH) * a.nqg))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[tc::kMaxDevices];
  cudaError_t attr_e = tc::set_smem_attr_once(reinterpret_cast<const void*>(attn_single_kernel), kSmem1Bytes, attr_set);
  if (attr_e != cudaSuccess) return attr_e;
  SingleParams p{};
  p.work = a.work;
  p.entries = a.entries;
  p.items = a.pairs;
  p.n_items = a.n_pairs;
  p.srest = a.srest;
  p.o = a.o;
  p.q_rows = a.q_rows;
  p.nqg = a.nqg;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.test_timeout = a.test_timeout;
  p.phi = a.phi;
  p.redo_count = redo_count;
  p.redo_items = redo_items;
  const int grid = a.n_pairs < num_sms ? a.n_pairs : num_sms;
  return launch_pdl(attn_single_kernel, dim3(grid), dim3(NT1), kSmem1Bytes, s, mq, mk, mv, ms, p);
}

}  // namespace hyat
