// Tensor-core hybrid attention for bf16, d = 128, on sm_100a: the pair schedule with two
// softmax warps per row.
//
// The method and the accumulator's start are those of attn_tc.cu (ReHyAt, Abstract; Hybrid
// Forcing, Section 2.A): O = phi(Q) S_rest, l = phi(q) . z_rest, then the softmax over the
// window tiles, with one normaliser. A CTA owns a pair of query tiles ("slots") as there, with
// the same TMA producer, MMA issue order, TMEM layout (S0 | S1 | O0 | O1) and pair schedule
// (shared key lists, split pairs). What differs is the softmax:
//   * each slot has two warpgroups; warp w of a slot's first warpgroup and warp w of its
//     second share an SM sub-partition and a TMEM lane quarter, and split each row's 128 keys:
//     the first takes keys 0-63, the second keys 64-127. With one warp per row the exp phase
//     of a tile ran a sub-partition's MUFU at about two thirds of its rate; two warps keep it
//     busier, which shortens each slot's softmax -> P.V -> Q.K^T chain;
//   * a thread's P (bf16 pairs) overwrites the first half of its own S columns (keys 0-63 go
//     to S columns 0-31, keys 64-127 to columns 64-95), so neither half writes where the other
//     still has to read; the P.V and linear-term MMAs address the two halves of the A operand
//     accordingly. phi(Q) (the linear term's A operand) is laid out the same way;
//   * exponents use the fixed reference m = 0 (p = 2^(s * scale * log2 e)), so the two halves
//     of a row need no common running max. A row whose sum leaves [2^-100, 2^100) (scores far
//     above 0, or every score far below 0 with no linear term) marks its query tile for the
//     redo list, and attn_tc_kernel, which moves its reference max, recomputes those tiles
//     after this kernel. For the workloads' unit-scale inputs the list stays empty;
//   * the epilogue adds the two halves' row sums through shared memory, and each thread
//     normalises and stores its 64 columns of O (the split-pair merge adds slot 1's halves).
// Roles: warps 0-7 slot 0, warps 8-15 slot 1 (softmax), warp 16 TMA, warp 17 MMA (warp-wide,
// elect.sync issue), warps 18-19 idle. Every mbarrier wait is bounded (%globaltimer).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyat_internal.h"
#include "tc_common.cuh"

namespace hyat {
namespace {

using namespace tc;
constexpr int NSW = 5;                           // K/V stage ring
constexpr int NTW = 640;                         // 5 warpgroups
constexpr int TMA_WARP = 16, MMA_WARP_W = 17;
constexpr float kSafeW = 1.2676506e30f;          // 2^100
constexpr float kTinyW = 7.8886091e-31f;         // 2^-100

// instruction descriptor, kind::f16: D f32, A/B bf16, M = 128, N = 128
constexpr uint32_t kIdescW = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescWKK = kIdescW;               // B K-major
constexpr uint32_t kIdescWKMN = kIdescW | (1u << 16);  // B MN-major

struct __align__(1024) SmemW {
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[NSW][TILE_BYTES];
  uint64_t kv_full[NSW], kv_empty[NSW];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t xfull, o1_free;       // split pairs: slot 1's row sums handed over; O1 read out
  uint64_t ex1[2], ex2[2];       // per slot: the second half's row sum written; the total written
  uint64_t drain;
  uint64_t never;                // test hook: a barrier nothing arrives on
  float lsum[2][128];            // [slot][row]: the second half's row sum, then the row total
  int32_t bad[2][2];             // [slot][pair parity]: a row of the tile left the safe range
  uint32_t tmem_base;
  int32_t abort_flag;
  unsigned long long timeout_ns;
};

struct WideParams {
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
  int32_t test_timeout;
  int32_t phi;
  int32_t* redo_count;     // query tiles for attn_tc_kernel to recompute: count, then entries
  int4* redo_items;
  int32_t redo_cap;
};

__device__ __forceinline__ bool wwait(uint64_t* b, uint32_t parity, SmemW* sm, uint32_t* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_suspend(b, parity, 1000000u)) return true;
    if (*reinterpret_cast<volatile int32_t*>(&sm->abort_flag)) return false;
    if (globaltimer() - t0 > sm->timeout_ns) {
      atomicOr(status, kStatusTimeout);
      *reinterpret_cast<volatile int32_t*>(&sm->abort_flag) = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool wwait_warp(uint64_t* b, uint32_t parity, SmemW* sm, uint32_t* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(b, parity))) return true;
  return __all_sync(0xffffffffu, wwait(b, parity, sm, status));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// p = 2^(s * sl) for 32 scores; P (bf16 pairs) -> 16 TMEM columns at tP. Returns the sum.
__device__ __forceinline__ float exp32(const uint32_t* r, float sl, uint32_t tP) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float p0 = ex2(u2f(r[2 * i]) * sl);
    const float p1 = ex2(u2f(r[2 * i + 1]) * sl);
    acc[(2 * i) & 3] += p0;
    acc[(2 * i + 1) & 3] += p1;
    pk[i] = pack_bf16(p0, p1);
  }
  tmem_st16(tP, pk);
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

struct PairViewW {
  int item[2];
  int eb[2];
  int n[2];
  bool has1, shared, split;
};

__device__ __forceinline__ PairViewW pair_view_w(const WideParams& p, int pi) {
  const int4 pr = p.pairs[pi];
  PairViewW v;
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

// The softmax of slot s, keys hf * 64 .. hf * 64 + 63 of row `row` (TMEM lane).
__device__ __forceinline__ void softmax_wide(SmemW* sm, const WideParams& p, uint32_t tmem, int warp) {
  const int s = warp >> 3, hf = (warp >> 2) & 1;
  const int lane = threadIdx.x & 31;
  const int row = (warp & 3) * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tS = tmem + s * 128 + lane_off;
  const uint32_t tMine = tS + hf * 64;           // this thread's S columns; P goes to the first 32
  const uint32_t tO = tmem + 256 + s * 128 + lane_off;
  uint64_t* q_full = &sm->q_full[s];
  uint64_t* s_full = &sm->s_full[s];
  uint64_t* p_full = &sm->p_full[s];
  uint64_t* pv_done = &sm->pv_done[s];
  const float sl = p.scale_log2;
  uint32_t qph = 0, sph = 0, xph = 0, pv_phase = 0, par = 0, e1ph = 0, e2ph = 0;
  bool o1_busy = false;
  for (int pi = blockIdx.x; pi < p.n_pairs; pi += gridDim.x) {
    const PairViewW pv = pair_view_w(p, pi);
    if (s == 1 && !pv.has1) continue;
    const WorkItem wi = p.work[s == 0 ? pv.item[0] : pv.item[1]];
    const int n = s == 0 ? pv.n[0] : pv.n[1];
    const Entry* ent = p.entries + (s == 0 ? pv.eb[0] : pv.eb[1]);
    const bool lin = !(pv.split && s == 1);
    int klen_next = n > 0 ? ent[0].k_len : 128;
    if (!wwait_warp(q_full, qph, sm, p.status)) return;
    qph ^= 1u;
    if (o1_busy) {
      // O1 is rewritten by this slot's first P.V: wait until slot 0 has read out the previous
      // split pair's O1 and row sums
      if (!wwait_warp(&sm->o1_free, xph ^ 1u, sm, p.status)) return;
      o1_busy = false;
    }
    float l = 0.0f;
    if (lin) {
      // phi(q) of this row's features hf * 64 .. + 63 -> TMEM (bf16 pairs), l = phi(q) . z
      const float4 zq = __ldg(reinterpret_cast<const float4*>(
          p.srest + (static_cast<int64_t>(wi.bh) * p.nqg + wi.state_group) * (D * D + D) + D * D) + lane);
      const float zreg[4] = {zq.x, zq.y, zq.z, zq.w};
      const uint8_t* qrow = sm->q[s] + row * 128;
      float lz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int cc = 0; cc < 8; ++cc) {           // 8 features per step
        const int c = hf * 8 + cc;
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
        tmem_st4(tMine + 4 * cc, pk);
      }
      l = (lz[0] + lz[1]) + (lz[2] + lz[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);        // one arrival per warp (its stores are done)
    }
    if (s == 0 && hf == 0 && p.test_timeout && !wwait_warp(&sm->never, 0, sm, p.status)) return;
    for (int j = 0; j < n; ++j) {
      const int klen = klen_next;
      if (j + 1 < n) klen_next = ent[j + 1].k_len;
      if (!wwait_warp(s_full, sph, sm, p.status)) return;
      sph ^= 1u;
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32p(tMine, r);
      tmem_ld32p(tMine + 32, r + 32);
      tmem_wait_ld();
      if (klen < 128) {
        const int lim = klen - hf * 64;
#pragma unroll
        for (int i = 0; i < 64; ++i) r[i] = i < lim ? r[i] : 0xff800000u;   // -inf
      }
      // keys hf * 64 + 0..31 -> P columns 0..15 of this thread's S columns, + 32..63 -> 16..31
      // (both were read into registers above)
      const float rs = exp32(r, sl, tMine) + exp32(r + 32, sl, tMine + 16);
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);        // one arrival per warp (its stores are done)
    }
    const uint32_t n_commits = static_cast<uint32_t>(n) + (lin ? 1u : 0u);
    if (!wwait_warp(pv_done, (pv_phase + n_commits - 1) & 1u, sm, p.status)) return;
    pv_phase += n_commits;
    tc_fence_after();
    // The halves' row sums meet in shared memory: the second half writes its sum, the first
    // half adds its own (and, for a split pair's slot 0, slot 1's total) and writes the total
    // back. The waits are bounded mbarrier waits, so a thread that gives up elsewhere cannot
    // leave the others blocked here.
    if (hf == 1) sm->lsum[s][row] = l;
    mbar_arrive(&sm->ex1[s]);
    if (!wwait_warp(&sm->ex1[s], e1ph, sm, p.status)) return;
    e1ph ^= 1u;
    if (pv.split && s == 1) {
      // slot 1 hands its row totals and O1 to slot 0, which merges and stores the tile
      if (hf == 0) {
        sm->lsum[1][row] = l + sm->lsum[1][row];
        tc_fence_before();
        mbar_arrive(&sm->xfull);
      }
      xph ^= 1u;
      o1_busy = true;
      continue;
    }
    float lt = 0.0f;
    if (hf == 0) {
      lt = l + sm->lsum[s][row];
      if (pv.split) {
        if (!wwait_warp(&sm->xfull, xph, sm, p.status)) return;
        tc_fence_after();
        lt += sm->lsum[1][row];
      }
      sm->lsum[s][row] = lt;
      if (row < wi.q_len && !(lt < kSafeW && lt >= kTinyW)) sm->bad[s][par] = 1;
    }
    if (pv.split) xph ^= 1u;
    tc_fence_before();
    mbar_arrive(&sm->ex2[s]);
    if (!wwait_warp(&sm->ex2[s], e2ph, sm, p.status)) return;
    e2ph ^= 1u;
    tc_fence_after();                    // O (and for split pairs O1) is read below
    if (hf == 1) lt = sm->lsum[s][row];
    if (hf == 0 && row == 0) {
      if (sm->bad[s][par]) {
        // the tile goes to the redo list (once; its output is rewritten there)
        const int k = atomicAdd(p.redo_count, 1);
        if (k < p.redo_cap) p.redo_items[k] = make_int4(s == 0 ? pv.item[0] : pv.item[1], -1, 0, 0);
        else atomicOr(p.status, kStatusBadTile);
        sm->bad[s][par] = 0;
      }
    }
    par ^= 1u;
    // epilogue: o = O / l (plus slot 1's O1 for split pairs), bf16, 16-byte stores, 64 columns
    const float inv = 1.0f / lt;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                          (static_cast<int64_t>(wi.bh) * p.q_rows + wi.q_row + row) * D + hf * 64);
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {                 // 32 columns at a time
      uint32_t o[32];
      tmem_ld32p(tO + hf * 64 + h * 32, o);
      if (pv.split) {
        uint32_t o1[32];
        tmem_ld32p(tO + 128 + hf * 64 + h * 32, o1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) + u2f(o1[i]));
      } else {
        tmem_wait_ld();
      }
      if (row < wi.q_len) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          w.x = pack_bf16(u2f(o[8 * v + 0]) * inv, u2f(o[8 * v + 1]) * inv);
          w.y = pack_bf16(u2f(o[8 * v + 2]) * inv, u2f(o[8 * v + 3]) * inv);
          w.z = pack_bf16(u2f(o[8 * v + 4]) * inv, u2f(o[8 * v + 5]) * inv);
          w.w = pack_bf16(u2f(o[8 * v + 6]) * inv, u2f(o[8 * v + 7]) * inv);
          dst[h * 4 + v] = w;
        }
      }
    }
    tc_fence_before();
    if (pv.split) mbar_arrive(&sm->o1_free);
  }
}

__global__ void __launch_bounds__(NTW, 1)
    attn_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                     const WideParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemW* sm = reinterpret_cast<SmemW*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NSW; ++i) {
      mbar_init(&sm->kv_full[i], 1);
      mbar_init(&sm->kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm->q_full[s], 1);
      mbar_init(&sm->q_empty[s], 1);
      mbar_init(&sm->s_full[s], 1);
      mbar_init(&sm->p_full[s], 8);             // one arrival per softmax warp of the slot
      mbar_init(&sm->pv_done[s], 1);
      mbar_init(&sm->ex1[s], 256);
      mbar_init(&sm->ex2[s], 256);
      sm->bad[s][0] = sm->bad[s][1] = 0;
    }
    mbar_init(&sm->xfull, 128);
    mbar_init(&sm->o1_free, 256);
    mbar_init(&sm->drain, 1);
    mbar_init(&sm->never, 1);
    sm->abort_flag = 0;
    sm->timeout_ns = p.test_timeout ? 20000000ull : kTimeoutNs;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == MMA_WARP_W) {
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

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, qph0 = 0, qph1 = 0, pending = 0, pending_ph = 0;
      bool ok = true;
      auto take = [&](const CUtensorMap* tm, int row, int z) -> bool {
        if (!wwait(&sm->kv_empty[st], ph ^ 1u, sm, p.status)) return false;
        tma_tile(sm->kv[st], tm, row, z, &sm->kv_full[st]);
        pending |= 1u << st;
        pending_ph = (pending_ph & ~(1u << st)) | (ph << st);
        if (++st == NSW) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int pi = blockIdx.x; pi < p.n_pairs && ok; pi += gridDim.x) {
        const PairViewW pv = pair_view_w(p, pi);
        const bool has1 = pv.has1, shared = pv.shared;
        const WorkItem w0 = p.work[pv.item[0]];
        const WorkItem w1 = has1 ? p.work[pv.item[1]] : w0;
        const int n0 = pv.n[0], n1 = pv.n[1];
        const Entry* e0 = p.entries + pv.eb[0];
        const Entry* e1 = p.entries + pv.eb[1];
        if (!(ok = wwait(&sm->q_empty[0], qph0 ^ 1u, sm, p.status))) break;
        qph0 ^= 1u;
        tma_tile(sm->q[0], &tmQ, w0.q_row, w0.bh, &sm->q_full[0]);
        if (has1) {
          if (!(ok = wwait(&sm->q_empty[1], qph1 ^ 1u, sm, p.status))) break;
          qph1 ^= 1u;
          tma_tile(sm->q[1], &tmQ, w1.q_row, w1.bh, &sm->q_full[1]);
        }
        ok = take(&tmS, 0, w0.bh * p.nqg + w0.state_group);
        if (ok && n0 > 0) ok = take(&tmK, e0[0].k_row, w0.bh);
        if (ok && has1) {
          if (!pv.split) ok = take(&tmS, 0, w1.bh * p.nqg + w1.state_group);
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
        for (int i = 0; i < NSW; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->kv_full[i], (pending_ph >> i) & 1u) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == MMA_WARP_W) {
    int st = 0;
    uint32_t ph = 0, qph0 = 0, qph1 = 0, pph0 = 0, pph1 = 0;
    bool ok = true;
    auto next_stage = [&](int& out) -> bool {
      if (!wwait_warp(&sm->kv_full[st], ph, sm, p.status)) return false;
      tc_fence_after();
      out = st;
      if (++st == NSW) { st = 0; ph ^= 1u; }
      return true;
    };
    auto wait_p = [&](uint64_t* bar, uint32_t& phase) -> bool {
      if (!wwait_warp(bar, phase, sm, p.status)) return false;
      phase ^= 1u;
      tc_fence_after();
      return true;
    };
    const uint64_t dQ0 = sdesc(smem_u32(sm->q[0]), 16, 1024), dQ1 = sdesc(smem_u32(sm->q[1]), 16, 1024);
    const uint64_t dK0 = sdesc(smem_u32(sm->kv[0]), 16, 1024);
    const uint64_t dV0 = sdesc(smem_u32(sm->kv[0]), HALF_BYTES, 1024);
    constexpr uint64_t kStageStep = TILE_BYTES >> 4;
    auto koff = [](int kk) -> uint64_t { return static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4); };
    auto qk = [&](uint32_t tS, uint64_t dq, int stage, uint64_t* done) {
      const uint64_t dk = dK0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) mma_ss_elect(tS, dq + koff(kk), dk + koff(kk), kIdescWKK, kk > 0);
      mma_commit_elect(done);
    };
    // O (+)= A . B: A = the slot's P (or phi(Q)), 16 keys (features) per MMA, keys 0-63 in S
    // columns 0-31 and keys 64-127 in S columns 64-95; B = the stage as MN-major
    auto pv = [&](uint32_t tO, uint32_t tS, int stage, uint64_t* done, bool init) {
      const uint64_t dv = dV0 + static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_elect(tO, tS + kk * 8 + (kk >= 4 ? 32 : 0), dv + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescWKMN,
                     (init && kk == 0) ? 0 : 1);
      mma_commit_elect(done);
    };
    const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
    for (int pi = blockIdx.x; pi < p.n_pairs && ok; pi += gridDim.x) {
      const PairViewW pvw = pair_view_w(p, pi);
      const bool has1 = pvw.has1, shared = pvw.shared, split = pvw.split;
      const int n0 = pvw.n[0], n1 = pvw.n[1];
      int k0 = -1, k1 = -1, v0 = -1, v1 = -1, sst = -1;
      ok = wait_p(&sm->p_full[0], pph0) && next_stage(sst);
      if (!ok) break;
      pv(tO0, tS0, sst, &sm->pv_done[0], true);       // O0 = phi(Q0) S_rest
      mma_commit_elect(&sm->kv_empty[sst]);
      if (!(ok = wwait_warp(&sm->q_full[0], qph0, sm, p.status))) break;
      qph0 ^= 1u;
      tc_fence_after();
      if (n0 > 0) {
        if (!(ok = next_stage(k0))) break;
        qk(tS0, dQ0, k0, &sm->s_full[0]);
        if (!shared) mma_commit_elect(&sm->kv_empty[k0]);
      }
      if (n0 <= 1) mma_commit_elect(&sm->q_empty[0]);
      if (has1) {
        if (!split) {
          ok = wait_p(&sm->p_full[1], pph1) && next_stage(sst);
          if (!ok) break;
          pv(tO1, tS1, sst, &sm->pv_done[1], true);
          mma_commit_elect(&sm->kv_empty[sst]);
        }
        if (!(ok = wwait_warp(&sm->q_full[1], qph1, sm, p.status))) break;
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
    mma_commit_elect(&sm->drain);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
    }
    __syncwarp();
  } else if (warp < 16) {
    softmax_wide(sm, p, tmem, warp);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP_W) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

constexpr size_t kSmemWBytes = sizeof(SmemW) + 1024;
static_assert(kSmemWBytes <= 232448, "shared memory above the 227 KB a CTA can have");

}  // namespace

cudaError_t launch_attn_wide(const AttnArgs& a, int32_t* redo_count, int4* redo_items, int32_t redo_cap, int num_sms,
                             cudaStream_t s) {
  if (a.n_pairs == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ms;
  if (!make_map(&mq, a.q, a.q_rows, a.BH) || !make_map(&mk, a.k, a.k_rows, a.BH) ||
      !make_map(&mv, a.v, a.k_rows, a.BH) || !make_map(&ms, a.srest_bf16, D, int64_t(a.BH) * a.nqg))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[tc::kMaxDevices];
  cudaError_t attr_e = tc::set_smem_attr_once(reinterpret_cast<const void*>(attn_wide_kernel), kSmemWBytes, attr_set);
  if (attr_e != cudaSuccess) return attr_e;
  WideParams p{};
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
  p.redo_count = redo_count;
  p.redo_items = redo_items;
  p.redo_cap = redo_cap;
  const int grid = a.n_pairs < num_sms ? a.n_pairs : num_sms;
  return launch_pdl(attn_wide_kernel, dim3(grid), dim3(NTW), kSmemWBytes, s, mq, mk, mv, ms, p);
}

}  // namespace hyat
