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
//     ("slots"), so the softmax of one slot overlaps the MMAs of the other;
//   * warp 8 issues TMA loads (Q tiles, K/V tiles, S_rest^T) into 128B-swizzled
//     shared memory through a 5-stage ring; warp 9 issues tcgen05.mma (one
//     thread) with fp32 accumulators in TMEM; warps 0-3 / 4-7 run the softmax
//     of slot 0 / 1, one query row per thread, reading S from TMEM and writing
//     P (bf16) back into TMEM, where it is the A operand of the P.V MMA;
//   * TMEM (512 columns): S0 | S1 | O0 | O1, each 128 columns; P and phi(Q)
//     alias the first 64 columns of S;
//   * the running max is only moved when it grows by more than 8 (log2
//     units): the rescale of O in TMEM is rare and the result is exact;
//   * every mbarrier wait is bounded (%globaltimer); a wait that gives up sets
//     the status word, and all roles drain and free TMEM before exiting.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "hyat_internal.h"

namespace hyat {
namespace {

constexpr int D = 128;
constexpr int TILE_BYTES = 128 * D * 2;          // one 128 x 128 bf16 tile
constexpr int HALF_BYTES = TILE_BYTES / 2;       // 64 columns (128 B rows)
constexpr int NS = 5;                            // K/V stage ring
constexpr int NUM_THREADS = 320;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr float kRescaleThreshold = 8.0f;        // log2 units
constexpr unsigned long long kTimeoutNs = 2000000000ull;

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
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct TcParams {
  const WorkItem* work;
  const Entry* entries;
  const int4* pairs;       // {item0, item1 (-1 = none), shared key list, 0}
  int32_t n_pairs;
  const float* srest;      // [groups][d*d + d] fp32; z at offset d*d
  void* o;
  int64_t q_rows;
  int32_t nqg;
  float scale_log2;
  uint32_t* status;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on a phase parity. Returns false if the kernel is aborting.
__device__ __noinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Smem* sm, uint32_t* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(b, parity)) return true;
    if ((it & 63u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&sm->abort_flag)) return false;
      if (globaltimer() - t0 > kTimeoutNs) {
        atomicOr(status, kStatusTimeout);
        *reinterpret_cast<volatile int32_t*>(&sm->abort_flag) = 1;
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if all lanes saw
// the phase (the TMEM instructions that follow are .sync.aligned).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* b, uint32_t parity, Smem* sm, uint32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait(b, parity, sm, status));
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// a 128-row x 128-column bf16 tile = two boxes of 64 columns (128-byte rows)
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* tm, int row, int z, uint64_t* bar) {
  mbar_expect_tx(bar, TILE_BYTES);
  tma_load_3d(smem_u32(dst), tm, 0, row, z, bar);
  tma_load_3d(smem_u32(dst + HALF_BYTES), tm, 64, row, z, bar);
}

// shared-memory matrix descriptor, 128-byte swizzle, sm100 version bits
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand (rows = M or N, 128 columns of K in two 64-column halves); K step kk of 16
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk) {
  return sdesc(base + (kk >> 2) * HALF_BYTES + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K, 128 columns of N in two 64-column halves); K step kk of 16 rows
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int kk) {
  return sdesc(base + kk * 2048, HALF_BYTES, 1024);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#define HYAT_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define HYAT_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : HYAT_R8(0), HYAT_R8(8), HYAT_R8(16), HYAT_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      HYAT_W8(0), HYAT_W8(8), HYAT_W8(16), HYAT_W8(24)
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float phi_elu1(float x) {
  return x > 0.0f ? x + 1.0f : ex2(x * 1.4426950408889634f);
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                   const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm->kv_full[i], 1);
      mbar_init(&sm->kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm->q_full[s], 1);
      mbar_init(&sm->q_empty[s], 1);
      mbar_init(&sm->s_full[s], 1);
      mbar_init(&sm->p_full[s], 128);
      mbar_init(&sm->pv_done[s], 1);
    }
    mbar_init(&sm->drain, 1);
    sm->abort_flag = 0;
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

  if (warp == PRODUCER_WARP) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int st = 0;
      uint32_t ph = 0;
      uint32_t qph[2] = {0, 0};
      uint32_t pending = 0;               // stages holding a load not yet seen complete
      uint32_t pending_ph[NS];
      bool ok = true;
      auto take = [&](const CUtensorMap* tm, int row, int z) -> bool {
        if (!mbar_wait(&sm->kv_empty[st], ph ^ 1u, sm, p.status)) return false;
        tma_tile(sm->kv[st], tm, row, z, &sm->kv_full[st]);
        pending |= 1u << st;
        pending_ph[st] = ph;
        if (++st == NS) { st = 0; ph ^= 1u; }
        return true;
      };
      for (int pi = blockIdx.x; pi < p.n_pairs && ok; pi += gridDim.x) {
        const int4 pr = p.pairs[pi];
        const int items[2] = {pr.x, pr.y};
        const bool shared = pr.z != 0;
        WorkItem wi[2];
        int n[2] = {0, 0};
        for (int s = 0; s < 2; ++s) {
          if (items[s] < 0) continue;
          wi[s] = p.work[items[s]];
          n[s] = wi[s].entry_end - wi[s].entry_begin;
          if (!mbar_wait(&sm->q_empty[s], qph[s] ^ 1u, sm, p.status)) { ok = false; break; }
          qph[s] ^= 1u;
          tma_tile(sm->q[s], &tmQ, wi[s].q_row, wi[s].bh, &sm->q_full[s]);
        }
        if (!ok) break;
        for (int s = 0; s < 2 && ok; ++s) {
          if (items[s] < 0) continue;
          ok = take(&tmS, 0, wi[s].bh * p.nqg + wi[s].state_group);
          if (ok && n[s] > 0 && (s == 0 || !shared))
            ok = take(&tmK, p.entries[wi[s].entry_begin].k_row, wi[s].bh);
        }
        const int nmax = n[0] > n[1] ? n[0] : n[1];
        for (int j = 0; j < nmax && ok; ++j) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (items[s] < 0 || j >= n[s] || (s == 1 && shared)) continue;
            const Entry* e = p.entries + wi[s].entry_begin;
            ok = take(&tmV, e[j].k_row, wi[s].bh);
            if (ok && j + 1 < n[s]) ok = take(&tmK, e[j + 1].k_row, wi[s].bh);
          }
        }
      }
      if (!ok) {
        // drain: wait (bounded) for every load this thread issued
        for (int i = 0; i < NS; ++i) {
          if (!(pending & (1u << i))) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&sm->kv_full[i], pending_ph[i]) && globaltimer() - t0 < kTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int st = 0;
      uint32_t ph = 0;
      uint32_t qph[2] = {0, 0}, pph[2] = {0, 0};
      bool ok = true;
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 384};
      auto next_stage = [&](int* out) -> bool {
        if (!mbar_wait(&sm->kv_full[st], ph, sm, p.status)) return false;
        tc_fence_after();
        *out = st;
        if (++st == NS) { st = 0; ph ^= 1u; }
        return true;
      };
      auto wait_p = [&](int s) -> bool {
        if (!mbar_wait(&sm->p_full[s], pph[s], sm, p.status)) return false;
        pph[s] ^= 1u;
        tc_fence_after();
        return true;
      };
      auto qk = [&](int s, int stage) {
        const uint32_t qa = smem_u32(sm->q[s]), kb = smem_u32(sm->kv[stage]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(tS[s], desc_kmajor(qa, kk), desc_kmajor(kb, kk), kIdescKK, kk > 0);
        mma_commit(&sm->s_full[s]);
      };
      auto pv = [&](int s, int stage) {
        const uint32_t vb = smem_u32(sm->kv[stage]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ts(tO[s], tS[s] + kk * 8, desc_mnmajor(vb, kk), kIdescKMN, 1);
        mma_commit(&sm->pv_done[s]);
      };
      for (int pi = blockIdx.x; pi < p.n_pairs && ok; pi += gridDim.x) {
        const int4 pr = p.pairs[pi];
        const int items[2] = {pr.x, pr.y};
        const bool shared = pr.z != 0;
        int n[2] = {0, 0};
        for (int s = 0; s < 2; ++s)
          if (items[s] >= 0) n[s] = p.work[items[s]].entry_end - p.work[items[s]].entry_begin;
        int kst[2] = {-1, -1};
        // linear branch: O_s = phi(Q_s) S_rest^T, then the first QK
        for (int s = 0; s < 2 && ok; ++s) {
          if (items[s] < 0) continue;
          int sst;
          ok = wait_p(s) && next_stage(&sst);
          if (!ok) break;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) mma_ts(tO[s], tS[s] + kk * 8, desc_kmajor(smem_u32(sm->kv[sst]), kk), kIdescKK, kk > 0);
          mma_commit(&sm->pv_done[s]);
          mma_commit(&sm->kv_empty[sst]);
          if (n[s] > 0) {
            if (!mbar_wait(&sm->q_full[s], qph[s], sm, p.status)) { ok = false; break; }
            tc_fence_after();
            if (s == 1 && shared) kst[1] = kst[0];
            else if (!next_stage(&kst[s])) { ok = false; break; }
            qk(s, kst[s]);
            if (!(s == 0 && shared)) mma_commit(&sm->kv_empty[kst[s]]);
            if (n[s] == 1) mma_commit(&sm->q_empty[s]);
          } else {
            if (!mbar_wait(&sm->q_full[s], qph[s], sm, p.status)) { ok = false; break; }
            mma_commit(&sm->q_empty[s]);
          }
          qph[s] ^= 1u;
        }
        const int nmax = n[0] > n[1] ? n[0] : n[1];
        int vst0 = -1;
        for (int j = 0; j < nmax && ok; ++j) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (items[s] < 0 || j >= n[s]) continue;
            int vst;
            if (!wait_p(s)) { ok = false; break; }
            if (s == 1 && shared) vst = vst0;
            else if (!next_stage(&vst)) { ok = false; break; }
            if (s == 0) vst0 = vst;
            pv(s, vst);
            if (!(s == 0 && shared)) mma_commit(&sm->kv_empty[vst]);
            if (j + 1 < n[s]) {
              if (s == 1 && shared) kst[1] = kst[0];
              else if (!next_stage(&kst[s])) { ok = false; break; }
              qk(s, kst[s]);
              if (!(s == 0 && shared)) mma_commit(&sm->kv_empty[kst[s]]);
              if (j + 2 == n[s]) mma_commit(&sm->q_empty[s]);
            }
          }
        }
      }
      // wait for every issued MMA before TMEM is released
      mma_commit(&sm->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&sm->drain, 0) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int s = warp >> 2;                          // slot of this warpgroup
    const int row = threadIdx.x & 127;                // query row in the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + s * 128 + lane_off;
    const uint32_t tO = tmem + 256 + s * 128 + lane_off;
    uint32_t qph = 0, sph = 0;
    uint32_t pv_phase = 0;                            // pv_done phases completed before this pair
    for (int pi = blockIdx.x; pi < p.n_pairs; pi += gridDim.x) {
      const int4 pr = p.pairs[pi];
      const int item = s == 0 ? pr.x : pr.y;
      if (item < 0) continue;
      const WorkItem wi = p.work[item];
      const int n = wi.entry_end - wi.entry_begin;
      if (!mbar_wait_warp(&sm->q_full[s], qph, sm, p.status)) break;
      qph ^= 1u;
      // phi(q) of this row -> TMEM (bf16 pairs), l = phi(q) . z
      const float* z = p.srest + (static_cast<int64_t>(wi.bh) * p.nqg + wi.state_group) * (D * D + D) + D * D;
      float l = 0.0f, m = 0.0f;
      {
        const uint8_t* qrow = sm->q[s] + row * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t packed[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4*>(qrow + half * HALF_BYTES + ((c ^ (row & 7)) << 4));
            const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&w4[e]);
              const float2 f = __bfloat1622float2(b2);
              const float f0 = phi_elu1(f.x), f1 = phi_elu1(f.y);
              const int col = half * 64 + c * 8 + e * 2;
              l = fmaf(f0, __ldg(z + col), l);
              l = fmaf(f1, __ldg(z + col + 1), l);
              packed[c * 4 + e] = pack_bf16(f0, f1);
            }
          }
          tmem_st32(tS + half * 32, packed);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm->p_full[s]);
      }
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        if (!mbar_wait_warp(&sm->s_full[s], sph, sm, p.status)) { ok = false; break; }
        sph ^= 1u;
        tc_fence_after();
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tS + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
        }
        const int klen = p.entries[wi.entry_begin + j].k_len;
        if (klen < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= klen) sv[i] = -INFINITY;
        }
        float mx = sv[0];
#pragma unroll
        for (int i = 1; i < 128; ++i) mx = fmaxf(mx, sv[i]);
        const float m_cand = mx * p.scale_log2;
        if (__any_sync(0xffffffffu, m_cand > m + kRescaleThreshold)) {
          const float m_new = fmaxf(m, m_cand);
          const float alpha = ex2(m - m_new);
          // the previous P.V (or the linear-branch MMA) must be complete before O is rescaled
          if (!mbar_wait_warp(&sm->pv_done[s], (pv_phase + j) & 1u, sm, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
          tmem_wait_st();
          l *= alpha;
          m = m_new;
        }
        float rs = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t packed[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2(fmaf(sv[c * 64 + 2 * i], p.scale_log2, -m));
            const float p1 = ex2(fmaf(sv[c * 64 + 2 * i + 1], p.scale_log2, -m));
            rs += p0 + p1;
            packed[i] = pack_bf16(p0, p1);
          }
          tmem_st32(tS + c * 32, packed);
        }
        l += rs;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm->p_full[s]);
      }
      if (!ok) break;
      // epilogue: o = O / l, bf16, 16-byte stores of the valid rows
      if (!mbar_wait_warp(&sm->pv_done[s], (pv_phase + n) & 1u, sm, p.status)) break;
      pv_phase += n + 1;
      tc_fence_after();
      const float inv = 1.0f / l;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (static_cast<int64_t>(wi.bh) * p.q_rows + wi.q_row + row) * D;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
        if (row < wi.q_len) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
            dst[v] = w;
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 tensor [z][rows][128] as a 3-D map with 64 x 128 boxes and 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t zdim) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(zdim)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

}  // namespace

bool attn_tc_supported(int d, int dtype) { return d == D && dtype == HYAT_BF16; }

cudaError_t launch_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t s) {
  if (a.n_pairs == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ms;
  if (!make_map(&mq, a.q, a.q_rows, a.BH) || !make_map(&mk, a.k, a.k_rows, a.BH) ||
      !make_map(&mv, a.v, a.k_rows, a.BH) || !make_map(&ms, a.srest_t, D, int64_t(a.BH) * a.nqg))
    return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
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
  const int grid = a.n_pairs < num_sms ? a.n_pairs : num_sms;
  attn_tc_kernel<<<grid, NUM_THREADS, kSmemBytes, s>>>(mq, mk, mv, ms, p);
  return cudaGetLastError();
}

}  // namespace hyat
