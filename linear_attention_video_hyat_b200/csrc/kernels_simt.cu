// CUDA-core kernels of libhyat: segment states, complement reduction, state
// transpose, and the fp32 hybrid-attention kernel. The fp32 workload runs
// entirely here (the tensor cores have no fp32 operand kind, and tf32 is too
// coarse for a 1e-5 bound); the bf16 path uses the tensor-core attention kernel
// and these kernels for its linear state.
//
// Linear-state formation follows Hybrid Forcing, Section 2.A ("Hybrid
// Attention": evicted key/value states aggregated into a compact state) and
// ReHyAt, Abstract (chunk-wise recurrent reformulation).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyat_internal.h"

namespace hyat {
namespace {

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// phi(x) = elu(x) + 1 with alpha = 1
// Feature maps of the linear branch (hyat_phi): 0 elu + 1, 1 ReLU, 2 exp.
__device__ __forceinline__ float phi_map(float x, int kind) {
  if (kind == 1) return fmaxf(x, 0.0f);
  if (kind == 2) return expf(x);
  return x > 0.0f ? x + 1.0f : expf(x);
}

// four consecutive elements as floats (p must be 8-byte (bf16) / 16-byte (f32) aligned)
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

// --------------------------------------------------------------------------
// Segment states: out[bh][g] = ( S_g = sum_j phi(k_j) v_j^T  (d x d, [a][b]),
//                               z_g = sum_j phi(k_j) (d) )
// grid (D/64 * D/64, nseg, BH), 256 threads, each a 4x4 block of a 64x64 tile.
// --------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) seg_state_kernel(SegStateArgs a) {
  constexpr int CH = 32, W = 64 + 4;
  __shared__ __align__(16) float Ks[CH][W];
  __shared__ __align__(16) float Vs[CH][W];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int at = blockIdx.x / (D / 64), bt = blockIdx.x % (D / 64);
  const int g = blockIdx.y, bh = blockIdx.z;
  const int64_t start = a.seg_base + static_cast<int64_t>(g) * a.seg_stride;
  int64_t len64 = a.rows_per_bh - start;
  if (len64 > a.seg_len) len64 = a.seg_len;
  const int len = len64 > 0 ? static_cast<int>(len64) : 0;
  const T* K = static_cast<const T*>(a.k) + (static_cast<int64_t>(bh) * a.rows_per_bh + start) * D;
  const T* V = static_cast<const T*>(a.v) + (static_cast<int64_t>(bh) * a.rows_per_bh + start) * D;
  float acc[4][4] = {};
  float zacc[4] = {};
  for (int t0 = 0; t0 < len; t0 += CH) {
    __syncthreads();
    for (int idx = tid; idx < CH * 16; idx += 256) {
      const int r = idx >> 4, c4 = (idx & 15) * 4;
      float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
      if (t0 + r < len) {
        kk = ld4(K + static_cast<int64_t>(t0 + r) * D + 64 * at + c4);
        kk = make_float4(phi_map(kk.x, a.phi), phi_map(kk.y, a.phi), phi_map(kk.z, a.phi), phi_map(kk.w, a.phi));
        vv = ld4(V + static_cast<int64_t>(t0 + r) * D + 64 * bt + c4);
      }
      *reinterpret_cast<float4*>(&Ks[r][c4]) = kk;
      *reinterpret_cast<float4*>(&Vs[r][c4]) = vv;
    }
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < CH; ++r) {
      const float4 kk = *reinterpret_cast<const float4*>(&Ks[r][4 * ty]);
      const float4 vv = *reinterpret_cast<const float4*>(&Vs[r][4 * tx]);
      const float kr[4] = {kk.x, kk.y, kk.z, kk.w};
      const float vr[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(kr[i], vr[j], acc[i][j]);
        zacc[i] += kr[i];
      }
    }
  }
  const int64_t E = static_cast<int64_t>(D) * D + D;
  float* out = a.out + (static_cast<int64_t>(bh) * a.nseg + g) * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float* row = out + static_cast<int64_t>(64 * at + 4 * ty + i) * D + 64 * bt + 4 * tx;
    float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    if (a.accumulate) {
      const float4 o = *reinterpret_cast<const float4*>(row);
      v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
    }
    *reinterpret_cast<float4*>(row) = v;
  }
  if (bt == 0 && tx == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float* zp = out + static_cast<int64_t>(D) * D + 64 * at + 4 * ty + i;
      *zp = a.accumulate ? *zp + zacc[i] : zacc[i];
    }
  }
}

// --------------------------------------------------------------------------
// Complement reduction: srest[bh][g] = sum_s cm[hm][g][s] * sseg[bh][s]
// (the 0/1 matrix cm marks the segments in a group's linear set).
// grid (ceil(E/256), ceil(nqg/G), BH), 256 threads: one column, G groups each; segment values
// are loaded SB at a time before the sums so that the loads overlap.
// --------------------------------------------------------------------------
template <int G, int SB>
__global__ void __launch_bounds__(256) complement_kernel(ComplementArgs a) {
  // Programmatic dependent launch: wait for the state kernel's results (a no-op when this
  // kernel was launched without the attribute), then let the attention kernel launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float cms[G][SB + 1];
  const int tid = threadIdx.x;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + tid;
  const int g0 = blockIdx.y * G, bh = blockIdx.z;
  const int hm = a.cm_heads == 1 ? 0 : bh % a.H;
  const float* S = a.sseg + static_cast<int64_t>(bh) * a.nseg * a.E;
  const float* cm = a.cm + static_cast<int64_t>(hm) * a.nqg * a.nseg;
  float acc[G];
#pragma unroll
  for (int i = 0; i < G; ++i) acc[i] = 0.0f;
  for (int s0 = 0; s0 < a.nseg; s0 += SB) {
    __syncthreads();
    for (int idx = tid; idx < G * SB; idx += 256) {
      const int gg = idx / SB, ss = idx % SB;
      cms[gg][ss] = (g0 + gg < a.nqg && s0 + ss < a.nseg)
                        ? cm[static_cast<int64_t>(g0 + gg) * a.nseg + s0 + ss] : 0.0f;
    }
    __syncthreads();
    float sv[SB];
#pragma unroll
    for (int ss = 0; ss < SB; ++ss)
      sv[ss] = (e < a.E && s0 + ss < a.nseg) ? __ldg(S + static_cast<int64_t>(s0 + ss) * a.E + e) : 0.0f;
#pragma unroll
    for (int ss = 0; ss < SB; ++ss)
#pragma unroll
      for (int gg = 0; gg < G; ++gg) acc[gg] = fmaf(cms[gg][ss], sv[ss], acc[gg]);
  }
  if (e < a.E) {
    const int64_t dd = static_cast<int64_t>(a.d) * a.d;
    const bool is_s = e < dd;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      if (g0 + gg >= a.nqg) continue;
      const int64_t grp = static_cast<int64_t>(bh) * a.nqg + g0 + gg;
      if (!is_s || a.write_f32_s) a.srest[grp * a.E + e] = acc[gg];
      if (is_s && a.srest_bf16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(acc[gg]);
        a.srest_bf16[grp * dd + e] = *reinterpret_cast<const uint16_t*>(&h);
      }
    }
  }
}

// S [a][b] fp32 (group stride d*d + d) -> bf16 S [a][b] (group stride d*d)
__global__ void state_to_bf16_kernel(const float* __restrict__ s, uint16_t* __restrict__ out, int64_t n, int32_t d) {
  const int64_t dd = static_cast<int64_t>(d) * d;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t g = i / dd, e = i % dd;
    const __nv_bfloat16 h = __float2bfloat16_rn(s[g * (dd + d) + e]);
    out[i] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

// --------------------------------------------------------------------------
// Hybrid attention on CUDA cores (fp32 arithmetic).
// One CTA = 64 query rows (half of a 128-row work item), key sub-tiles of 64.
// Thread (tx, ty): score block rows 4ty..4ty+3 x keys 4tx..4tx+3; output rows
// 4ty..4ty+3 x columns {4tx + 64u + j}.
// The accumulator starts from the linear term with running max 0:
//   acc = phi(Q) S_rest, l = phi(Q) z_rest, m = 0   (log2 domain)
// and each key tile rescales it online, which yields the joint normaliser.
// --------------------------------------------------------------------------
template <int D>
struct SimtSmem {
  static constexpr int BQ = 64, BK = 64, PQ = BQ + 4, PK = BK + 4, PD = D + 4;
  static constexpr size_t bytes = sizeof(float) * (size_t(D) * PQ + size_t(D) * PK + size_t(BK) * PD + size_t(BK) * PQ);
};

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
  using SM = SimtSmem<D>;
  constexpr int BQ = SM::BQ, BK = SM::BK, PQ = SM::PQ, PK = SM::PK, PD = SM::PD, NU = D / 64;
  extern __shared__ __align__(16) float smem[];
  float* Qs = smem;               // [D][PQ]  Q transposed
  float* Ks = Qs + D * PQ;        // [D][PK]  K transposed
  float* Vs = Ks + D * PK;        // [BK][PD]
  float* Ps = Vs + BK * PD;       // [BK][PQ] P transposed
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const WorkItem w = a.work[blockIdx.x >> 1];
  const int half = blockIdx.x & 1;
  const int q0 = w.q_row + half * BQ;
  const int qlen = min(BQ, w.q_len - half * BQ);
  if (qlen <= 0) return;
  const T* Q = static_cast<const T*>(a.q) + static_cast<int64_t>(w.bh) * a.q_rows * D;
  const T* K = static_cast<const T*>(a.k) + static_cast<int64_t>(w.bh) * a.k_rows * D;
  const T* V = static_cast<const T*>(a.v) + static_cast<int64_t>(w.bh) * a.k_rows * D;
  T* O = static_cast<T*>(a.o) + static_cast<int64_t>(w.bh) * a.q_rows * D;

  for (int idx = tid; idx < BQ * (D / 4); idx += 256) {
    const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < qlen) x = ld4(Q + static_cast<int64_t>(q0 + r) * D + c4);
    Qs[(c4 + 0) * PQ + r] = x.x;
    Qs[(c4 + 1) * PQ + r] = x.y;
    Qs[(c4 + 2) * PQ + r] = x.z;
    Qs[(c4 + 3) * PQ + r] = x.w;
  }

  // ---- linear term: acc = phi(Q) S, l = phi(Q) z ----
  const int64_t E = static_cast<int64_t>(D) * D + D;
  const float* Sr = a.srest + (static_cast<int64_t>(w.bh) * a.nqg + w.state_group) * E;
  float acc[4][4 * NU];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4 * NU; ++c) acc[i][c] = 0.0f;
  float l[4] = {0.f, 0.f, 0.f, 0.f}, m[4] = {0.f, 0.f, 0.f, 0.f};
  for (int a0 = 0; a0 < D; a0 += BK) {
    __syncthreads();
    for (int idx = tid; idx < BK * (D / 4); idx += 256) {
      const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
      *reinterpret_cast<float4*>(&Vs[r * PD + c4]) = ld4(Sr + static_cast<int64_t>(a0 + r) * D + c4);
    }
    __syncthreads();
    for (int r = 0; r < BK; ++r) {
      const float4 qv = *reinterpret_cast<const float4*>(&Qs[(a0 + r) * PQ + 4 * ty]);
      const float pq[4] = {phi_map(qv.x, a.phi), phi_map(qv.y, a.phi), phi_map(qv.z, a.phi), phi_map(qv.w, a.phi)};
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        const float4 sv = *reinterpret_cast<const float4*>(&Vs[r * PD + 4 * tx + 64 * u]);
        const float sr[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][4 * u + j] = fmaf(pq[i], sr[j], acc[i][4 * u + j]);
      }
    }
  }
  {
    const float* z = Sr + static_cast<int64_t>(D) * D;
    constexpr int PER = D / 16;
    for (int r = 0; r < PER; ++r) {
      const int c = tx * PER + r;
      const float4 qv = *reinterpret_cast<const float4*>(&Qs[c * PQ + 4 * ty]);
      const float zc = z[c];
      l[0] = fmaf(phi_map(qv.x, a.phi), zc, l[0]);
      l[1] = fmaf(phi_map(qv.y, a.phi), zc, l[1]);
      l[2] = fmaf(phi_map(qv.z, a.phi), zc, l[2]);
      l[3] = fmaf(phi_map(qv.w, a.phi), zc, l[3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) l[i] += __shfl_xor_sync(0xffffffffu, l[i], off);
  }

  // ---- softmax window ----
  for (int e = w.entry_begin; e < w.entry_end; ++e) {
    const Entry en = a.entries[e];
    for (int sub = 0; sub < en.k_len; sub += BK) {
      const int kv0 = en.k_row + sub;
      const int klen = min(BK, en.k_len - sub);
      __syncthreads();
      for (int idx = tid; idx < BK * (D / 4); idx += 256) {
        const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
        float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
        if (r < klen) {
          kk = ld4(K + static_cast<int64_t>(kv0 + r) * D + c4);
          vv = ld4(V + static_cast<int64_t>(kv0 + r) * D + c4);
        }
        Ks[(c4 + 0) * PK + r] = kk.x;
        Ks[(c4 + 1) * PK + r] = kk.y;
        Ks[(c4 + 2) * PK + r] = kk.z;
        Ks[(c4 + 3) * PK + r] = kk.w;
        *reinterpret_cast<float4*>(&Vs[r * PD + c4]) = vv;
      }
      __syncthreads();
      float s[4][4] = {};
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        const float4 qv = *reinterpret_cast<const float4*>(&Qs[c * PQ + 4 * ty]);
        const float4 kv = *reinterpret_cast<const float4*>(&Ks[c * PK + 4 * tx]);
        const float qr[4] = {qv.x, qv.y, qv.z, qv.w};
        const float kr[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) s[i][j] = fmaf(qr[i], kr[j], s[i][j]);
      }
      float p[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[i][j] = (4 * tx + j < klen) ? s[i][j] * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[i][j]);
        }
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m[i], mx);
        const float alpha = exp2f(m[i] - m_new);
        m[i] = m_new;
        float rs = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          p[i][j] = exp2f(s[i][j] - m_new);
          rs += p[i][j];
        }
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
        l[i] = l[i] * alpha + rs;
#pragma unroll
        for (int c = 0; c < 4 * NU; ++c) acc[i][c] *= alpha;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(&Ps[(4 * tx + j) * PQ + 4 * ty]) = make_float4(p[0][j], p[1][j], p[2][j], p[3][j]);
      __syncthreads();
      for (int j = 0; j < klen; ++j) {
        const float4 pv = *reinterpret_cast<const float4*>(&Ps[j * PQ + 4 * ty]);
        const float pr[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const float4 vv = *reinterpret_cast<const float4*>(&Vs[j * PD + 4 * tx + 64 * u]);
          const float vr[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) acc[i][4 * u + jj] = fmaf(pr[i], vr[jj], acc[i][4 * u + jj]);
        }
      }
    }
  }

  // ---- normalise and store ----
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 4 * ty + i;
    if (r >= qlen) continue;
    const float inv = 1.0f / l[i];
    T* orow = O + static_cast<int64_t>(q0 + r) * D;
#pragma unroll
    for (int u = 0; u < NU; ++u)
#pragma unroll
      for (int j = 0; j < 4; ++j) orow[4 * tx + 64 * u + j] = from_f<T>(acc[i][4 * u + j] * inv);
  }
}

template <typename T, int D>
cudaError_t launch_attn_simt_t(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = SimtSmem<D>::bytes;
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.n_work == 0) return cudaSuccess;
  attn_simt_kernel<T, D><<<a.n_work * 2, 256, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_seg_state_t(const SegStateArgs& a, cudaStream_t s) {
  if (a.nseg == 0) return cudaSuccess;
  dim3 grid((D / 64) * (D / 64), a.nseg, a.BH);
  seg_state_kernel<T, D><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_seg_state(const SegStateArgs& a, cudaStream_t s) {
  if (a.dtype == HYAT_F32) return a.d == 64 ? launch_seg_state_t<float, 64>(a, s) : launch_seg_state_t<float, 128>(a, s);
  return a.d == 64 ? launch_seg_state_t<__nv_bfloat16, 64>(a, s) : launch_seg_state_t<__nv_bfloat16, 128>(a, s);
}

cudaError_t launch_complement(const ComplementArgs& a, cudaStream_t s) {
  if (a.nqg == 0 || a.BH == 0) return cudaSuccess;
  const bool few = a.nqg <= 8;      // chunk windows: a handful of groups per head
  dim3 grid((a.E + 255) / 256, (a.nqg + (few ? 7 : 31)) / (few ? 8 : 32), a.BH);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return few ? cudaLaunchKernelEx(&cfg, complement_kernel<8, 24>, a) : cudaLaunchKernelEx(&cfg, complement_kernel<32, 16>, a);
}

cudaError_t launch_state_to_bf16(const float* srest, uint16_t* out, int64_t n_groups, int32_t d, cudaStream_t s) {
  const int64_t n = n_groups * d * d;
  if (n == 0) return cudaSuccess;
  const int blocks = static_cast<int>((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048);
  state_to_bf16_kernel<<<blocks, 256, 0, s>>>(srest, out, n, d);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s) {
  if (a.dtype == HYAT_F32) return a.d == 64 ? launch_attn_simt_t<float, 64>(a, s) : launch_attn_simt_t<float, 128>(a, s);
  return a.d == 64 ? launch_attn_simt_t<__nv_bfloat16, 64>(a, s) : launch_attn_simt_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace hyat
