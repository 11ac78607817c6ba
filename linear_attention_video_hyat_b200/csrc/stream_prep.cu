// The work of a streaming step between the fold's state kernel and the attention kernel, in one
// launch (Long-Horizon Streaming Video Generation via Hybrid Attention with Decoupled
// Distillation, Section 2.A: frames that leave the window are folded into the linear state,
// the window keeps the latest frames for block-sparse softmax attention; Section 2.C: the
// temporal RoPE index is a capped offset). Four independent jobs, each on its own range of
// blocks:
//   * fold reduce: S, z += the fold's partial states, summed in a fixed order (so a run is
//     bit-reproducible), and the bf16 copy of S that the attention's linear-term MMA reads;
//   * ring copy: the chunk's K and V into its ring slot, 16-byte vectors; with the fused RoPE,
//     K is turned on its way in (the copy reads and writes every K vector anyway);
//   * Q rotation (fused RoPE only): Q turned into a workspace copy that the attention reads;
//   * layout: one warp per (b, h, query tile) compacts its row of the step's tile mask into
//     the key-tile list (ring rows), and checks that the diagonal tile of the newest chunk is
//     kept; with split pairs, the last layout block to finish deals the pairs out to the
//     attention's persistent CTAs from this step's key-tile counts.
// The kernel streams its bytes once (HBM-bound); its copy blocks wait for the fold's partial
// states (and for the fold to have read the ring slot they overwrite) with a programmatic-launch
// wait, and it lets the attention kernel start its prologue early.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyat_internal.h"
#include "rope_common.cuh"

namespace hyat {
namespace {

constexpr int kPrepThreads = 256;
constexpr int kPrepUnroll = 4;        // vectors a thread moves at a time (memory parallelism)

template <typename T>
__device__ __forceinline__ void turn_vector(uint4& v, int col, int half_t, const float2* cs) {
  constexpr int E = RopeLanes<T>::kElems, P = E / 2;
  const int pair0 = col * P;
  if (pair0 >= half_t) return;
  float f[E];
  RopeLanes<T>::to_f32(v, f);
#pragma unroll
  for (int k = 0; k < P; ++k)
    if (pair0 + k < half_t) rope_turn(f[2 * k], f[2 * k + 1], cs[pair0 + k].x, cs[pair0 + k].y);
  v = RopeLanes<T>::from_f32(f);
}

// Split pairs dealt out from this step's key-tile counts, the way the host deals the pairs of
// the bidirectional layouts. Largest count first, the list is rows of `grid` pairs (pair
// r * grid + c runs on CTA c); two ways of placing each row's pairs are weighed, and the one
// whose busiest CTA holds less work wins (ties: the first):
//   * serpentine: left to right in even rows, right to left in odd rows;
//   * least loaded first: each row's pairs, largest first, to the CTAs in ascending order of
//     the work they already hold (longest-processing-time first, a row at a time).
// A pair's work is its key tiles plus one for its set-up. The layout blocks count themselves
// done; the last one (it sees every work item: each thread fences its writes before the count)
// sorts the items with a counting sort in shared memory and deals the rows there, so that the
// only global traffic is one read of the counts and one write of the list. Items of equal
// count may land in any order: every pair is computed on its own, so the output does not
// depend on it.
struct OrderSmem {
  int32_t bins[kMaxStreamOrderBins];    // histogram of counts, then first sorted position
  int32_t sorted[kMaxStreamOrderItems]; // count << 20 | item, largest count first
  int32_t load[kMaxStreamOrderGrid + 4];
  int32_t dealt[kMaxStreamOrderItems];  // least-loaded-first: sorted position of each pair
  int32_t is_last, serp_max;
};

__device__ __forceinline__ int sorted_cost(const OrderSmem& o, int k) { return (o.sorted[k] >> 20) + 1; }

// Longest-processing-time dealing of the rows: dealt[r0 + c] = sorted position that goes to CTA
// c in the row at r0. Returns the busiest CTA's work.
__device__ __forceinline__ int deal_least_loaded(OrderSmem& o, int n_items, int grid) {
  constexpr int kPer = (kMaxStreamOrderGrid + kPrepThreads - 1) / kPrepThreads;
  for (int c = threadIdx.x; c < grid + 4; c += kPrepThreads) o.load[c] = 0;
  __syncthreads();
  for (int r0 = 0; r0 < n_items; r0 += grid) {
    const int len = min(grid, n_items - r0);        // a partial last row: CTAs 0 .. len - 1
    int add[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int c = threadIdx.x + u * kPrepThreads;
      add[u] = 0;
      if (c >= len) continue;
      const int lc = o.load[c];
      int rank = 0;                                 // CTAs holding less work (ties: lower index)
      for (int c2 = 0; c2 < len; c2 += 4) {        // reads up to load[len + 2] < load[grid + 4]
        const int4 l4 = *reinterpret_cast<const int4*>(&o.load[c2]);
        rank += (c2 < len) & ((l4.x < lc) | ((l4.x == lc) & (c2 < c)));
        rank += (c2 + 1 < len) & ((l4.y < lc) | ((l4.y == lc) & (c2 + 1 < c)));
        rank += (c2 + 2 < len) & ((l4.z < lc) | ((l4.z == lc) & (c2 + 2 < c)));
        rank += (c2 + 3 < len) & ((l4.w < lc) | ((l4.w == lc) & (c2 + 3 < c)));
      }
      o.dealt[r0 + c] = r0 + rank;
      add[u] = sorted_cost(o, r0 + rank);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int c = threadIdx.x + u * kPrepThreads;
      if (c < len) o.load[c] += add[u];
    }
    __syncthreads();
  }
  int mx = 0;
  for (int c = 0; c < grid; ++c) mx = max(mx, o.load[c]);
  return mx;
}

__device__ __forceinline__ void order_split_pairs(const StreamPrepArgs& a) {
  __shared__ __align__(16) OrderSmem o;
  __threadfence();                                  // this thread's work item, before the count
  __syncthreads();
  if (threadIdx.x == 0) o.is_last = atomicAdd(a.done_counter, 1u) == static_cast<uint32_t>(a.nb_layout - 1);
  __syncthreads();
  if (!o.is_last) return;
  __threadfence();
  const int n_items = a.BH * a.nqt, grid = a.grid;
  const int nb = a.cap_entries + 1;                 // counts 0 .. cap_entries
  for (int b = threadIdx.x; b < nb; b += kPrepThreads) o.bins[b] = 0;
  if (threadIdx.x == 0) o.serp_max = 0;
  __syncthreads();
  constexpr int kItemsPer = kMaxStreamOrderItems / kPrepThreads;
  int cnt[kItemsPer];
#pragma unroll
  for (int u = 0; u < kItemsPer; ++u) {             // every count read in one round trip
    const int it = threadIdx.x + u * kPrepThreads;
    cnt[u] = it < n_items ? __ldcg(&a.work[it].entry_end) - __ldcg(&a.work[it].entry_begin) : -1;
  }
#pragma unroll
  for (int u = 0; u < kItemsPer; ++u)
    if (cnt[u] >= 0) atomicAdd(&o.bins[cnt[u]], 1);
  __syncthreads();
  // exclusive scan from the largest count down: bins[n] = number of items with a larger count
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, per = (nb + 31) / 32;
    const int hi = nb - 1 - lane * per;             // this lane's bins: hi, hi - 1, ..., > hi - per
    int sum = 0;
    for (int k = 0; k < per; ++k)
      if (hi - k >= 0) sum += o.bins[hi - k];
    int excl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, excl, off);
      if (lane >= off) excl += t;
    }
    excl -= sum;
    for (int k = 0; k < per; ++k) {
      if (hi - k < 0) break;
      const int c = o.bins[hi - k];
      o.bins[hi - k] = excl;
      excl += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kItemsPer; ++u) {
    const int it = threadIdx.x + u * kPrepThreads;
    if (cnt[u] >= 0) o.sorted[atomicAdd(&o.bins[cnt[u]], 1)] = (cnt[u] << 20) | it;
  }
  __syncthreads();
  // the serpentine's busiest CTA
  for (int c = threadIdx.x; c < grid; c += kPrepThreads) {
    int l = 0;
    for (int r0 = 0, r = 0; r0 < n_items; r0 += grid, ++r) {
      const int len = min(grid, n_items - r0);
      if (c < len) l += sorted_cost(o, r0 + ((r & 1) ? len - 1 - c : c));
    }
    atomicMax(&o.serp_max, l);
  }
  const bool lpt = deal_least_loaded(o, n_items, grid) < o.serp_max;
  for (int k = threadIdx.x; k < n_items; k += kPrepThreads) {
    int src;
    if (lpt) {
      src = o.dealt[k];
    } else {
      const int r = k / grid, r0 = r * grid, len = min(grid, n_items - r0), c = k - r0;
      src = r0 + ((r & 1) ? len - 1 - c : c);
    }
    const int it = o.sorted[src] & 0xfffff;
    a.pairs[k] = make_int4(it, it, 0, 1);
  }
  if (threadIdx.x == 0) *a.done_counter = 0u;       // for the next step
}

// One row of the step's tile mask (one warp per (bh, query tile)) compacted into its key-tile
// list as ring rows; the diagonal tile of the newest chunk must be kept.
__device__ __forceinline__ void layout_row(const StreamPrepArgs& a, int item) {
  const int lane = threadIdx.x & 31;
  const int bh = item / a.nqt, i = item % a.nqt;
  const int hm = a.mask_heads == 1 ? 0 : bh % a.H;
  const uint8_t* row = a.mask + (static_cast<int64_t>(hm) * a.nqt + i) * a.nkt;
  const int64_t base = static_cast<int64_t>(item) * a.cap_entries;
  int count = 0;
  for (int kt0 = 0; kt0 < a.nkt; kt0 += 32) {
    const int kt = kt0 + lane;
    const bool keep = kt < a.nkt && __ldcg(row + kt) != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = count + __popc(bal & ((1u << lane) - 1u));
      const int w = kt / a.nqt, t = kt % a.nqt;
      const int slot = w < a.n_sink_visible ? a.nwc + w : (a.first_window_mod + w - a.n_sink_visible) % a.nwc;
      a.entries[base + pos] = Entry{slot * a.L + t * kTile, min(kTile, a.L - t * kTile)};
    }
    count += __popc(bal);
  }
  if (lane == 0) {
    if (__ldcg(row + (a.nkt - a.nqt + i)) == 0) atomicOr(a.status, kStatusBadMask);
    a.work[item] = WorkItem{bh, i * kTile, min(kTile, a.L - i * kTile), 0, static_cast<int32_t>(base),
                            static_cast<int32_t>(base + count), 0, 0};
  }
}

template <typename T>
__global__ void __launch_bounds__(kPrepThreads) stream_prep_kernel(const StreamPrepArgs a) {
  extern __shared__ float2 cs_table[];            // [chunk frame][pair]: (cos, sin)
  int b = blockIdx.x;

  // ---- layout: one warp per (bh, query tile). These blocks come first in the grid. The
  // layout reads the step's mask and writes the tables that the previous step's attention
  // read; the fold's state kernel writes neither. With `layout_early` the host states that the
  // kernel ahead of this one is the fold, which lets this grid start only after its own
  // programmatic wait, i.e. once everything enqueued before the call (that attention, a kernel
  // that wrote the mask) has finished; so these blocks skip the wait and run, pair ordering
  // included, while the fold still runs. They read the mask past L1 (`__ldcg`).
  if (b < a.nb_layout) {
    if (!a.layout_early) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int item = b * (kPrepThreads / 32) + (threadIdx.x >> 5);
    if (item < a.BH * a.nqt) layout_row(a, item);
    if (a.pairs) order_split_pairs(a);              // every thread of the block takes part
    return;
  }
  b -= a.nb_layout;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int E = RopeLanes<T>::kElems;
  const int cols = a.d / E;                       // 16-byte vectors per row
  const int64_t row_vecs = static_cast<int64_t>(a.L) * cols;

  // ---- fold reduce: srest[bh] += sum_r partial[bh][r], r in order; bf16 copy of S
  if (b < a.nb_fold) {
    const int64_t E4 = (static_cast<int64_t>(a.d) * a.d + a.d) / 4, dd4 = static_cast<int64_t>(a.d) * a.d / 4;
    for (int64_t i = static_cast<int64_t>(b) * kPrepThreads + threadIdx.x; i < E4 * a.BH;
         i += static_cast<int64_t>(a.nb_fold) * kPrepThreads) {
      const int64_t bh = i / E4, e4 = i % E4;
      float4* dst = reinterpret_cast<float4*>(a.srest) + bh * E4 + e4;
      float4 acc = *dst;
      const float4* src = reinterpret_cast<const float4*>(a.partial) + bh * a.parts * E4 + e4;
      for (int r = 0; r < a.parts; ++r) {
        const float4 v = src[r * E4];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      *dst = acc;
      if (e4 < dd4) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&lo);
        w.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(a.srest_bf16)[bh * dd4 + e4] = w;
      }
    }
    return;
  }
  b -= a.nb_fold;

  // ---- K, V into the ring (K turned), or Q turned into its workspace copy
  const bool is_kv = b < a.nb_kv;
  if (is_kv || b < a.nb_kv + a.nb_q) {
    const int nb = is_kv ? a.nb_kv : a.nb_q;
    const int bb = is_kv ? b : b - a.nb_kv;
    const bool turn = a.half_t > 0;
    if (turn) {
      // (cos, sin) of every (chunk frame, pair): frame f of the chunk sits at the capped
      // offset min(p0 + f, cap - 1) from the reference frame
      for (int i = threadIdx.x; i < a.chunk_frames * a.half_t; i += kPrepThreads) {
        const int f = i / a.half_t, pr = i % a.half_t;
        const int p = min(a.p0 + f, a.cap - 1);
        float c, s;
        rope_cos_sin(p, a.theta[pr], &c, &s);
        cs_table[i] = make_float2(c, s);
      }
      __syncthreads();
    }
    const int64_t total = row_vecs * a.BH;
    const int64_t stride = static_cast<int64_t>(nb) * kPrepThreads;
    // kPrepUnroll vectors per thread at a time: every load is issued before the first store
    for (int64_t i0 = static_cast<int64_t>(bb) * kPrepThreads + threadIdx.x; i0 < total; i0 += stride * kPrepUnroll) {
      uint4 x[kPrepUnroll], y[kPrepUnroll];
#pragma unroll
      for (int u = 0; u < kPrepUnroll; ++u) {
        const int64_t i = i0 + u * stride;
        if (i >= total) break;
        if (is_kv) {
          x[u] = reinterpret_cast<const uint4*>(a.k)[i];
          y[u] = reinterpret_cast<const uint4*>(a.v)[i];
        } else {
          x[u] = reinterpret_cast<const uint4*>(a.q)[i];
        }
      }
#pragma unroll
      for (int u = 0; u < kPrepUnroll; ++u) {
        const int64_t i = i0 + u * stride;
        if (i >= total) break;
        const int64_t bh = i / row_vecs, off = i % row_vecs;
        const int col = static_cast<int>(off % cols);
        const float2* cs = cs_table + (static_cast<int>(off / cols) / a.tokens_per_frame) * a.half_t;
        if (turn) turn_vector<T>(x[u], col, a.half_t, cs);
        if (is_kv) {
          const int64_t dst = (bh * a.nslots + a.slot) * row_vecs + off;
          reinterpret_cast<uint4*>(a.ring_k)[dst] = x[u];
          reinterpret_cast<uint4*>(a.ring_v)[dst] = y[u];
        } else {
          reinterpret_cast<uint4*>(a.q_out)[i] = x[u];
        }
      }
    }
    return;
  }
}

int blocks_for(int64_t n, int cap) {
  const int64_t b = (n + kPrepThreads - 1) / kPrepThreads;
  return static_cast<int>(b < cap ? b : cap);
}

}  // namespace

cudaError_t launch_stream_prep(StreamPrepArgs a, int num_sms, cudaStream_t s) {
  const int E = a.elem_bytes == 4 ? 4 : 8;
  if (a.d % E != 0 || (a.half_t > 0 && a.chunk_frames * a.half_t * 8 > 48 * 1024)) return cudaErrorInvalidValue;
  if (a.pairs && (a.cap_entries + 1 > kMaxStreamOrderBins || a.grid < 1 || a.grid > kMaxStreamOrderGrid ||
                  a.BH * a.nqt > kMaxStreamOrderItems || !a.done_counter)) return cudaErrorInvalidValue;
  const int64_t vecs = static_cast<int64_t>(a.L) * (a.d / E) * a.BH;
  a.nb_fold = a.partial ? blocks_for((static_cast<int64_t>(a.d) * a.d + a.d) / 4 * a.BH, 2 * num_sms) : 0;
  a.nb_kv = blocks_for((vecs + kPrepUnroll - 1) / kPrepUnroll, 8 * num_sms);
  a.nb_q = a.q_out ? blocks_for((vecs + kPrepUnroll - 1) / kPrepUnroll, 4 * num_sms) : 0;
  a.nb_layout = (a.BH * a.nqt + kPrepThreads / 32 - 1) / (kPrepThreads / 32);
  const int grid = a.nb_fold + a.nb_kv + a.nb_q + a.nb_layout;
  const size_t smem = a.half_t > 0 ? sizeof(float2) * a.chunk_frames * a.half_t : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPrepThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return a.elem_bytes == 4 ? cudaLaunchKernelEx(&cfg, stream_prep_kernel<float>, a)
                           : cudaLaunchKernelEx(&cfg, stream_prep_kernel<__nv_bfloat16>, a);
}

}  // namespace hyat
