// C ABI of libhyat: handles, workspace planning, argument validation and
// launch sequencing on the caller's stream.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "hyat_internal.h"

using namespace hyat;

namespace {

constexpr int kKinds = 5;  // state, complement, attention, stream fold, stream prep
enum Kind { K_STATE = 0, K_COMPLEMENT = 1, K_ATTN = 2, K_FOLD = 3, K_PREP = 4 };

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int32_t nseg_pad64(int32_t n) { return (n + 63) / 64 * 64; }

struct Plan {
  size_t status = 0, work = 0, entries = 0, pairs = 0, cm = 0, cm_bf16 = 0, sseg = 0, srest = 0, srest_bf16 = 0;
  size_t ring_k = 0, ring_v = 0, mask = 0, fold_partial = 0, q_rot = 0, redo = 0, total = 0;
  int64_t n_work = 0, n_entries = 0;
};

int64_t elem_bytes(const hyat_config& c) { return c.dtype == HYAT_F32 ? 4 : 2; }

// The streaming fold splits the evicted chunk of every (b, h) into token ranges so that the
// state kernel fills the GPU (one range per SM, about); the workspace holds up to
// kFoldPartsMax ranges per (b, h), enough for 256 SMs.
constexpr int32_t kFoldPartsMax = 32;
int32_t fold_parts_cap(const hyat_config& c) {
  const int64_t BH = int64_t(c.B) * c.H;
  const int64_t by_sms = std::max<int64_t>(1, 256 / std::max<int64_t>(BH, 1));
  const int64_t by_len = (stream_chunk_tokens(c) + 127) / 128;
  return static_cast<int32_t>(std::min<int64_t>({by_sms, by_len, kFoldPartsMax}));
}

// Offsets of every region in the caller's workspace.
Plan make_plan(const hyat_config& c, int64_t n_work, int64_t n_entries, const Layout& L) {
  Plan p;
  const int64_t BH = int64_t(c.B) * c.H;
  const int64_t E = int64_t(c.d) * c.d + c.d;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 256); return o; };
  p.n_work = n_work;
  p.n_entries = n_entries;
  p.status = take(256);
  p.work = take(sizeof(WorkItem) * std::max<int64_t>(n_work, 1));
  p.entries = take(sizeof(Entry) * std::max<int64_t>(n_entries, 1));
  p.pairs = take(sizeof(int4) * std::max<int64_t>(n_work, 1));
  if (c.mode == HYAT_MODE_STREAM) {
    const int64_t Lc = stream_chunk_tokens(c), slots = stream_ring_slots(c), nqt = tiles(Lc);
    p.srest = take(sizeof(float) * BH * E);
    p.srest_bf16 = take(2 * BH * c.d * c.d);
    p.ring_k = take(size_t(BH * slots * Lc * c.d * elem_bytes(c)));
    p.ring_v = take(size_t(BH * slots * Lc * c.d * elem_bytes(c)));
    p.mask = take(size_t(c.mask_heads) * nqt * nqt * slots);
    p.fold_partial = take(sizeof(float) * BH * fold_parts_cap(c) * E);
    if (c.rope_t_dims > 0) p.q_rot = take(size_t(BH * Lc * c.d * elem_bytes(c)));
    p.redo = take(sizeof(int4) * std::max<int64_t>(n_work, 1));
  } else {
    p.cm = take(sizeof(float) * size_t(L.cm_heads) * L.nqg * L.nseg);
    if (c.mode == HYAT_MODE_BLOCKMASK || c.mode == HYAT_MODE_RADIAL)
      p.cm_bf16 = take(2 * size_t(L.cm_heads) * L.nqg * nseg_pad64(L.nseg));
    p.sseg = take(sizeof(float) * BH * L.nseg * E);
    p.srest = take(sizeof(float) * BH * L.nqg * E);
    p.srest_bf16 = take(2 * BH * L.nqg * c.d * c.d);
    p.redo = take(sizeof(int4) * std::max<int64_t>(n_work, 1));
  }
  p.total = off;
  return p;
}

// Counts of work items and entries (exact, or an upper bound for BLOCKMASK without a mask).
bool plan_counts(const hyat_config& c, const uint8_t* host_mask, Layout* L, int64_t* n_work,
                 int64_t* n_entries, std::string* err) {
  if (c.mode == HYAT_MODE_STREAM) {
    *err = build_layout(c, nullptr, L);
    const int64_t nqt = tiles(stream_chunk_tokens(c));
    *n_work = int64_t(c.B) * c.H * nqt;
    *n_entries = *n_work * nqt * stream_ring_slots(c);
    return err->empty();
  }
  if (c.mode == HYAT_MODE_BLOCKMASK && host_mask == nullptr) {
    const int64_t nT = tiles(rows_q(c));
    L->nseg = static_cast<int32_t>(nT);
    L->nqg = static_cast<int32_t>(nT);
    L->cm_heads = c.mask_heads;
    *n_work = int64_t(c.B) * c.H * nT;
    *n_entries = int64_t(c.mask_heads) * nT * nT;
    return true;
  }
  *err = build_layout(c, host_mask, L);
  if (!err->empty()) return false;
  *n_work = static_cast<int64_t>(L->work.size());
  *n_entries = static_cast<int64_t>(L->entries.size());
  return true;
}

}  // namespace

struct hyat_ctx {
  hyat_config cfg{};
  Layout lay;
  Plan plan;
  int32_t BH = 0, E = 0;
  int64_t rq = 0, rk = 0;
  char* ws = nullptr;
  uint32_t* d_status = nullptr;
  WorkItem* d_work = nullptr;
  Entry* d_entries = nullptr;
  int4* d_pairs = nullptr;
  int32_t n_pairs = 0;
  // one query tile per CTA (attn_single_kernel) with its redo list; the two counters live in
  // the zeroed status region
  bool single = false;
  bool wide = false;                 // two softmax warps per row (the default), with a redo list
  bool order_on_device = false;      // streaming split pairs, ordered by the prep kernel each step
  uint32_t* d_order_done = nullptr;  // the prep kernel's count of finished layout blocks
  int4* d_redo = nullptr;
  int32_t* d_redo_count = nullptr;
  uint32_t* d_redo_done = nullptr;
  float* d_cm = nullptr;
  uint16_t* d_cm_bf16 = nullptr;
  bool use_gemm = false;             // tensor-core complement (block masks)
  float* d_sseg = nullptr;
  float* d_srest = nullptr;
  uint16_t* d_srest_bf16 = nullptr;
  void* d_ring_k = nullptr;
  void* d_ring_v = nullptr;
  uint8_t* d_mask = nullptr;
  int32_t step = 0;
  int32_t folded_step = -1;          // step whose evicted chunk is already in S, z
  int32_t last_step = -1;            // step of the last streaming call (its layout is on the device)
  void* d_q_rot = nullptr;           // fused RoPE: the turned Q of the current call
  double rope_theta[64] = {};        // fused RoPE: base^(-2i / t_dims)
  // graph replay of steady streaming steps: one captured step per (ring phase, fold, pointers)
  struct StepGraph {
    cudaGraphExec_t exec;
    int32_t phase;
    bool fold;
    const void *q, *k, *v, *o, *mask;
  };
  std::vector<StepGraph> graphs;
  cudaStream_t cap_stream = nullptr;
  float* d_fold_partial = nullptr;
  int32_t fold_parts = 1, fold_part_len = 0;
  bool use_tc = false;
  int num_sms = 148;
  cudaStream_t last_stream = nullptr;
  std::string err;
  bool profiling = false;
  struct Rec { int kind; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> free_events;
  double ms[kKinds] = {};
  int64_t launches[kKinds] = {};
};

namespace {

hyat_status fail(hyat_ctx* h, hyat_status s, const std::string& msg) {
  if (h) h->err = msg;
  return s;
}

hyat_status cuda_fail(hyat_ctx* h, cudaError_t e, const char* what) {
  return fail(h, HYAT_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

cudaEvent_t get_event(hyat_ctx* h) {
  if (!h->free_events.empty()) {
    cudaEvent_t e = h->free_events.back();
    h->free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Times the launches issued by `fn` when profiling is on.
template <typename Fn>
cudaError_t timed(hyat_ctx* h, int kind, cudaStream_t s, Fn&& fn) {
  if (!h->profiling) return fn();
  cudaEvent_t a = get_event(h), b = get_event(h);
  if (a) cudaEventRecord(a, s);
  cudaError_t e = fn();
  if (b) cudaEventRecord(b, s);
  if (a && b) h->recs.push_back({kind, a, b});
  return e;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hyat_status check_ptrs(hyat_ctx* h, const void* q, const void* k, const void* v, const void* o) {
  if (!q || !k || !v || !o) return fail(h, HYAT_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(h, HYAT_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return HYAT_OK;
}

AttnArgs attn_args(hyat_ctx* h, const void* q, const void* k, const void* v, void* o, int64_t n_work,
                   int32_t nqg) {
  AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.o = o;
  a.q_rows = h->rq;
  a.k_rows = h->rk;
  a.work = h->d_work;
  a.n_work = static_cast<int32_t>(n_work);
  a.entries = h->d_entries;
  a.pairs = h->d_pairs;
  a.n_pairs = h->n_pairs;
  a.srest = h->d_srest;
  a.srest_bf16 = h->d_srest_bf16;
  a.nqg = nqg;
  a.d = h->cfg.d;
  a.dtype = h->cfg.dtype;
  a.BH = h->BH;
  const float scale = h->cfg.scale > 0.0f ? h->cfg.scale : 1.0f / std::sqrt(float(h->cfg.d));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = h->d_status;
  a.test_timeout = (h->cfg.flags & HYAT_FLAG_TEST_DEVICE_TIMEOUT) ? 1 : 0;
  a.phi = h->cfg.phi;
  return a;
}

hyat_status launch_attention(hyat_ctx* h, const AttnArgs& a, cudaStream_t s) {
  cudaError_t e = timed(h, K_ATTN, s, [&] {
    if (!h->use_tc) return launch_attn_simt(a, s);
    if (h->wide) {
      cudaError_t r = launch_attn_wide(a, h->d_redo_count, h->d_redo, static_cast<int32_t>(h->plan.n_work),
                                       h->num_sms, s);
      if (r == cudaSuccess) r = launch_attn_tc_redo(a, h->d_redo, h->d_redo_count, h->d_redo_done, h->num_sms, s);
      return r;
    }
    if (!h->single) return launch_attn_tc(a, h->num_sms, s);
    cudaError_t r = launch_attn_single(a, h->d_redo_count, h->d_redo, h->num_sms, s);
    if (r == cudaSuccess) r = launch_attn_tc_redo(a, h->d_redo, h->d_redo_count, h->d_redo_done, h->num_sms, s);
    return r;
  });
  if (e != cudaSuccess) return cuda_fail(h, e, "attention kernel");
  return HYAT_OK;
}

}  // namespace

extern "C" {

const char* hyat_status_string(hyat_status s) {
  switch (s) {
    case HYAT_OK: return "ok";
    case HYAT_ERR_INVALID_ARG: return "invalid argument";
    case HYAT_ERR_UNSUPPORTED: return "unsupported";
    case HYAT_ERR_CUDA: return "CUDA error";
    case HYAT_ERR_DEVICE_TIMEOUT: return "device timeout";
    case HYAT_ERR_STATE: return "bad stream state";
  }
  return "unknown status";
}

const char* hyat_last_error(hyat_handle h) { return h ? h->err.c_str() : "null handle"; }

size_t hyat_workspace_bytes(const hyat_config* cfg) {
  if (!cfg || !validate_config(*cfg).empty()) return 0;
  Layout L;
  int64_t nw = 0, ne = 0;
  std::string err;
  if (!plan_counts(*cfg, nullptr, &L, &nw, &ne, &err)) return 0;
  return make_plan(*cfg, nw, ne, L).total;
}

hyat_status hyat_create(const hyat_config* cfg, void* workspace, size_t workspace_bytes,
                        const uint8_t* host_mask, hyat_handle* out) {
  if (!out) return HYAT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return HYAT_ERR_INVALID_ARG;
  const std::string verr = validate_config(*cfg);
  if (!verr.empty()) return HYAT_ERR_INVALID_ARG;
  if (cfg->mode == HYAT_MODE_BLOCKMASK && !host_mask) return HYAT_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return HYAT_ERR_INVALID_ARG;

  hyat_ctx* h = new (std::nothrow) hyat_ctx();
  if (!h) return HYAT_ERR_CUDA;
  h->cfg = *cfg;
  h->BH = cfg->B * cfg->H;
  h->E = cfg->d * cfg->d + cfg->d;
  h->rq = rows_q(*cfg);
  h->rk = rows_k(*cfg);
  int64_t nw = 0, ne = 0;
  std::string err;
  if (!plan_counts(*cfg, host_mask, &h->lay, &nw, &ne, &err)) {
    delete h;
    return HYAT_ERR_INVALID_ARG;
  }
  h->plan = make_plan(*cfg, nw, ne, h->lay);
  const size_t bound = hyat_workspace_bytes(cfg);
  if (workspace_bytes < h->plan.total || workspace_bytes < bound) {
    delete h;
    return HYAT_ERR_INVALID_ARG;
  }
  char* ws = static_cast<char*>(workspace);
  h->ws = ws;
  h->d_status = reinterpret_cast<uint32_t*>(ws + h->plan.status);
  h->d_work = reinterpret_cast<WorkItem*>(ws + h->plan.work);
  h->d_entries = reinterpret_cast<Entry*>(ws + h->plan.entries);
  h->d_pairs = reinterpret_cast<int4*>(ws + h->plan.pairs);
  h->d_srest = reinterpret_cast<float*>(ws + h->plan.srest);
  h->d_srest_bf16 = reinterpret_cast<uint16_t*>(ws + h->plan.srest_bf16);
  if (cfg->mode == HYAT_MODE_STREAM) {
    h->d_ring_k = ws + h->plan.ring_k;
    h->d_ring_v = ws + h->plan.ring_v;
    h->d_mask = reinterpret_cast<uint8_t*>(ws + h->plan.mask);
    h->d_fold_partial = reinterpret_cast<float*>(ws + h->plan.fold_partial);
    if (h->plan.q_rot) h->d_q_rot = ws + h->plan.q_rot;
    h->d_redo = reinterpret_cast<int4*>(ws + h->plan.redo);
    if (cfg->rope_t_dims > 0) {
      const double base = cfg->rope_base > 0.0f ? static_cast<double>(cfg->rope_base) : 10000.0;
      for (int i = 0; i < cfg->rope_t_dims / 2; ++i) h->rope_theta[i] = std::pow(base, -2.0 * i / cfg->rope_t_dims);
    }
  } else {
    h->d_cm = reinterpret_cast<float*>(ws + h->plan.cm);
    if (h->plan.cm_bf16) h->d_cm_bf16 = reinterpret_cast<uint16_t*>(ws + h->plan.cm_bf16);
    h->d_sseg = reinterpret_cast<float*>(ws + h->plan.sseg);
    h->d_redo = reinterpret_cast<int4*>(ws + h->plan.redo);
  }
  h->d_redo_count = reinterpret_cast<int32_t*>(ws + h->plan.status + 64);
  h->d_redo_done = reinterpret_cast<uint32_t*>(ws + h->plan.status + 128);
  h->d_order_done = reinterpret_cast<uint32_t*>(ws + h->plan.status + 192);

  int dev = 0, major = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) {
    delete h;
    return HYAT_ERR_CUDA;
  }
  h->use_tc = cfg->dtype == HYAT_BF16 && !(cfg->flags & HYAT_FLAG_SIMT) && major == 10 &&
              attn_tc_supported(cfg->d, cfg->dtype);
  h->use_gemm = h->use_tc && h->d_cm_bf16 != nullptr && complement_tc_supported(cfg->d, h->lay.nqg);
  h->wide = h->use_tc && !(cfg->flags & (HYAT_FLAG_SINGLE_TILE | HYAT_FLAG_PAIR_ONE_WARP));
  if (cfg->mode == HYAT_MODE_STREAM) {
    // token ranges of the fold: about one per SM, whole 64-token stages
    const int32_t Lc = stream_chunk_tokens(*cfg);
    const int32_t want = std::max<int32_t>(1, std::min<int32_t>(fold_parts_cap(*cfg), h->num_sms / std::max(h->BH, 1)));
    const int32_t stages = (Lc + 63) / 64;
    h->fold_part_len = (stages + want - 1) / want * 64;
    h->fold_parts = (Lc + h->fold_part_len - 1) / h->fold_part_len;
  }

  // test hook: every query tile without softmax keys, so a call returns the linear branch
  if (cfg->flags & HYAT_FLAG_TEST_LINEAR_BRANCH)
    for (WorkItem& w : h->lay.work) w.entry_end = w.entry_begin;

  // layout tables and zeroed state
  e = cudaMemset(ws, 0, h->plan.status + 256);
  if (e == cudaSuccess && !h->lay.work.empty())
    e = cudaMemcpy(h->d_work, h->lay.work.data(), sizeof(WorkItem) * h->lay.work.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !h->lay.entries.empty())
    e = cudaMemcpy(h->d_entries, h->lay.entries.data(), sizeof(Entry) * h->lay.entries.size(),
                   cudaMemcpyHostToDevice);
  std::vector<int4> pairs;
  if (cfg->mode == HYAT_MODE_STREAM) {
    const int32_t nqt = tiles(stream_chunk_tokens(*cfg));
    pairs = build_stream_pairs(h->BH, nqt);
    if (prefer_split_pairs(pairs.size(), h->num_sms)) {
      pairs = build_split_pairs(size_t(h->BH) * nqt);
      // the key-tile counts change with every step's mask: the prep kernel deals the pairs
      // out largest first (a table of one bin per possible count)
      h->order_on_device = h->use_tc && nqt * stream_ring_slots(*cfg) + 1 <= kMaxStreamOrderBins &&
                           h->num_sms <= kMaxStreamOrderGrid && int64_t(h->BH) * nqt <= kMaxStreamOrderItems;
    }
  } else if (h->use_tc && (cfg->flags & HYAT_FLAG_SINGLE_TILE)) {
    pairs = build_single_items(h->lay.work, h->num_sms);
    h->single = true;
  } else {
    pairs = choose_pairs(h->lay.work, h->num_sms);
  }
  h->n_pairs = static_cast<int32_t>(pairs.size());
  if (e == cudaSuccess && !pairs.empty())
    e = cudaMemcpy(h->d_pairs, pairs.data(), sizeof(int4) * pairs.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !h->lay.cm.empty())
    e = cudaMemcpy(h->d_cm, h->lay.cm.data(), sizeof(float) * h->lay.cm.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && h->d_cm_bf16) {
    // the 0/1 complement matrix as bf16 (exact), rows padded to a multiple of 64 segments
    const int32_t np = nseg_pad64(h->lay.nseg);
    std::vector<uint16_t> cmb(size_t(h->lay.cm_heads) * h->lay.nqg * np, 0);
    for (int32_t m = 0; m < h->lay.cm_heads; ++m)
      for (int32_t g = 0; g < h->lay.nqg; ++g)
        for (int32_t sg = 0; sg < h->lay.nseg; ++sg)
          if (h->lay.cm[(size_t(m) * h->lay.nqg + g) * h->lay.nseg + sg] != 0.0f)
            cmb[(size_t(m) * h->lay.nqg + g) * np + sg] = 0x3F80;   // bf16 1.0
    e = cudaMemcpy(h->d_cm_bf16, cmb.data(), 2 * cmb.size(), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess && cfg->mode == HYAT_MODE_STREAM)
    e = cudaMemset(ws + h->plan.srest, 0, h->plan.total - h->plan.srest);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    delete h;
    return HYAT_ERR_CUDA;
  }
  *out = h;
  return HYAT_OK;
}

hyat_status hyat_destroy(hyat_handle h) {
  if (!h) return HYAT_OK;
  for (auto& r : h->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->free_events) cudaEventDestroy(e);
  for (auto& g : h->graphs) cudaGraphExecDestroy(g.exec);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  delete h;
  return HYAT_OK;
}

hyat_status hyat_fwd_bidir(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                           void* stream) {
  if (!h) return HYAT_ERR_INVALID_ARG;
  if (h->cfg.mode == HYAT_MODE_STREAM) return fail(h, HYAT_ERR_INVALID_ARG, "handle is in STREAM mode");
  hyat_status st = check_ptrs(h, q, k, v, o);
  if (st != HYAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  const Layout& L = h->lay;
  SegStateArgs sa{};
  sa.k = k; sa.v = v; sa.rows_per_bh = h->rk;
  sa.BH = h->BH; sa.d = h->cfg.d; sa.dtype = h->cfg.dtype; sa.phi = h->cfg.phi;
  sa.nseg = L.nseg; sa.seg_base = 0; sa.seg_stride = L.seg_stride; sa.seg_len = L.seg_len;
  sa.out = h->d_sseg; sa.accumulate = 0; sa.status = h->d_status;
  if (h->use_gemm) {        // hi/lo bf16 parts for the tensor-core complement, in the same bytes
    sa.out_hi = reinterpret_cast<uint16_t*>(h->d_sseg);
    sa.out_lo = sa.out_hi + size_t(h->BH) * L.nseg * h->E;
  }
  cudaError_t e = timed(h, K_STATE, s, [&] {
    return h->use_tc ? launch_seg_state_tc(sa, h->num_sms, s) : launch_seg_state(sa, s);
  });
  if (e != cudaSuccess) return cuda_fail(h, e, "segment state kernel");
  ComplementArgs ca{};
  ca.sseg = h->d_sseg; ca.cm = h->d_cm; ca.srest = h->d_srest;
  ca.srest_bf16 = h->use_tc ? h->d_srest_bf16 : nullptr;
  ca.write_f32_s = h->use_tc ? 0 : 1;       // the tensor-core path reads S as bf16, z as fp32
  ca.BH = h->BH; ca.H = h->cfg.H; ca.cm_heads = L.cm_heads; ca.nseg = L.nseg; ca.nqg = L.nqg; ca.E = h->E;
  ca.d = h->cfg.d;
  if (h->use_gemm) {
    ComplementTcArgs ga{};
    ga.cm_bf16 = h->d_cm_bf16;
    ga.seg_hi = sa.out_hi;
    ga.seg_lo = sa.out_lo;
    ga.srest = h->d_srest;
    ga.srest_bf16 = h->d_srest_bf16;
    ga.write_f32_s = 0;
    ga.BH = h->BH; ga.H = h->cfg.H; ga.mask_heads = L.cm_heads; ga.nqg = L.nqg; ga.nseg = L.nseg;
    ga.nseg_pad = nseg_pad64(L.nseg); ga.E = h->E; ga.status = h->d_status;
    e = timed(h, K_COMPLEMENT, s, [&] { return launch_complement_tc(ga, h->num_sms, s); });
  } else {
    e = timed(h, K_COMPLEMENT, s, [&] { return launch_complement(ca, s); });
  }
  if (e != cudaSuccess) return cuda_fail(h, e, "complement kernel");
  if (h->cfg.flags & HYAT_FLAG_TEST_SOFTMAX_BRANCH) {
    // test hook: no linear state, so the call returns the softmax branch alone
    e = cudaMemsetAsync(h->d_srest, 0, sizeof(float) * size_t(h->BH) * L.nqg * h->E, s);
    if (e == cudaSuccess && h->d_srest_bf16)
      e = cudaMemsetAsync(h->d_srest_bf16, 0, 2 * size_t(h->BH) * L.nqg * h->cfg.d * h->cfg.d, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "branch test hook");
  }
  return launch_attention(h, attn_args(h, q, k, v, o, h->plan.n_work, L.nqg), s);
}

namespace {

// Launches of one streaming call for the current chunk, all on `s` and all capturable: the
// fold of the chunk leaving the window (if `fold`), the prep kernel (fold reduce, K and V into
// the ring slot, the fused RoPE, the step's layout from the device mask `mask`), then the
// attention. Every argument is a function of the step's ring phase once the window is full.
hyat_status enqueue_stream_call(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                                const uint8_t* mask, bool fold, const StreamGeometry& g, int32_t step,
                                cudaStream_t s) {
  const hyat_config& c = h->cfg;
  const int32_t Lc = stream_chunk_tokens(c), nwc = stream_window_chunks(c), nqt = tiles(Lc);
  const int32_t slot = g.write_slot;
  cudaError_t e = timed(h, K_FOLD, s, [&]() -> cudaError_t {
    if (!fold) return cudaSuccess;
    // chunk s - nwc leaves the window: its slot is the one this call writes
    SegStateArgs sa{};
    sa.k = h->d_ring_k; sa.v = h->d_ring_v; sa.rows_per_bh = h->rk;
    sa.BH = h->BH; sa.d = c.d; sa.dtype = c.dtype; sa.phi = c.phi;
    sa.nseg = 1; sa.seg_base = slot * Lc; sa.seg_stride = Lc; sa.seg_len = Lc;
    sa.out = h->d_srest; sa.accumulate = 1; sa.status = h->d_status;
    if (!h->use_tc) return launch_seg_state(sa, s);
    // token ranges in parallel; the prep kernel sums them in order into S, z
    sa.parts = h->fold_parts; sa.part_len = h->fold_part_len; sa.partial = h->d_fold_partial;
    return launch_seg_state_tc(sa, h->num_sms, s);
  });
  if (e != cudaSuccess) return cuda_fail(h, e, "stream fold");
  StreamPrepArgs pa{};
  pa.BH = h->BH; pa.L = Lc; pa.d = c.d; pa.elem_bytes = static_cast<int32_t>(elem_bytes(c));
  if (fold && h->use_tc) {
    pa.partial = h->d_fold_partial; pa.srest = h->d_srest; pa.srest_bf16 = h->d_srest_bf16; pa.parts = h->fold_parts;
  }
  pa.k = k; pa.v = v; pa.ring_k = h->d_ring_k; pa.ring_v = h->d_ring_v;
  pa.nslots = stream_ring_slots(c); pa.slot = slot;
  if (c.rope_t_dims > 0) {
    pa.q = q; pa.q_out = h->d_q_rot;
    pa.half_t = c.rope_t_dims / 2; pa.chunk_frames = c.chunk_frames; pa.tokens_per_frame = c.tokens_per_frame;
    // offset of the chunk's first frame from the first frame of the oldest rolling-window
    // chunk (0 while the window holds none yet: a sink chunk at its own step)
    pa.p0 = step >= g.first_window ? (step - g.first_window) * c.chunk_frames : 0;
    pa.cap = c.rope_cap;
    for (int i = 0; i < pa.half_t; ++i) pa.theta[i] = h->rope_theta[i];
  }
  pa.mask = mask; pa.work = h->d_work; pa.entries = h->d_entries; pa.status = h->d_status;
  pa.H = c.H; pa.mask_heads = c.mask_heads; pa.nqt = nqt; pa.nkt = nqt * g.n_visible;
  pa.cap_entries = nqt * stream_ring_slots(c); pa.nwc = nwc;
  pa.n_sink_visible = g.n_sink_visible; pa.first_window_mod = g.first_window % nwc;
  if (h->order_on_device) {
    pa.pairs = h->d_pairs; pa.grid = std::min(h->n_pairs, h->num_sms); pa.done_counter = h->d_order_done;
  }
  // When this call folds, the kernel ahead of the prep kernel is the fold's state kernel,
  // which triggers the prep grid only after its own programmatic wait: by then everything
  // enqueued before this call (the previous step's attention, a kernel that wrote a device
  // mask) has finished, so the prep kernel's layout blocks need not wait. Without a fold the
  // kernel ahead could be anything the caller enqueued, so they wait.
  pa.layout_early = (h->use_tc && fold) ? 1 : 0;
  e = timed(h, K_PREP, s, [&] { return launch_stream_prep(pa, h->num_sms, s); });
  if (e != cudaSuccess) return cuda_fail(h, e, "stream prep kernel");
  const void* qa = c.rope_t_dims > 0 ? h->d_q_rot : q;
  return launch_attention(h, attn_args(h, qa, h->d_ring_k, h->d_ring_v, o, int64_t(h->BH) * nqt, 1), s);
}

enum class MaskSrc { kHost, kDevice, kGraph };
constexpr size_t kMaxStepGraphs = 16;

// One streaming call for the current chunk. The first call of a chunk folds the chunk that
// leaves the window into S, z; every call writes its K, V into the chunk's ring slot and
// attends. `commit` marks the chunk's final call: the step counter then advances, and the
// K, V just written stay in the window.
hyat_status stream_call(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                        const uint8_t* step_mask, MaskSrc src, void* stream, bool commit) {
  if (!h) return HYAT_ERR_INVALID_ARG;
  if (h->cfg.mode != HYAT_MODE_STREAM) return fail(h, HYAT_ERR_INVALID_ARG, "handle is not in STREAM mode");
  hyat_status st = check_ptrs(h, q, k, v, o);
  if (st != HYAT_OK) return st;
  const hyat_config& c = h->cfg;
  const int32_t Lc = stream_chunk_tokens(c), nwc = stream_window_chunks(c), nqt = tiles(Lc);
  const int32_t s_ = h->step;
  const StreamGeometry g = stream_geometry(c, s_);
  const int32_t nkt = nqt * g.n_visible;
  const size_t mask_bytes = size_t(c.mask_heads) * nqt * nkt;
  if (src == MaskSrc::kHost && step_mask) {
    for (int32_t m = 0; m < c.mask_heads; ++m)
      for (int32_t i = 0; i < nqt; ++i)
        if (!step_mask[(size_t(m) * nqt + i) * nkt + nqt * (g.n_visible - 1) + i])
          return fail(h, HYAT_ERR_INVALID_ARG, "step mask: diagonal tile of the newest chunk must be kept");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  const bool fold = g.evicted >= 0 && h->folded_step != s_;
  const bool steady = g.n_window == nwc && g.n_sink_visible == stream_sink_chunks(c);
  if (src == MaskSrc::kGraph && steady && !h->profiling) {
    const int32_t phase = s_ % nwc;
    auto it = std::find_if(h->graphs.begin(), h->graphs.end(), [&](const hyat_ctx::StepGraph& x) {
      return x.phase == phase && x.fold == fold && x.q == q && x.k == k && x.v == v && x.o == o && x.mask == step_mask;
    });
    if (it == h->graphs.end()) {
      // capture this step; the cache keeps the kMaxStepGraphs most recent captures (callers
      // that rotate a few input buffers reuse one graph per phase and buffer set)
      if (h->graphs.size() >= kMaxStepGraphs) {
        cudaGraphExecDestroy(h->graphs.front().exec);
        h->graphs.erase(h->graphs.begin());
      }
      cudaError_t e = cudaSuccess;
      if (!h->cap_stream) e = cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking);
      if (e != cudaSuccess) return cuda_fail(h, e, "capture stream");
      e = cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal);
      if (e != cudaSuccess) return cuda_fail(h, e, "begin capture");
      if (!step_mask) e = cudaMemsetAsync(h->d_mask, 1, mask_bytes, h->cap_stream);
      st = e == cudaSuccess
               ? enqueue_stream_call(h, q, k, v, o, step_mask ? step_mask : h->d_mask, fold, g, s_, h->cap_stream)
               : cuda_fail(h, e, "step mask fill");
      cudaGraph_t graph = nullptr;
      const cudaError_t e2 = cudaStreamEndCapture(h->cap_stream, &graph);
      if (st != HYAT_OK) {
        if (graph) cudaGraphDestroy(graph);
        return st;
      }
      if (e2 != cudaSuccess) return cuda_fail(h, e2, "end capture");
      cudaGraphExec_t exec = nullptr;
      e = cudaGraphInstantiate(&exec, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess) return cuda_fail(h, e, "graph instantiate");
      h->graphs.push_back({exec, phase, fold, q, k, v, o, step_mask});
      it = h->graphs.end() - 1;
    }
    const cudaError_t e = cudaGraphLaunch(it->exec, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "graph launch");
  } else {
    const uint8_t* m = step_mask;
    cudaError_t e = cudaSuccess;
    if (src == MaskSrc::kHost && step_mask)
      e = cudaMemcpyAsync(h->d_mask, step_mask, mask_bytes, cudaMemcpyHostToDevice, s);
    else if (!step_mask)
      e = cudaMemsetAsync(h->d_mask, 1, mask_bytes, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "step mask upload");
    if (src == MaskSrc::kHost || !step_mask) m = h->d_mask;
    st = enqueue_stream_call(h, q, k, v, o, m, fold, g, s_, s);
    if (st != HYAT_OK) return st;
  }
  if (fold) h->folded_step = s_;
  h->last_step = s_;
  if (commit) h->step += 1;
  return HYAT_OK;
}

}  // namespace

hyat_status hyat_fwd_stream_step(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                                 const uint8_t* host_step_mask, void* stream) {
  return stream_call(h, q, k, v, o, host_step_mask, MaskSrc::kHost, stream, true);
}

hyat_status hyat_fwd_stream_denoise(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                                    const uint8_t* host_step_mask, void* stream) {
  return stream_call(h, q, k, v, o, host_step_mask, MaskSrc::kHost, stream, false);
}

hyat_status hyat_fwd_stream_step_dev(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                                     const uint8_t* dev_step_mask, void* stream) {
  return stream_call(h, q, k, v, o, dev_step_mask, MaskSrc::kDevice, stream, true);
}

hyat_status hyat_fwd_stream_step_graph(hyat_handle h, const void* q, const void* k, const void* v, void* o,
                                       const uint8_t* dev_step_mask, void* stream) {
  return stream_call(h, q, k, v, o, dev_step_mask, MaskSrc::kGraph, stream, true);
}

hyat_status hyat_stream_get_layout(hyat_handle h, int32_t* work, size_t work_cap, int32_t* entries,
                                   size_t entries_cap, int32_t* info, size_t info_len, int64_t* counts) {
  if (!h || !counts) return HYAT_ERR_INVALID_ARG;
  if (h->cfg.mode != HYAT_MODE_STREAM) return fail(h, HYAT_ERR_INVALID_ARG, "handle is not in STREAM mode");
  if (h->last_step < 0) return fail(h, HYAT_ERR_STATE, "no streaming call yet");
  const int32_t nqt = tiles(stream_chunk_tokens(h->cfg)), slots = stream_ring_slots(h->cfg);
  const int64_t n_work = int64_t(h->BH) * nqt, n_ent = n_work * nqt * slots;
  counts[0] = n_work;
  counts[1] = n_ent;
  counts[2] = h->last_step;
  if (!work || !entries || !info) return HYAT_OK;
  if (work_cap < size_t(n_work) * 8 || entries_cap < size_t(n_ent) * 2)
    return fail(h, HYAT_ERR_INVALID_ARG, "layout buffers too small");
  if (hyat_stream_plan(&h->cfg, h->last_step, info, info_len) != HYAT_OK)
    return fail(h, HYAT_ERR_INVALID_ARG, "info buffer too small");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(work, h->d_work, sizeof(WorkItem) * n_work, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(entries, h->d_entries, sizeof(Entry) * n_ent, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "layout copy");
  return HYAT_OK;
}

hyat_status hyat_get_pairs(hyat_handle h, int32_t* pairs, size_t cap, int64_t* n_pairs) {
  if (!h || !n_pairs) return HYAT_ERR_INVALID_ARG;
  *n_pairs = h->n_pairs;
  if (!pairs) return HYAT_OK;
  if (cap < size_t(h->n_pairs) * 4) return fail(h, HYAT_ERR_INVALID_ARG, "pair buffer too small");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess && h->n_pairs > 0)
    e = cudaMemcpy(pairs, h->d_pairs, sizeof(int4) * h->n_pairs, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "pair copy");
  return HYAT_OK;
}

hyat_status hyat_sync(hyat_handle h) {
  if (!h) return HYAT_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
  uint32_t status = 0;
  e = cudaMemcpy(&status, h->d_status, sizeof(status), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "status read");
  if (status) {
    // The status region also holds the single-tile schedule's redo count and its finish
    // counter; a launch that gave up may have left them set, so the next call starts clean.
    cudaMemset(h->d_status, 0, 256);
    if (status & kStatusTimeout) return fail(h, HYAT_ERR_DEVICE_TIMEOUT, "a device-side wait timed out");
    if (status & kStatusBadTile) return fail(h, HYAT_ERR_DEVICE_TIMEOUT, "a device-side bounds check failed");
    return fail(h, HYAT_ERR_INVALID_ARG, "device step mask: a diagonal tile of the newest chunk was not kept");
  }
  return HYAT_OK;
}

hyat_status hyat_plan_layout(const hyat_config* cfg, const uint8_t* host_mask, int32_t* work, size_t work_cap,
                             int32_t* entries, size_t entries_cap, int64_t* counts) {
  if (!cfg || !counts) return HYAT_ERR_INVALID_ARG;
  if (!validate_config(*cfg).empty() || cfg->mode == HYAT_MODE_STREAM) return HYAT_ERR_INVALID_ARG;
  if (cfg->mode == HYAT_MODE_BLOCKMASK && !host_mask) return HYAT_ERR_INVALID_ARG;
  Layout L;
  if (!build_layout(*cfg, host_mask, &L).empty()) return HYAT_ERR_INVALID_ARG;
  counts[0] = static_cast<int64_t>(L.work.size());
  counts[1] = static_cast<int64_t>(L.entries.size());
  if (!work || !entries) return HYAT_OK;  // size query
  if (work_cap < L.work.size() * 8 || entries_cap < L.entries.size() * 2) return HYAT_ERR_INVALID_ARG;
  std::memcpy(work, L.work.data(), sizeof(WorkItem) * L.work.size());
  std::memcpy(entries, L.entries.data(), sizeof(Entry) * L.entries.size());
  return HYAT_OK;
}

hyat_status hyat_radial_mask(int32_t n_frames, int32_t tokens_per_frame, uint8_t* out, size_t out_bytes) {
  if (n_frames < 1 || tokens_per_frame < 1 || !out) return HYAT_ERR_INVALID_ARG;
  const int64_t nT = tiles(int64_t(n_frames) * tokens_per_frame);
  if (out_bytes < size_t(nT * nT)) return HYAT_ERR_INVALID_ARG;
  radial_tile_mask(n_frames, tokens_per_frame, out);
  return HYAT_OK;
}

hyat_status hyat_lvsa_mask(int32_t n_frames, int32_t tokens_per_frame, int32_t window_frames,
                           int32_t anchor_stride, int32_t rotation, uint8_t* out, size_t out_bytes) {
  if (n_frames < 1 || tokens_per_frame < 1 || !out || window_frames < 1 || window_frames % 2 == 0 ||
      anchor_stride < 0 || rotation < 0)
    return HYAT_ERR_INVALID_ARG;
  const int64_t nT = tiles(int64_t(n_frames) * tokens_per_frame);
  if (out_bytes < size_t(nT * nT)) return HYAT_ERR_INVALID_ARG;
  lvsa_tile_mask(n_frames, tokens_per_frame, window_frames, anchor_stride, rotation, out);
  return HYAT_OK;
}

hyat_status hyat_stream_plan(const hyat_config* cfg, int32_t step, int32_t* info, size_t info_len) {
  if (!cfg || !info || step < 0 || cfg->mode != HYAT_MODE_STREAM || !validate_config(*cfg).empty())
    return HYAT_ERR_INVALID_ARG;
  const int32_t slots = stream_ring_slots(*cfg);
  if (info_len < size_t(4 + slots)) return HYAT_ERR_INVALID_ARG;
  const StreamGeometry g = stream_geometry(*cfg, step);
  info[0] = g.first_window;
  info[1] = g.n_visible;
  info[2] = g.evicted;
  info[3] = g.write_slot;
  for (int32_t w = 0; w < slots; ++w) {
    const int32_t chunk = w < g.n_sink_visible ? w : g.first_window + (w - g.n_sink_visible);
    info[4 + w] = w < g.n_visible ? stream_slot_of_chunk(*cfg, chunk) : -1;
  }
  return HYAT_OK;
}

// state blob: header, then S/z (fp32 [BH][E]), ring K, ring V
namespace {
struct StateHeader {
  uint32_t magic, version;
  int32_t step, BH, d, L, nwc, dtype;
  int32_t folded_step, reserved[3];   // version 2: the step whose evicted chunk is in S, z;
                                      // reserved[0]: sink chunks
};
constexpr uint32_t kMagic = 0x54415948u;  // "HYAT"
}  // namespace

size_t hyat_stream_state_bytes(hyat_handle h) {
  if (!h || h->cfg.mode != HYAT_MODE_STREAM) return 0;
  const size_t ring = size_t(h->BH) * stream_ring_slots(h->cfg) * stream_chunk_tokens(h->cfg) * h->cfg.d *
                      elem_bytes(h->cfg);
  return sizeof(StateHeader) + sizeof(float) * size_t(h->BH) * h->E + 2 * ring;
}

hyat_status hyat_stream_get_state(hyat_handle h, void* dst_host, size_t bytes) {
  if (!h || !dst_host) return HYAT_ERR_INVALID_ARG;
  if (h->cfg.mode != HYAT_MODE_STREAM) return fail(h, HYAT_ERR_INVALID_ARG, "handle is not in STREAM mode");
  if (bytes < hyat_stream_state_bytes(h)) return fail(h, HYAT_ERR_INVALID_ARG, "state buffer too small");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronize");
  StateHeader hd{kMagic, 2, h->step, h->BH, h->cfg.d, stream_chunk_tokens(h->cfg), stream_window_chunks(h->cfg),
                 h->cfg.dtype, h->folded_step, {stream_sink_chunks(h->cfg), 0, 0}};
  char* p = static_cast<char*>(dst_host);
  std::memcpy(p, &hd, sizeof(hd));
  p += sizeof(hd);
  const size_t sb = sizeof(float) * size_t(h->BH) * h->E;
  const size_t rb = (hyat_stream_state_bytes(h) - sizeof(hd) - sb) / 2;
  e = cudaMemcpy(p, h->d_srest, sb, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(p + sb, h->d_ring_k, rb, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(p + sb + rb, h->d_ring_v, rb, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "state copy");
  return HYAT_OK;
}

hyat_status hyat_stream_set_state(hyat_handle h, const void* src_host, size_t bytes) {
  if (!h || !src_host) return HYAT_ERR_INVALID_ARG;
  if (h->cfg.mode != HYAT_MODE_STREAM) return fail(h, HYAT_ERR_INVALID_ARG, "handle is not in STREAM mode");
  if (bytes < hyat_stream_state_bytes(h)) return fail(h, HYAT_ERR_STATE, "state buffer too small");
  StateHeader hd;
  std::memcpy(&hd, src_host, sizeof(hd));
  if (hd.magic != kMagic || hd.version != 2 || hd.BH != h->BH || hd.d != h->cfg.d ||
      hd.L != stream_chunk_tokens(h->cfg) || hd.nwc != stream_window_chunks(h->cfg) || hd.dtype != h->cfg.dtype ||
      hd.reserved[0] != stream_sink_chunks(h->cfg) ||
      hd.step < 0 || hd.folded_step > hd.step)
    return fail(h, HYAT_ERR_STATE, "state blob does not match this handle");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronize");
  const char* p = static_cast<const char*>(src_host) + sizeof(hd);
  const size_t sb = sizeof(float) * size_t(h->BH) * h->E;
  const size_t rb = (hyat_stream_state_bytes(h) - sizeof(hd) - sb) / 2;
  e = cudaMemcpy(h->d_srest, p, sb, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->d_ring_k, p + sb, rb, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->d_ring_v, p + sb + rb, rb, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && h->use_tc) e = launch_state_to_bf16(h->d_srest, h->d_srest_bf16, h->BH, h->cfg.d, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(h, e, "state copy");
  h->step = hd.step;
  h->folded_step = hd.folded_step;
  return HYAT_OK;
}

hyat_status hyat_set_profiling(hyat_handle h, int enable) {
  if (!h) return HYAT_ERR_INVALID_ARG;
  h->profiling = enable != 0;
  return HYAT_OK;
}

hyat_status hyat_kernel_times(hyat_handle h, double* ms, int64_t* launches, int n_kinds) {
  if (!h || !ms || !launches || n_kinds < 1) return HYAT_ERR_INVALID_ARG;
  for (auto& r : h->recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(h, e, "event synchronize");
    float t = 0.0f;
    e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(h, e, "event elapsed time");
    h->ms[r.kind] += t;
    h->launches[r.kind] += 1;
    h->free_events.push_back(r.a);
    h->free_events.push_back(r.b);
  }
  h->recs.clear();
  for (int i = 0; i < n_kinds; ++i) {
    ms[i] = i < kKinds ? h->ms[i] : 0.0;
    launches[i] = i < kKinds ? h->launches[i] : 0;
  }
  for (int i = 0; i < kKinds; ++i) {
    h->ms[i] = 0.0;
    h->launches[i] = 0;
  }
  return HYAT_OK;
}

}  // extern "C"
