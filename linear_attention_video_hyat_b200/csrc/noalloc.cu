// Allocation-free bidirectional forward.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: code that runs while a caching allocator (PyTorch's included) must not
// be re-entered, plug-in hosts whose memory is owned by another runtime, and
// real-time loops that forbid cudaMalloc/cudaFree because those calls can
// synchronise the device and stall for milliseconds. For them this file keeps
// the forward's scratch (layout tables, per-frame / per-tile linear states,
// complement states) in one file-scope __device__ array, reserved once per GPU
// when the library is loaded and held until the process exits. The caller
// passes only Q, K, V and O.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "hyat_internal.h"

namespace hyat {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per GPU
constexpr int kMaxDevices = 64;

// The scratch. In host code `g_noalloc_scratch` is a host-side stand-in, not a
// device address: it is never passed to a kernel directly; the device address
// is obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
int g_major[kMaxDevices] = {};

// Resolve the scratch address, SM count and compute-capability major of the current device
// (once per device).
cudaError_t scratch_for_current_device(void** addr, int* num_sms, int* major) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    int sms = 0, mj = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&mj, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    g_num_sms[dev] = sms;
    g_major[dev] = mj;
  }
  *addr = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  *major = g_major[dev];
  return cudaSuccess;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace hyat

using namespace hyat;

extern "C" HYAT_API hyat_status hyat_fwd_bidir_noalloc(const hyat_config* cfg, const void* q, const void* k,
                                                       const void* v, void* o, void* stream) {
  if (!cfg || !q || !k || !v || !o) return HYAT_ERR_INVALID_ARG;
  if (!validate_config(*cfg).empty()) return HYAT_ERR_INVALID_ARG;
  if (cfg->mode != HYAT_MODE_WINDOW && cfg->mode != HYAT_MODE_RADIAL) return HYAT_ERR_INVALID_ARG;
  if (cfg->flags & (HYAT_FLAG_TEST_SOFTMAX_BRANCH | HYAT_FLAG_TEST_LINEAR_BRANCH)) return HYAT_ERR_UNSUPPORTED;
  for (const void* p : {q, k, v, static_cast<const void*>(o)})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return HYAT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The layout tables travel from pageable host vectors that die when this call returns; a
  // captured copy would read them at replay. So the call refuses stream capture.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return HYAT_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) return HYAT_ERR_UNSUPPORTED;

  Layout L;
  if (!build_layout(*cfg, nullptr, &L).empty()) return HYAT_ERR_INVALID_ARG;
  const int64_t BH = int64_t(cfg->B) * cfg->H;
  const int64_t E = int64_t(cfg->d) * cfg->d + cfg->d;
  const int64_t rows = rows_q(*cfg);
  const int32_t nseg_pad = (L.nseg + 63) / 64 * 64;

  void* base = nullptr;
  int num_sms = 0, major = 0;
  if (scratch_for_current_device(&base, &num_sms, &major) != cudaSuccess) return HYAT_ERR_CUDA;
  // the same kernels as hyat_fwd_bidir on a handle of this configuration
  const bool use_tc = cfg->dtype == HYAT_BF16 && !(cfg->flags & HYAT_FLAG_SIMT) && major == 10 &&
                      attn_tc_supported(cfg->d, cfg->dtype);
  const bool use_gemm = use_tc && cfg->mode == HYAT_MODE_RADIAL && complement_tc_supported(cfg->d, L.nqg);

  // carve the static scratch
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o2 = off; off = up256(off + bytes); return o2; };
  const size_t o_status = take(256);
  const size_t o_work = take(sizeof(WorkItem) * L.work.size());
  const size_t o_entries = take(sizeof(Entry) * (L.entries.empty() ? 1 : L.entries.size()));
  const size_t o_pairs = take(sizeof(int4) * (L.work.empty() ? 1 : L.work.size()));
  const size_t o_cm = take(sizeof(float) * L.cm.size());
  const size_t o_cm_bf16 = use_gemm ? take(2 * size_t(L.cm_heads) * L.nqg * nseg_pad) : 0;
  const size_t o_sseg = take(sizeof(float) * size_t(BH) * L.nseg * E);   // or its bf16 hi/lo parts
  const size_t o_srest = take(sizeof(float) * size_t(BH) * L.nqg * E);
  const size_t o_srest_bf16 = take(2 * size_t(BH) * L.nqg * cfg->d * cfg->d);
  const size_t o_redo = take(sizeof(int4) * (L.work.empty() ? 1 : L.work.size()));   // redo list
  if (off > kNoAllocScratchBytes) return HYAT_ERR_UNSUPPORTED;  // needs more than the static scratch

  const std::vector<int4> pairs = choose_pairs(L.work, num_sms);   // at most one per work item
  std::vector<uint16_t> cmb;
  if (use_gemm) {   // the 0/1 complement matrix in bf16 (exact), rows padded to 64 segments
    cmb.assign(size_t(L.cm_heads) * L.nqg * nseg_pad, 0);
    for (int32_t m = 0; m < L.cm_heads; ++m)
      for (int32_t g = 0; g < L.nqg; ++g)
        for (int32_t sg = 0; sg < L.nseg; ++sg)
          if (L.cm[(size_t(m) * L.nqg + g) * L.nseg + sg] != 0.0f) cmb[(size_t(m) * L.nqg + g) * nseg_pad + sg] = 0x3F80;
  }
  char* ws = static_cast<char*>(base);

  // layout tables: pageable host -> scratch (the copy has consumed the vectors when it returns);
  // the status region (status word, redo count and its finish counter) starts at zero on every
  // call
  cudaError_t e = cudaMemsetAsync(ws + o_status, 0, 256, s);
  if (e == cudaSuccess && !L.work.empty())
    e = cudaMemcpyAsync(ws + o_work, L.work.data(), sizeof(WorkItem) * L.work.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !L.entries.empty())
    e = cudaMemcpyAsync(ws + o_entries, L.entries.data(), sizeof(Entry) * L.entries.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !pairs.empty())
    e = cudaMemcpyAsync(ws + o_pairs, pairs.data(), sizeof(int4) * pairs.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !L.cm.empty())
    e = cudaMemcpyAsync(ws + o_cm, L.cm.data(), sizeof(float) * L.cm.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && use_gemm)
    e = cudaMemcpyAsync(ws + o_cm_bf16, cmb.data(), 2 * cmb.size(), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return HYAT_ERR_CUDA;

  uint32_t* status = reinterpret_cast<uint32_t*>(ws + o_status);
  SegStateArgs sa{};
  sa.k = k; sa.v = v; sa.rows_per_bh = rows;
  sa.BH = static_cast<int32_t>(BH); sa.d = cfg->d; sa.dtype = cfg->dtype; sa.phi = cfg->phi;
  sa.nseg = L.nseg; sa.seg_base = 0; sa.seg_stride = L.seg_stride; sa.seg_len = L.seg_len;
  sa.out = reinterpret_cast<float*>(ws + o_sseg); sa.accumulate = 0; sa.status = status;
  if (use_gemm) {           // hi/lo bf16 parts for the tensor-core complement, in the same bytes
    sa.out_hi = reinterpret_cast<uint16_t*>(ws + o_sseg);
    sa.out_lo = sa.out_hi + size_t(BH) * L.nseg * E;
  }
  e = use_tc ? launch_seg_state_tc(sa, num_sms, s) : launch_seg_state(sa, s);
  if (e != cudaSuccess) return HYAT_ERR_CUDA;

  float* srest = reinterpret_cast<float*>(ws + o_srest);
  uint16_t* srest_bf16 = reinterpret_cast<uint16_t*>(ws + o_srest_bf16);
  if (use_gemm) {
    ComplementTcArgs ga{};
    ga.cm_bf16 = reinterpret_cast<const uint16_t*>(ws + o_cm_bf16);
    ga.seg_hi = sa.out_hi; ga.seg_lo = sa.out_lo;
    ga.srest = srest; ga.srest_bf16 = srest_bf16; ga.write_f32_s = 0;
    ga.BH = static_cast<int32_t>(BH); ga.H = cfg->H; ga.mask_heads = L.cm_heads; ga.nqg = L.nqg; ga.nseg = L.nseg;
    ga.nseg_pad = nseg_pad; ga.E = static_cast<int32_t>(E); ga.status = status;
    e = launch_complement_tc(ga, num_sms, s);
  } else {
    ComplementArgs ca{};
    ca.sseg = sa.out; ca.cm = reinterpret_cast<const float*>(ws + o_cm);
    ca.srest = srest;
    ca.srest_bf16 = use_tc ? srest_bf16 : nullptr;
    ca.write_f32_s = use_tc ? 0 : 1;        // the tensor-core path reads S as bf16, z as fp32
    ca.BH = static_cast<int32_t>(BH); ca.H = cfg->H; ca.cm_heads = L.cm_heads; ca.nseg = L.nseg; ca.nqg = L.nqg;
    ca.E = static_cast<int32_t>(E); ca.d = cfg->d;
    e = launch_complement(ca, s);
  }
  if (e != cudaSuccess) return HYAT_ERR_CUDA;

  AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.o = o;
  a.q_rows = rows; a.k_rows = rows;
  a.work = reinterpret_cast<const WorkItem*>(ws + o_work);
  a.n_work = static_cast<int32_t>(L.work.size());
  a.entries = reinterpret_cast<const Entry*>(ws + o_entries);
  a.pairs = reinterpret_cast<const int4*>(ws + o_pairs);
  a.n_pairs = static_cast<int32_t>(pairs.size());
  a.srest = srest;
  a.srest_bf16 = srest_bf16;
  a.nqg = L.nqg; a.d = cfg->d; a.dtype = cfg->dtype; a.BH = static_cast<int32_t>(BH);
  const float scale = cfg->scale > 0.0f ? cfg->scale : 1.0f / sqrtf(float(cfg->d));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = status;
  a.phi = cfg->phi;
  if (!use_tc) {
    e = launch_attn_simt(a, s);
  } else {
    // the default schedule of hyat_fwd_bidir: two softmax warps per row, then the redo pass
    int32_t* redo_count = reinterpret_cast<int32_t*>(ws + o_status + 64);
    uint32_t* redo_done = reinterpret_cast<uint32_t*>(ws + o_status + 128);
    int4* redo = reinterpret_cast<int4*>(ws + o_redo);
    e = launch_attn_wide(a, redo_count, redo, static_cast<int32_t>(L.work.size()), num_sms, s);
    if (e == cudaSuccess) e = launch_attn_tc_redo(a, redo, redo_count, redo_done, num_sms, s);
  }
  return e == cudaSuccess ? HYAT_OK : HYAT_ERR_CUDA;
}
