// Internal declarations shared by the host runtime and the kernels of libhyat.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/hyat.h"

namespace hyat {

constexpr int kTile = 128;          // query / key tile edge (rows)

// Device status word bits (workspace offset 0).
constexpr uint32_t kStatusTimeout = 1u;     // a bounded wait gave up
constexpr uint32_t kStatusBadTile = 2u;     // a tile descriptor failed its bounds check
constexpr uint32_t kStatusBadMask = 4u;     // a device step mask lacks a diagonal tile

// A work item: one query tile and the key tiles of its softmax window.
struct WorkItem {
  int32_t bh, q_row, q_len, state_group, entry_begin, entry_end, pad0, pad1;
};
static_assert(sizeof(WorkItem) == 32, "work item is 8 int32");

// A key tile of a window: rows [k_row, k_row + k_len) of one (b, h).
struct Entry {
  int32_t k_row, k_len;
};

// Host-side layout of a configuration.
struct Layout {
  // uniform key segments whose linear states are formed: segment g covers
  // rows [seg_base + g * seg_stride, + min(seg_len, rows_k - start))
  int32_t nseg = 0, seg_stride = 0, seg_len = 0;
  int32_t nqg = 0;                 // state groups (chunks, query tiles or 1)
  int32_t cm_heads = 1;            // heads of the complement matrix
  std::vector<float> cm;           // [cm_heads][nqg][nseg]: 1 = segment is in the linear set
  std::vector<WorkItem> work;
  std::vector<Entry> entries;
};

// Validate a configuration; returns an empty string if valid.
std::string validate_config(const hyat_config& c);
int64_t rows_q(const hyat_config& c);           // query rows per (b, h)
int64_t rows_k(const hyat_config& c);           // key rows per (b, h) (ring for STREAM)
int32_t stream_chunk_tokens(const hyat_config& c);
int32_t stream_window_chunks(const hyat_config& c);   // rolling window, in chunks
int32_t stream_sink_chunks(const hyat_config& c);     // leading chunks kept for good
int32_t stream_ring_slots(const hyat_config& c);      // window + sink slots per (b, h)
// Chunks visible at a streaming step: the sink chunks [0, n_sink_visible) first, then the
// rolling window [first_window, step]; key tiles follow that order.
struct StreamGeometry {
  int32_t n_sink_visible, first_window, n_window, n_visible;
  int32_t evicted;      // chunk folded into S, z at this step (-1: none)
  int32_t write_slot;   // ring slot of this step's chunk
};
StreamGeometry stream_geometry(const hyat_config& c, int32_t step);
int32_t stream_slot_of_chunk(const hyat_config& c, int32_t chunk);
int32_t tiles(int64_t rows);

// Host layout builders (layout.cpp).
std::string build_layout(const hyat_config& c, const uint8_t* host_mask, Layout* out);
// Pair consecutive work items of the same (b, h) into units of two query tiles;
// `shared` marks pairs whose key lists are identical (loaded once for both).
std::vector<int4> build_pairs(const std::vector<WorkItem>& work);
// Reorder pairs so that a persistent grid of `grid` CTAs, taking pair k on CTA k mod grid,
// gets nearly equal work: largest pairs first, each row of `grid` pairs dealt to the CTAs in
// ascending order of the work they already hold.
std::vector<int4> order_pairs_for_grid(const std::vector<int4>& pairs, const std::vector<WorkItem>& work,
                                       int32_t grid);
std::vector<int4> build_stream_pairs(int32_t BH, int32_t nqt);
// One split pair {i, i, 0, 1} per work item: both slots of a CTA run the same query tile,
// each over half of its key tiles, and the halves are merged in the epilogue.
std::vector<int4> build_split_pairs(size_t n_items);
// Split pairs when ordinary pairs would give the persistent grid fewer than four waves.
bool prefer_split_pairs(size_t n_ordinary_pairs, int32_t num_sms);
// build_pairs or build_split_pairs (by prefer_split_pairs), then order_pairs_for_grid.
std::vector<int4> choose_pairs(const std::vector<WorkItem>& work, int32_t num_sms);
void radial_tile_mask(int32_t n_frames, int32_t tokens_per_frame, uint8_t* out);
// Structured window plus rotating global anchors on the 128-token tile grid: tile (a, b) is
// kept iff some query token of a and key token of b are at most (window_frames - 1) / 2 frames
// apart, or b holds a token of an anchor frame f ((f + rotation) % anchor_stride == 0).
void lvsa_tile_mask(int32_t n_frames, int32_t tokens_per_frame, int32_t window_frames, int32_t anchor_stride,
                    int32_t rotation, uint8_t* out);

// ---- kernel launch wrappers (kernels_simt.cu, attn_tc.cu) ----
struct SegStateArgs {
  const void* k; const void* v; int64_t rows_per_bh;
  int32_t BH, d, dtype;
  int32_t nseg, seg_base, seg_stride, seg_len;
  float* out;                 // [BH][nseg][E], E = d*d + d (S row-major [a][b], then z[a])
  int32_t accumulate;         // out += instead of out =
  uint32_t* status;           // device status word (tensor-core kernel's bounded waits)
  uint16_t* out_hi;           // tensor-core kernel only: if set, write bf16 hi = bf16(x) and
  uint16_t* out_lo;           // lo = bf16(x - hi) ([BH][nseg][E] each) instead of fp32 `out`
  // tensor-core kernel only: split each segment into `parts` token ranges of `part_len`
  // tokens (a multiple of 64); the state of range r of segment g of bh goes to
  // partial[((bh * nseg + g) * parts + r) * E] (plain store), and `out` is not written.
  int32_t parts;
  int32_t part_len;
  float* partial;
  int32_t phi;                // hyat_phi
};
cudaError_t launch_seg_state(const SegStateArgs& a, cudaStream_t s);

cudaError_t launch_seg_state_tc(const SegStateArgs& a, int num_sms, cudaStream_t s);

struct ComplementArgs {
  const float* sseg;          // [BH][nseg][E]
  const float* cm;            // [cm_heads][nqg][nseg]
  float* srest;               // [BH][nqg][E]: z always; S only if write_f32_s
  uint16_t* srest_bf16;       // [BH][nqg][d][d] bf16 S (natural [a][b] layout) or null
  int32_t write_f32_s;
  int32_t BH, H, cm_heads, nseg, nqg, E, d;
};
cudaError_t launch_complement(const ComplementArgs& a, cudaStream_t s);

// Tensor-core complement for block masks (d = 128, more than 8 groups): a GEMM of the bf16
// 0/1 complement matrix with the hi/lo bf16 segment states (gemm_tc.cu).
struct ComplementTcArgs {
  const uint16_t* cm_bf16;    // [mask_heads][nqg][nseg_pad] bf16 0/1, rows padded with zeros
  const uint16_t* seg_hi;     // [BH][nseg][E]
  const uint16_t* seg_lo;     // [BH][nseg][E]
  float* srest;               // [BH][nqg][E]: z always; S only if write_f32_s
  uint16_t* srest_bf16;       // [BH][nqg][d][d]
  int32_t write_f32_s;
  int32_t BH, H, mask_heads, nqg, nseg, nseg_pad, E;
  uint32_t* status;
};
bool complement_tc_supported(int d, int nqg);
cudaError_t launch_complement_tc(const ComplementTcArgs& a, int num_sms, cudaStream_t s);

// S (fp32 [a][b], group stride d*d + d) -> bf16 S [a][b] (group stride d*d) for the
// tensor-core linear term, where S in its natural layout is the MN-major B operand.
cudaError_t launch_state_to_bf16(const float* srest, uint16_t* out, int64_t n_groups, int32_t d,
                                 cudaStream_t s);

struct AttnArgs {
  const void* q; const void* k; const void* v; void* o;
  int64_t q_rows, k_rows;     // rows per (b, h)
  const WorkItem* work; int32_t n_work;
  const Entry* entries;
  const int4* pairs; int32_t n_pairs;   // tensor-core path: {item0, item1 or -1, shared list, 0}
  const float* srest;         // [BH][nqg][E]
  const uint16_t* srest_bf16; // [BH][nqg][d][d] bf16 S, natural layout (tensor-core path)
  int32_t nqg, d, dtype, BH;
  float scale_log2;           // scale * log2(e)
  uint32_t* status;
  int32_t test_timeout;       // HYAT_FLAG_TEST_DEVICE_TIMEOUT (tensor-core path)
  int32_t phi;                // hyat_phi
};
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t s);
// One query tile per CTA at a time (a.pairs = {item, -1, 0, 0} in processing order, a.n_pairs
// of them). Tiles whose row sums leave the safe range are appended to redo_items (count at
// *redo_count, at most a.n_pairs); launch_attn_tc_redo then recomputes them with
// attn_tc_kernel, reading the count on the device and resetting it (and *done_count) to 0.
cudaError_t launch_attn_single(const AttnArgs& a, int32_t* redo_count, int4* redo_items, int num_sms,
                               cudaStream_t s);
// The pair schedule with two softmax warps per row (attn_tc_wide.cu): fixed reference max 0;
// query tiles whose row sums leave [2^-100, 2^100) are appended to redo_items (at most
// redo_cap) for launch_attn_tc_redo.
cudaError_t launch_attn_wide(const AttnArgs& a, int32_t* redo_count, int4* redo_items, int32_t redo_cap, int num_sms,
                             cudaStream_t s);
cudaError_t launch_attn_tc_redo(const AttnArgs& a, const int4* redo_items, int32_t* redo_count,
                                uint32_t* done_count, int num_sms, cudaStream_t s);
std::vector<int4> build_single_items(const std::vector<WorkItem>& work, int32_t num_sms);
bool attn_tc_supported(int d, int dtype);

// A streaming step's work between the fold's state kernel and the attention (stream_prep.cu):
// fold reduce, ring copy (K turned by the fused RoPE), Q turned into a workspace copy, and the
// step's layout, in one launch. Every argument is the same for steps of the same ring phase
// once the window is full, so a captured step replays for each of them.
struct StreamPrepArgs {
  int32_t nb_fold, nb_kv, nb_q, nb_layout;    // block ranges (set by launch_stream_prep)
  int32_t BH, L, d, elem_bytes;
  // fold reduce (partial = null: this step folds nothing)
  const float* partial;           // [BH][parts][E]
  float* srest;                   // [BH][E]
  uint16_t* srest_bf16;           // [BH][d][d]
  int32_t parts;
  // ring copy
  const void* k; const void* v;   // [BH][L][d]
  void* ring_k; void* ring_v;     // [BH][nslots][L][d]
  int32_t nslots, slot;
  // fused RoPE (half_t = 0: none): frame f of the chunk turns by min(p0 + f, cap - 1) * theta
  const void* q;                  // [BH][L][d]
  void* q_out;                    // null: Q is not turned (no fused RoPE)
  int32_t half_t, chunk_frames, tokens_per_frame, p0, cap;
  double theta[64];               // base^(-2i / t_dims), i < half_t
  // layout
  const uint8_t* mask;            // [mask_heads][nqt][nkt] (device)
  WorkItem* work;                 // [BH][nqt]
  Entry* entries;                 // [BH][nqt][cap_entries]
  uint32_t* status;               // kStatusBadMask if a diagonal tile of the newest chunk is off
  int32_t H, mask_heads, nqt, nkt, cap_entries, nwc;
  int32_t n_sink_visible;         // visible chunks 0..n_sink_visible-1 sit in slots nwc + c
  int32_t first_window_mod;       // first window chunk mod nwc: window chunk w sits in slot
                                  // (first_window_mod + w - n_sink_visible) % nwc
  // Split-pair order (pairs != null): the last layout block to finish writes one split pair
  // {item, item, 0, 1} per work item into pairs, largest key-tile count first, each row of
  // `grid` pairs dealt to the attention's persistent CTAs least-loaded first (pair k runs on
  // CTA k mod grid); done_counter counts finished layout blocks and is reset by the last one.
  int4* pairs;
  int32_t grid;
  uint32_t* done_counter;
  // Nonzero: the kernel ahead of this one on the stream is the fold's state kernel, which lets
  // this grid start only after its own programmatic wait (everything enqueued before the call
  // has finished by then), so the layout blocks need not wait.
  int32_t layout_early;
};
constexpr int32_t kMaxStreamOrderBins = 1024;   // split-pair ordering: key-tile counts 0..1023
constexpr int32_t kMaxStreamOrderGrid = 1024;   // persistent grids of up to 1024 CTAs
constexpr int32_t kMaxStreamOrderItems = 2048;  // and up to 2048 work items
cudaError_t launch_stream_prep(StreamPrepArgs a, int num_sms, cudaStream_t s);

}  // namespace hyat
