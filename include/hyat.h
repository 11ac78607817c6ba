/*
 * hyat.h -- C interface of libhyat, hybrid softmax-window + linear-state
 * attention (forward) for video diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * The operation (ReHyAt: Recurrent Hybrid Attention for Video Diffusion
 * Transformers, Abstract; Long-Horizon Streaming Video Generation via Hybrid
 * Attention with Decoupled Distillation, Section 2.A "Hybrid Attention";
 * Radial Attention: O(n log n) Sparse Attention with Energy Decay for Long
 * Video Generation, Abstract): each query i takes exact softmax attention over
 * the keys of its window W_i and reaches every other key j in its linear set
 * R_i through the linear-attention state S = sum phi(k_j) v_j^T, z = sum phi(k_j),
 * under one normaliser:
 *
 *   o_i = ( sum_{j in W_i} e^{s_ij - m_i} v_j + e^{-m_i} phi(q_i)^T S )
 *       / ( sum_{j in W_i} e^{s_ij - m_i}     + e^{-m_i} phi(q_i)^T z ),
 *   s_ij = scale * q_i . k_j,   phi(x) = elu(x) + 1 (or ReLU, exp: hyat_phi),
 *   m_i = max(0, max_j s_ij).
 *
 * Modes (hyat_config.mode):
 *   WINDOW     bidirectional; frames of tokens_per_frame tokens are grouped in
 *              chunks of chunk_frames; a query's window is its chunk plus
 *              halo_frames frames on each side, clipped to the video; R_i is
 *              every other token (token-exact).
 *   BLOCKMASK  bidirectional; W_i is the union of the 128x128 tiles that a
 *              caller mask keeps on the absolute tile grid; R_i is the rest.
 *   RADIAL     BLOCKMASK with the static radial mask built by the library: a
 *              tile is kept iff it holds a near pair (same frame, or
 *              2*|p_j - p_i| < tokens_per_frame >> floor(log2 t) at frame
 *              distance t, p = raster index inside the frame).
 *   STREAM     causal streaming in chunks of chunk_frames frames; the KV window
 *              holds the latest window_frames frames (a multiple of
 *              chunk_frames); chunks that leave the window are folded into the
 *              recurrent state (S, z); queries of the current chunk attend to
 *              the kept 128x128 tiles of the window (per-step mask) and to the
 *              state. Dropped window tiles reach neither branch.
 *
 * Conventions shared by every entry point:
 *   - Tensors Q, K, V, O are row-major [B, H, N, d] (N = tokens), contiguous,
 *     device memory, 16-byte aligned, dtype = hyat_config.dtype. O has Q's
 *     shape. The caller owns them.
 *   - The workspace is device memory owned by the caller, at least
 *     hyat_workspace_bytes() bytes, 256-byte aligned, untouched by the caller
 *     while the handle lives. The library never calls cudaMalloc on a
 *     forward call.
 *   - Every forward call is enqueued on the given stream (a cudaStream_t
 *     passed as void*; NULL = legacy default stream) and returns without
 *     waiting for the GPU. A device-side timeout (a bounded wait that gave up)
 *     sets a status word in the workspace; hyat_sync() reports it as
 *     HYAT_ERR_DEVICE_TIMEOUT.
 *   - Nothing aborts or prints. Every failure returns a status; the text of
 *     the last failure on a handle is hyat_last_error(handle).
 *   - A handle is not thread-safe. Different handles are independent.
 */
#ifndef HYAT_H_
#define HYAT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYAT_API __attribute__((visibility("default")))
#else
#define HYAT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HYAT_OK = 0,
  HYAT_ERR_INVALID_ARG = 1,     /* bad shape, pointer, alignment, mask or call order */
  HYAT_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. d not in {64,128}) */
  HYAT_ERR_CUDA = 3,            /* a CUDA runtime call failed; see hyat_last_error */
  HYAT_ERR_DEVICE_TIMEOUT = 4,  /* a device-side bounded wait gave up */
  HYAT_ERR_STATE = 5            /* stream state blob malformed or mismatched */
} hyat_status;

typedef enum { HYAT_F32 = 0, HYAT_BF16 = 1 } hyat_dtype;
/* Feature map of the linear branch. The pages leave it open (the hybrid normaliser
 * needs phi >= 0); elu + 1 is the default. ReLU and exp are the other maps of the
 * linear-attention literature the pages cite (Transformers are RNNs; Hedgehog). */
typedef enum { HYAT_PHI_ELU1 = 0, HYAT_PHI_RELU = 1, HYAT_PHI_EXP = 2 } hyat_phi;
typedef enum {
  HYAT_MODE_WINDOW = 0,
  HYAT_MODE_BLOCKMASK = 1,
  HYAT_MODE_RADIAL = 2,
  HYAT_MODE_STREAM = 3
} hyat_mode;

/* Flags (hyat_config.flags). */
#define HYAT_FLAG_SIMT 1u        /* run bf16 through the CUDA-core path (cross-check) */
/* Test hook for the device-timeout path, which must work without faulting a GPU: the
 * tensor-core attention kernel also waits once on a barrier that nothing signals, with a
 * 20 ms limit. The wait gives up, every role drains and frees TMEM, the status word is set,
 * and hyat_sync() returns HYAT_ERR_DEVICE_TIMEOUT; later calls on any handle work. */
#define HYAT_FLAG_TEST_DEVICE_TIMEOUT 2u
/* Schedules of the tensor-core attention. By default a CTA runs a pair of query tiles (the
 * streaming mode, a split pair of one tile), with two softmax warps per row, each taking 64 of
 * a key tile's 128 keys, a fixed reference max of 0 and a redo list: query tiles whose row sums
 * leave [2^-100, 2^100) (scores far above 0, or all far below 0 with no linear term) are
 * recomputed right after by the one-warp-per-row pair kernel, which moves its reference max.
 * HYAT_FLAG_SINGLE_TILE (bidirectional modes) runs one query tile per CTA at a time (three S
 * buffers in TMEM; two softmax warpgroups on alternate key tiles), with the same redo list.
 * HYAT_FLAG_PAIR_ONE_WARP runs the pair schedule with one softmax warp per row and an exact
 * moving reference max (no redo list). All give results within the same tolerance; the
 * default is the fastest on B200, the others are kept for cross-checks and timing. */
#define HYAT_FLAG_SINGLE_TILE 4u
#define HYAT_FLAG_PAIR_ONE_WARP 8u
/* Test hooks for branch-wise parity (WINDOW, BLOCKMASK and RADIAL; STREAM and the
 * allocation-free call reject them). A query row's output is (N_soft + N_lin) / (D_soft +
 * D_lin): the softmax branch over its window keys and the linear branch over the rest (ReHyAt
 * abstract; Hybrid Forcing, Section 2.A). With unit-variance inputs the linear branch carries
 * most of the weight, so the hybrid output alone says little about the softmax branch.
 * HYAT_FLAG_TEST_SOFTMAX_BRANCH zeroes the linear state between the complement and the
 * attention kernel: the call returns N_soft / D_soft. HYAT_FLAG_TEST_LINEAR_BRANCH empties
 * every query tile's key list when the handle is created: the call returns N_lin / D_lin =
 * phi(q) S_rest / phi(q) z_rest. At most one of the two may be set. */
#define HYAT_FLAG_TEST_SOFTMAX_BRANCH 16u
#define HYAT_FLAG_TEST_LINEAR_BRANCH 32u

typedef struct {
  int32_t B, H, d;               /* d in {64, 128} */
  int32_t tokens_per_frame;      /* F */
  int32_t n_frames;              /* T (bidirectional modes); ignored by STREAM */
  int32_t chunk_frames;          /* WINDOW: chunk; STREAM: frames per step */
  int32_t halo_frames;           /* WINDOW: frames added on each side of a chunk */
  int32_t window_frames;         /* STREAM: frames kept in the KV window */
  int32_t mode;                  /* hyat_mode */
  int32_t dtype;                 /* hyat_dtype */
  int32_t phi;                   /* hyat_phi */
  int32_t mask_heads;            /* BLOCKMASK / STREAM masks: 1 (shared) or H */
  uint32_t flags;                /* HYAT_FLAG_* */
  float scale;                   /* softmax logit scale; 0 => 1/sqrt(d) */
  int32_t sink_frames;           /* STREAM: leading frames kept in the window for good (an
                                    attention sink); a multiple of chunk_frames, 0 = none */
  /* STREAM: the capped temporal RoPE of hyat_rope_temporal, fused into the step (Long-Horizon
   * Streaming Video Generation via Hybrid Attention with Decoupled Distillation, Section 2.C,
   * the relative RoPE constraint). rope_t_dims = 0: none. Otherwise each call turns the first
   * rope_t_dims dimensions of its Q and K exactly as hyat_rope_temporal would, with the
   * reference frame the first frame of the oldest rolling-window chunk (the call's own chunk
   * while the window holds none yet) and the index capped at rope_cap - 1: K on its way into
   * the KV ring, Q into a workspace copy that the attention reads. The caller's Q and K are
   * not modified. Needs rope_t_dims even and <= d, rope_cap >= 1, chunk_frames * rope_t_dims
   * <= 8192. */
  int32_t rope_t_dims;
  int32_t rope_cap;
  float rope_base;               /* frequency base; 0 => 10000 */
} hyat_config;

typedef struct hyat_ctx* hyat_handle;

/* Bytes of device workspace a handle of this configuration needs (an upper
 * bound independent of the mask). Returns 0 if the configuration is invalid. */
HYAT_API size_t hyat_workspace_bytes(const hyat_config* cfg);

/* Create a handle. `host_mask` is read only by BLOCKMASK: uint8
 * [mask_heads, nT, nT], nT = ceil(N/128), nonzero = tile kept; NULL elsewhere.
 * Builds the layout on the host (and the radial mask for RADIAL), copies it
 * into the workspace (synchronously, on the legacy stream) and zeroes the
 * stream state. On failure *out is NULL. */
HYAT_API hyat_status hyat_create(const hyat_config* cfg, void* workspace, size_t workspace_bytes,
                                 const uint8_t* host_mask, hyat_handle* out);

/* Bidirectional forward (WINDOW, BLOCKMASK, RADIAL): O = hybrid(Q, K, V).
 * Q, K, V, O: [B, H, T*F, d] device pointers. Enqueues the state kernel, the
 * complement reduction and the attention kernel on `stream`. */
HYAT_API hyat_status hyat_fwd_bidir(hyat_handle h, const void* q, const void* k, const void* v,
                           void* o, void* stream);

/* One streaming step (STREAM): Q, K, V, O are the current chunk,
 * [B, H, L, d], L = chunk_frames * F. `host_step_mask` is uint8
 * [mask_heads, nQT, nQT * nwin] on the host (nQT = ceil(L/128), nwin = number
 * of window chunks visible at this step = min(step + 1, window_frames /
 * chunk_frames), key tiles ordered oldest chunk first), or NULL for all tiles
 * kept. Its diagonal tiles of the newest chunk must be set. Steps run in order;
 * the step counter lives in the handle. Before attention, the chunk leaving
 * the window (if any) is folded into S, z and the new K, V enter its ring slot. */
HYAT_API hyat_status hyat_fwd_stream_step(hyat_handle h, const void* q, const void* k, const void* v,
                                 void* o, const uint8_t* host_step_mask, void* stream);

/* A non-final call for the current streaming chunk: one denoising step of it.
 * Streaming video models denoise a chunk in several calls and keep only the
 * last call's keys and values in the cache (Hybrid Forcing, Section 2.A: the
 * window holds the frames already generated). A chunk's calls are any number
 * of hyat_fwd_stream_denoise calls followed by one hyat_fwd_stream_step,
 * which is the final call and advances the step counter. Every call sees the
 * committed window chunks, the folded state and its own Q, K, V as the
 * newest chunk; arguments, layouts and the mask are those of
 * hyat_fwd_stream_step. The chunk leaving the window is folded once, at the
 * chunk's first call. */
HYAT_API hyat_status hyat_fwd_stream_denoise(hyat_handle h, const void* q, const void* k, const void* v,
                                    void* o, const uint8_t* host_step_mask, void* stream);

/* hyat_fwd_stream_step with the step mask already in device memory: `dev_step_mask` has the
 * layout of host_step_mask (NULL = every tile kept) and must stay valid until the step has
 * run. Nothing is copied from the host, so the call can be captured in a CUDA graph by the
 * library (hyat_fwd_stream_step_graph). The diagonal tiles are checked on the device: a
 * missing one is computed as given and reported by hyat_sync() as HYAT_ERR_INVALID_ARG. */
HYAT_API hyat_status hyat_fwd_stream_step_dev(hyat_handle h, const void* q, const void* k, const void* v,
                                     void* o, const uint8_t* dev_step_mask, void* stream);

/* hyat_fwd_stream_step_dev replayed from a CUDA graph. Once the window is full, a step's
 * launches depend only on its ring phase (step mod window_frames / chunk_frames) and on the
 * pointers q, k, v, o and dev_step_mask: the first such step of each phase is captured (on a
 * stream of the handle) into a graph, and later steps of that phase with the same pointers
 * launch the graph on `stream` with one call. New pointers capture again; the handle keeps
 * the 16 most recent graphs, so a caller that rotates a few input buffers reuses them. Steps
 * before the window is full, and calls with profiling on, run as hyat_fwd_stream_step_dev.
 * Results equal hyat_fwd_stream_step_dev's bit for bit. */
HYAT_API hyat_status hyat_fwd_stream_step_graph(hyat_handle h, const void* q, const void* k, const void* v,
                                       void* o, const uint8_t* dev_step_mask, void* stream);

/* Wait for the last call's stream and report device-side errors. */
HYAT_API hyat_status hyat_sync(hyat_handle h);

/* Release a handle (does not free the caller's workspace). NULL is accepted. */
HYAT_API hyat_status hyat_destroy(hyat_handle h);

HYAT_API const char* hyat_last_error(hyat_handle h);
HYAT_API const char* hyat_status_string(hyat_status s);

/* ---- inspection and test hooks (host-only unless stated) ---- */

/* Host-only layout of a bidirectional configuration, without a GPU.
 * Work items are 8 int32 each: {bh, q_row, q_len, state_group, entry_begin,
 * entry_end, 0, 0}; entries are 2 int32 each: {k_row, k_len}. Counts are
 * written to counts[0] (work items) and counts[1] (entries); if a capacity is
 * too small the arrays are not written and HYAT_ERR_INVALID_ARG returned. */
HYAT_API hyat_status hyat_plan_layout(const hyat_config* cfg, const uint8_t* host_mask,
                             int32_t* work, size_t work_cap, int32_t* entries,
                             size_t entries_cap, int64_t* counts);

/* Host-only radial tile mask: out = uint8 [nT, nT], nT = ceil(T*F/128). */
HYAT_API hyat_status hyat_radial_mask(int32_t n_frames, int32_t tokens_per_frame, uint8_t* out,
                             size_t out_bytes);

/* Host-only structured-window + rotating-anchor tile mask, for BLOCKMASK
 * handles (Long Video Sparse Attention, Abstract: a structured window pattern
 * with rotating global anchors). The pages do not define the pattern; this
 * reading keeps tile (a, b) iff
 *   - some query token of tile a and key token of tile b lie at most
 *     (window_frames - 1) / 2 frames apart (window_frames odd), or
 *   - tile b holds a token of an anchor frame f: (f + rotation) % anchor_stride
 *     == 0 (anchor_stride 0: no anchors).
 * The caller advances `rotation` (e.g. with the denoising step) so the anchor
 * grid moves. Everything the mask drops reaches the query through the linear
 * state. out = uint8 [nT, nT], nT = ceil(T*F/128). */
HYAT_API hyat_status hyat_lvsa_mask(int32_t n_frames, int32_t tokens_per_frame, int32_t window_frames,
                           int32_t anchor_stride, int32_t rotation, uint8_t* out, size_t out_bytes);

/* Host-only streaming bookkeeping of step `step`: info[0] = first visible
 * chunk, info[1] = number of visible chunks, info[2] = chunk folded into the
 * state before this step's attention (-1 if none), info[3] = ring slot
 * receiving this step's K/V, info[4 + w] = ring slot of visible chunk w. */
HYAT_API hyat_status hyat_stream_plan(const hyat_config* cfg, int32_t step, int32_t* info,
                             size_t info_len);

/* Test hook (STREAM): the layout the last streaming call built on the device, copied to the
 * host (synchronises the device). work: n_work x 8 int32 per (b, h, query tile)
 * {bh, q_row, q_len, 0, entry_begin, entry_end, 0, 0}; entries: n_work x cap slots of 2 int32
 * {k_row, k_len}, item t's key tiles at [entry_begin, entry_end), k_row a row of the KV ring
 * (slot * L + offset in the chunk); info (4 + ring slots int32): hyat_stream_plan of that
 * call's step. counts[0] = n_work, counts[1] = entry slots, counts[2] = that step. Null
 * arrays: counts only. HYAT_ERR_STATE before the first streaming call. */
HYAT_API hyat_status hyat_stream_get_layout(hyat_handle h, int32_t* work, size_t work_cap, int32_t* entries,
                                   size_t entries_cap, int32_t* info, size_t info_len, int64_t* counts);

/* Test hook: the persistent attention kernel's pair list as the last forward or streaming
 * call left it, copied to the host (synchronises the device). 4 int32 per pair {item0,
 * item1, shared, split}, items indexing the work list: pair k runs on CTA k mod
 * min(n_pairs, SMs); item1 = -1 when the pair holds one query tile; shared = 1 when both
 * query tiles have the same key-tile list (one K/V load serves both); split = 1 when the
 * pair's two halves are item0's key tiles cut in two.
 * The list holds the pairs largest first (key tiles of both items + 2), in rows of
 * min(n_pairs, SMs) pairs, each row placed in a serpentine or least loaded first (the row's
 * pairs to the CTAs holding the least work so far), whichever leaves the busiest CTA less
 * work. In STREAM mode with split pairs the prep kernel rewrites the list every step by the
 * same rule from that step's key-tile counts (cost: key tiles + 1), as long as the step has at
 * most 2048 query tiles, 1023 key tiles per query tile and 1024 CTAs; otherwise the list keeps
 * its creation order. *n_pairs always receives the count; a null `pairs` copies nothing;
 * HYAT_ERR_INVALID_ARG if cap < 4 * n_pairs. */
HYAT_API hyat_status hyat_get_pairs(hyat_handle h, int32_t* pairs, size_t cap, int64_t* n_pairs);

/* Stream state (S, z, KV ring, step, and whether the current chunk's fold
 * has run) to / from a host buffer: a 48-byte header, then S, z as fp32
 * [B*H][d*d + d], then the K and V rings. The size is
 * hyat_stream_state_bytes(); both calls synchronise the device. */
HYAT_API size_t hyat_stream_state_bytes(hyat_handle h);
HYAT_API hyat_status hyat_stream_get_state(hyat_handle h, void* dst_host, size_t bytes);
HYAT_API hyat_status hyat_stream_set_state(hyat_handle h, const void* src_host, size_t bytes);

/* Kernel timing: when enabled, each forward call records CUDA events around
 * its launches; hyat_kernel_times() returns the summed milliseconds and
 * launch counts per kernel kind since the last reset (kinds: 0 state,
 * 1 complement, 2 attention, 3 stream fold, 4 stream prep: fold reduce, ring copy, fused
 * RoPE and layout).
 * Reading the times synchronises the device. */
HYAT_API hyat_status hyat_set_profiling(hyat_handle h, int enable);
HYAT_API hyat_status hyat_kernel_times(hyat_handle h, double* ms, int64_t* launches, int n_kinds);

/* ---- allocation-free forward ----
 * No passage of the pages corresponds to this entry point; it exists for
 * callers that cannot allocate device memory where they run the layer (code
 * running while a caching allocator must not be re-entered, plug-in hosts
 * whose device memory belongs to another runtime, real-time loops where
 * cudaMalloc/cudaFree would synchronise the device).
 *
 * Same operation and tensor conventions as hyat_fwd_bidir, for WINDOW and
 * RADIAL configurations, without a handle or a workspace: the scratch lives in
 * one static 32 MiB __device__ array that every GPU loading the library holds
 * until the process exits. It runs the same kernels, in the same order and with
 * the same work order, as hyat_fwd_bidir on a handle of the same configuration,
 * so its output equals that call's bit for bit. No cudaMalloc, cudaFree or
 * allocating library call is made. Returns HYAT_ERR_UNSUPPORTED when the configuration needs more than
 * 32 MiB of scratch (for example, 12 heads x 21 frames of 1560 tokens at
 * d = 128 need about 25 MiB), HYAT_ERR_INVALID_ARG for other modes, bad
 * configurations or pointers that are not 16-byte aligned.
 * The first call on a device resolves the array's device address; make that
 * first call before any stream capture. The call copies its layout tables from
 * host memory that it releases on return, so it returns HYAT_ERR_UNSUPPORTED
 * (nothing enqueued) when `stream` is being captured. Every call reuses the same array and
 * leaves the previous call's contents in it (the status word is cleared on
 * each call): calls that overlap on the GPU -- on different streams, or from
 * different threads -- race on it and must be serialised by the caller.
 * Device-side timeouts of this path are not reported (there is no handle). The attention
 * always runs the pair schedule (HYAT_FLAG_SINGLE_TILE is ignored here). */
HYAT_API hyat_status hyat_fwd_bidir_noalloc(const hyat_config* cfg, const void* q, const void* k,
                                            const void* v, void* o, void* stream);

/* ---- the step before attention ---- */

/* Temporal rotary position embedding with a capped relative index (Long-Horizon Streaming
 * Video Generation via Hybrid Attention with Decoupled Distillation, Section 2.C, the relative
 * RoPE constraint: the temporal RoPE index is written relative to a reference frame and held
 * below an upper bound, so that generation of any length stays inside the index range the
 * pretrained model has seen). The pages give no formula; this reading applies rotary pairs in
 * their usual form to the first t_dims dimensions of each head:
 *   (x[2i], x[2i+1]) turns by the angle p * base^(-2i / t_dims) for i < t_dims / 2,
 *   p = min(frame - ref_frame, cap - 1),  frame = first_frame + token / tokens_per_frame,
 * and leaves dimensions t_dims .. d-1 unchanged (a 3-D embedding rotates them by spatial
 * position, which the cap does not concern). Apply it to Q and K before the attention call.
 *   x, y    device tensors [BH, n_tokens, d] of dtype (HYAT_F32 or HYAT_BF16), 16-byte
 *           aligned, owned by the caller; y == x works in place (then only the band is
 *           rewritten), other overlaps are not allowed;
 *   d       64 or 128; t_dims even, 0 <= t_dims <= d; cap >= 1; base > 0 and finite;
 *           first_frame >= ref_frame; BH <= 65535.
 * Angles and their sines and cosines are formed in double, the rotation in fp32. Enqueued
 * on `stream`; returns HYAT_ERR_INVALID_ARG (nothing enqueued) on bad arguments and
 * HYAT_ERR_CUDA if the launch fails. BH or n_tokens 0 is a no-op. */
HYAT_API hyat_status hyat_rope_temporal(const void* x, void* y, int32_t BH, int32_t n_tokens, int32_t d,
                                        int32_t dtype, int32_t tokens_per_frame, int32_t first_frame,
                                        int32_t ref_frame, int32_t cap, int32_t t_dims, float base,
                                        void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HYAT_H_ */
