// Host layout builder: which key tiles each query tile attends to by softmax,
// and which key segments reach it through the linear state.
//
// Window rules follow the hybrid attention of ReHyAt (Abstract: chunk-wise
// softmax + linear attention) and the block-sparse window of Hybrid Forcing
// (Section 2.A); the radial mask follows Radial Attention (Abstract: each
// token attends to spatially near tokens, the window shrinking with temporal
// distance).
#include <algorithm>
#include <cmath>
#include <string>

#include "hyat_internal.h"

namespace hyat {

int32_t tiles(int64_t rows) { return static_cast<int32_t>((rows + kTile - 1) / kTile); }

int32_t stream_chunk_tokens(const hyat_config& c) { return c.chunk_frames * c.tokens_per_frame; }
int32_t stream_window_chunks(const hyat_config& c) { return c.window_frames / c.chunk_frames; }
int32_t stream_sink_chunks(const hyat_config& c) { return c.sink_frames / c.chunk_frames; }
int32_t stream_ring_slots(const hyat_config& c) { return stream_window_chunks(c) + stream_sink_chunks(c); }

StreamGeometry stream_geometry(const hyat_config& c, int32_t step) {
  StreamGeometry g;
  const int32_t nwc = stream_window_chunks(c), ns = stream_sink_chunks(c);
  g.n_sink_visible = std::min(ns, step + 1);
  g.first_window = std::max(ns, step - nwc + 1);
  g.n_window = step >= g.first_window ? step - g.first_window + 1 : 0;
  g.n_visible = g.n_sink_visible + g.n_window;
  g.evicted = step - nwc >= ns ? step - nwc : -1;
  g.write_slot = stream_slot_of_chunk(c, step);
  return g;
}

int32_t stream_slot_of_chunk(const hyat_config& c, int32_t chunk) {
  const int32_t nwc = stream_window_chunks(c);
  return chunk < stream_sink_chunks(c) ? nwc + chunk : chunk % nwc;
}

int64_t rows_q(const hyat_config& c) {
  if (c.mode == HYAT_MODE_STREAM) return stream_chunk_tokens(c);
  return static_cast<int64_t>(c.n_frames) * c.tokens_per_frame;
}

int64_t rows_k(const hyat_config& c) {
  if (c.mode == HYAT_MODE_STREAM)
    return static_cast<int64_t>(stream_ring_slots(c)) * stream_chunk_tokens(c);
  return static_cast<int64_t>(c.n_frames) * c.tokens_per_frame;
}

std::string validate_config(const hyat_config& c) {
  if (c.B < 1 || c.H < 1) return "B and H must be >= 1";
  if (c.d != 64 && c.d != 128) return "d must be 64 or 128";
  if (c.tokens_per_frame < 1) return "tokens_per_frame must be >= 1";
  if (c.dtype != HYAT_F32 && c.dtype != HYAT_BF16) return "dtype must be HYAT_F32 or HYAT_BF16";
  if (c.phi != HYAT_PHI_ELU1 && c.phi != HYAT_PHI_RELU && c.phi != HYAT_PHI_EXP)
    return "phi must be HYAT_PHI_ELU1, HYAT_PHI_RELU or HYAT_PHI_EXP";
  if (!(c.scale >= 0.0f) || std::isinf(c.scale)) return "scale must be finite and >= 0";
  switch (c.mode) {
    case HYAT_MODE_WINDOW:
      if (c.n_frames < 1) return "n_frames must be >= 1";
      if (c.chunk_frames < 1) return "chunk_frames must be >= 1";
      if (c.halo_frames < 0) return "halo_frames must be >= 0";
      break;
    case HYAT_MODE_BLOCKMASK:
      if (c.n_frames < 1) return "n_frames must be >= 1";
      if (c.mask_heads != 1 && c.mask_heads != c.H) return "mask_heads must be 1 or H";
      break;
    case HYAT_MODE_RADIAL:
      if (c.n_frames < 1) return "n_frames must be >= 1";
      break;
    case HYAT_MODE_STREAM:
      if (c.chunk_frames < 1) return "chunk_frames must be >= 1";
      if (c.window_frames < c.chunk_frames || c.window_frames % c.chunk_frames != 0)
        return "window_frames must be a positive multiple of chunk_frames";
      if (c.mask_heads != 1 && c.mask_heads != c.H) return "mask_heads must be 1 or H";
      if (c.sink_frames < 0 || c.sink_frames % c.chunk_frames != 0)
        return "sink_frames must be a non-negative multiple of chunk_frames";
      break;
    default:
      return "unknown mode";
  }
  const uint32_t branch = c.flags & (HYAT_FLAG_TEST_SOFTMAX_BRANCH | HYAT_FLAG_TEST_LINEAR_BRANCH);
  if (branch == (HYAT_FLAG_TEST_SOFTMAX_BRANCH | HYAT_FLAG_TEST_LINEAR_BRANCH))
    return "at most one of the branch test flags";
  if (branch && c.mode == HYAT_MODE_STREAM) return "the branch test flags are for the bidirectional modes";
  if (c.rope_t_dims != 0) {
    if (c.mode != HYAT_MODE_STREAM) return "the fused temporal RoPE is a STREAM option";
    if (c.rope_t_dims < 0 || c.rope_t_dims > c.d || c.rope_t_dims % 2 != 0)
      return "rope_t_dims must be even and at most d";
    if (c.rope_cap < 1) return "rope_cap must be >= 1";
    if (!(c.rope_base >= 0.0f) || std::isinf(c.rope_base)) return "rope_base must be finite and >= 0";
    if (static_cast<int64_t>(c.chunk_frames) * c.rope_t_dims > 8192) return "chunk_frames * rope_t_dims must be <= 8192";
  }
  const int64_t n = rows_k(c) > rows_q(c) ? rows_k(c) : rows_q(c);
  if (n * c.d >= (int64_t(1) << 31)) return "rows * d per head must be < 2^31";
  if (static_cast<int64_t>(c.B) * c.H * n * c.d >= (int64_t(1) << 40)) return "tensor too large";
  return "";
}

// Radial tile mask by interval marking: for every query tile and every
// frame piece it covers, the keys near that piece in key frame fk form one
// position interval [p0 - r, p1 + r] (r = largest integer with 2r < w); the
// tiles that interval touches are kept.
void radial_tile_mask(int32_t n_frames, int32_t F, uint8_t* out) {
  const int64_t N = static_cast<int64_t>(n_frames) * F;
  const int32_t nT = tiles(N);
  std::fill(out, out + static_cast<size_t>(nT) * nT, uint8_t(0));
  for (int32_t a = 0; a < nT; ++a) {
    const int64_t r0 = static_cast<int64_t>(a) * kTile;
    const int64_t r1 = std::min<int64_t>(N, r0 + kTile);  // exclusive
    for (int64_t r = r0; r < r1;) {
      const int32_t fq = static_cast<int32_t>(r / F);
      const int64_t piece_end = std::min<int64_t>(r1, static_cast<int64_t>(fq + 1) * F);
      const int64_t p0 = r - static_cast<int64_t>(fq) * F;
      const int64_t p1 = piece_end - 1 - static_cast<int64_t>(fq) * F;
      for (int32_t fk = 0; fk < n_frames; ++fk) {
        const int32_t t = fq > fk ? fq - fk : fk - fq;
        int64_t lo, hi;  // key positions inside frame fk, inclusive
        if (t == 0) {
          lo = 0;
          hi = F - 1;
        } else {
          int lg = 0;
          while ((2 << lg) <= t) ++lg;           // floor(log2 t)
          const int64_t w = static_cast<int64_t>(F) >> lg;
          if (w <= 0) continue;
          const int64_t rad = (w - 1) / 2;        // 2*|dp| < w  <=>  |dp| <= (w-1)/2
          lo = std::max<int64_t>(0, p0 - rad);
          hi = std::min<int64_t>(F - 1, p1 + rad);
          if (lo > hi) continue;
        }
        const int64_t k0 = static_cast<int64_t>(fk) * F + lo;
        const int64_t k1 = static_cast<int64_t>(fk) * F + hi;
        for (int64_t b = k0 / kTile; b <= k1 / kTile; ++b) out[static_cast<size_t>(a) * nT + b] = 1;
      }
      r = piece_end;
    }
  }
}

void lvsa_tile_mask(int32_t n_frames, int32_t F, int32_t window_frames, int32_t anchor_stride, int32_t rotation,
                    uint8_t* out) {
  const int64_t N = static_cast<int64_t>(n_frames) * F;
  const int32_t nT = tiles(N);
  const int32_t half = (window_frames - 1) / 2;
  // frames covered by each tile, and whether a tile holds a token of an anchor frame
  std::vector<int32_t> f_lo(nT), f_hi(nT);
  std::vector<uint8_t> has_anchor(nT, 0);
  for (int32_t t = 0; t < nT; ++t) {
    const int64_t r0 = static_cast<int64_t>(t) * kTile, r1 = std::min<int64_t>(N, r0 + kTile) - 1;
    f_lo[t] = static_cast<int32_t>(r0 / F);
    f_hi[t] = static_cast<int32_t>(r1 / F);
    if (anchor_stride > 0)
      for (int32_t f = f_lo[t]; f <= f_hi[t]; ++f)
        if ((f + rotation) % anchor_stride == 0) has_anchor[t] = 1;
  }
  for (int32_t a = 0; a < nT; ++a)
    for (int32_t b = 0; b < nT; ++b) {
      const int32_t gap = std::max(0, std::max(f_lo[b] - f_hi[a], f_lo[a] - f_hi[b]));
      out[static_cast<size_t>(a) * nT + b] = (gap <= half || has_anchor[b]) ? 1 : 0;
    }
}

// The key tiles of [k_lo, k_hi), first key first, or last tile first when `descending`.
static void push_window_entries(int64_t k_lo, int64_t k_hi, bool descending, std::vector<Entry>* e) {
  const size_t first = e->size();
  for (int64_t k = k_lo; k < k_hi; k += kTile)
    e->push_back(Entry{static_cast<int32_t>(k), static_cast<int32_t>(std::min<int64_t>(kTile, k_hi - k))});
  if (descending) std::reverse(e->begin() + static_cast<std::ptrdiff_t>(first), e->end());
}

std::string build_layout(const hyat_config& c, const uint8_t* host_mask, Layout* L) {
  *L = Layout();
  const int32_t BH = c.B * c.H;
  const int64_t N = rows_q(c);
  const int32_t F = c.tokens_per_frame;
  if (c.mode == HYAT_MODE_WINDOW) {
    const int32_t T = c.n_frames, C = c.chunk_frames, h = c.halo_frames;
    const int32_t n_chunks = (T + C - 1) / C;
    L->nseg = T;
    L->seg_stride = F;
    L->seg_len = F;
    L->nqg = n_chunks;
    L->cm_heads = 1;
    L->cm.assign(static_cast<size_t>(n_chunks) * T, 0.0f);
    std::vector<int32_t> eb(n_chunks), ee(n_chunks);
    for (int32_t ch = 0; ch < n_chunks; ++ch) {
      const int32_t lo = std::max(0, ch * C - h);
      const int32_t hi = std::min(T, (ch + 1) * C + h);
      for (int32_t f = 0; f < T; ++f)
        L->cm[static_cast<size_t>(ch) * T + f] = (f < lo || f >= hi) ? 1.0f : 0.0f;
      eb[ch] = static_cast<int32_t>(L->entries.size());
      // Neighbouring windows share the halo frames: the end of one window is the start of the
      // next. Odd chunks walk their window last tile first, so the CTAs of two neighbouring
      // chunks, which run at the same time, reach the shared frames at the same time and the
      // second read of those K, V tiles hits L2 instead of HBM. (The sum over keys does not
      // depend on their order beyond rounding.)
      push_window_entries(static_cast<int64_t>(lo) * F, static_cast<int64_t>(hi) * F, (ch & 1) != 0, &L->entries);
      ee[ch] = static_cast<int32_t>(L->entries.size());
    }
    for (int32_t bh = 0; bh < BH; ++bh)
      for (int32_t ch = 0; ch < n_chunks; ++ch) {
        const int64_t q0 = static_cast<int64_t>(ch) * C * F;
        const int64_t q1 = std::min<int64_t>(N, static_cast<int64_t>(ch + 1) * C * F);
        for (int64_t q = q0; q < q1; q += kTile)
          L->work.push_back(WorkItem{bh, static_cast<int32_t>(q),
                                     static_cast<int32_t>(std::min<int64_t>(kTile, q1 - q)), ch,
                                     eb[ch], ee[ch], 0, 0});
      }
    return "";
  }
  if (c.mode == HYAT_MODE_BLOCKMASK || c.mode == HYAT_MODE_RADIAL) {
    const int32_t nT = tiles(N);
    std::vector<uint8_t> radial;
    const uint8_t* mask = host_mask;
    int32_t mh = c.mask_heads;
    if (c.mode == HYAT_MODE_RADIAL) {
      radial.resize(static_cast<size_t>(nT) * nT);
      radial_tile_mask(c.n_frames, F, radial.data());
      mask = radial.data();
      mh = 1;
    } else if (mask == nullptr) {
      return "BLOCKMASK needs a host mask";
    }
    L->nseg = nT;
    L->seg_stride = kTile;
    L->seg_len = kTile;
    L->nqg = nT;
    L->cm_heads = mh;
    L->cm.assign(static_cast<size_t>(mh) * nT * nT, 0.0f);
    std::vector<int32_t> eb(static_cast<size_t>(mh) * nT), ee(static_cast<size_t>(mh) * nT);
    for (int32_t m = 0; m < mh; ++m)
      for (int32_t i = 0; i < nT; ++i) {
        const size_t row = (static_cast<size_t>(m) * nT + i) * nT;
        eb[static_cast<size_t>(m) * nT + i] = static_cast<int32_t>(L->entries.size());
        for (int32_t b = 0; b < nT; ++b) {
          if (mask[row + b]) {
            L->entries.push_back(Entry{b * kTile, static_cast<int32_t>(std::min<int64_t>(kTile, N - int64_t(b) * kTile))});
          } else {
            L->cm[row + b] = 1.0f;
          }
        }
        ee[static_cast<size_t>(m) * nT + i] = static_cast<int32_t>(L->entries.size());
      }
    for (int32_t bh = 0; bh < BH; ++bh) {
      const int32_t m = (mh == 1) ? 0 : bh % c.H;
      for (int32_t i = 0; i < nT; ++i)
        L->work.push_back(WorkItem{bh, i * kTile, static_cast<int32_t>(std::min<int64_t>(kTile, N - int64_t(i) * kTile)),
                                   i, eb[static_cast<size_t>(m) * nT + i], ee[static_cast<size_t>(m) * nT + i], 0, 0});
    }
    return "";
  }
  if (c.mode == HYAT_MODE_STREAM) {
    // work items and entries are produced on the device each step
    L->nseg = 1;
    L->seg_stride = stream_chunk_tokens(c);
    L->seg_len = stream_chunk_tokens(c);
    L->nqg = 1;
    return "";
  }
  return "unknown mode";
}

std::vector<int4> build_pairs(const std::vector<WorkItem>& work) {
  std::vector<int4> pairs;
  for (size_t i = 0; i < work.size();) {
    if (i + 1 < work.size() && work[i + 1].bh == work[i].bh) {
      const bool shared = work[i].entry_begin == work[i + 1].entry_begin && work[i].entry_end == work[i + 1].entry_end;
      pairs.push_back(make_int4(static_cast<int>(i), static_cast<int>(i + 1), shared ? 1 : 0, 0));
      i += 2;
    } else {
      pairs.push_back(make_int4(static_cast<int>(i), -1, 0, 0));
      i += 1;
    }
  }
  return pairs;
}

std::vector<int4> order_pairs_for_grid(const std::vector<int4>& pairs, const std::vector<WorkItem>& work,
                                       int32_t grid) {
  if (grid <= 1 || pairs.size() <= static_cast<size_t>(grid)) return pairs;
  // cost of a pair: its key tiles (both slots) plus two tiles' worth of per-pair set-up
  auto n_of = [&](int item) { return item < 0 ? 0 : work[item].entry_end - work[item].entry_begin; };
  std::vector<int64_t> cost(pairs.size());
  for (size_t i = 0; i < pairs.size(); ++i) cost[i] = n_of(pairs[i].x) + n_of(pairs[i].y) + 2;
  std::vector<size_t> idx(pairs.size());
  for (size_t i = 0; i < idx.size(); ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](size_t a, size_t b) { return cost[a] > cost[b]; });
  // The kernel hands pair k to CTA k mod grid, so the list is rows of `grid` pairs, one per
  // CTA, largest first. Two ways of placing each row's pairs are weighed, and the one whose
  // busiest CTA holds less work wins (ties: the first):
  //   * serpentine: left to right in even rows, right to left in odd rows;
  //   * least loaded first: the row's pairs, largest first, to the CTAs in ascending order of
  //     the work they already hold (ties: lower CTA), a longest-processing-time rule.
  // Neither wins everywhere: with a few distinct costs the serpentine balances better, with
  // widely spread costs the second.
  const size_t n = idx.size();
  std::vector<int4> serp(n), lpt(n);
  std::vector<int64_t> load_s(grid, 0), load_l(grid, 0);
  std::vector<int32_t> by_load(grid);
  for (size_t r0 = 0, r = 0; r0 < n; r0 += grid, ++r) {
    const size_t len = std::min<size_t>(grid, n - r0);   // a partial row: CTAs 0 .. len - 1
    for (size_t j = 0; j < len; ++j) {
      const size_t c = (r & 1) ? len - 1 - j : j;
      serp[r0 + c] = pairs[idx[r0 + j]];
      load_s[c] += cost[idx[r0 + j]];
    }
    for (size_t c = 0; c < len; ++c) by_load[c] = static_cast<int32_t>(c);
    std::stable_sort(by_load.begin(), by_load.begin() + len, [&](int32_t a, int32_t b) { return load_l[a] < load_l[b]; });
    for (size_t j = 0; j < len; ++j) {
      const int32_t c = by_load[j];
      lpt[r0 + c] = pairs[idx[r0 + j]];
      load_l[c] += cost[idx[r0 + j]];
    }
  }
  const int64_t max_s = *std::max_element(load_s.begin(), load_s.end());
  const int64_t max_l = *std::max_element(load_l.begin(), load_l.end());
  return max_l < max_s ? lpt : serp;
}

std::vector<int4> build_split_pairs(size_t n_items) {
  std::vector<int4> pairs(n_items);
  for (size_t i = 0; i < n_items; ++i) pairs[i] = make_int4(static_cast<int>(i), static_cast<int>(i), 0, 1);
  return pairs;
}

bool prefer_split_pairs(size_t n_ordinary_pairs, int32_t num_sms) {
  return n_ordinary_pairs < static_cast<size_t>(4) * static_cast<size_t>(num_sms > 0 ? num_sms : 1);
}

std::vector<int4> choose_pairs(const std::vector<WorkItem>& work, int32_t num_sms) {
  std::vector<int4> pairs = build_pairs(work);
  if (prefer_split_pairs(pairs.size(), num_sms)) pairs = build_split_pairs(work.size());
  return order_pairs_for_grid(pairs, work, num_sms);
}

std::vector<int4> build_single_items(const std::vector<WorkItem>& work, int32_t num_sms) {
  std::vector<int4> items(work.size());
  for (size_t i = 0; i < work.size(); ++i) items[i] = make_int4(static_cast<int>(i), -1, 0, 0);
  return order_pairs_for_grid(items, work, num_sms);
}

std::vector<int4> build_stream_pairs(int32_t BH, int32_t nqt) {
  std::vector<int4> pairs;
  for (int32_t bh = 0; bh < BH; ++bh)
    for (int32_t i = 0; i < nqt; i += 2)
      pairs.push_back(make_int4(bh * nqt + i, i + 1 < nqt ? bh * nqt + i + 1 : -1, 0, 0));
  return pairs;
}

}  // namespace hyat
