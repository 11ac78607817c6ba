"""Hybrid attention written out from its definition, in float64, on the CPU.

TEST INFRASTRUCTURE: see the package docstring. Nothing here is tuned; rows are
evaluated in blocks only to bound memory, and each row is independent by
definition.

The operation (ReHyAt: Recurrent Hybrid Attention for Video Diffusion
Transformers, Abstract; Long-Horizon Streaming Video Generation via Hybrid
Attention with Decoupled Distillation, §2.A "Hybrid Attention"): every query i
splits the keys into a softmax set W_i (its local or block-sparse window) and a
linear set R_i (everything the window does not reach: all other tokens for a
bidirectional transformer, only the evicted frames when streaming). With
s_ij = q_i.k_j * scale and a feature map phi, the weights are

    w_ij = exp(s_ij)              for j in W_i
    w_ij = phi(q_i) . phi(k_j)    for j in R_i
    w_ij = 0                      otherwise

and o_i = sum_j w_ij v_j / sum_j w_ij. Shifting every weight of row i by the
same factor exp(-m_i) leaves o_i unchanged, which is how the chunk-wise form
(exp(s - m) over the window, exp(-m) phi(q)^T S and exp(-m) phi(q)^T z for the
linear state S = sum phi(k) v^T, z = sum phi(k)) reaches exactly this result.
Here m_i = max(0, max_{j in W_i} s_ij) only keeps exp() in range.

Readings taken where the pages are silent (each is listed with its reason in
the design notes):
  * phi = elu + 1 with alpha = 1 by default (ReLU and exp on request), on raw q
    and k; the scale multiplies softmax logits only.
  * bidirectional window: chunk c covers frames [c*C, (c+1)*C); its window is
    frames [c*C - halo, (c+1)*C + halo) clipped to the video.
  * radial mask: tile kept iff any token pair in it is "near"; near means same
    frame, or 2*|p_j - p_i| < F >> floor(log2 t) with t the frame distance and
    p the raster index inside the frame.
  * streaming: at step s the window is the chunks [s - n_win + 1, s]; older
    chunks are evicted into the linear set; window tiles the mask drops are
    dropped (they reach neither branch). With n_sink sink chunks, chunks
    [0, n_sink) stay visible for good and the window starts no earlier than
    n_sink; a denoising call of chunk s is the same computation with that
    call's own K, V as chunk s.
  * structured window + rotating anchors (Long Video Sparse Attention): keys
    within (window_frames - 1) / 2 frames of the query, plus every key of an
    anchor frame f with (f + rotation) % anchor_stride == 0.
"""
from __future__ import annotations

import numpy as np

ROW_BLOCK = 256


# --------------------------------------------------------------------------
# feature map
# --------------------------------------------------------------------------
def phi_elu1(x):
    """phi(x) = elu(x) + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def phi_relu(x):
    """phi(x) = max(x, 0)."""
    return np.maximum(np.asarray(x, dtype=np.float64), 0.0)


def phi_exp(x):
    """phi(x) = exp(x), elementwise."""
    return np.exp(np.asarray(x, dtype=np.float64))


# The pages leave the feature map open (only phi >= 0 is needed for one normaliser);
# elu + 1 is the default, ReLU and exp are the alternatives of the linear-attention papers
# the pages cite.
FEATURE_MAPS = {"elu1": phi_elu1, "relu": phi_relu, "exp": phi_exp}


def feature_map(phi):
    """A feature map given by name ("elu1", "relu", "exp") or as a function."""
    return FEATURE_MAPS[phi] if isinstance(phi, str) else phi


# --------------------------------------------------------------------------
# the definition, for a block of rows
# --------------------------------------------------------------------------
def hybrid_rows(q_rows, k, v, soft, lin, scale, phi=phi_elu1):
    """Outputs of the rows in ``q_rows`` [R,d] against keys k [N,d], values v [N,d].

    ``soft`` and ``lin`` are disjoint boolean masks [R,N]: the softmax set and
    the linear set of each row. Returns (o [R,d], num_soft, den_soft, num_lin,
    den_lin), all shifted by the same exp(-m_i) per row, so the branch-wise
    numerators and denominators can be checked separately.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    assert not np.any(soft & lin), "softmax and linear sets must be disjoint"
    s = (q_rows @ k.T) * scale
    s_win = np.where(soft, s, -np.inf)
    m = np.maximum(0.0, np.max(s_win, axis=1, initial=-np.inf))
    e_soft = np.exp(s_win - m[:, None])                 # 0 outside the window
    lin_w = (phi(q_rows) @ phi(k).T) * np.exp(-m)[:, None]
    e_lin = np.where(lin, lin_w, 0.0)
    num_soft = e_soft @ v
    den_soft = e_soft.sum(axis=1)
    num_lin = e_lin @ v
    den_lin = e_lin.sum(axis=1)
    o = (num_soft + num_lin) / (den_soft + den_lin)[:, None]
    return o, num_soft, den_soft, num_lin, den_lin


def _run_rows(q, k, v, rows, sets_fn, scale, with_branches=False, phi="elu1"):
    """Apply hybrid_rows per (batch, head) over the requested rows.

    q: [B,H,Nq,d]; k, v: [B,H,Nk,d]; sets_fn(h, rows) -> (soft, lin).
    """
    B, H, Nq, d = q.shape
    if rows is None:
        rows = np.arange(Nq)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, H, len(rows), d))
    br = [np.zeros((B, H, len(rows), d)), np.zeros((B, H, len(rows))),
          np.zeros((B, H, len(rows), d)), np.zeros((B, H, len(rows)))]
    for b in range(B):
        for h in range(H):
            kb = np.asarray(k[b, h], dtype=np.float64)
            vb = np.asarray(v[b, h], dtype=np.float64)
            for r0 in range(0, len(rows), ROW_BLOCK):
                rr = rows[r0:r0 + ROW_BLOCK]
                soft, lin = sets_fn(h, rr)
                qb = np.asarray(q[b, h, rr], dtype=np.float64)
                o, ns, ds, nl, dl = hybrid_rows(qb, kb, vb, soft, lin, scale, feature_map(phi))
                out[b, h, r0:r0 + len(rr)] = o
                if with_branches:
                    br[0][b, h, r0:r0 + len(rr)] = ns
                    br[1][b, h, r0:r0 + len(rr)] = ds
                    br[2][b, h, r0:r0 + len(rr)] = nl
                    br[3][b, h, r0:r0 + len(rr)] = dl
    if with_branches:
        return out, br
    return out


def _default_scale(d, scale):
    return 1.0 / np.sqrt(d) if scale is None else float(scale)


# --------------------------------------------------------------------------
# bidirectional chunk window (ReHyAt, Abstract: chunk-wise hybrid attention)
# --------------------------------------------------------------------------
def bidir_window_interval(frame, n_frames, chunk_frames, halo_frames):
    """Window of the chunk holding ``frame``, as a frame interval [lo, hi)."""
    c = frame // chunk_frames
    lo = max(0, c * chunk_frames - halo_frames)
    hi = min(n_frames, (c + 1) * chunk_frames + halo_frames)
    return lo, hi


def bidir_sets(rows, tokens_per_frame, n_frames, chunk_frames, halo_frames):
    """Softmax and linear sets of the given query rows (token-exact)."""
    N = tokens_per_frame * n_frames
    rows = np.asarray(rows, dtype=np.int64)
    j = np.arange(N)[None, :]
    lo = np.empty(len(rows), dtype=np.int64)
    hi = np.empty(len(rows), dtype=np.int64)
    for n, i in enumerate(rows):
        f_lo, f_hi = bidir_window_interval(int(i) // tokens_per_frame, n_frames,
                                           chunk_frames, halo_frames)
        lo[n], hi[n] = f_lo * tokens_per_frame, f_hi * tokens_per_frame
    soft = (j >= lo[:, None]) & (j < hi[:, None])
    return soft, ~soft


def bidir_window_attention(q, k, v, tokens_per_frame, n_frames, chunk_frames,
                           halo_frames, scale=None, rows=None, with_branches=False, phi="elu1"):
    """Bidirectional hybrid attention: window = chunk +/- halo frames, the rest linear."""
    sc = _default_scale(q.shape[-1], scale)
    fn = lambda h, rr: bidir_sets(rr, tokens_per_frame, n_frames, chunk_frames, halo_frames)
    return _run_rows(q, k, v, rows, fn, sc, with_branches, phi)


# --------------------------------------------------------------------------
# tile masks (block-sparse window; Hybrid Forcing §2.A block-sparse SWA)
# --------------------------------------------------------------------------
def tile_mask_sets(h, rows, tile_mask, N, tile=128):
    """Softmax set = tokens of kept key tiles of the row's query tile; linear = the rest.

    tile_mask: uint8/bool [Hm, nQT, nKT] on the absolute tile grid (Hm = 1 or H).
    """
    tm = np.asarray(tile_mask).astype(bool)
    hm = 0 if tm.shape[0] == 1 else h
    rows = np.asarray(rows, dtype=np.int64)
    key_tile = np.arange(N) // tile
    soft = tm[hm][rows // tile][:, key_tile]
    return soft, ~soft


def blockmask_attention(q, k, v, tile_mask, scale=None, rows=None, tile=128,
                        with_branches=False, phi="elu1"):
    N = q.shape[2]
    sc = _default_scale(q.shape[-1], scale)
    fn = lambda h, rr: tile_mask_sets(h, rr, tile_mask, N, tile)
    return _run_rows(q, k, v, rows, fn, sc, with_branches, phi)


# --------------------------------------------------------------------------
# radial mask (Radial Attention, Abstract: spatial window shrinking with
# temporal distance)
# --------------------------------------------------------------------------
def radial_window(t, tokens_per_frame):
    """Spatial window (tokens) at frame distance t >= 1: F >> floor(log2 t)."""
    t = int(t)
    assert t >= 1
    return tokens_per_frame >> (t.bit_length() - 1)


def radial_token_near(i, j, tokens_per_frame):
    """Token-level radial predicate (vectorised over broadcastable i, j)."""
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    fi, pi = np.divmod(i, tokens_per_frame)
    fj, pj = np.divmod(j, tokens_per_frame)
    t = np.abs(fi - fj)
    # floor(log2 t) for integer t >= 1: frexp gives t = m * 2**e with m in [0.5, 1)
    lg = np.frexp(np.maximum(t, 1).astype(np.float64))[1].astype(np.int64) - 1
    w = np.right_shift(np.int64(tokens_per_frame), lg)
    return (t == 0) | (2 * np.abs(pj - pi) < w)


def _tile_frame_segments(n_tiles, N, tokens_per_frame, tile):
    """(tile, frame, p_lo, p_hi) pieces: each tile split at frame boundaries."""
    segs = []
    for a in range(n_tiles):
        r0, r1 = a * tile, min((a + 1) * tile, N)
        r = r0
        while r < r1:
            f = r // tokens_per_frame
            end = min(r1, (f + 1) * tokens_per_frame)
            segs.append((a, f, r - f * tokens_per_frame, end - 1 - f * tokens_per_frame))
            r = end
    return np.array(segs, dtype=np.int64)


def radial_tile_mask(n_frames, tokens_per_frame, tile=128):
    """Kept tiles [nT, nT] (uint8): a tile is kept iff some token pair in it is near.

    For a query piece (frame fq, positions [a0, a1]) and a key piece (frame fk,
    positions [b0, b1]) the closest pair has |p_j - p_i| = gap of the two
    intervals, so the piece pair holds a near pair iff fq == fk or
    2 * gap < F >> floor(log2 |fq - fk|).
    """
    N = n_frames * tokens_per_frame
    nT = -(-N // tile)
    seg = _tile_frame_segments(nT, N, tokens_per_frame, tile)
    qa, qf, q0, q1 = (seg[:, c][:, None] for c in range(4))
    ka, kf, k0, k1 = (seg[:, c][None, :] for c in range(4))
    t = np.abs(qf - kf)
    gap = np.maximum(0, np.maximum(k0 - q1, q0 - k1))
    wt = np.zeros_like(t)
    for tt in np.unique(t):
        if tt > 0:
            wt[t == tt] = radial_window(int(tt), tokens_per_frame)
    near = (t == 0) | (2 * gap < wt)
    mask = np.zeros((nT, nT), dtype=np.uint8)
    qi, ki = np.nonzero(near)
    mask[seg[qi, 0], seg[ki, 0]] = 1
    return mask


# --------------------------------------------------------------------------
# structured window + rotating global anchors (Long Video Sparse Attention,
# Abstract). Reading (the pages give no rule): keys within (window_frames - 1)/2
# frames of the query, plus every key of an anchor frame f with
# (f + rotation) % anchor_stride == 0; a 128-token tile pair is kept iff it holds
# such a token pair.
# --------------------------------------------------------------------------
def lvsa_token_near(i, j, tokens_per_frame, window_frames, anchor_stride, rotation):
    """Token-level predicate (vectorised over broadcastable i, j)."""
    fi = np.asarray(i, dtype=np.int64) // tokens_per_frame
    fj = np.asarray(j, dtype=np.int64) // tokens_per_frame
    near = np.abs(fi - fj) <= (window_frames - 1) // 2
    if anchor_stride > 0:
        near = near | ((fj + rotation) % anchor_stride == 0)
    return near


def lvsa_tile_mask(n_frames, tokens_per_frame, window_frames, anchor_stride, rotation=0, tile=128):
    """Kept tiles [nT, nT] (uint8). A tile pair holds a near token pair iff the frames of
    the two tiles come within the window, or the key tile touches an anchor frame."""
    N = n_frames * tokens_per_frame
    nT = -(-N // tile)
    frames_of = [set(range((a * tile) // tokens_per_frame, (min(N, (a + 1) * tile) - 1) // tokens_per_frame + 1))
                 for a in range(nT)]
    half = (window_frames - 1) // 2
    anchor = np.array([anchor_stride > 0 and any((f + rotation) % anchor_stride == 0 for f in fr)
                       for fr in frames_of])
    lo = np.array([min(fr) for fr in frames_of])
    hi = np.array([max(fr) for fr in frames_of])
    gap = np.maximum(0, np.maximum(lo[None, :] - hi[:, None], lo[:, None] - hi[None, :]))
    return ((gap <= half) | anchor[None, :]).astype(np.uint8)


def radial_attention(q, k, v, n_frames, tokens_per_frame, scale=None, rows=None,
                     tile=128, with_branches=False, phi="elu1"):
    mask = radial_tile_mask(n_frames, tokens_per_frame, tile)[None]
    return blockmask_attention(q, k, v, mask, scale, rows, tile, with_branches, phi)


# --------------------------------------------------------------------------
# streaming (Hybrid Forcing §2.A: evicted frames feed a linear state; the
# recent window is block-sparse softmax)
# --------------------------------------------------------------------------
def stream_visible_chunks(step, n_window_chunks, n_sink_chunks=0):
    """Chunks visible at ``step``, oldest first: the sink chunks that exist, then the latest
    n_window_chunks chunks after them."""
    sinks = list(range(min(n_sink_chunks, step + 1)))
    first = max(n_sink_chunks, step - n_window_chunks + 1)
    return sinks + list(range(first, step + 1))


def stream_sets(h, rows, step, chunk_tokens, n_window_chunks, tile_mask, tile=128, n_sink_chunks=0):
    """Sets for query rows (chunk-local) of chunk ``step`` over keys of chunks 0..step.

    Key j is the global token index over the generated chunks; the mask is
    [Hm, nQT, nQT * n_visible] with key tiles ordered oldest visible chunk first.
    """
    tm = np.asarray(tile_mask).astype(bool)
    hm = 0 if tm.shape[0] == 1 else h
    rows = np.asarray(rows, dtype=np.int64)
    nqt = -(-chunk_tokens // tile)
    vis = stream_visible_chunks(step, n_window_chunks, n_sink_chunks)
    rank = {c: r for r, c in enumerate(vis)}
    n_keys = (step + 1) * chunk_tokens
    j = np.arange(n_keys)
    c_of_j = j // chunk_tokens
    visible = np.isin(c_of_j, vis)
    kt_of_j = np.array([rank.get(int(c), 0) for c in c_of_j], dtype=np.int64) * nqt + (j % chunk_tokens) // tile
    soft = np.zeros((len(rows), n_keys), dtype=bool)
    soft[:, visible] = tm[hm][rows // tile][:, kt_of_j[visible]]
    lin = np.broadcast_to(~visible, soft.shape).copy()
    return soft, lin


def stream_step_attention(q_chunk, k_hist, v_hist, step, chunk_tokens, n_window_chunks,
                          tile_mask, scale=None, rows=None, tile=128, with_branches=False, phi="elu1",
                          n_sink_chunks=0):
    """Output of chunk ``step``; k_hist, v_hist hold chunks 0..step ([B,H,(step+1)L,d])."""
    assert k_hist.shape[2] == (step + 1) * chunk_tokens
    sc = _default_scale(q_chunk.shape[-1], scale)
    fn = lambda h, rr: stream_sets(h, rr, step, chunk_tokens, n_window_chunks, tile_mask, tile, n_sink_chunks)
    return _run_rows(q_chunk, k_hist, v_hist, rows, fn, sc, with_branches, phi)


def stream_evicted_state(k_hist, v_hist, step, chunk_tokens, n_window_chunks, phi="elu1", n_sink_chunks=0):
    """Linear state used at ``step``: S = sum phi(k) v^T, z = sum phi(k) over evicted chunks
    (chunks that are neither sinks nor in the window).

    Returns S [B,H,d,d] and z [B,H,d] in float64 (zero before anything is evicted).
    """
    lo = n_sink_chunks * chunk_tokens
    hi = max(n_sink_chunks, step - n_window_chunks + 1) * chunk_tokens
    k = np.asarray(k_hist[:, :, lo:hi], dtype=np.float64)
    v = np.asarray(v_hist[:, :, lo:hi], dtype=np.float64)
    pk = feature_map(phi)(k)
    S = np.einsum("bhna,bhnc->bhac", pk, v)
    z = pk.sum(axis=2)
    return S, z


# --------------------------------------------------------------------------
# work counts for the effective-FLOP metric
# --------------------------------------------------------------------------
def effective_pairs_bidir(tokens_per_frame, n_frames, chunk_frames, halo_frames):
    """Number of (query, key) pairs inside the softmax windows, per head."""
    total = 0
    for f in range(n_frames):
        lo, hi = bidir_window_interval(f, n_frames, chunk_frames, halo_frames)
        total += tokens_per_frame * (hi - lo) * tokens_per_frame
    return total


def effective_pairs_tile_mask(tile_mask, n_q, n_k, tile=128):
    """Valid (query, key) pairs inside kept tiles, per mask head."""
    tm = np.asarray(tile_mask).astype(np.int64)
    nqt, nkt = tm.shape[-2], tm.shape[-1]
    qlen = np.minimum(tile, n_q - tile * np.arange(nqt))
    klen = np.minimum(tile, n_k - tile * np.arange(nkt))
    return np.einsum("...ij,i,j->...", tm, qlen, klen)
