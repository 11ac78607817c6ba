"""GPU tests of the streaming step's device-side pieces, through the C ABI.

- The layout a step builds on the device (its key tiles per query tile, as ring rows) read
  back and compared bit for bit with the oracle's token sets (Hybrid Forcing, Section 2.A:
  block-sparse softmax over the window, evicted frames through the linear state), with the
  ring slot of every visible chunk checked against the ring's contents.
- The capped temporal RoPE fused into the step (Section 2.C) against the standalone
  hyat_rope_temporal followed by the step, and against the oracle.
- The device-mask call and its CUDA-graph replay against the host-mask call, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_parity, f64

pytestmark = pytest.mark.gpu

ROPE = {"t_dims": 44, "cap": 5, "base": 10000.0}


def _dev(*ts):
    return [t.cuda() for t in ts]


def _ring_k(h, cfg):
    """The K ring from the state blob: [BH, slots, L, d] bf16 bits as uint16."""
    blob = h.get_state()
    BH, d = cfg.B * cfg.H, cfg.d
    L = cfg.chunk_frames * cfg.tokens_per_frame
    slots = cfg.window_frames // cfg.chunk_frames + cfg.sink_frames // cfg.chunk_frames
    off = 48 + 4 * BH * (d * d + d)
    n = BH * slots * L * d
    return np.frombuffer(blob[off:off + 2 * n], np.uint16).reshape(BH, slots, L, d)


@pytest.mark.parametrize("sink_frames", [0, 3])
@pytest.mark.parametrize("mask_heads", [1, 2])
def test_stream_device_layout_bit_exact(sink_frames, mask_heads):
    """Steps 0 to 12 of a 3-tile chunk with a 3-chunk window: the device key-tile list of every
    (head, query tile) covers exactly the oracle's softmax keys, in mask order, and each
    visible chunk sits in the ring slot the step reports."""
    w = wl.Workload("stream_layout", "stream", 1, 2, 128, 100, 45, chunk_frames=3, window_frames=9,
                    n_steps=13, seed=12, sink_frames=sink_frames)
    cfg = hyat.config_from_workload(w, mask_heads=mask_heads)
    h = hyat.Hyat(cfg)
    L, nqt, nwc, ns = w.chunk_tokens, 3, 3, sink_frames // 3
    k_bits = []
    for s in range(13):
        q, k, v, mask = wl.gen_stream_step(w, s)
        mask = mask[:mask_heads]
        h.stream_step(*_dev(q, k, v), mask=mask)
        k_bits.append(k.view(torch.int16).numpy().view(np.uint16))
        work, ent, info, step = h.stream_layout()
        assert step == s
        vis = oracle.stream_visible_chunks(s, nwc, ns)
        assert info[1] == len(vis)
        slots = [int(x) for x in info[4:4 + len(vis)]]
        ring = _ring_k(h, cfg)
        for wv, c in enumerate(vis):          # the slot really holds that chunk's K
            assert np.array_equal(ring[:, slots[wv]], k_bits[c][0]), (s, c)
        cap = ent.shape[1]
        for bh in range(2):
            for i in range(nqt):
                item = bh * nqt + i
                q_len = min(128, L - 128 * i)
                assert [int(x) for x in work[item][[0, 1, 2, 3, 4, 6, 7]]] == [bh, 128 * i, q_len, 0, item * cap, 0, 0]
                n = work[item][5] - work[item][4]
                got = np.zeros((s + 1) * L, bool)
                order = []
                for k_row, k_len in ent[item, :n]:
                    slot, t = divmod(int(k_row), L)
                    assert t % 128 == 0 and k_len == min(128, L - t)
                    wv = slots.index(slot)
                    order.append(wv * nqt + t // 128)
                    j0 = vis[wv] * L + t
                    assert not got[j0:j0 + k_len].any()
                    got[j0:j0 + k_len] = True
                assert order == sorted(order)
                soft, _ = oracle.stream_sets(bh, np.array([128 * i]), s, L, nwc, mask, n_sink_chunks=ns)
                assert np.array_equal(got, soft[0]), (s, bh, i)
    h.close()


def _rope_ref_frames(w, s):
    """The fused RoPE's frames for step s: the chunk's first frame and the reference frame
    (the first frame of the oldest rolling-window chunk, or the chunk's own while the window
    holds none)."""
    nwc, ns = w.window_frames // w.chunk_frames, w.sink_frames // w.chunk_frames
    first_window = max(ns, s - nwc + 1)
    f0 = s * w.chunk_frames
    return f0, (first_window * w.chunk_frames if s >= first_window else f0)


@pytest.mark.parametrize("sink_frames", [0, 3])
def test_stream_fused_rope_equals_standalone_then_step(sink_frames):
    """Steps 0 to 10 with the RoPE fused into the step give the same bits as the standalone
    hyat_rope_temporal on Q and K followed by a plain step; sampled steps also match the
    oracle (oracle RoPE, then the oracle's streaming step)."""
    w = wl.Workload("stream_rope", "stream", 1, 2, 128, 200, 33, chunk_frames=3, window_frames=9,
                    n_steps=11, seed=19, sink_frames=sink_frames)
    hf = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2, rope=ROPE))
    hs = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2))
    L, nwc, ns = w.chunk_tokens, 3, sink_frames // 3
    kh, vh = [], []
    for s in range(11):
        q, k, v, mask = wl.gen_stream_step(w, s)
        qd, kd, vd = _dev(q, k, v)
        f0, ref = _rope_ref_frames(w, s)
        qr = hyat.rope_temporal(qd, w.tokens_per_frame, f0, ref, ROPE["cap"], ROPE["t_dims"], ROPE["base"])
        kr = hyat.rope_temporal(kd, w.tokens_per_frame, f0, ref, ROPE["cap"], ROPE["t_dims"], ROPE["base"])
        of = hf.stream_step(qd, kd, vd, mask=mask)
        os_ = hs.stream_step(qr, kr, vd, mask=mask)
        torch.cuda.synchronize()
        assert torch.equal(of, os_), s
        assert torch.equal(qd.cpu(), q) and torch.equal(kd.cpu(), k)      # the caller's Q, K untouched
        # the RoPE step's outputs are bf16 tensors: the attention sees the turned Q and K
        # rounded to bf16 (and the cache keeps K so)
        bf = lambda x: torch.from_numpy(x).to(torch.bfloat16).double().numpy()
        qo = bf(oracle.rope_temporal(f64(q), w.tokens_per_frame, f0, ref, ROPE["cap"], ROPE["t_dims"], ROPE["base"]))
        ko = bf(oracle.rope_temporal(f64(k), w.tokens_per_frame, f0, ref, ROPE["cap"], ROPE["t_dims"], ROPE["base"]))
        kh.append(ko)
        vh.append(v.float().numpy())
        if s in (0, 4, 10):
            want = oracle.stream_step_attention(qo, np.concatenate(kh, axis=2), np.concatenate(vh, axis=2), s, L,
                                                nwc, mask, n_sink_chunks=ns)
            assert_parity("bf16", f64(of.cpu()), want, f"step {s}")
    hf.sync()
    hs.sync()
    hf.close()
    hs.close()


def test_stream_graph_replay_equals_eager_steps():
    """14 steps through three handles: host mask, device mask, and device mask replayed from
    CUDA graphs (fixed input buffers, as graph replay needs); every output bit for bit equal.
    Midway the output buffer changes, which captures again."""
    w = wl.Workload("stream_graph", "stream", 1, 2, 128, 200, 42, chunk_frames=3, window_frames=9,
                    n_steps=14, seed=27)
    cfg = hyat.config_from_workload(w, mask_heads=2)
    ha, hb, hc = hyat.Hyat(cfg), hyat.Hyat(cfg), hyat.Hyat(cfg)
    q0, k0, v0, m0 = wl.gen_stream_step(w, 13)
    qb, kb, vb = (torch.empty_like(t, device="cuda") for t in (q0, k0, v0))
    mbuf = torch.zeros(m0.size, dtype=torch.uint8, device="cuda")
    ob = [torch.empty_like(qb), torch.empty_like(qb)]
    for s in range(14):
        q, k, v, mask = wl.gen_stream_step(w, s)
        qd, kd, vd = _dev(q, k, v)
        oa = ha.stream_step(qd, kd, vd, mask=mask)
        md = torch.from_numpy(np.ascontiguousarray(mask)).cuda()
        o_b = hb.stream_step_dev(qd, kd, vd, mask=md)
        qb.copy_(qd); kb.copy_(kd); vb.copy_(vd)
        mflat = torch.from_numpy(np.ascontiguousarray(mask).reshape(-1)).cuda()
        mbuf[:mflat.numel()].copy_(mflat)
        o_c = hc.stream_step_dev(qb, kb, vb, mask=mbuf[:mflat.numel()], out=ob[s >= 9], graph=True)
        torch.cuda.synchronize()
        assert torch.equal(oa, o_b), f"device mask, step {s}"
        assert torch.equal(oa, o_c), f"graph replay, step {s}"
    for h in (ha, hb, hc):
        h.sync()
        h.close()


def test_stream_device_mask_without_diagonal_is_reported():
    w = wl.Workload("stream_badmask", "stream", 1, 2, 128, 200, 9, chunk_frames=3, window_frames=9,
                    n_steps=2, seed=4)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2))
    q, k, v, mask = wl.gen_stream_step(w, 0)
    mask = mask.copy()
    mask[1, 2, 2] = 0                      # head 1, query tile 2: its diagonal tile
    h.stream_step_dev(*_dev(q, k, v), mask=torch.from_numpy(mask).cuda())
    with pytest.raises(hyat.HyatError) as ei:
        h.sync()
    assert ei.value.status == hyat.ERR_INVALID_ARG
    # the handle stays usable
    q, k, v, mask = wl.gen_stream_step(w, 1)
    h.stream_step(*_dev(q, k, v), mask=mask)
    h.sync()
    h.close()


def _deal_max_loads(sorted_costs, G):
    """Busiest CTA's work under the two ways of dealing rows of G pairs (serpentine; least
    loaded first), for costs sorted largest first."""
    n = len(sorted_costs)
    ls, ll = np.zeros(G, np.int64), np.zeros(G, np.int64)
    for r, r0 in enumerate(range(0, n, G)):
        m = min(G, n - r0)
        row = sorted_costs[r0:r0 + m]
        ls[:m] += row[::-1] if r & 1 else row
        by_load = sorted(range(m), key=lambda c: (ll[c], c))
        for j, c in enumerate(by_load):
            ll[c] += row[j]
    return ls.max(), ll.max()


def test_stream_split_pairs_ordered_largest_first_on_device():
    """With more query tiles than SMs' worth of pairs, the streaming attention runs split pairs,
    and the prep kernel deals them out every step from that step's key-tile counts: each work
    item once, in rows of G = min(n, SMs) pairs (pair r * G + c on CTA c) that hold the counts
    largest first. Within a row the pairs follow whichever rule leaves the busiest CTA less work
    (key tiles + 1 per pair): a serpentine, or the larger counts to the CTAs holding less work so
    far. The outputs still match the oracle."""
    w = wl.Workload("stream_order", "stream", 1, 60, 128, 100, 33, chunk_frames=3, window_frames=9,
                    n_steps=7, seed=31)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=w.H))
    L, nwc = w.chunk_tokens, 3
    G0 = torch.cuda.get_device_properties(0).multi_processor_count
    kh, vh = [], []
    for s in range(7):
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        work, _, _, _ = h.stream_layout()
        pairs = h.pairs()
        n = len(work)
        assert len(pairs) == n and n > G0
        assert sorted(pairs[:, 0].tolist()) == list(range(n))
        assert (pairs[:, 1] == pairs[:, 0]).all() and (pairs[:, 2] == 0).all() and (pairs[:, 3] == 1).all()
        G = min(n, G0)
        counts = (work[:, 5] - work[:, 4]).astype(np.int64)
        want_rows = np.sort(counts)[::-1]
        serp_max, lpt_max = _deal_max_loads(want_rows + 1, G)
        lpt = lpt_max < serp_max
        load = np.zeros(G, np.int64)
        for r, r0 in enumerate(range(0, n, G)):
            m = min(G, n - r0)
            got = counts[pairs[r0:r0 + m, 0]]
            assert np.array_equal(np.sort(got)[::-1], want_rows[r0:r0 + m]), (s, r0)
            if lpt:
                dealt = got[sorted(range(m), key=lambda c: (load[c], c))]
            else:
                dealt = got[::-1] if r & 1 else got
            assert all(a >= b for a, b in zip(dealt, dealt[1:])), (s, r0, lpt)
            load[:m] += got + 1
        assert load.max() == min(serp_max, lpt_max)
        if s in (0, 6):
            heads = [0, 1, 59]
            got = f64(o.cpu())[:, heads]
            want = oracle.stream_step_attention(f64(q)[:, heads], np.concatenate(kh, axis=2)[:, heads],
                                                np.concatenate(vh, axis=2)[:, heads], s, L, nwc,
                                                mask[heads], n_sink_chunks=0)
            assert_parity("bf16", got, want, f"step {s}")
    h.sync()
    h.close()


def test_stream_split_pairs_beyond_the_device_order_limit():
    """A window of 28 chunks: a query tile may keep up to 37 x 28 = 1036 key tiles, more
    counts than the prep kernel's ordering table holds (1024), so the split pairs keep their
    list order; the steps still match the oracle."""
    w = wl.Workload("stream_long_window", "stream", 1, 2, 128, 1560, 6, chunk_frames=3, window_frames=84,
                    n_steps=2, seed=41)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=w.H))
    L, nwc = w.chunk_tokens, 28
    kh, vh = [], []
    for s in range(2):
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        pairs = h.pairs()
        n = 2 * 37
        assert len(pairs) == n and np.array_equal(pairs[:, 0], np.arange(n)) and (pairs[:, 3] == 1).all()
        rows = np.unique(np.concatenate([np.arange(0, L, 61), [L - 1]]))
        want = oracle.stream_step_attention(f64(q), np.concatenate(kh, axis=2), np.concatenate(vh, axis=2), s, L,
                                            nwc, mask, rows=rows, n_sink_chunks=0)
        assert_parity("bf16", f64(o.cpu())[:, :, rows], want, f"step {s}")
    h.sync()
    h.close()
