"""GPU parity of the pair schedule with one softmax warp per row (HYAT_FLAG_PAIR_ONE_WARP).

The default schedule (two softmax warps per row, fixed reference max, redo list) is what the
other GPU test files run; this one keeps the one-warp kernel covered on its own. That kernel
moves its reference max exactly (it is also the redo pass of the other schedules); the cases
below cover ragged tiles, every window geometry, both limits (all tiles kept = softmax
attention), block masks, split pairs (streaming), scores far above 0 and every score far
below 0 with no linear term.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_bf16_peaked, assert_parity, f64, sample_rows

pytestmark = pytest.mark.gpu
ONE = hyat.FLAG_PAIR_ONE_WARP


def _dev(*ts):
    return [t.cuda() for t in ts]


def _run(w, mask=None, mask_heads=1, qkv=None):
    h = hyat.Hyat(hyat.config_from_workload(w, flags=ONE, mask_heads=mask_heads), mask)
    q, k, v = wl.gen_qkv(w) if qkv is None else qkv
    o = h.forward(*_dev(q, k, v))
    h.sync()
    out = o.cpu()
    h.close()
    return out, (q, k, v)


def _window_ref(w, q, k, v, rows=None):
    return oracle.bidir_window_attention(f64(q), f64(k), f64(v), w.tokens_per_frame, w.n_frames,
                                         w.chunk_frames, w.halo_frames, rows=rows)


@pytest.mark.parametrize("T,F,C,h,H", [(7, 200, 2, 1, 2), (4, 64, 1, 0, 2), (3, 130, 3, 0, 1), (6, 1560, 3, 1, 1),
                                       (1, 100, 1, 0, 1), (3, 100, 1, 1, 1), (5, 300, 3, 1, 3)])
def test_one_warp_window_small(T, F, C, h, H):
    w = wl.Workload("one_warp", "window", 1, H, 128, F, T, C, h, seed=T * 31 + F)
    o, (q, k, v) = _run(w)
    assert_parity("bf16", f64(o), _window_ref(w, q, k, v), (T, F, C, h, H))


@pytest.mark.parametrize("kind", ["random", "zeros", "ones"])
def test_one_warp_blockmask(kind):
    T, F, H = 5, 230, 2
    nT = -(-T * F // 128)
    mask = {"random": wl.gen_tile_mask(H, nT, nT, seed=4),
            "zeros": np.zeros((H, nT, nT), np.uint8),
            "ones": np.ones((H, nT, nT), np.uint8)}[kind]
    w = wl.Workload("bm", "blockmask", 1, H, 128, F, T, seed=5)
    o, (q, k, v) = _run(w, mask=mask, mask_heads=H)
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), mask), kind)
    if kind == "ones":      # window = all tokens: exact softmax attention
        sdpa = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(f64(q)), torch.from_numpy(f64(k)), torch.from_numpy(f64(v))).numpy()
        assert_parity("bf16", f64(o), sdpa, "ones vs sdpa")


def test_one_warp_radial_and_lvsa_small():
    w = wl.Workload("radial_small", "radial", 1, 2, 128, 300, 9, seed=6)
    o, (q, k, v) = _run(w)
    assert_parity("bf16", f64(o), oracle.radial_attention(f64(q), f64(k), f64(v), 9, 300), "radial")
    w = wl.Workload("lvsa_small", "lvsa", 1, 2, 128, 300, 9, window_frames=3, anchor_stride=3, rotation=1, seed=37)
    mask = hyat.lvsa_mask(w.n_frames, w.tokens_per_frame, 3, 3, 1)[None]
    o, (q, k, v) = _run(w, mask=mask)
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), mask), "lvsa")


@pytest.mark.parametrize("sigma", [6.0, 20.0])
def test_one_warp_large_logits(sigma):
    """Scores far above the starting reference max: the kernel moves it and rescales exactly;
    twice on one handle, then a unit-scale call."""
    w = wl.Workload("large_logits", "window", 1, 2, 128, 300, 4, 2, 1, seed=17)
    q, k, v = wl.gen_qkv(w)
    q = (q.float() * sigma).to(torch.bfloat16)
    k = (k.float() * sigma).to(torch.bfloat16)
    h = hyat.Hyat(hyat.config_from_workload(w, flags=ONE))
    for _ in range(2):
        o = h.forward(*_dev(q, k, v))
        h.sync()
        assert_bf16_peaked(f64(o.cpu()), _window_ref(w, q, k, v), f64(v), sigma)
    q2, k2, v2 = wl.gen_qkv(w.with_(seed=18))
    o2 = h.forward(*_dev(q2, k2, v2))
    h.sync()
    assert_parity("bf16", f64(o2.cpu()), _window_ref(w, q2, k2, v2), "after redo")
    h.close()


def test_one_warp_far_negative_logits():
    T, F, H = 5, 230, 2
    nT = -(-T * F // 128)
    mask = np.ones((H, nT, nT), np.uint8)
    w = wl.Workload("bm_neg", "blockmask", 1, H, 128, F, T, seed=9)
    q, k, v = wl.gen_qkv(w)
    q = (q.float() + 3.0).to(torch.bfloat16)
    k = (k.float() - 3.0).to(torch.bfloat16)
    o, _ = _run(w, mask=mask, mask_heads=H, qkv=(q, k, v))
    assert np.all(np.isfinite(f64(o)))
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), mask), "far negative")


def test_one_warp_stream_split_pairs():
    """Streaming steps run split pairs (both slots on one query tile, merged in the epilogue)."""
    w = wl.Workload("stream_one_warp", "stream", 1, 2, 128, 200, 24, chunk_frames=3, window_frames=9,
                    n_steps=7, seed=13)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2, flags=ONE))
    L, nwc = w.chunk_tokens, 3
    kh, vh = [], []
    for s in range(7):
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        h.sync()
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        ref = oracle.stream_step_attention(f64(q), np.concatenate(kh, axis=2), np.concatenate(vh, axis=2), s, L,
                                           nwc, mask)
        assert_parity("bf16", f64(o.cpu()), ref, f"step {s}")
    h.close()


def test_one_warp_device_timeout_is_reported_and_recoverable():
    w = wl.Workload("timeout", "window", 1, 2, 128, 200, 4, 2, 1, seed=2)
    q, k, v = _dev(*wl.gen_qkv(w))
    h = hyat.Hyat(hyat.config_from_workload(w, flags=ONE | hyat.FLAG_TEST_DEVICE_TIMEOUT))
    h.forward(q, k, v)
    with pytest.raises(hyat.HyatError) as ei:
        h.sync()
    assert ei.value.status == hyat.ERR_DEVICE_TIMEOUT
    h.close()
    o, _ = _run(w, qkv=tuple(t.cpu() for t in (q, k, v)))
    assert_parity("bf16", f64(o), _window_ref(w, *(t.cpu() for t in (q, k, v))), "after a device timeout")


@pytest.mark.slow
def test_one_warp_full_wan13b_sampled():
    w = wl.WAN13B_BIDIR
    o, (q, k, v) = _run(w)
    C = w.chunk_tokens
    tiles = [(c0 + t, min(c0 + t + 128, c0 + C, w.N)) for c0 in range(0, w.N, C) for t in (0, 128 * 36)]
    rows = sample_rows(w.N, tiles, per_tile=2, seed=3)
    heads = [0, 5, 11]
    ref = _window_ref(w, q[:, heads], k[:, heads], v[:, heads], rows=rows)
    assert_parity("bf16", f64(o[:, heads][:, :, rows]), ref, "wan1.3b one warp per row")
