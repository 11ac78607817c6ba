"""GPU parity of libhyat against the fp64 oracle, through the C ABI.

Small geometries compare every output element; they span several 128-row
tiles with ragged tails (frames and chunks that are not multiples of 128).
The full-size workloads compare sampled rows (first and last rows of query
tiles, chunk edges, random rows) that the oracle evaluates one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_bf16_peaked, assert_parity, f64, sample_rows, errors

pytestmark = pytest.mark.gpu


def _dev(*ts):
    return [t.cuda() for t in ts]


def _bidir(w, mask=None, flags=0, mask_heads=1, qkv=None):
    cfg = hyat.config_from_workload(w, flags=flags, mask_heads=mask_heads)
    q, k, v = wl.gen_qkv(w) if qkv is None else qkv
    h = hyat.Hyat(cfg, mask)
    o = h.forward(*_dev(q, k, v))
    h.sync()
    out = o.cpu()
    h.close()
    return out, (q, k, v)


def _window_ref(w, q, k, v, rows=None):
    return oracle.bidir_window_attention(f64(q), f64(k), f64(v), w.tokens_per_frame, w.n_frames,
                                         w.chunk_frames, w.halo_frames, rows=rows)


# ------------------------------------------------------------------ small, full output
def test_tiny_f32_workload_full():
    w = wl.TINY_F32
    o, (q, k, v) = _bidir(w)
    assert_parity("f32", f64(o), _window_ref(w, q, k, v), w.name)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,F,C,h,d,H", [(7, 200, 2, 1, 128, 2), (5, 300, 3, 1, 64, 3), (4, 64, 1, 0, 128, 2),
                                         (3, 130, 3, 0, 128, 1), (6, 1560, 3, 1, 128, 1), (1, 100, 1, 0, 128, 1)])
def test_window_small(dtype, T, F, C, h, d, H):
    w = wl.Workload("small", "window", 1, H, d, F, T, C, h, dtype=dtype, seed=T * 1000 + F)
    o, (q, k, v) = _bidir(w)
    assert_parity(dtype, f64(o), _window_ref(w, q, k, v), (T, F, C, h, d, H))


@pytest.mark.parametrize("sigma", [6.0, 20.0])
def test_window_large_logits(sigma):
    """Scores far above the reference max (sigma 20: |s| * log2(e) / sqrt(d) reaches ~250):
    the kernel must move its reference max and rescale the accumulator exactly.

    These inputs lie outside the five workloads (unit or U[0.5, 2] per-head scales): their
    softmax is nearly one-hot, so a row's output is close to one value row and the fixed
    2e-2 bound stops following from the bf16 arithmetic. The bound checked is the derived
    peaked-input bound of assert_bf16_peaked."""
    w = wl.Workload("large_logits", "window", 1, 2, 128, 300, 4, 2, 1, seed=17)
    q, k, v = wl.gen_qkv(w)
    q = (q.float() * sigma).to(torch.bfloat16)
    k = (k.float() * sigma).to(torch.bfloat16)
    o, _ = _bidir(w, qkv=(q, k, v))
    assert_bf16_peaked(f64(o), _window_ref(w, q, k, v), f64(v), sigma)


@pytest.mark.parametrize("flags", [0, hyat.FLAG_SINGLE_TILE], ids=["pair", "single"])
def test_all_kept_far_negative_logits(flags):
    """Every tile kept (no linear term) and every logit near -100: relative to the starting
    reference m = 0 each exponential flushes to zero, so the kernels must move m down to the
    row's scale instead of dividing by a zero row sum."""
    T, F, H = 5, 230, 2
    nT = -(-T * F // 128)
    mask = np.ones((H, nT, nT), np.uint8)
    w = wl.Workload("bm_neg", "blockmask", 1, H, 128, F, T, seed=9)
    q, k, v = wl.gen_qkv(w)
    q = (q.float() + 3.0).to(torch.bfloat16)      # q . k ~ -9 d: logits ~ -102 +- 4
    k = (k.float() - 3.0).to(torch.bfloat16)
    o, _ = _bidir(w, mask=mask, mask_heads=H, flags=flags, qkv=(q, k, v))
    assert np.all(np.isfinite(f64(o)))
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), mask), "far negative")


def test_window_batch2_per_head_std():
    w = wl.Workload("small_b2", "window", 2, 3, 128, 250, 6, 3, 1, per_head_std=True, seed=11)
    o, (q, k, v) = _bidir(w)
    assert_parity("bf16", f64(o), _window_ref(w, q, k, v), w.name)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("kind", ["random", "zeros", "ones"])
def test_blockmask_small(dtype, kind):
    T, F, H = 5, 230, 2
    N = T * F
    nT = -(-N // 128)
    mask = {"random": wl.gen_tile_mask(H, nT, nT, seed=4),
            "zeros": np.zeros((H, nT, nT), np.uint8),
            "ones": np.ones((H, nT, nT), np.uint8)}[kind]
    w = wl.Workload("bm", "blockmask", 1, H, 128, F, T, dtype=dtype, seed=5)
    o, (q, k, v) = _bidir(w, mask=mask, mask_heads=H)
    ref = oracle.blockmask_attention(f64(q), f64(k), f64(v), mask)
    assert_parity(dtype, f64(o), ref, kind)
    if kind == "ones":      # window = all tokens: exact softmax attention
        sdpa = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(f64(q)), torch.from_numpy(f64(k)), torch.from_numpy(f64(v))).numpy()
        assert_parity(dtype, f64(o), sdpa, "ones vs sdpa")
    if kind == "zeros":     # empty window: pure linear attention
        pq, pk = oracle.phi_elu1(f64(q)), oracle.phi_elu1(f64(k))
        S = np.einsum("bhna,bhnc->bhac", pk, f64(v))
        lin = np.einsum("bhna,bhac->bhnc", pq, S) / np.einsum("bhna,bha->bhn", pq, pk.sum(2))[..., None]
        assert_parity(dtype, f64(o), lin, "zeros vs linear")


@pytest.mark.parametrize("T,F", [(9, 300), (6, 200)])
def test_radial_small(T, F):
    w = wl.Workload("radial_small", "radial", 1, 2, 128, F, T, seed=6)
    o, (q, k, v) = _bidir(w)
    ref = oracle.radial_attention(f64(q), f64(k), f64(v), T, F)
    assert_parity("bf16", f64(o), ref, w.name)


# ------------------------------------------------------------------ streaming
STATE_HEADER_BYTES = 48   # magic, version, step, BH, d, L, nwc, dtype, folded step, 3 reserved


def _state_from_blob(blob, BH, d):
    hdr = np.frombuffer(blob[:STATE_HEADER_BYTES], np.int32)
    E = d * d + d
    s = np.frombuffer(blob[STATE_HEADER_BYTES:STATE_HEADER_BYTES + 4 * BH * E], np.float32).reshape(BH, E)
    return int(hdr[2]), s[:, :d * d].reshape(BH, d, d), s[:, d * d:]


def _run_stream(w, steps, check_steps=None, rows=None, mask_heads=None, handle=None, start=0, hist=None):
    mh = w.H if mask_heads is None else mask_heads
    cfg = hyat.config_from_workload(w, mask_heads=mh)
    h = hyat.Hyat(cfg) if handle is None else handle
    L = w.chunk_tokens
    nwc = w.window_frames // w.chunk_frames
    kh, vh = hist if hist is not None else ([], [])
    outs = {}
    for s in range(start, start + steps):
        q, k, v, mask = wl.gen_stream_step(w, s)
        mask = mask[:mh]
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        kh.append(k.float().numpy())                    # exact copies of the bf16 values
        vh.append(v.float().numpy())
        if check_steps is None or s in check_steps:
            h.sync()
            k_all, v_all = np.concatenate(kh, axis=2), np.concatenate(vh, axis=2)
            ref = oracle.stream_step_attention(f64(q), k_all, v_all, s, L, nwc, mask, rows=rows)
            got = f64(o) if rows is None else f64(o)[:, :, rows]
            outs[s] = (got, ref)
    h.sync()
    return h, outs, (kh, vh)


def test_stream_small_steps_and_state():
    w = wl.Workload("stream_small", "stream", 1, 2, 128, 200, 24, chunk_frames=3, window_frames=9,
                    n_steps=8, seed=3)
    h, outs, (kh, vh) = _run_stream(w, 8)
    for s, (got, ref) in outs.items():
        assert_parity("bf16", got, ref, f"step {s}")
    step, S, z = _state_from_blob(h.get_state(), 2, 128)
    assert step == 8
    k_all, v_all = np.concatenate(kh, axis=2), np.concatenate(vh, axis=2)
    # after step 7 the state holds phi(k) v^T of every chunk evicted up to step 7
    S_ref, z_ref = oracle.stream_evicted_state(k_all, v_all, 7, w.chunk_tokens, 3)
    # The tensor-core fold takes phi(k) as a bf16 operand: each product phi(k)_a v_b carries a
    # relative rounding error <= 2^-8 (v is exact), so |S - S*|_ab <= 2^-8 sum_j |phi(k_j)_a v_jb|;
    # fp32 accumulation adds at most 1e-5 of the largest entry.
    n_ev = (7 - 3 + 1) * w.chunk_tokens
    pk = oracle.phi_elu1(k_all[:, :, :n_ev])
    bound_S = 2.0 ** -8 * np.einsum("bhna,bhnc->bhac", pk, np.abs(v_all[:, :, :n_ev]))
    bound_z = 2.0 ** -8 * pk.sum(axis=2)
    err_S = np.abs(S.reshape(1, 2, 128, 128) - S_ref)
    err_z = np.abs(z.reshape(1, 2, 128) - z_ref)
    assert np.all(err_S <= bound_S + 1e-5 * np.abs(S_ref).max()), float((err_S / bound_S).max())
    assert np.all(err_z <= bound_z + 1e-5 * np.abs(z_ref).max()), float((err_z / bound_z).max())
    # and the error is the random rounding kind: its rms is far below the worst case
    assert np.sqrt((err_S ** 2).mean()) < 0.1 * np.sqrt((bound_S ** 2).mean())
    h.close()


def test_stream_shared_mask_and_f32():
    w = wl.Workload("stream_f32", "stream", 1, 3, 64, 130, 15, chunk_frames=2, window_frames=4,
                    n_steps=5, dtype="f32", seed=8)
    h, outs, _ = _run_stream(w, 5, mask_heads=1)
    for s, (got, ref) in outs.items():
        assert_parity("f32", got, ref, f"step {s}")
    h.close()


def test_stream_checkpoint_resume_bit_identical():
    w = wl.Workload("stream_ckpt", "stream", 1, 2, 128, 200, 30, chunk_frames=3, window_frames=9,
                    n_steps=10, seed=21)
    cfg = hyat.config_from_workload(w, mask_heads=2)
    h1 = hyat.Hyat(cfg)
    ref_outs = []
    for s in range(10):
        q, k, v, mask = wl.gen_stream_step(w, s)
        ref_outs.append(h1.stream_step(*_dev(q, k, v), mask=mask).cpu())
        if s == 5:
            h1.sync()
            blob = h1.get_state()
    h1.close()
    h2 = hyat.Hyat(cfg)
    h2.set_state(blob)
    for s in range(6, 10):
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h2.stream_step(*_dev(q, k, v), mask=mask).cpu()
        assert torch.equal(o, ref_outs[s]), s
    h2.close()


def test_stream_denoise_calls_then_final_call():
    """Several denoising calls per chunk, then the final call: every call attends to the
    committed window, the folded state and its own K, V; only the final K, V stay."""
    w = wl.Workload("stream_denoise", "stream", 1, 2, 128, 200, 24, chunk_frames=3, window_frames=9,
                    n_steps=6, seed=5)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2))
    L, nwc = w.chunk_tokens, w.window_frames // w.chunk_frames
    kh, vh = [], []
    for s in range(6):
        for call in range(2):
            q, k, v, mask = wl.gen_stream_step(w, s, call=call)
            o = h.stream_denoise(*_dev(q, k, v), mask=mask)
            h.sync()
            k_all = np.concatenate(kh + [k.float().numpy()], axis=2)
            v_all = np.concatenate(vh + [v.float().numpy()], axis=2)
            ref = oracle.stream_step_attention(f64(q), k_all, v_all, s, L, nwc, mask)
            assert_parity("bf16", f64(o), ref, f"chunk {s} denoising call {call}")
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        h.sync()
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        ref = oracle.stream_step_attention(f64(q), np.concatenate(kh, axis=2), np.concatenate(vh, axis=2),
                                           s, L, nwc, mask)
        assert_parity("bf16", f64(o), ref, f"chunk {s} final call")
    step, S, z = _state_from_blob(h.get_state(), 2, 128)
    assert step == 6
    # the folded state holds the final K, V of chunks 0..2 only; the bound is the one of
    # test_stream_small_steps_and_state (bf16 phi(k) operand, fp32 accumulation)
    k_all, v_all = np.concatenate(kh, axis=2), np.concatenate(vh, axis=2)
    S_ref, z_ref = oracle.stream_evicted_state(k_all, v_all, 5, L, 3)
    n_ev = 3 * L
    pk = oracle.phi_elu1(k_all[:, :, :n_ev])
    bound_S = 2.0 ** -8 * np.einsum("bhna,bhnc->bhac", pk, np.abs(v_all[:, :, :n_ev]))
    bound_z = 2.0 ** -8 * pk.sum(axis=2)
    assert np.all(np.abs(S.reshape(1, 2, 128, 128) - S_ref) <= bound_S + 1e-5 * np.abs(S_ref).max())
    assert np.all(np.abs(z.reshape(1, 2, 128) - z_ref) <= bound_z + 1e-5 * np.abs(z_ref).max())
    h.close()


def test_stream_checkpoint_between_denoising_calls_bit_identical():
    """A state saved after a chunk's denoising call (its fold done) resumes exactly."""
    w = wl.Workload("stream_ckpt_mid", "stream", 1, 2, 128, 200, 24, chunk_frames=3, window_frames=9,
                    n_steps=6, seed=9)
    cfg = hyat.config_from_workload(w, mask_heads=2)
    h1 = hyat.Hyat(cfg)
    for s in range(4):
        h1.stream_step(*_dev(*wl.gen_stream_step(w, s)[:3]), mask=wl.gen_stream_step(w, s)[3])
    q, k, v, mask = wl.gen_stream_step(w, 4, call=0)
    h1.stream_denoise(*_dev(q, k, v), mask=mask)        # chunk 4: folds chunk 1
    h1.sync()
    blob = h1.get_state()
    seq = [("denoise", wl.gen_stream_step(w, 4, call=1)), ("step", wl.gen_stream_step(w, 4)),
           ("step", wl.gen_stream_step(w, 5))]
    ref = []
    for kind, (q, k, v, mask) in seq:
        fn = h1.stream_denoise if kind == "denoise" else h1.stream_step
        ref.append(fn(*_dev(q, k, v), mask=mask).cpu())
    h1.close()
    h2 = hyat.Hyat(cfg)
    h2.set_state(blob)
    for (kind, (q, k, v, mask)), r in zip(seq, ref):
        fn = h2.stream_denoise if kind == "denoise" else h2.stream_step
        assert torch.equal(fn(*_dev(q, k, v), mask=mask).cpu(), r), kind
    h2.close()


def test_stream_with_attention_sink():
    """The first chunk stays in the window for good; the chunks between it and the rolling
    window are folded into the state; denoising calls see the sink too."""
    w = wl.Workload("stream_sink", "stream", 1, 2, 128, 200, 27, chunk_frames=3, window_frames=6,
                    n_steps=8, seed=41, sink_frames=3)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2))
    L, nwc, ns = w.chunk_tokens, 2, 1
    kh, vh = [], []
    for s in range(8):
        if s in (2, 5):
            q, k, v, mask = wl.gen_stream_step(w, s, call=0)
            o = h.stream_denoise(*_dev(q, k, v), mask=mask)
            h.sync()
            ref = oracle.stream_step_attention(f64(q), np.concatenate(kh + [k.float().numpy()], axis=2),
                                               np.concatenate(vh + [v.float().numpy()], axis=2), s, L, nwc,
                                               mask, n_sink_chunks=ns)
            assert_parity("bf16", f64(o), ref, f"denoising call, chunk {s}")
        q, k, v, mask = wl.gen_stream_step(w, s)
        assert mask.shape[2] == (-(-L // 128)) * len(oracle.stream_visible_chunks(s, nwc, ns))
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        h.sync()
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        ref = oracle.stream_step_attention(f64(q), np.concatenate(kh, axis=2), np.concatenate(vh, axis=2),
                                           s, L, nwc, mask, n_sink_chunks=ns)
        assert_parity("bf16", f64(o), ref, f"chunk {s}")
    step, S, z = _state_from_blob(h.get_state(), 2, 128)
    assert step == 8
    k_all, v_all = np.concatenate(kh, axis=2), np.concatenate(vh, axis=2)
    S_ref, z_ref = oracle.stream_evicted_state(k_all, v_all, 7, L, nwc, n_sink_chunks=ns)   # chunks 1..5
    pk = oracle.phi_elu1(k_all[:, :, L:6 * L])
    bound_S = 2.0 ** -8 * np.einsum("bhna,bhnc->bhac", pk, np.abs(v_all[:, :, L:6 * L]))
    assert np.all(np.abs(S.reshape(1, 2, 128, 128) - S_ref) <= bound_S + 1e-5 * np.abs(S_ref).max())
    assert np.all(np.abs(z.reshape(1, 2, 128) - z_ref) <= 2.0 ** -8 * pk.sum(axis=2) + 1e-5 * np.abs(z_ref).max())
    h.close()


# ------------------------------------------------------------------ feature maps
@pytest.mark.parametrize("phi", ["relu", "exp"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_feature_map_window(phi, dtype):
    w = wl.Workload("phi_window", "window", 1, 2, 128, 300, 6, 2, 1, dtype=dtype, seed=23, phi=phi)
    o, (q, k, v) = _bidir(w)
    ref = oracle.bidir_window_attention(f64(q), f64(k), f64(v), w.tokens_per_frame, w.n_frames,
                                        w.chunk_frames, w.halo_frames, phi=phi)
    assert_parity(dtype, f64(o), ref, (phi, dtype))


@pytest.mark.parametrize("phi", ["relu", "exp"])
def test_feature_map_blockmask(phi):
    """Diagonal tile mask with query tile 0 left empty (pure linear attention for its rows)."""
    T, F, H = 4, 230, 2
    nT = -(-T * F // 128)
    mask = np.zeros((H, nT, nT), np.uint8)
    mask[:, np.arange(nT), np.arange(nT)] = 1
    mask[:, 0, :] = 0
    w = wl.Workload("phi_bm", "blockmask", 1, H, 128, F, T, seed=29, phi=phi)
    o, (q, k, v) = _bidir(w, mask=mask, mask_heads=H)
    ref = oracle.blockmask_attention(f64(q), f64(k), f64(v), mask, phi=phi)
    assert_parity("bf16", f64(o), ref, phi)


@pytest.mark.parametrize("phi", ["relu", "exp"])
def test_feature_map_stream(phi):
    w = wl.Workload("phi_stream", "stream", 1, 2, 128, 200, 18, chunk_frames=3, window_frames=9,
                    n_steps=6, seed=31, phi=phi)
    h = hyat.Hyat(hyat.config_from_workload(w, mask_heads=2))
    L, nwc = w.chunk_tokens, w.window_frames // w.chunk_frames
    kh, vh = [], []
    for s in range(6):
        q, k, v, mask = wl.gen_stream_step(w, s)
        o = h.stream_step(*_dev(q, k, v), mask=mask)
        h.sync()
        kh.append(k.float().numpy())
        vh.append(v.float().numpy())
        ref = oracle.stream_step_attention(f64(q), np.concatenate(kh, axis=2), np.concatenate(vh, axis=2),
                                           s, L, nwc, mask, phi=phi)
        assert_parity("bf16", f64(o), ref, (phi, s))
    h.close()


# ------------------------------------------------------------------ errors
def test_invalid_calls_return_errors_and_handle_stays_usable():
    w = wl.Workload("err", "stream", 1, 2, 64, 100, 9, chunk_frames=3, window_frames=6, n_steps=2, seed=1)
    cfg = hyat.config_from_workload(w, mask_heads=1)
    h = hyat.Hyat(cfg)
    q, k, v, mask = wl.gen_stream_step(w, 0)
    bad = mask[:1].copy()
    bad[0, 0, 0] = 0                                    # diagonal tile dropped
    with pytest.raises(hyat.HyatError) as ei:
        h.stream_step(*_dev(q, k, v), mask=bad)
    assert ei.value.status == hyat.ERR_INVALID_ARG
    qd, kd, vd = _dev(q, k, v)
    st = hyat.lib.hyat_fwd_stream_step(h.handle, qd.data_ptr() + 2, kd.data_ptr(), vd.data_ptr(),
                                       qd.data_ptr(), None, None)
    assert st == hyat.ERR_INVALID_ARG                   # misaligned pointer
    st = hyat.lib.hyat_fwd_bidir(h.handle, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), qd.data_ptr(), None)
    assert st == hyat.ERR_INVALID_ARG                   # bidirectional call on a stream handle
    o = h.stream_step(qd, kd, vd, mask=mask[:1])        # still works at step 0
    h.sync()
    ref = oracle.stream_step_attention(f64(q), f64(k), f64(v), 0, 300, 2, mask[:1])
    assert_parity("bf16", f64(o), ref, "after errors")
    h.close()


def test_device_timeout_is_reported_and_recoverable():
    """The timeout path without faulting the GPU: a wait on a signal that never comes gives up
    after 20 ms, the call reports HYAT_ERR_DEVICE_TIMEOUT, and later calls work."""
    w = wl.Workload("timeout", "window", 1, 2, 128, 200, 4, 2, 1, seed=2)
    q, k, v = _dev(*wl.gen_qkv(w))
    h = hyat.Hyat(hyat.config_from_workload(w, flags=hyat.FLAG_TEST_DEVICE_TIMEOUT))
    h.forward(q, k, v)
    with pytest.raises(hyat.HyatError) as ei:
        h.sync()
    assert ei.value.status == hyat.ERR_DEVICE_TIMEOUT
    h.sync()                                            # the status word was cleared
    h.close()
    h2 = hyat.Hyat(hyat.config_from_workload(w))
    o = h2.forward(q, k, v)
    h2.sync()
    ref = _window_ref(w, *(t.cpu() for t in (q, k, v)))
    assert_parity("bf16", f64(o.cpu()), ref, "after a device timeout")
    h2.close()


# ------------------------------------------------------------------ full-size workloads
def _lvsa_masks(w):
    """(library mask for the handle, oracle mask for the reference); equal bit for bit."""
    lib_mask = hyat.lvsa_mask(w.n_frames, w.tokens_per_frame, w.window_frames, w.anchor_stride, w.rotation)
    ref_mask = oracle.lvsa_tile_mask(w.n_frames, w.tokens_per_frame, w.window_frames, w.anchor_stride, w.rotation)
    assert np.array_equal(lib_mask, ref_mask)
    return lib_mask[None], ref_mask[None]


def _bidir_sampled(w, heads, per_tile=2, seed=0, flags=0):
    lib_mask = ref_mask = None
    if w.mode == "lvsa":
        lib_mask, ref_mask = _lvsa_masks(w)
    o, (q, k, v) = _bidir(w, mask=lib_mask, flags=flags)
    N = w.N
    if w.mode == "window":
        C = w.chunk_tokens
        tiles = [(c0 + t, min(c0 + t + 128, c0 + C, N)) for c0 in range(0, N, C) for t in (0, 128 * 36)]
    else:
        tiles = [(t, min(t + 128, N)) for t in range(0, N, 128 * 97)] + [(N - 96, N)]
    rows = sample_rows(N, tiles, per_tile=per_tile, seed=seed)
    qs, ks, vs = q[:, heads], k[:, heads], v[:, heads]
    if w.mode == "window":
        ref = _window_ref(w, qs, ks, vs, rows=rows)
    elif w.mode == "lvsa":
        ref = oracle.blockmask_attention(f64(qs), f64(ks), f64(vs), ref_mask, rows=rows)
    else:
        ref = oracle.radial_attention(f64(qs), f64(ks), f64(vs), w.n_frames, w.tokens_per_frame, rows=rows)
    got = f64(o[:, heads][:, :, rows])
    return got, ref


@pytest.mark.slow
def test_full_wan13b_bidir_sampled():
    got, ref = _bidir_sampled(wl.WAN13B_BIDIR, heads=[0, 5, 11])
    assert_parity("bf16", got, ref, "wan1.3b")


@pytest.mark.slow
def test_full_wan13b_bidir_whole_head():
    """One head of the full Wan-1.3B layer, all 32760 rows, element by element against the
    fp64 oracle (rows in blocks of one chunk)."""
    w = wl.WAN13B_BIDIR
    o, (q, k, v) = _bidir(w)
    head = [7]
    qs, ks, vs = q[:, head], k[:, head], v[:, head]
    got = f64(o[:, head])
    C = w.chunk_tokens
    ref = np.concatenate([_window_ref(w, qs, ks, vs, rows=np.arange(c0, min(c0 + C, w.N)))
                          for c0 in range(0, w.N, C)], axis=2)
    assert ref.shape == got.shape == (1, 1, w.N, w.d)
    assert_parity("bf16", got, ref, "wan1.3b head 7, every row")


@pytest.mark.slow
def test_full_wan14b_bidir_sampled():
    got, ref = _bidir_sampled(wl.WAN14B_BIDIR, heads=[0, 17, 39], per_tile=2)
    assert_parity("bf16", got, ref, "wan14b")


@pytest.mark.slow
def test_full_radial_sampled():
    got, ref = _bidir_sampled(wl.RADIAL_84F, heads=[0, 11], per_tile=2)
    assert_parity("bf16", got, ref, "radial")


@pytest.mark.slow
def test_full_lvsa_sampled():
    got, ref = _bidir_sampled(wl.LVSA_126F, heads=[0, 7], per_tile=2)
    assert_parity("bf16", got, ref, "lvsa")


@pytest.mark.parametrize("wf,stride,rot", [(3, 3, 1), (5, 4, 0), (1, 2, 3), (3, 0, 0)])
def test_lvsa_small(wf, stride, rot):
    w = wl.Workload("lvsa_small", "lvsa", 1, 2, 128, 300, 9, window_frames=wf, anchor_stride=stride,
                    rotation=rot, seed=37)
    lib_mask, ref_mask = _lvsa_masks(w)
    o, (q, k, v) = _bidir(w, mask=lib_mask)
    ref = oracle.blockmask_attention(f64(q), f64(k), f64(v), ref_mask)
    assert_parity("bf16", f64(o), ref, (wf, stride, rot))


@pytest.mark.slow
def test_full_stream_sampled():
    w = wl.STREAM_HF
    rows = sample_rows(w.chunk_tokens, [(0, 128), (128 * 36, w.chunk_tokens)], per_tile=4,
                       extra=[1000, 2345, 4000])
    h, outs, _ = _run_stream(w, w.n_steps, check_steps={0, 1, 2, 3, 4, 17, 39}, rows=rows)
    for s, (got, ref) in outs.items():
        assert_parity("bf16", got, ref, f"step {s}")
    h.close()


# ------------------------------------------------------------------ single-tile schedule
# HYAT_FLAG_SINGLE_TILE: one query tile per CTA, two softmax warpgroups on alternate key
# tiles, three S buffers, fixed reference max with a redo list for tiles out of range.
SINGLE = hyat.FLAG_SINGLE_TILE


@pytest.mark.parametrize("T,F,C,h,H", [(7, 200, 2, 1, 2), (4, 64, 1, 0, 2), (3, 130, 3, 0, 1), (6, 1560, 3, 1, 1),
                                       (1, 100, 1, 0, 1), (3, 100, 1, 1, 1), (5, 100, 2, 1, 1), (8, 100, 4, 1, 1)])
def test_single_tile_window_small(T, F, C, h, H):
    """Query tiles of 1 to 61 key tiles: every count of S-buffer fills mod 3 and both warpgroups
    with no tile at all (a query tile with one key tile leaves warpgroup 1 only the linear term)."""
    w = wl.Workload("single", "window", 1, H, 128, F, T, C, h, seed=T * 100 + F)
    o, (q, k, v) = _bidir(w, flags=SINGLE)
    assert_parity("bf16", f64(o), _window_ref(w, q, k, v), (T, F, C, h, H))


@pytest.mark.parametrize("sigma", [6.0, 20.0])
def test_single_tile_large_logits_take_the_redo_list(sigma):
    """Row sums beyond 2^100 under the fixed reference max: those query tiles are recomputed by
    the pair kernel, which moves its reference max; the result must be as exact as there.
    Like test_window_large_logits, these nearly one-hot inputs lie outside the five workloads
    and are held to the derived peaked-input bound."""
    w = wl.Workload("large_logits", "window", 1, 2, 128, 300, 4, 2, 1, seed=17)
    q, k, v = wl.gen_qkv(w)
    q = (q.float() * sigma).to(torch.bfloat16)
    k = (k.float() * sigma).to(torch.bfloat16)
    h = hyat.Hyat(hyat.config_from_workload(w, flags=SINGLE))
    for rep in range(2):            # the second call finds the redo list emptied by the first
        o = h.forward(*_dev(q, k, v))
        h.sync()
        assert_bf16_peaked(f64(o.cpu()), _window_ref(w, q, k, v), f64(v), sigma)
    # and a unit-scale call on the same handle after that is exact too
    q2, k2, v2 = wl.gen_qkv(w.with_(seed=18))
    o2 = h.forward(*_dev(q2, k2, v2))
    h.sync()
    assert_parity("bf16", f64(o2.cpu()), _window_ref(w, q2, k2, v2), "after redo")
    h.close()


@pytest.mark.parametrize("kind", ["random", "zeros", "ones"])
def test_single_tile_blockmask(kind):
    T, F, H = 5, 230, 2
    nT = -(-T * F // 128)
    mask = {"random": wl.gen_tile_mask(H, nT, nT, seed=4),
            "zeros": np.zeros((H, nT, nT), np.uint8),
            "ones": np.ones((H, nT, nT), np.uint8)}[kind]
    w = wl.Workload("bm", "blockmask", 1, H, 128, F, T, seed=5)
    o, (q, k, v) = _bidir(w, mask=mask, mask_heads=H, flags=SINGLE)
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), mask), kind)


@pytest.mark.parametrize("phi", ["relu", "exp"])
def test_single_tile_feature_maps(phi):
    w = wl.Workload("single_phi", "window", 1, 2, 128, 200, 7, 2, 1, seed=8, phi=phi)
    o, (q, k, v) = _bidir(w, flags=SINGLE)
    ref = oracle.bidir_window_attention(f64(q), f64(k), f64(v), 200, 7, 2, 1, phi=phi)
    assert_parity("bf16", f64(o), ref, phi)


def test_single_tile_radial_and_lvsa_small():
    w = wl.Workload("radial_small", "radial", 1, 2, 128, 300, 9, seed=6)
    o, (q, k, v) = _bidir(w, flags=SINGLE)
    assert_parity("bf16", f64(o), oracle.radial_attention(f64(q), f64(k), f64(v), 9, 300), "radial")
    w = wl.Workload("lvsa_small", "lvsa", 1, 2, 128, 300, 9, window_frames=3, anchor_stride=3, rotation=1, seed=37)
    lib_mask, ref_mask = _lvsa_masks(w)
    o, (q, k, v) = _bidir(w, mask=lib_mask, flags=SINGLE)
    assert_parity("bf16", f64(o), oracle.blockmask_attention(f64(q), f64(k), f64(v), ref_mask), "lvsa")


def test_single_tile_device_timeout_is_reported_and_recoverable():
    w = wl.Workload("timeout", "window", 1, 2, 128, 200, 4, 2, 1, seed=2)
    q, k, v = _dev(*wl.gen_qkv(w))
    h = hyat.Hyat(hyat.config_from_workload(w, flags=SINGLE | hyat.FLAG_TEST_DEVICE_TIMEOUT))
    h.forward(q, k, v)
    with pytest.raises(hyat.HyatError) as ei:
        h.sync()
    assert ei.value.status == hyat.ERR_DEVICE_TIMEOUT
    h.close()
    o, _ = _bidir(w, flags=SINGLE, qkv=tuple(t.cpu() for t in (q, k, v)))
    assert_parity("bf16", f64(o), _window_ref(w, *(t.cpu() for t in (q, k, v))), "after a device timeout")


@pytest.mark.slow
def test_single_tile_full_wan13b_sampled():
    got, ref = _bidir_sampled(wl.WAN13B_BIDIR, heads=[0, 5, 11], flags=SINGLE)
    assert_parity("bf16", got, ref, "wan1.3b single tile")


# ------------------------------------------------------------------ capped temporal RoPE
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,t_dims,F,f0,ref,cap", [(128, 44, 100, 5, 3, 4), (64, 64, 37, 0, 0, 21),
                                                   (128, 128, 1560, 40, 31, 21), (128, 0, 50, 2, 2, 1),
                                                   (128, 2, 7, 9, 0, 3), (64, 18, 1, 3, 3, 40)])
def test_rope_temporal(dtype, d, t_dims, F, f0, ref, cap):
    """Against the oracle on 700 tokens (5.5 blocks of 128): the band within one bf16 rounding
    of the exact rotation (fp32: within 1e-6 of the row scale), the rest bit for bit; in place
    gives the same."""
    rng = np.random.default_rng(d + t_dims + F)
    x = torch.from_numpy(rng.standard_normal((2, 3, 700, d), dtype=np.float32))
    x = x.to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    xd = x.cuda()
    y = hyat.rope_temporal(xd, F, f0, ref, cap, t_dims, base=10000.0)
    y2 = hyat.rope_temporal(xd.clone(), F, f0, ref, cap, t_dims, base=10000.0)
    xi = xd.clone()
    hyat.rope_temporal(xi, F, f0, ref, cap, t_dims, base=10000.0, out=xi)
    torch.cuda.synchronize()
    want = oracle.rope_temporal(f64(x), F, f0, ref, cap, t_dims, base=10000.0)
    got = f64(y.cpu())
    scale = np.abs(f64(x)).max()
    bound = (2.0 ** -8 * np.abs(want) + 1e-6 * scale) if dtype == "bf16" else 1e-6 * scale
    assert np.all(np.abs(got - want) <= bound), float(np.abs(got - want).max())
    np.testing.assert_array_equal(got[..., t_dims:], f64(x)[..., t_dims:])
    assert torch.equal(y, y2) and torch.equal(y, xi)
