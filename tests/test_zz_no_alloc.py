"""The allocation-free forward (hyat_fwd_bidir_noalloc), called through the C ABI.

It serves callers that cannot allocate device memory where they run the layer (code inside a
caching allocator's critical section, plug-in hosts whose device memory belongs to another
runtime, real-time loops where cudaMalloc / cudaFree would synchronise the device); its
scratch is a static device array shared by every call. It runs the same kernels in the same
order as the handle-based hyat_fwd_bidir, so each of two calls in a row (different inputs, so
stale scratch would show) must equal the handle's output bit for bit; sampled rows are also
held to the fp64 oracle. This file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_parity, f64, sample_rows

pytestmark = pytest.mark.gpu


def _noalloc(cfg, q, k, v):
    o = torch.empty_like(q)
    st = hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         o.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == hyat.OK, hyat.lib.hyat_status_string(st)
    return o


def _oracle_rows(w, q, k, v, rows):
    qs, ks, vs = f64(q[:, :1]), f64(k[:, :1]), f64(v[:, :1])
    if w.mode == "window":
        return oracle.bidir_window_attention(qs, ks, vs, w.tokens_per_frame, w.n_frames, w.chunk_frames,
                                             w.halo_frames, rows=rows)
    return oracle.radial_attention(qs, ks, vs, w.n_frames, w.tokens_per_frame, rows=rows)


@pytest.mark.parametrize("w", [wl.WAN13B_BIDIR, wl.TINY_F32,
                               wl.Workload("radial_small", "radial", 1, 2, 128, 300, 9, seed=6)],
                         ids=lambda w: w.name)
def test_noalloc_matches_handle_forward_twice(w):
    cfg = hyat.config_from_workload(w)
    h = hyat.Hyat(cfg)
    for seed in (w.seed + 101, w.seed + 202):
        qh, kh, vh = wl.gen_qkv(w, seed=seed)
        q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
        ref = h.forward(q, k, v)
        got = _noalloc(cfg, q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"{w.name} seed {seed}: differs from the handle forward"
        rows = sample_rows(w.N, [(0, min(w.N, 128)), (max(0, w.N - 128), w.N)], per_tile=4, seed=seed)
        assert_parity(w.dtype, f64(got[:, :1, rows].cpu()), _oracle_rows(w, qh, kh, vh, rows),
                      f"{w.name} seed {seed} vs oracle")
    h.close()


def test_noalloc_rejects_configs_beyond_its_scratch():
    cfg = hyat.config_from_workload(wl.WAN14B_BIDIR)       # needs ~55 MiB of linear states
    st = hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), 16, 16, 16, 16, None)
    assert st == hyat.ERR_UNSUPPORTED
    cfg = hyat.config_from_workload(wl.STREAM_HF)
    assert hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), 16, 16, 16, 16, None) == hyat.ERR_INVALID_ARG


def test_noalloc_refuses_stream_capture():
    """Its layout tables are copied from host memory that the call frees on return, so a
    captured call could not be replayed: it returns HYAT_ERR_UNSUPPORTED while capturing."""
    w = wl.Workload("small", "window", 1, 2, 128, 200, 4, 2, 1, seed=3)
    cfg = hyat.config_from_workload(w)
    q, k, v = (t.cuda() for t in wl.gen_qkv(w))
    o = torch.empty_like(q)
    _noalloc(cfg, q, k, v)          # resolves the scratch address before any capture
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        g.capture_begin()
        st = hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             o.data_ptr(), s.cuda_stream)
        g.capture_end()
    assert st == hyat.ERR_UNSUPPORTED
