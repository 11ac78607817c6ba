"""The allocation-free forward (hyat_fwd_bidir_noalloc), called through the C ABI.

It serves callers that cannot allocate device memory where they run the layer;
its scratch is a static device array shared by every call. Each of two calls
in a row (different inputs, so stale scratch would show) must match the
handle-based hyat_fwd_bidir within the parity tolerance of the other tests.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_parity, f64

pytestmark = pytest.mark.gpu


def _noalloc(cfg, q, k, v):
    o = torch.empty_like(q)
    st = hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         o.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == hyat.OK, hyat.lib.hyat_status_string(st)
    return o


@pytest.mark.parametrize("w", [wl.WAN13B_BIDIR, wl.TINY_F32,
                               wl.Workload("radial_small", "radial", 1, 2, 128, 300, 9, seed=6)],
                         ids=lambda w: w.name)
def test_noalloc_matches_handle_forward_twice(w):
    cfg = hyat.config_from_workload(w)
    h = hyat.Hyat(cfg)
    for seed in (w.seed + 101, w.seed + 202):
        q, k, v = (t.cuda() for t in wl.gen_qkv(w, seed=seed))
        ref = h.forward(q, k, v)
        got = _noalloc(cfg, q, k, v)
        torch.cuda.synchronize()
        assert_parity(w.dtype, f64(got.cpu()), f64(ref.cpu()), f"{w.name} seed {seed}")
    h.close()


def test_noalloc_rejects_configs_beyond_its_scratch():
    cfg = hyat.config_from_workload(wl.WAN14B_BIDIR)       # needs ~55 MiB of linear states
    st = hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), 16, 16, 16, 16, None)
    assert st == hyat.ERR_UNSUPPORTED
    cfg = hyat.config_from_workload(wl.STREAM_HF)
    assert hyat.lib.hyat_fwd_bidir_noalloc(ctypes.byref(cfg), 16, 16, 16, 16, None) == hyat.ERR_INVALID_ARG
