"""Branch-wise GPU parity: each branch of the hybrid output against the oracle's.

A query row's output is (N_soft + N_lin) / (D_soft + D_lin), the exact softmax over its
window keys and the linear-attention term over the rest (ReHyAt abstract; Hybrid Forcing,
Section 2.A). With unit-variance inputs the linear branch carries most of the weight, so a
slip confined to the softmax branch could hide under the hybrid output's tolerance. The
handle's test flags return one branch at a time (HYAT_FLAG_TEST_SOFTMAX_BRANCH zeroes the
linear state; HYAT_FLAG_TEST_LINEAR_BRANCH empties every key list), and the oracle returns
both branches' numerators and denominators (`with_branches=True`).
"""
import numpy as np
import pytest

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl
from parity import assert_parity, f64, sample_rows

pytestmark = pytest.mark.gpu

BRANCHES = {"softmax": hyat.FLAG_TEST_SOFTMAX_BRANCH, "linear": hyat.FLAG_TEST_LINEAR_BRANCH}


def _run(w, flags, mask=None, mask_heads=1):
    cfg = hyat.config_from_workload(w, flags=flags, mask_heads=mask_heads)
    q, k, v = wl.gen_qkv(w)
    h = hyat.Hyat(cfg, mask)
    o = h.forward(q.cuda(), k.cuda(), v.cuda())
    h.sync()
    h.close()
    return f64(o), (q, k, v)


def check_branch(o, br, which, dtype="bf16", what=""):
    """Compare the GPU branch with the oracle's on the rows where that branch has any weight
    (a row whose mask keeps every key tile has no linear branch: 0 / 0 on both sides)."""
    ns, ds, nl, dl = br
    num, den = (ns, ds) if which == "softmax" else (nl, dl)
    rows = den > 0                                    # [B, H, rows]
    assert rows.mean() > 0.5, (what, "too few rows with this branch")
    ref = num[rows] / den[rows][:, None]
    assert_parity(dtype, o[rows][None, None], ref[None, None], (what, which))


@pytest.mark.parametrize("which", ["softmax", "linear"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,F,C,h", [(7, 200, 2, 1), (5, 300, 3, 1), (6, 1560, 3, 1)])
def test_window_branch(which, dtype, T, F, C, h):
    w = wl.Workload("branch", "window", 1, 2, 128, F, T, C, h, dtype=dtype, seed=31 * T + F)
    o, (q, k, v) = _run(w, BRANCHES[which])
    _, br = oracle.bidir_window_attention(f64(q), f64(k), f64(v), F, T, C, h, with_branches=True)
    check_branch(o, br, which, dtype, (T, F, C, h))


@pytest.mark.parametrize("which", ["softmax", "linear"])
@pytest.mark.parametrize("schedule", [hyat.FLAG_PAIR_ONE_WARP, hyat.FLAG_SINGLE_TILE], ids=["one-warp", "single"])
def test_window_branch_other_schedules(which, schedule):
    w = wl.Workload("branch_sched", "window", 1, 2, 128, 300, 5, 3, 1, seed=77)
    o, (q, k, v) = _run(w, BRANCHES[which] | schedule)
    _, br = oracle.bidir_window_attention(f64(q), f64(k), f64(v), 300, 5, 3, 1, with_branches=True)
    check_branch(o, br, which, what="schedule")


@pytest.mark.parametrize("which", ["softmax", "linear"])
def test_blockmask_branch(which):
    T, F, H = 5, 230, 2
    nT = -(-T * F // 128)
    mask = wl.gen_tile_mask(H, nT, nT, seed=8)
    mask[:, np.arange(nT), np.arange(nT)] = 1          # every row keeps a tile: D_soft > 0
    w = wl.Workload("bm_branch", "blockmask", 1, H, 128, F, T, seed=12)
    o, (q, k, v) = _run(w, BRANCHES[which], mask=mask, mask_heads=H)
    _, br = oracle.blockmask_attention(f64(q), f64(k), f64(v), mask, with_branches=True)
    check_branch(o, br, which, what="blockmask")


@pytest.mark.parametrize("which", ["softmax", "linear"])
def test_radial_branch(which):
    """12 frames of 1560 tokens (the radial rule keeps 56 % of the tiles), sampled rows."""
    w = wl.Workload("radial_branch", "radial", 1, 1, 128, 1560, 12, seed=13)
    o, (q, k, v) = _run(w, BRANCHES[which])
    rows = sample_rows(w.N, [(t, min(t + 128, w.N)) for t in range(0, w.N, 128)], per_tile=1, seed=3)
    _, br = oracle.radial_attention(f64(q), f64(k), f64(v), 12, 1560, rows=rows, with_branches=True)
    check_branch(o[:, :, rows], br, which, what="radial")


@pytest.mark.slow
@pytest.mark.parametrize("which", ["softmax", "linear"])
def test_full_wan13b_branch_sampled(which):
    """The headline layer, both branches, sampled rows (the first and last row of every query
    tile plus a random one) of three heads."""
    w = wl.WAN13B_BIDIR
    o, (q, k, v) = _run(w, BRANCHES[which])
    chunk = w.chunk_frames * w.tokens_per_frame
    tiles = [(c0 + t, min(c0 + t + 128, c0 + chunk, w.N)) for c0 in range(0, w.N, chunk)
             for t in range(0, min(chunk, w.N - c0), 128)]
    rows = sample_rows(w.N, tiles, per_tile=1, seed=5)
    heads = [0, 5, 11]
    _, br = oracle.bidir_window_attention(f64(q[:, heads]), f64(k[:, heads]), f64(v[:, heads]), w.tokens_per_frame,
                                          w.n_frames, w.chunk_frames, w.halo_frames, rows=rows, with_branches=True)
    check_branch(o[:, heads][:, :, rows], br, which, what="wan1.3b")


def test_branch_flags_rejected_where_they_do_not_apply():
    both = hyat.FLAG_TEST_SOFTMAX_BRANCH | hyat.FLAG_TEST_LINEAR_BRANCH
    w = wl.Workload("branch_bad", "window", 1, 1, 128, 100, 3, 1, 0, seed=1)
    with pytest.raises(hyat.HyatError):
        hyat.Hyat(hyat.config_from_workload(w, flags=both))
    ws = wl.Workload("branch_stream", "stream", 1, 2, 128, 200, 9, chunk_frames=3, window_frames=9, n_steps=2, seed=2)
    with pytest.raises(hyat.HyatError):
        hyat.Hyat(hyat.config_from_workload(ws, flags=hyat.FLAG_TEST_SOFTMAX_BRANCH))
