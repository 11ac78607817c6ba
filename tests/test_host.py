"""Host-side tests of libhyat (no GPU): exported symbols, layout and eviction
indexing bit-exact against the oracle's window rules, and argument validation."""
import os
import re

import numpy as np
import torch
import pytest

import oracle
from linear_attention_video_hyat_b200 import hyat, workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_symbol():
    header = open(os.path.join(ROOT, "include", "hyat.h")).read()
    declared = sorted(set(re.findall(r"HYAT_API [^;]*?\b(hyat_\w+)\(", header)))
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(hyat.lib, name), name
    assert sorted(hyat.EXPORTED) == declared


def test_binding_constants_match_the_header():
    """Every HYAT_FLAG_*, status and enum value the binding names has the header's value."""
    header = open(os.path.join(ROOT, "include", "hyat.h")).read()
    flags = dict(re.findall(r"#define HYAT_FLAG_(\w+) (\d+)u", header))
    assert len(flags) >= 6
    for name, val in flags.items():
        assert getattr(hyat, "FLAG_" + name) == int(val), name
    enums = dict((n, int(v)) for n, v in re.findall(r"\bHYAT_(\w+) = (\d+)", header))
    for name in ("OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_DEVICE_TIMEOUT", "ERR_STATE",
                 "F32", "BF16", "MODE_WINDOW", "MODE_BLOCKMASK", "MODE_RADIAL", "MODE_STREAM"):
        if name in enums:
            assert getattr(hyat, name) == enums[name], name


def _window_rows_from_layout(work, ent, bh=0):
    """Map query row -> sorted array of softmax keys, from the C++ layout."""
    rows = {}
    for w in work:
        if w[0] != bh:
            continue
        keys = np.sort(np.concatenate([np.arange(e[0], e[0] + e[1]) for e in ent[w[4]:w[5]]])) \
            if w[5] > w[4] else np.zeros(0, np.int64)
        for r in range(w[1], w[1] + w[2]):
            assert r not in rows
            rows[r] = keys
    return rows


@pytest.mark.parametrize("T,F,C,h", [(21, 1560, 3, 1), (4, 64, 1, 0), (7, 200, 2, 1), (5, 300, 3, 2),
                                     (3, 100, 5, 0), (21, 3600, 3, 1)])
def test_window_layout_matches_oracle(T, F, C, h):
    cfg = hyat.make_config("window", 1, 2, 128, F, T, C, h)
    work, ent = hyat.plan_layout(cfg)
    N = T * F
    assert set(np.unique(work[:, 0])) == {0, 1}
    rows = _window_rows_from_layout(work, ent)
    assert sorted(rows) == list(range(N))
    sample = np.unique(np.concatenate([np.arange(0, N, max(1, N // 97)), [N - 1]]))
    soft, lin = oracle.bidir_sets(sample, F, T, C, h)
    for n, r in enumerate(sample):
        np.testing.assert_array_equal(rows[r], np.nonzero(soft[n])[0])
    # every key tile is at most 128 keys, every query tile lies inside one chunk
    assert np.all((ent[:, 1] >= 1) & (ent[:, 1] <= 128))
    for w in work:
        assert (w[1] // F) // C == ((w[1] + w[2] - 1) // F) // C
        # even chunks list their key tiles first key first, odd chunks last tile first, with
        # no gap or overlap between consecutive tiles
        starts = ent[w[4]:w[5], 0]
        step = np.diff(starts) if w[3] % 2 == 0 else -np.diff(starts)
        assert np.all(step == 128), (w, starts[:4])


def test_window_layout_tile_counts_wan13b():
    cfg = hyat.config_from_workload(wl.WAN13B_BIDIR)
    work, ent = hyat.plan_layout(cfg)
    assert len(work) == 12 * 7 * 37                     # 37 query tiles per 4680-token chunk
    per_chunk = [w[5] - w[4] for w in work[:7 * 37:37]]
    assert per_chunk == [49, 61, 61, 61, 61, 61, 49]    # 6240- and 7800-key windows
    assert sorted(set(work[:, 2])) == [72, 128]


@pytest.mark.parametrize("T,F", [(84, 1560), (12, 300), (9, 100), (5, 64), (7, 130), (1, 50), (21, 3600)])
def test_radial_mask_bit_exact(T, F):
    np.testing.assert_array_equal(hyat.radial_mask(T, F), oracle.radial_tile_mask(T, F))


def test_radial_layout_counts():
    cfg = hyat.config_from_workload(wl.RADIAL_84F)
    work, ent = hyat.plan_layout(cfg)
    m = oracle.radial_tile_mask(84, 1560)
    assert len(ent) == int(m.sum()) == 290972
    for w in work[[0, 1, 500, 1023]]:
        kt = ent[w[4]:w[5], 0] // 128
        np.testing.assert_array_equal(kt, np.nonzero(m[w[1] // 128])[0])


def test_blockmask_layout_per_head():
    H, T, F = 3, 5, 100
    nT = -(-T * F // 128)
    mask = wl.gen_tile_mask(H, nT, nT, seed=9)
    cfg = hyat.make_config("blockmask", 2, H, 64, F, T, mask_heads=H)
    work, ent = hyat.plan_layout(cfg, mask)
    assert len(work) == 2 * H * nT
    for w in work:
        h = w[0] % H
        soft, _ = oracle.tile_mask_sets(h, [w[1]], mask, T * F)
        keys = np.concatenate([np.arange(e[0], e[0] + e[1]) for e in ent[w[4]:w[5]]]) \
            if w[5] > w[4] else np.zeros(0, np.int64)
        np.testing.assert_array_equal(keys, np.nonzero(soft[0])[0])


def test_stream_plan_eviction_indexing():
    w = wl.STREAM_HF
    cfg = hyat.config_from_workload(w)
    nwc = 3
    slot_of = {}
    for s in range(w.n_steps):
        p = hyat.stream_plan(cfg, s)
        first = max(0, s - nwc + 1)
        assert p["first_visible"] == first and p["n_visible"] == s - first + 1
        assert p["evicted"] == (s - nwc if s >= nwc else -1)
        # the chunk written at step s goes to the slot freed by the evicted chunk
        if p["evicted"] >= 0:
            assert slot_of[p["evicted"]] == p["write_slot"]
        slot_of[s] = p["write_slot"]
        assert p["slots"] == [slot_of[c] for c in range(first, s + 1)]
        # evicted frames are exactly the frames the oracle sends to the linear set
        L = w.chunk_tokens
        _, lin = oracle.stream_sets(0, [0], s, L, nwc, np.ones((1, 37, 37 * (s - first + 1)), np.uint8))
        assert int(lin.sum()) == first * L


@pytest.mark.parametrize("bad", [dict(d=96), dict(B=0), dict(tokens_per_frame=0), dict(mode=9),
                                 dict(mode="stream", window_frames=8), dict(mode="blockmask", mask_heads=3),
                                 dict(dtype=7), dict(scale=-1.0), dict(phi=3), dict(phi=-1),
                                 dict(flags=hyat.FLAG_TEST_SOFTMAX_BRANCH | hyat.FLAG_TEST_LINEAR_BRANCH),
                                 dict(mode="stream", flags=hyat.FLAG_TEST_SOFTMAX_BRANCH),
                                 dict(mode="stream", flags=hyat.FLAG_TEST_LINEAR_BRANCH)])
def test_invalid_configs_rejected(bad):
    kw = dict(mode="window", B=1, H=2, d=64, tokens_per_frame=64, n_frames=4, chunk_frames=1,
              window_frames=9)
    kw.update(bad)
    if kw["mode"] == "stream":
        kw["chunk_frames"] = 3
    cfg = hyat.make_config(**kw)
    assert hyat.workspace_bytes(cfg) == 0


@pytest.mark.parametrize("flags", [0, hyat.FLAG_TEST_SOFTMAX_BRANCH, hyat.FLAG_TEST_LINEAR_BRANCH])
def test_branch_flags_accepted_in_bidirectional_modes(flags):
    for mode in ("window", "radial"):
        cfg = hyat.make_config(mode, 1, 2, 64, 64, 4, 1, 0, flags=flags)
        assert hyat.workspace_bytes(cfg) > 0


@pytest.mark.parametrize("rope,ok", [({"t_dims": 44, "cap": 21}, True), ({"t_dims": 128, "cap": 1, "base": 500.0}, True),
                                     ({"t_dims": 43, "cap": 21}, False), ({"t_dims": 130, "cap": 21}, False),
                                     ({"t_dims": 44, "cap": 0}, False), ({"t_dims": -2, "cap": 3}, False),
                                     ({"t_dims": 44, "cap": 3, "base": -1.0}, False),
                                     ({"t_dims": 44, "cap": 3, "base": float("inf")}, False)])
def test_fused_rope_config_validation(rope, ok):
    """The fused temporal RoPE is a STREAM option with an even band of at most d dimensions and
    a cap of at least 1; its workspace adds the turned Q of one chunk."""
    cfg = hyat.config_from_workload(wl.STREAM_HF, rope=rope)
    plain = hyat.workspace_bytes(hyat.config_from_workload(wl.STREAM_HF))
    n = hyat.workspace_bytes(cfg)
    if ok:
        q_bytes = wl.STREAM_HF.B * wl.STREAM_HF.H * wl.STREAM_HF.chunk_tokens * wl.STREAM_HF.d * 2
        assert plain + q_bytes <= n <= plain + q_bytes + 256
    else:
        assert n == 0
    # never on a bidirectional handle
    assert hyat.workspace_bytes(hyat.config_from_workload(wl.WAN13B_BIDIR, rope={"t_dims": 44, "cap": 21})) == 0


def test_workspace_sizes():
    for w in (wl.TINY_F32, wl.WAN13B_BIDIR, wl.WAN14B_BIDIR, wl.STREAM_HF, wl.RADIAL_84F):
        n = hyat.workspace_bytes(hyat.config_from_workload(w))
        assert 0 < n < 4 << 30, (w.name, n)


def test_peaked_bf16_bound_accepts_rounding_and_rejects_a_planted_error():
    """The large-logit tolerance admits bf16 rounding of o and P, and no more."""
    import pytest as _pt
    from parity import assert_bf16_peaked
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 1, 64, 16))
    s = 40.0 * rng.standard_normal((1, 1, 8, 64))           # nearly one-hot softmax rows
    p = np.exp(s - s.max(axis=3, keepdims=True))
    ref = (p @ v[0, 0]) / p.sum(axis=3, keepdims=True)
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()
    o = bf((bf(p) @ v[0, 0]) / p.sum(axis=3, keepdims=True))  # P and o rounded to bf16
    assert_bf16_peaked(o, ref, v)
    bad = o.copy()
    bad[0, 0, 3, 5] += 2.0 ** -8 * (abs(ref[0, 0, 3, 5]) + np.abs(v).max()) * 1.5
    with _pt.raises(AssertionError):
        assert_bf16_peaked(bad, ref, v)


@pytest.mark.parametrize("phi", ["elu1", "relu", "exp"])
def test_feature_maps_accepted(phi):
    cfg = hyat.make_config("window", 1, 2, 64, 64, 4, 1, 0, phi=phi)
    assert hyat.workspace_bytes(cfg) > 0


@pytest.mark.parametrize("T,F,wf,stride,rot", [(21, 1560, 5, 4, 0), (21, 1560, 11, 3, 2), (126, 1560, 11, 4, 1),
                                               (9, 300, 1, 0, 0), (7, 130, 3, 2, 5)])
def test_lvsa_mask_matches_oracle(T, F, wf, stride, rot):
    got = hyat.lvsa_mask(T, F, wf, stride, rot)
    ref = oracle.lvsa_tile_mask(T, F, wf, stride, rot)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("bad", [dict(window_frames=4), dict(window_frames=0), dict(anchor_stride=-1),
                                 dict(rotation=-1)])
def test_lvsa_mask_rejects_bad_arguments(bad):
    kw = dict(n_frames=5, tokens_per_frame=100, window_frames=3, anchor_stride=2, rotation=0)
    kw.update(bad)
    with pytest.raises(hyat.HyatError):
        hyat.lvsa_mask(**kw)


@pytest.mark.parametrize("sink_frames", [3, 6])
def test_stream_plan_with_sink(sink_frames):
    """Sink chunks keep their own slots for good; the rolling window cycles the others."""
    w = wl.STREAM_HF.with_(sink_frames=sink_frames)
    cfg = hyat.config_from_workload(w)
    nwc, ns = 3, sink_frames // 3
    slot_of = {}
    for s in range(20):
        p = hyat.stream_plan(cfg, s)
        vis = oracle.stream_visible_chunks(s, nwc, ns)
        assert p["n_visible"] == len(vis) == wl.stream_window_chunks(w, s)
        assert p["first_visible"] == max(ns, s - nwc + 1)
        assert p["evicted"] == (s - nwc if s - nwc >= ns else -1)
        if p["evicted"] >= 0:
            assert slot_of[p["evicted"]] == p["write_slot"]
        slot_of[s] = p["write_slot"]
        assert p["slots"] == [slot_of[c] for c in vis]
        assert len(set(p["slots"])) == len(vis)
        assert all(slot_of[c] == nwc + c for c in range(min(ns, s + 1)))


def test_bench_work_counts_match_the_oracle_pair_counts():
    """The effective FLOPs the bench reports come from the library layout; they must equal
    4 d times the oracle's count of in-window (query, key) pairs plus the state FLOPs."""
    import bench
    w = wl.WAN13B_BIDIR
    c = bench.work_counts(w)
    pairs = oracle.effective_pairs_bidir(w.tokens_per_frame, w.n_frames, w.chunk_frames, w.halo_frames)
    assert c["pairs_per_head"] == pairs
    BH, d, N = w.B * w.H, w.d, w.N
    assert c["total_flops"] == 4 * d * pairs * BH + BH * N * (2 * d * d + d) + BH * N * (2 * d * d + 2 * d)
    # radial: pairs inside kept tiles, counted on the oracle's own mask
    wr = wl.RADIAL_84F.with_(n_frames=12)
    cr = bench.work_counts(wr)
    tm = oracle.radial_tile_mask(wr.n_frames, wr.tokens_per_frame)[None]
    assert cr["pairs_per_head"] == int(oracle.effective_pairs_tile_mask(tm, wr.N, wr.N)[0])


def test_bench_stream_step_flops_by_brute_force():
    import bench
    w = wl.STREAM_HF
    mask = wl.gen_stream_step(w, 5)[3]
    flops, attn = bench.stream_step_flops(w, mask, True)
    L, d, H = w.chunk_tokens, w.d, w.H
    qlen = [min(128, L - 128 * i) for i in range(37)]
    pairs = sum(int(mask[h, i, j]) * qlen[i] * qlen[j % 37] for h in range(H) for i in range(37)
                for j in range(mask.shape[2]))
    assert attn == 4 * d * pairs + H * L * (2 * d * d + 2 * d)
    assert flops == attn + H * L * (2 * d * d + d)


def test_rope_temporal_validates_before_touching_the_gpu():
    """Bad arguments return HYAT_ERR_INVALID_ARG and empty tensors are a no-op, with no launch."""
    f = hyat.lib.hyat_rope_temporal
    good = dict(BH=2, n=10, d=128, dt=hyat.BF16, F=5, f0=3, ref=1, cap=4, t=44, base=10000.0)

    def call(x=None, y=None, **kw):
        a = dict(good, **kw)
        return f(x, y, a["BH"], a["n"], a["d"], a["dt"], a["F"], a["f0"], a["ref"], a["cap"], a["t"], a["base"], None)
    assert call(BH=0) == hyat.OK and call(n=0) == hyat.OK
    assert call() == hyat.ERR_INVALID_ARG                                      # null tensors
    for bad in (dict(d=96), dict(dt=7), dict(F=0), dict(cap=0), dict(t=45), dict(t=130), dict(t=-2),
                dict(base=0.0), dict(base=float("inf")), dict(f0=0, ref=1), dict(BH=-1), dict(BH=70000)):
        assert call(**bad) == hyat.ERR_INVALID_ARG, bad
