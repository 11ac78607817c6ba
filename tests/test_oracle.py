"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a library
routine computing a special case (softmax attention, elu), an associativity
re-evaluation (pure linear attention), brute-force loops over the explicit
weight matrix, hand-derived closed forms, invariances, and token-level brute
force of the tile rules. A plausible slip (a dropped branch, a wrong window
edge, a swapped operand, a wrong phi) fails at least one of them.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_video_hyat_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- feature map
def test_phi_is_elu_plus_one():
    x = np.concatenate([_rand(2000, 1, 3.0), [0.0, -0.0, 1e-30, -1e-30, -40.0, 40.0]])
    ref = torch.nn.functional.elu(torch.from_numpy(x), alpha=1.0).numpy() + 1.0
    # torch evaluates expm1(x) + 1, which rounds differently from exp(x): absolute 1e-15
    np.testing.assert_allclose(oracle.phi_elu1(x), ref, rtol=1e-15, atol=1e-15)
    assert np.all(oracle.phi_elu1(x) > 0)


def test_phi_relu_and_exp_closed_forms():
    x = np.concatenate([_rand(2000, 2, 3.0), [0.0, -0.0, 1e-300, -1e-300, -40.0, 40.0]])
    # ReLU: (x + |x|) / 2, zero exactly on x <= 0
    np.testing.assert_array_equal(oracle.phi_relu(x), (x + np.abs(x)) / 2)
    assert np.all(oracle.phi_relu(x[x <= 0]) == 0.0)
    # exp: exp(0) = 1, exp(ln 2) = 2, and exp(a) exp(b) = exp(a + b)
    assert oracle.phi_exp(0.0) == 1.0
    np.testing.assert_allclose(oracle.phi_exp(np.log(2.0)), 2.0, rtol=1e-15)
    a, b = _rand(500, 3), _rand(500, 4)
    np.testing.assert_allclose(oracle.phi_exp(a) * oracle.phi_exp(b), oracle.phi_exp(a + b), rtol=1e-14)
    assert oracle.feature_map("elu1") is oracle.phi_elu1 and set(oracle.FEATURE_MAPS) == {"elu1", "relu", "exp"}


# ------------------------------------------------------------------- limits
def test_window_all_is_softmax_attention():
    """One chunk spanning the whole video: the linear set is empty."""
    B, H, T, F, d = 1, 2, 3, 32, 16
    q, k, v = (_rand((B, H, T * F, d), s) for s in (1, 2, 3))
    o = oracle.bidir_window_attention(q, k, v, F, T, chunk_frames=T, halo_frames=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-13)
    # the same through an all-ones tile mask
    nT = -(-T * F // 8)
    o2 = oracle.blockmask_attention(q, k, v, np.ones((1, nT, nT), np.uint8), tile=8)
    np.testing.assert_allclose(o2, ref, rtol=1e-11, atol=1e-13)


_TORCH_PHI = {"elu1": lambda t: torch.nn.functional.elu(t) + 1, "relu": torch.relu, "exp": torch.exp}


@pytest.mark.parametrize("phi", ["elu1", "relu", "exp"])
def test_empty_window_is_linear_attention(phi):
    """An all-zero tile mask: every key reaches the query through phi(q).phi(k)."""
    B, H, N, d = 1, 3, 80, 16
    q, k, v = (_rand((B, H, N, d), s) for s in (4, 5, 6))
    o = oracle.blockmask_attention(q, k, v, np.zeros((H, 10, 10), np.uint8), tile=8, phi=phi)
    pq = _TORCH_PHI[phi](torch.from_numpy(q)).numpy()
    pk = _TORCH_PHI[phi](torch.from_numpy(k)).numpy()
    S = np.einsum("bhna,bhnc->bhac", pk, v)          # associativity: (phi K)^T V first
    z = pk.sum(axis=2)
    ref = np.einsum("bhna,bhac->bhnc", pq, S) / np.einsum("bhna,bha->bhn", pq, z)[..., None]
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-13)


# -------------------------------------------------------------- brute force
def _phi_scalar(x, phi):
    if phi == "relu":
        return x if x > 0 else 0.0
    if phi == "exp":
        return float(np.e) ** x
    return x + 1 if x > 0 else np.exp(x)


def _bruteforce(q, k, v, in_soft, in_lin, scale, phi="elu1"):
    """Explicit N x N weight matrix with plain loops, no stabiliser."""
    n, d = q.shape
    out = np.zeros((n, v.shape[1]))
    for i in range(n):
        num = np.zeros(v.shape[1])
        den = 0.0
        for j in range(k.shape[0]):
            if in_soft(i, j):
                w = np.exp(sum(q[i, a] * k[j, a] for a in range(d)) * scale)
            elif in_lin(i, j):
                w = 0.0
                for a in range(d):
                    w += _phi_scalar(q[i, a], phi) * _phi_scalar(k[j, a], phi)
            else:
                w = 0.0
            num += w * v[j]
            den += w
        out[i] = num / den
    return out


@pytest.mark.parametrize("phi", ["elu1", "relu", "exp"])
def test_bruteforce_bidir_window(phi):
    T, F, d = 5, 6, 4
    N = T * F
    q, k, v = (_rand((1, 1, N, d), s) for s in (7, 8, 9))
    C, h = 2, 1
    o = oracle.bidir_window_attention(q, k, v, F, T, C, h, phi=phi)[0, 0]

    def soft(i, j):
        c = (i // F) // C
        return max(0, c * C - h) * F <= j < min(T, (c + 1) * C + h) * F

    ref = _bruteforce(q[0, 0], k[0, 0], v[0, 0], soft, lambda i, j: not soft(i, j), 0.5, phi)
    np.testing.assert_allclose(o, ref, rtol=1e-12)


def test_bruteforce_tile_mask():
    N, d, tile = 27, 4, 4
    nT = -(-N // tile)
    q, k, v = (_rand((1, 2, N, d), s) for s in (10, 11, 12))
    mask = wl.gen_tile_mask(2, nT, nT, seed=3)
    o = oracle.blockmask_attention(q, k, v, mask, tile=tile)
    for h in range(2):
        soft = lambda i, j: bool(mask[h, i // tile, j // tile])
        ref = _bruteforce(q[0, h], k[0, h], v[0, h], soft, lambda i, j: not soft(i, j), 0.5)
        np.testing.assert_allclose(o[0, h], ref, rtol=1e-12)


def test_bruteforce_stream_step():
    L, d, tile, nwin = 10, 4, 4, 2
    nqt = -(-L // tile)
    step = 3                                            # chunks 0,1 evicted; 2,3 visible
    rng = np.random.default_rng(13)
    kh, vh = rng.standard_normal((1, 1, 4 * L, d)), rng.standard_normal((1, 1, 4 * L, d))
    qc = rng.standard_normal((1, 1, L, d))
    mask = (rng.random((1, nqt, nqt * nwin)) < 0.5).astype(np.uint8)
    mask[0, np.arange(nqt), nqt + np.arange(nqt)] = 1
    o = oracle.stream_step_attention(qc, kh, vh, step, L, nwin, mask, tile=tile)[0, 0]

    def soft(i, j):
        c = j // L
        if c < step - nwin + 1:
            return False
        kt = (c - (step - nwin + 1)) * nqt + (j % L) // tile
        return bool(mask[0, i // tile, kt])

    lin = lambda i, j: j // L < step - nwin + 1
    ref = _bruteforce(qc[0, 0], kh[0, 0], vh[0, 0], soft, lin, 0.5)
    np.testing.assert_allclose(o, ref, rtol=1e-12)


def test_bruteforce_stream_step_with_sink():
    """Sink chunk 0 stays visible; chunk 1 is evicted; chunks 2, 3 form the window."""
    L, d, tile, nwin, n_sink = 10, 4, 4, 2, 1
    nqt = -(-L // tile)
    step = 3
    rng = np.random.default_rng(17)
    kh, vh = rng.standard_normal((1, 1, 4 * L, d)), rng.standard_normal((1, 1, 4 * L, d))
    qc = rng.standard_normal((1, 1, L, d))
    vis = [0, 2, 3]
    assert oracle.stream_visible_chunks(step, nwin, n_sink) == vis
    mask = (rng.random((1, nqt, nqt * len(vis))) < 0.5).astype(np.uint8)
    mask[0, np.arange(nqt), nqt * 2 + np.arange(nqt)] = 1
    o = oracle.stream_step_attention(qc, kh, vh, step, L, nwin, mask, tile=tile, n_sink_chunks=n_sink)[0, 0]

    def soft(i, j):
        c = j // L
        if c not in vis:
            return False
        return bool(mask[0, i // tile, vis.index(c) * nqt + (j % L) // tile])

    ref = _bruteforce(qc[0, 0], kh[0, 0], vh[0, 0], soft, lambda i, j: j // L == 1, 0.5)
    np.testing.assert_allclose(o, ref, rtol=1e-12)
    # the evicted state holds chunk 1 only
    S, z = oracle.stream_evicted_state(kh, vh, step, L, nwin, n_sink_chunks=n_sink)
    pk = np.where(kh[0, 0, L:2 * L] > 0, kh[0, 0, L:2 * L] + 1, np.exp(kh[0, 0, L:2 * L]))
    np.testing.assert_allclose(S[0, 0], pk.T @ vh[0, 0, L:2 * L], rtol=1e-13)
    np.testing.assert_allclose(z[0, 0], pk.sum(0), rtol=1e-13)


# ------------------------------------------------------------- closed forms
def _frame_indicator_v(T, F, d):
    v = np.zeros((1, 1, T * F, d))
    for f in range(T):
        v[0, 0, f * F:(f + 1) * F, f] = 1.0
    return v


def test_closed_form_tiny_golden():
    """q = k = 0 on the tiny workload's geometry; expected values from the golden file."""
    T, F, d = 4, 64, 64
    z = np.zeros((1, 1, T * F, d))
    o = oracle.bidir_window_attention(z, z, _frame_indicator_v(T, F, d), F, T, 1, 0)[0, 0]
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "closed_form_q0k0_tiny.txt"))
            if ln.strip() and not ln.startswith("#")]
    for r in rows:
        f = int(r[0])
        exp = np.array([eval(x) for x in r[1:]])
        np.testing.assert_allclose(o[f * F:(f + 1) * F, :T], np.broadcast_to(exp, (F, T)),
                                   rtol=1e-14)
        assert np.all(o[f * F:(f + 1) * F, T:] == 0)


def test_closed_form_chunk_halo_window():
    """q = k = 0 with 3-frame chunks and a 1-frame halo (the Wan geometry, fewer tokens)."""
    T, F, d = 21, 5, 32
    z = np.zeros((1, 1, T * F, d))
    o = oracle.bidir_window_attention(z, z, _frame_indicator_v(T, F, d), F, T, 3, 1)[0, 0]
    for i in range(T * F):
        c = (i // F) // 3
        lo, hi = max(0, 3 * c - 1), min(T, 3 * c + 4)
        wts = np.array([1.0 if lo <= f < hi else float(d) for f in range(T)]) * F
        np.testing.assert_allclose(o[i, :T], wts / wts.sum(), rtol=1e-13)
    # edge chunks see 4 frames, interior chunks 5
    assert oracle.bidir_window_interval(0, 21, 3, 1) == (0, 4)
    assert oracle.bidir_window_interval(10, 21, 3, 1) == (8, 13)
    assert oracle.bidir_window_interval(20, 21, 3, 1) == (17, 21)


def test_closed_form_stream():
    """q = k = 0: kept window keys weigh 1, evicted keys weigh d, dropped tiles 0."""
    L, d, tile, nwin, step = 12, 8, 4, 3, 5
    nqt = 3
    v = np.zeros((1, 1, (step + 1) * L, d))
    for c in range(step + 1):
        v[0, 0, c * L:(c + 1) * L, c] = 1.0
    z = np.zeros((1, 1, (step + 1) * L, d))
    mask = wl.gen_tile_mask(1, nqt, nqt * nwin, seed=5)
    mask[0, np.arange(nqt), 2 * nqt + np.arange(nqt)] = 1
    o = oracle.stream_step_attention(z[:, :, :L], z, v, step, L, nwin, mask, tile=tile)[0, 0]
    for i in range(L):
        w = np.zeros(step + 1)
        for c in range(step + 1):
            if c < step - nwin + 1:
                w[c] = d * L
            else:
                w[c] = sum(mask[0, i // tile, (c - (step - nwin + 1)) * nqt + t] * min(tile, L - t * tile)
                           for t in range(nqt))
        np.testing.assert_allclose(o[i, :step + 1], w / w.sum(), rtol=1e-13)


def test_constant_values_and_convexity():
    B, H, T, F, d = 1, 2, 6, 10, 8
    q, k = _rand((B, H, T * F, d), 20, 2.0), _rand((B, H, T * F, d), 21, 2.0)
    c = _rand(d, 22)
    v = np.broadcast_to(c, (B, H, T * F, d)).copy()
    o = oracle.bidir_window_attention(q, k, v, F, T, 2, 1)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=1e-12)
    v = _rand((B, H, T * F, d), 23)
    o = oracle.bidir_window_attention(q, k, v, F, T, 2, 1)
    assert np.all(o.max(axis=2) <= v.max(axis=2) + 1e-12)
    assert np.all(o.min(axis=2) >= v.min(axis=2) - 1e-12)


def test_permutation_invariance_and_partition():
    """Permuting keys inside the linear set keeps o; moving a key across the window edge does not."""
    T, F, d = 6, 8, 8
    q, k, v = (_rand((1, 1, T * F, d), s) for s in (30, 31, 32))
    o = oracle.bidir_window_attention(q, k, v, F, T, 2, 0)
    # rows of chunk 0 (frames 0,1): frames 2..5 are linear; shuffle keys 16..47 together
    perm = np.arange(T * F)
    perm[16:48] = 16 + np.random.default_rng(3).permutation(32)
    o2 = oracle.bidir_window_attention(q, k[:, :, perm], v[:, :, perm], F, T, 2, 0)
    np.testing.assert_allclose(o2[0, 0, :16], o[0, 0, :16], rtol=1e-12)
    # swapping a window key (frame 1) with a linear key (frame 2) changes chunk 0's rows
    perm = np.arange(T * F)
    perm[[12, 20]] = perm[[20, 12]]
    o3 = oracle.bidir_window_attention(q, k[:, :, perm], v[:, :, perm], F, T, 2, 0)
    assert np.max(np.abs(o3[0, 0, :16] - o[0, 0, :16])) > 1e-6


def test_rows_subset_matches_full():
    q, k, v = (_rand((1, 2, 90, 8), s) for s in (40, 41, 42))
    full = oracle.bidir_window_attention(q, k, v, 15, 6, 3, 1)
    rows = np.array([0, 17, 44, 45, 89])
    sub = oracle.bidir_window_attention(q, k, v, 15, 6, 3, 1, rows=rows)
    np.testing.assert_array_equal(sub, full[:, :, rows])


def test_branches_sum_to_output():
    q, k, v = (_rand((1, 1, 60, 8), s) for s in (50, 51, 52))
    o, (ns, ds, nl, dl) = oracle.bidir_window_attention(q, k, v, 10, 6, 2, 0, with_branches=True)
    np.testing.assert_allclose(o, (ns + nl) / (ds + dl)[..., None], rtol=1e-14)
    assert np.all(ds > 0) and np.all(dl > 0)


# ----------------------------------------------------------------- radial
def test_radial_window_sequence():
    assert [oracle.radial_window(t, 1560) for t in (1, 2, 3, 4, 7, 8, 16, 32, 64, 83)] == \
        [1560, 780, 780, 390, 390, 195, 97, 48, 24, 24]


@pytest.mark.parametrize("T,F,tile", [(12, 300, 128), (9, 100, 32), (5, 64, 128), (7, 130, 64)])
def test_radial_tile_rule_matches_token_bruteforce(T, F, tile):
    N = T * F
    i = np.arange(N)
    near = oracle.radial_token_near(i[:, None], i[None, :], F)
    # direct per-pair check of the predicate on a sample, written with python ints
    rng = np.random.default_rng(0)
    for a, b in rng.integers(0, N, size=(300, 2)):
        fa, pa = divmod(int(a), F)
        fb, pb = divmod(int(b), F)
        t = abs(fa - fb)
        exp = t == 0 or 2 * abs(pb - pa) < (F >> (t.bit_length() - 1))
        assert bool(near[a, b]) == exp
    nT = -(-N // tile)
    pad = np.zeros((nT * tile, nT * tile), dtype=bool)
    pad[:N, :N] = near
    brute = pad.reshape(nT, tile, nT, tile).any(axis=(1, 3))
    np.testing.assert_array_equal(oracle.radial_tile_mask(T, F, tile).astype(bool), brute)


def test_radial_attention_is_tile_mask_attention():
    T, F = 5, 40
    q, k, v = (_rand((1, 1, T * F, 8), s) for s in (60, 61, 62))
    tm = oracle.radial_tile_mask(T, F, 16)
    np.testing.assert_array_equal(oracle.radial_attention(q, k, v, T, F, tile=16),
                                  oracle.blockmask_attention(q, k, v, tm[None], tile=16))


# ---------------------------------------------------------------- streaming
def test_stream_state_is_prefix_sum_of_evicted():
    L, d, nwin, steps = 6, 4, 3, 8
    rng = np.random.default_rng(70)
    kh, vh = rng.standard_normal((1, 2, steps * L, d)), rng.standard_normal((1, 2, steps * L, d))
    S = np.zeros((1, 2, d, d))
    z = np.zeros((1, 2, d))
    for s in range(steps):
        ev = s - nwin                                   # chunk evicted when step s starts
        if ev >= 0:
            for j in range(ev * L, (ev + 1) * L):
                pk = torch.nn.functional.elu(torch.from_numpy(kh[:, :, j])).numpy() + 1
                S += pk[..., :, None] * vh[:, :, j, None, :]
                z += pk
        S2, z2 = oracle.stream_evicted_state(kh[:, :, :(s + 1) * L], vh[:, :, :(s + 1) * L],
                                             s, L, nwin)
        np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(z2, z, rtol=1e-12, atol=1e-12)


def test_stream_without_eviction_is_block_causal_softmax():
    """Before any eviction, with every tile kept, chunk s attends to chunks 0..s by softmax."""
    L, d, tile, nwin = 8, 8, 4, 3
    rng = np.random.default_rng(80)
    kh, vh = rng.standard_normal((1, 1, 3 * L, d)), rng.standard_normal((1, 1, 3 * L, d))
    qh = rng.standard_normal((1, 1, 3 * L, d))
    for s in range(3):
        mask = np.ones((1, 2, 2 * (s + 1)), np.uint8)
        o = oracle.stream_step_attention(qh[:, :, s * L:(s + 1) * L], kh[:, :, :(s + 1) * L],
                                         vh[:, :, :(s + 1) * L], s, L, nwin, mask, tile=tile)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qh[:, :, s * L:(s + 1) * L]), torch.from_numpy(kh[:, :, :(s + 1) * L]),
            torch.from_numpy(vh[:, :, :(s + 1) * L])).numpy()
        np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-13)


def test_stream_workload_mask_shape_and_diagonal():
    w = wl.STREAM_HF
    for step in (0, 1, 2, 7):
        _, _, _, m = wl.gen_stream_step(w.with_(H=2), step)
        nwin = min(step + 1, 3)
        assert m.shape == (2, 37, 37 * nwin)
        assert np.all(m[:, np.arange(37), 37 * (nwin - 1) + np.arange(37)] == 1)


# -------------------------------------------------------------- work counts
def test_effective_pairs():
    assert oracle.effective_pairs_bidir(1560, 21, 3, 1) == 99 * 1560 ** 2
    assert oracle.effective_pairs_bidir(64, 4, 1, 0) == 4 * 64 ** 2
    tm = np.ones((1, 3, 3), np.uint8)
    assert oracle.effective_pairs_tile_mask(tm, 300, 300)[0] == 300 * 300


# -------------------------------------------------------------- LVSA mask
@pytest.mark.parametrize("F,T,wf,stride,rot", [(10, 7, 3, 3, 0), (10, 7, 1, 2, 1), (13, 5, 5, 0, 0), (6, 9, 3, 4, 2)])
def test_lvsa_tile_mask_is_token_bruteforce(F, T, wf, stride, rot):
    tile = 8
    N = T * F
    nT = -(-N // tile)
    m = oracle.lvsa_tile_mask(T, F, wf, stride, rot, tile=tile)
    for a in range(nT):
        for b in range(nT):
            i = np.arange(a * tile, min(N, (a + 1) * tile))[:, None]
            j = np.arange(b * tile, min(N, (b + 1) * tile))[None, :]
            # the predicate, evaluated from its definition with plain integer arithmetic
            near = any((abs(ii // F - jj // F) <= (wf - 1) // 2) or (stride > 0 and (jj // F + rot) % stride == 0)
                       for ii in i[:, 0] for jj in j[0])
            assert m[a, b] == int(near), (a, b)
    np.testing.assert_array_equal(
        m, np.array([[int(oracle.lvsa_token_near(np.arange(a * tile, min(N, (a + 1) * tile))[:, None],
                                                  np.arange(b * tile, min(N, (b + 1) * tile))[None, :],
                                                  F, wf, stride, rot).any())
                      for b in range(nT)] for a in range(nT)]))


def test_lvsa_tile_mask_invariants():
    T, F = 12, 50
    base = oracle.lvsa_tile_mask(T, F, 3, 4, 1, tile=16)
    np.testing.assert_array_equal(base, oracle.lvsa_tile_mask(T, F, 3, 4, 5, tile=16))   # period = stride
    assert np.all(np.diag(base) == 1)                                                     # own tile always kept
    assert np.all(oracle.lvsa_tile_mask(T, F, 2 * T + 1, 4, 1, tile=16) == 1)              # window covers all
    win = oracle.lvsa_tile_mask(T, F, 3, 0, 0, tile=16)                                    # no anchors: banded
    assert np.all(win == win.T)
    assert base.sum() > win.sum()


# ------------------------------------------------------------------ capped temporal RoPE
# Pins for oracle.rope_temporal from the mathematics of rotations, independent of its code.
def test_rope_complex_form_and_identities():
    """Pair i of a token of offset p, read as the complex number x[2i] + i x[2i+1], is
    multiplied by exp(i p theta_i); the band's width 0 and offset 0 leave x unchanged."""
    rng = np.random.default_rng(41)
    x = rng.standard_normal((2, 30, 16))
    F, f0, ref, cap, t, base = 4, 3, 1, 5, 10, 100.0
    got = oracle.rope_temporal(x, F, f0, ref, cap, t, base)
    p = np.minimum(f0 + np.arange(30) // F - ref, cap - 1)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    theta = np.array([base ** (-2.0 * i / t) if i < t // 2 else 0.0 for i in range(8)])
    zr = z * np.exp(1j * p[:, None] * theta[None, :])
    want = np.empty_like(x)
    want[..., 0::2], want[..., 1::2] = zr.real, zr.imag
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(oracle.rope_temporal(x, F, f0, ref, cap, 0, base), x)
    same = oracle.rope_temporal(x, F, ref, ref, cap, t, base)[:, :F]      # first frame: p = 0
    np.testing.assert_array_equal(same, x[:, :F])


def test_rope_is_relative_and_capped():
    """Inside the cap, q at offset a against k at offset b depends on a - b only; norms are
    kept; beyond the cap every frame turns like offset cap - 1."""
    rng = np.random.default_rng(42)
    d, t, F, cap = 8, 8, 1, 6
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    x = np.stack([q, k])[:, None, :].repeat(10, axis=1)                   # tokens = frames 0..9
    rq = oracle.rope_temporal(x[0], F, 0, 0, cap, t)
    rk = oracle.rope_temporal(x[1], F, 0, 0, cap, t)
    for a, b, a2, b2 in [(3, 1, 4, 2), (5, 5, 0, 0), (2, 4, 0, 2)]:
        assert abs(rq[a] @ rk[b] - rq[a2] @ rk[b2]) < 1e-12
    np.testing.assert_allclose(np.linalg.norm(rq, axis=1), np.linalg.norm(q), rtol=1e-13)
    for f in range(cap, 10):
        np.testing.assert_array_equal(rq[f], rq[cap - 1])
    assert np.abs(rq[cap - 1] - rq[cap - 2]).max() > 1e-3
    with pytest.raises(ValueError):
        oracle.rope_temporal(x[0], F, 0, 1, cap, t)                        # frame before the reference
    with pytest.raises(ValueError):
        oracle.rope_temporal(x[0], F, 0, 0, cap, 7)                        # odd band
