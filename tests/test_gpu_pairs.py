"""The persistent attention's pair list for bidirectional layouts, read back through the C ABI.

Pair k runs on CTA k mod G (G = min(pairs, SMs)). The host sorts the pairs by work (key tiles
of both query tiles + 2) largest first and places each row of G pairs either in a serpentine
or least loaded first, whichever leaves the busiest CTA less work. These tests check that
rule from the layout's work list, and that every work item is in exactly one pair.
"""
import numpy as np
import pytest
import torch

from linear_attention_video_hyat_b200 import hyat, workloads as wl
from test_gpu_stream import _deal_max_loads

pytestmark = pytest.mark.gpu


def _case(name):
    w = wl.WORKLOADS[name]
    mask = None
    if w.mode == "radial":
        mask = hyat.radial_mask(w.n_frames, w.tokens_per_frame)[None]
    if w.mode == "lvsa":
        mask = hyat.lvsa_mask(w.n_frames, w.tokens_per_frame, 11, 4)[None]
    return hyat.config_from_workload(w), mask


@pytest.mark.parametrize("name", ["wan1.3b_bidir_T21x1560", "radial_T84x1560", "lvsa_T126x1560_w11_s4"])
def test_bidir_pairs_dealt_by_the_better_rule(name):
    cfg, mask = _case(name)
    work, _ = hyat.plan_layout(cfg, mask)
    h = hyat.Hyat(cfg, mask=mask)
    pairs = h.pairs()
    h.close()
    n_of = lambda i: 0 if i < 0 else int(work[i, 5] - work[i, 4])
    items = [i for p in pairs for i in (p[0], p[1]) if i >= 0]
    assert sorted(items) == list(range(len(work)))
    cost = np.array([n_of(p[0]) + n_of(p[1]) + 2 for p in pairs], np.int64)
    G = min(len(pairs), torch.cuda.get_device_properties(0).multi_processor_count)
    want = np.sort(cost)[::-1]
    serp_max, lpt_max = _deal_max_loads(want, G)
    load = np.zeros(G, np.int64)
    for r, r0 in enumerate(range(0, len(pairs), G)):
        m = min(G, len(pairs) - r0)
        got = cost[r0:r0 + m]
        assert np.array_equal(np.sort(got)[::-1], want[r0:r0 + m])
        load[:m] += got
    assert load.max() == min(serp_max, lpt_max)
