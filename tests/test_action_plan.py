"""The NVFP4 read's work split, checked on the host (wam_debug_action_plan): every 128-key tile
of every (episode, head) is read by exactly one CTA, the parts of one head share their tile
boundaries, and the parts stay within the workspace's slots and the SM count."""

import itertools

import numpy as np
import pytest

from cached_kv_attention_b200 import synth, wam


def _parts(nv, k):
    """Tiles of the k parts of one (episode, head): part 0 the action tile (0) and video tiles
    [1, 1 + nv / k), part r the video tiles [1 + r nv / k, 1 + (r + 1) nv / k)."""
    out = []
    for r in range(k):
        t0 = 0 if r == 0 else 1 + r * nv // k
        t1 = 1 + (r + 1) * nv // k
        out.append(range(t0, t1))
    return out


def _check(B, H, T, F, pad, sms):
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    k, n_ctas, max_parts = wam.debug_action_plan(lay, sms)
    nvalid = (1 - np.asarray(pad)).sum(axis=1)
    nv = nvalid * (T // 128)
    assert n_ctas == H * int(k.sum()) and max_parts == int(k.max())
    for b in range(B):
        assert 1 <= k[b] <= max(nv[b], 1)
        tiles = [t for part in _parts(int(nv[b]), int(k[b])) for t in part]
        assert sorted(tiles) == list(range(1 + int(nv[b])))  # each tile once
        assert all(len(p) >= 1 for p in _parts(int(nv[b]), int(k[b])))
    if n_ctas > sms:  # only when even one part per head does not fit
        assert np.all(k == 1)
    return k, n_ctas


def test_bench_layouts():
    for name in ("ctx2.4s_bf16", "ctx19.2s_bf16", "ctx38.4s_bf16", "batched4_bf16"):
        w = synth.WORKLOADS[name]
        pad = synth.pad_mask(w).numpy()
        k, n = _check(w.B, w.H, w.T, w.F, pad, 148)
        assert n <= 148
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    k, n = _check(w.B, w.H, w.T, w.F, synth.pad_mask(w).numpy(), 148)
    assert list(k) == [6] and n == 144  # 42 video tiles per head: 6 parts of 7


@pytest.mark.parametrize("B,H", list(itertools.product([1, 2, 5], [1, 3, 24, 64])))
def test_many_layouts(B, H):
    rng = np.random.default_rng(B * 100 + H)
    for T, F in ((128, 3), (256, 9), (768, 6)):
        for sms in (7, 148):
            pad = (rng.random((B, F)) < 0.4).astype(np.uint8)
            pad[:, -1] = 0
            _check(B, H, T, F, pad, sms)
            _check(B, H, T, F, np.ones((B, F), np.uint8), sms)  # no valid frame: the action tile


def test_plan_rejects_bad_arguments():
    with pytest.raises(wam.WamError):
        wam.debug_action_plan(wam.VideoLayout(1, 2, 128, 64, 3), 148)   # T % 128 != 0
    with pytest.raises(wam.WamError):
        wam.debug_action_plan(wam.VideoLayout(1, 2, 128, 128, 3), 0)
