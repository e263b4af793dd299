"""Launch order of the tensor-core prefill's work items (host logic, CPU only).

The library picks the order in which a prefill call's work items (one valid query frame of one
episode) are launched by replaying the block scheduler's in-order dispatch onto one CTA per SM.
These tests read that order through `wam_debug_prefill_order` and check it against an
independent count of each item's key frames, against longest-first, and against a replay of
the dispatch written here."""

import heapq

import numpy as np
import pytest

from cached_kv_attention_b200 import synth, wam

B200_SMS = 148


def layout_of(name, T=None):
    w = synth.WORKLOADS[name]
    if T is not None:
        w = w.replace(T=T)
    return w, wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, synth.pad_mask(w).numpy())


def key_frames(w, b, f):
    """Valid frames an item of frame f reads: every non-padding frame up to f (one frame per
    attention block, the layouts' default)."""
    pad = synth.pad_mask(w).numpy()
    return int(sum(1 for u in range(f + 1) if not pad[b, u]))


def makespan(nk, w, sms):
    """In-order dispatch of every item's CTAs (ceil(T / 256) x H each, cost key tiles + 5) onto
    `sms` SMs, each CTA to the SM that frees first; returns when the last one ends."""
    per_item = (w.T // 128 + 1) // 2 * w.H
    free = [0] * sms
    end = 0
    for k in nk:
        cost = int(k) * (w.T // 128) + 5
        for _ in range(per_item):
            t = heapq.heappop(free) + cost
            heapq.heappush(free, t)
            end = max(end, t)
    return end


RANGES = {
    "history": lambda w: (0, w.F_h),
    "imagination": lambda w: (w.F_h, w.F),
    "all": lambda w: (0, w.F),
}


@pytest.mark.parametrize("name", ["ctx19.2s_bf16", "ctx2.4s_bf16", "ctx38.4s_bf16", "batched4_bf16"])
@pytest.mark.parametrize("rng", sorted(RANGES))
@pytest.mark.parametrize("sms", [0, 16, B200_SMS, 1000])
def test_order_is_a_permutation_no_worse_than_longest_first(name, rng, sms):
    w, lay = layout_of(name)
    f0, f1 = RANGES[rng](w)
    ep, fr, nk = wam.debug_prefill_order(lay, f0, f1, sms)
    ep0, fr0, nk0 = wam.debug_prefill_order(lay, f0, f1, 0)
    pad = synth.pad_mask(w).numpy()
    # every valid query frame of every episode exactly once, with its key-frame count
    want = sorted((b, f) for b in range(w.B) for f in range(f0, f1) if not pad[b, f])
    assert sorted(zip(ep.tolist(), fr.tolist())) == want
    for b, f, k in zip(ep, fr, nk):
        assert k == key_frames(w, int(b), int(f))
    # n_sms = 0 is longest first (ties in episode, frame order); any other order is a
    # permutation of it that the dispatch replay scores no worse
    assert np.all(np.diff(nk0) <= 0)
    assert sorted(zip(ep0.tolist(), fr0.tolist(), nk0.tolist())) == \
        sorted(zip(ep.tolist(), fr.tolist(), nk.tolist()))
    if sms > 0:
        assert makespan(nk, w, sms) <= makespan(nk0, w, sms)


def test_history_pass_of_the_19_2s_chunk_on_148_sms():
    # 5 valid history frames (19 of 24 padded): items of 5, 4, 3, 2, 1 key frames, 72 CTAs
    # each on 148 SMs.  Longest first leaves the 72 one-frame CTAs in a last wave; the order
    # picked runs the two-frame items right behind the five-frame ones.
    w, lay = layout_of("ctx19.2s_bf16")
    ep, fr, nk = wam.debug_prefill_order(lay, 0, w.F_h, B200_SMS)
    assert nk.tolist() == [5, 2, 4, 3, 1]
    assert fr.tolist() == [23, 20, 22, 21, 19] and ep.tolist() == [0] * 5
    assert makespan(nk, w, B200_SMS) < makespan(sorted(nk, reverse=True), w, B200_SMS)


def test_single_wave_keeps_longest_first():
    # the two imagined frames: 2 x 72 = 144 CTAs fit on 148 SMs at once
    w, lay = layout_of("ctx19.2s_bf16")
    ep, fr, nk = wam.debug_prefill_order(lay, w.F_h, w.F, B200_SMS)
    n_hist = w.F_h - int(synth.pad_mask(w).numpy()[0].sum())  # 5 valid history frames
    assert nk.tolist() == [n_hist + 2, n_hist + 1]  # each imagined frame also reads the ones before it
    assert fr.tolist() == [w.F - 1, w.F - 2]


def test_rejects_layouts_without_a_tensor_core_prefill():
    w, lay = layout_of("ctx19.2s_bf16", T=64)
    with pytest.raises(wam.WamError):
        wam.debug_prefill_order(lay, 0, w.F_h, B200_SMS)
    w, lay = layout_of("ctx19.2s_bf16")
    with pytest.raises(wam.WamError):
        wam.debug_prefill_order(lay, 3, 2, B200_SMS)


def test_repeated_and_alternating_calls_give_the_same_orders():
    # the library keeps its last answer for a repeated work list; alternating layouts and SM
    # counts must still get each one's own order
    cases = [("ctx19.2s_bf16", 0, B200_SMS), ("batched4_bf16", 0, B200_SMS),
             ("ctx19.2s_bf16", 0, 16), ("ctx38.4s_bf16", 0, B200_SMS)]
    first = {}
    for name, f0, sms in cases:
        w, lay = layout_of(name)
        first[(name, sms)] = [a.tolist() for a in wam.debug_prefill_order(lay, f0, w.F_h, sms)]
    for _ in range(2):
        for name, f0, sms in cases + cases[::-1]:
            w, lay = layout_of(name)
            got = [a.tolist() for a in wam.debug_prefill_order(lay, f0, w.F_h, sms)]
            assert got == first[(name, sms)]
            again = [a.tolist() for a in wam.debug_prefill_order(lay, f0, w.F_h, sms)]
            assert again == got


# ---- cross-frame pairing of one-wave calls


def test_one_wave_imagination_pass_pairs_its_two_frames():
    # 19.2 s: the 2 imagined frames read 7 and 6 key frames; 2 items x 3 CTAs x 24 heads = 144
    # CTAs fit on 148 SMs, so each CTA takes the same query tile of both frames
    w, lay = layout_of("ctx19.2s_bf16")
    ep, fr, nk, paired = wam.debug_prefill_order(lay, w.F_h, w.F, B200_SMS, with_pairing=True)
    assert paired
    assert list(ep) == [0, 0] and list(fr) == [w.F_h + 1, w.F_h] and list(nk) == [7, 6]


def test_multi_wave_calls_are_not_paired():
    w, lay = layout_of("ctx19.2s_bf16")
    assert not wam.debug_prefill_order(lay, 0, w.F_h, B200_SMS, with_pairing=True)[3]  # 360 CTAs
    assert not wam.debug_prefill_order(lay, w.F_h, w.F, 16, with_pairing=True)[3]      # 16 SMs
    assert not wam.debug_prefill_order(lay, w.F_h, w.F, 0, with_pairing=True)[3]


def _expected_pairing(ep, nk, T, H, sms):
    """The pairing rule restated: a one-wave call (all CTAs resident), an even number of
    128-row query tiles per frame, an even number of items in every episode, and some episode
    whose items read unequal numbers of key frames."""
    QT = T // 128
    n = len(ep)
    if QT % 2 or sms <= 0 or n < 2 or n * (QT // 2) * H > sms:
        return False
    per = {}
    for b, k in zip(ep.tolist(), nk.tolist()):
        per.setdefault(b, []).append(k)
    if any(len(v) % 2 for v in per.values()):
        return False
    return any(max(v) != min(v) for v in per.values())


def _random_call(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 4))
    H = int(rng.choice([1, 2, 4, 24]))
    T = int(rng.choice([128, 256, 384, 512, 768]))
    F = int(rng.integers(2, 9))
    pad = (rng.random((B, F)) < 0.3).astype(np.uint8)
    pad[:, -1] = 0
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    f0 = int(rng.integers(0, F - 1))
    sms = int(rng.choice([0, 16, B200_SMS, 1000, 1000]))
    return lay, f0, F, sms, T, H


@pytest.mark.parametrize("seed", range(48))
def test_pairing_rule_and_pairs(seed):
    lay, f0, F, sms, T, H = _random_call(seed)
    ep, fr, nk, paired = wam.debug_prefill_order(lay, f0, F, sms, with_pairing=True)
    ep0, fr0, nk0 = wam.debug_prefill_order(lay, f0, F, 0)
    assert paired == _expected_pairing(ep0, nk0, T, H, sms)
    # always a permutation of the longest-first items
    assert sorted(zip(ep.tolist(), fr.tolist(), nk.tolist())) == \
        sorted(zip(ep0.tolist(), fr0.tolist(), nk0.tolist()))
    if not paired:
        return
    # pairs (2i, 2i + 1): one episode, the first reading at least the second's key frames; in
    # each episode the i-th most with the i-th fewest
    per = {}
    for i in range(0, len(ep), 2):
        assert ep[i] == ep[i + 1] and nk[i] >= nk[i + 1]
        per.setdefault(int(ep[i]), []).append((int(nk[i]), int(nk[i + 1])))
    for b, pairs in per.items():
        ks = sorted((int(k) for e, k in zip(ep0, nk0) if e == b), reverse=True)
        assert sorted(pairs, reverse=True) == [(ks[i], ks[-1 - i]) for i in range(len(ks) // 2)]


def test_pairing_cases_are_exercised():
    # the random calls above include paired and unpaired ones
    flags = [wam.debug_prefill_order(*_random_call(s)[:4], with_pairing=True)[3] for s in range(48)]
    assert 5 <= sum(flags) <= 43


def test_grouped_future_frames_are_not_paired():
    # the two imagined frames in one attention block read the same key frames: equal counts,
    # nothing to balance, so the call keeps one frame per CTA pair of tiles
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    pad = synth.pad_mask(w).numpy()
    block = list(range(w.F_h)) + [w.F_h] * w.F_f
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad, block)
    ep, fr, nk, paired = wam.debug_prefill_order(lay, w.F_h, w.F, B200_SMS, with_pairing=True)
    assert not paired and list(nk) == [7, 7]
    # one frame per block (the default layout) pairs them
    lay1 = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    assert wam.debug_prefill_order(lay1, w.F_h, w.F, B200_SMS, with_pairing=True)[3]
