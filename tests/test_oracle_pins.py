"""Pins of the fp64 oracle to things other than itself: values written out by hand from the
pages (tests/golden), closed forms, library routines that the definition reduces to in special
cases, invariants, and brute force on tiny inputs.  CPU only."""

import math

import numpy as np
import pytest
import torch

from oracle import wam_oracle as O
from tests.golden import load

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- schedules

def test_video_schedule_lands_exactly_on_sigma_star():
    meta, _ = load("schedules.txt")
    n, end, *want = meta["video"]
    s = O.flow_schedule(n, end)
    assert s[0] == 1.0 and s[-1] == 0.9          # bit-exact endpoints
    assert np.all(np.diff(s) < 0)
    np.testing.assert_allclose(s, want, rtol=0, atol=1e-15)


def test_action_schedule_runs_one_to_zero():
    meta, _ = load("schedules.txt")
    n, end, *want = meta["action"]
    s = O.flow_schedule(n, end)
    assert s[0] == 1.0 and s[-1] == 0.0
    np.testing.assert_allclose(s, want, rtol=0, atol=1e-15)


def test_time_shift_closed_form():
    # s*u/(1+(s-1)u): endpoints fixed, u=1/2 -> s/(s+1)
    for s in (0.5, 3.0, 5.0):
        v = O.time_shift([0.0, 0.5, 1.0], s)
        assert v[0] == 0.0 and v[2] == 1.0
        assert abs(v[1] - s / (s + 1)) < 1e-15
    sched = O.flow_schedule(4, 0.9, shift=3.0)
    assert sched[0] == 1.0 and sched[-1] == 0.9


def test_schedule_rejects_zero_steps():
    with pytest.raises(ValueError):
        O.flow_schedule(0)


# ----------------------------------------------------------------------------- Euler

def test_euler_with_true_target_recovers_x0():
    # x_sigma = (1 - sigma) x0 + sigma eps, u = eps - x0: from x = eps at sigma = 1 the
    # full schedule must return x0 and the partial one the path point at sigma* = 0.9.
    x0, eps = RNG.standard_normal((5, 7)), RNG.standard_normal((5, 7))
    for n, end in ((10, 0.0), (4, 0.9), (2, 0.9), (3, 0.5)):
        s = O.flow_schedule(n, end)
        x = eps.copy()
        for i in range(n):
            x = O.euler_step(x, eps - x0, s[i + 1] - s[i])
        np.testing.assert_allclose(x, (1 - end) * x0 + end * eps, rtol=0, atol=1e-13)


def test_euler_with_state_dependent_field_is_exact_on_a_line():
    # For a single data point x0 the ideal velocity at x_sigma is (x_sigma - x0) / sigma;
    # trajectories are straight lines in sigma, so Euler is exact at every step.
    x0, eps = RNG.standard_normal(9), RNG.standard_normal(9)
    s = O.flow_schedule(10, 0.0)
    x = eps.copy()
    for i in range(10):
        x = O.euler_step(x, (x - x0) / s[i], s[i + 1] - s[i])
        np.testing.assert_allclose(x, (1 - s[i + 1]) * x0 + s[i + 1] * eps, atol=1e-13)


# ----------------------------------------------------------------------------- masks

@pytest.mark.parametrize("name", ["video_mask_F3_T2_pad100.txt",
                                  "video_mask_F3_T2_pad100_blocks011.txt",
                                  "video_mask_F4_T1_pad0100_call23.txt"])
def test_video_mask_matches_hand_written(name):
    meta, want = load(name)
    pad = np.array([meta["pad"]], dtype=np.uint8)
    F = pad.shape[1]
    T = want.shape[1] // F
    got = O.video_allowed(pad, meta["blocks"], T, meta["f_begin"][0], meta["f_end"][0])
    assert got.shape == (1,) + want.shape
    np.testing.assert_array_equal(got[0].astype(int), want)


def test_action_mask_matches_hand_written():
    meta, want = load("action_mask_F3_T2_pad100_nact2.txt")
    pad = np.array([meta["pad"]], dtype=np.uint8)
    got = O.action_key_allowed(pad, 2, meta["n_act"][0])
    np.testing.assert_array_equal(got.astype(int), want)
    assert O.action_key_allowed(pad, 2, 3, with_video=False).all()


@pytest.mark.parametrize("F,T,P", [(5, 3, 0), (6, 2, 2), (4, 4, 3)])
def test_video_mask_pair_counts(F, T, P):
    pad = np.zeros((2, F), np.uint8)
    pad[:, :P] = 1
    v = F - P
    m = O.video_allowed(pad, None, T, 0, F)
    assert m.sum() == 2 * T * T * v * (v + 1) // 2           # block lower triangle
    m1 = O.video_allowed(pad, [0] * F, T, 0, F)
    assert m1.sum() == 2 * (v * T) ** 2                      # one block: all valid pairs


def test_video_mask_call_slice_is_rows_of_full_call():
    pad = np.array([[1, 0, 0, 1, 0, 0]], np.uint8)
    full = O.video_allowed(pad, None, 3, 0, 6)
    part = O.video_allowed(pad, None, 3, 2, 5)
    np.testing.assert_array_equal(part[0], full[0, 6:15, :15])


def test_block_ids_validation():
    with pytest.raises(ValueError):
        O.block_ids([0, 2, 1], 3)
    with pytest.raises(ValueError):
        O.block_ids([0, 1], 3)


# ----------------------------------------------------------------------------- attention

def _sdpa(q, k, v, **kw):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), **kw)[0, 0].numpy()


def test_single_frame_is_textbook_attention():
    T, D = 12, 16
    q, k, v = (RNG.standard_normal((1, T, 1, D)) for _ in range(3))
    o = O.video_prefill(q, k, v, None, None, np.zeros((1, 1), np.uint8), None, T, 0, 1)
    np.testing.assert_allclose(o[0, :, 0], _sdpa(q[0, :, 0], k[0, :, 0], v[0, :, 0]),
                               rtol=1e-12, atol=1e-12)


def test_one_token_frames_are_causal_attention():
    F, D = 9, 8
    q, k, v = (RNG.standard_normal((1, F, 1, D)) for _ in range(3))
    o = O.video_prefill(q, k, v, None, None, np.zeros((1, F), np.uint8), None, 1, 0, F)
    np.testing.assert_allclose(o[0, :, 0], _sdpa(q[0, :, 0], k[0, :, 0], v[0, :, 0],
                                                 is_causal=True), rtol=1e-12, atol=1e-12)


def test_brute_force_tiny_with_padding_and_cache():
    # Pure-Python loops with math.exp over the predicate stated in words.
    B, H, D, T, F, fb = 2, 2, 4, 2, 4, 1
    pad = np.array([[0, 1, 0, 0], [1, 0, 0, 0]], np.uint8)
    q = RNG.standard_normal((B, (F - fb) * T, H, D))
    kn, vn = RNG.standard_normal((2, B, (F - fb) * T, H, D))
    kc, vc = RNG.standard_normal((2, B, F * T, H, D))
    got = O.video_prefill(q, kn, vn, kc, vc, pad, None, T, fb, F)
    for b in range(B):
        for h in range(H):
            for i in range(q.shape[1]):
                fq = fb + i // T
                num, den = np.zeros(D), 0.0
                for kt in range(F * T):
                    fk = kt // T
                    if pad[b, fq] or pad[b, fk] or fk > fq:
                        continue
                    kk = kc[b, kt, h] if fk < fb else kn[b, kt - fb * T, h]
                    vv = vc[b, kt, h] if fk < fb else vn[b, kt - fb * T, h]
                    w = math.exp(sum(q[b, i, h, d] * kk[d] for d in range(D)) / math.sqrt(D))
                    num, den = num + w * vv, den + w
                want = num / den if den else np.zeros(D)
                np.testing.assert_allclose(got[b, i, h], want, rtol=1e-12, atol=1e-12)


def test_two_key_closed_form_pins_the_scale():
    # q = a e1, keys +e1 and -e1, values 1 and 0: O = sigmoid(2 a / sqrt(D)).
    D, a = 16, 3.0
    q = np.zeros((1, D)); q[0, 0] = a
    k = np.zeros((2, D)); k[0, 0], k[1, 0] = 1.0, -1.0
    v = np.array([[1.0], [0.0]])
    o = O.masked_attention(q, k, v, np.ones((1, 2), bool), 1 / math.sqrt(D))
    assert abs(o[0, 0] - 1 / (1 + math.exp(-2 * a / math.sqrt(D)))) < 1e-15


def test_constant_values_and_padded_rows():
    B, H, D, T, F = 1, 1, 8, 3, 4
    pad = np.array([[1, 1, 0, 0]], np.uint8)
    q, k = RNG.standard_normal((2, B, F * T, H, D))
    v = np.full((B, F * T, H, D), 2.5)
    o = O.video_prefill(q, k, v, None, None, pad, None, T, 0, F)
    assert np.all(o[0, :2 * T] == 0.0)
    np.testing.assert_allclose(o[0, 2 * T:], 2.5, rtol=1e-14)


def test_padded_keys_and_later_frames_do_not_matter():
    B, H, D, T, F = 1, 2, 8, 2, 5
    pad = np.array([[1, 0, 1, 0, 0]], np.uint8)
    q, k, v = RNG.standard_normal((3, B, F * T, H, D))
    base = O.video_prefill(q, k, v, None, None, pad, None, T, 0, F)
    k2, v2 = k.copy(), v.copy()
    for f in (0, 2):
        k2[0, f * T:(f + 1) * T] = 1e3 * RNG.standard_normal((T, H, D))
        v2[0, f * T:(f + 1) * T] = -7.0
    np.testing.assert_array_equal(base, O.video_prefill(q, k2, v2, None, None, pad, None, T, 0, F))
    k3 = k.copy(); k3[0, 4 * T:] += 5.0
    o3 = O.video_prefill(q, k3, v, None, None, pad, None, T, 0, F)
    np.testing.assert_array_equal(base[0, :4 * T], o3[0, :4 * T])


def test_two_calls_through_the_cache_equal_one_call():
    B, H, D, T, F, Fh = 2, 2, 8, 3, 5, 3
    pad = np.array([[1, 0, 0, 0, 0], [0, 0, 0, 0, 0]], np.uint8)
    q, k, v = RNG.standard_normal((3, B, F * T, H, D))
    whole = O.video_prefill(q, k, v, None, None, pad, None, T, 0, F)
    kc = O.cache_store(np.zeros((B, F * T, H, D)), k[:, :Fh * T], pad, T, 0, Fh)
    vc = O.cache_store(np.zeros((B, F * T, H, D)), v[:, :Fh * T], pad, T, 0, Fh)
    fut = O.video_prefill(q[:, Fh * T:], k[:, Fh * T:], v[:, Fh * T:], kc, vc, pad, None, T, Fh, F)
    np.testing.assert_allclose(fut, whole[:, Fh * T:], rtol=1e-13, atol=1e-13)


def test_cache_store_skips_padding_only():
    pad = np.array([[1, 0, 0]], np.uint8)
    old = np.full((1, 6, 1, 1), -1.0)
    new = np.arange(6.0).reshape(1, 6, 1, 1)
    got = O.cache_store(old, new, pad, 2, 0, 3)
    np.testing.assert_array_equal(got.ravel(), [-1, -1, 2, 3, 4, 5])


# ----------------------------------------------------------------------------- fusion

def test_partition_of_thirty_layers_by_four():
    parts = O.interval_partition(30, 4)
    assert len(parts) == 8 and parts[0] == [0, 1, 2, 3] and parts[-1] == [28, 29]
    assert sum(len(p) for p in parts) == 30
    assert O.interaction_layers(30, 4) == [3, 7, 11, 15, 19, 23, 27, 29]
    assert O.interval_partition(4, 2) == [[0, 1], [2, 3]]
    assert O.interaction_layers(30, 1) == list(range(30))


def test_fuse_weights_closed_forms():
    w = O.fuse_weights([0.0, math.log(3.0)])
    np.testing.assert_allclose(w, [0.25, 0.75], rtol=1e-15)
    np.testing.assert_array_equal(O.fuse_weights([0.0, -np.inf, -np.inf]), [1.0, 0.0, 0.0])
    np.testing.assert_allclose(O.fuse_weights([2.0] * 4), [0.25] * 4, rtol=1e-15)
    x = RNG.standard_normal(4)
    assert abs(O.fuse_weights(x).sum() - 1.0) < 1e-15
    np.testing.assert_allclose(O.fuse_weights(x + 100.0), O.fuse_weights(x), rtol=1e-14)


def test_fusion_one_hot_reproduces_a_layer_exactly():
    layers = [RNG.standard_normal((1, 6, 2, 4)) for _ in range(4)]
    for j in range(4):
        w = np.zeros(4); w[j] = 1.0
        np.testing.assert_array_equal(O.fuse_interval(layers, w), layers[j])


def test_fusion_closed_form_and_mean():
    layers = [np.full((2, 3), float(j + 1)) for j in range(4)]
    w = np.array([0.1, 0.2, 0.3, 0.4])
    np.testing.assert_allclose(O.fuse_interval(layers, w), 3.0, rtol=1e-15)  # sum_j w_j (j+1)
    eq = O.fuse_interval(layers, O.fuse_weights([0.0] * 4))
    np.testing.assert_allclose(eq, 2.5, rtol=1e-15)
    assert O.fuse_interval(layers, w).shape == layers[0].shape       # one layer's length


# ----------------------------------------------------------------------------- action attention

def test_action_self_only_is_bidirectional_attention():
    B, n, H, D = 1, 6, 2, 8
    qa, ka, va = RNG.standard_normal((3, B, n, H, D))
    o = O.action_attention(qa, ka, va, None, None, np.zeros((1, 1), np.uint8), 4)
    for h in range(H):
        np.testing.assert_allclose(o[0, :, h], _sdpa(qa[0, :, h], ka[0, :, h], va[0, :, h]),
                                   rtol=1e-12, atol=1e-12)


def test_action_attention_equals_masked_library_attention():
    B, n, H, D, T, F = 2, 4, 2, 8, 3, 4
    pad = np.array([[1, 1, 0, 0], [0, 0, 1, 0]], np.uint8)
    qa, ka, va = RNG.standard_normal((3, B, n, H, D))
    fk, fv = RNG.standard_normal((2, B, F * T, H, D))
    o = O.action_attention(qa, ka, va, fk, fv, pad, T)
    for b in range(B):
        keep = np.concatenate([np.repeat(pad[b] == 0, T), np.ones(n, bool)])
        mask = torch.from_numpy(np.repeat(keep[None], n, axis=0))[None, None]
        for h in range(H):
            K = np.concatenate([fk[b, :, h], ka[b, :, h]])
            V = np.concatenate([fv[b, :, h], va[b, :, h]])
            want = _sdpa(qa[b, :, h], K, V, attn_mask=mask[0, 0])
            np.testing.assert_allclose(o[b, :, h], want, rtol=1e-12, atol=1e-12)


def test_action_two_buffer_merge_equals_concatenation():
    # One softmax over [video; action] equals two per-buffer softmaxes merged by their
    # log-sum-exp (the shared normalisation of Long-WAM Summary §4.2).
    n, D, Nv = 5, 8, 11
    q, ka, va = RNG.standard_normal((3, n, D))
    kv, vv = RNG.standard_normal((2, Nv, D))
    s = 1 / math.sqrt(D)
    whole = O.masked_attention(q, np.concatenate([kv, ka]), np.concatenate([vv, va]),
                               np.ones((n, Nv + n), bool), s)
    def part(k, v):
        z = s * q @ k.T
        m = z.max(1, keepdims=True)
        p = np.exp(z - m)
        return p @ v, p.sum(1, keepdims=True), m
    o1, l1, m1 = part(kv, vv)
    o2, l2, m2 = part(ka, va)
    m = np.maximum(m1, m2)
    merged = (o1 * np.exp(m1 - m) + o2 * np.exp(m2 - m)) / (l1 * np.exp(m1 - m) + l2 * np.exp(m2 - m))
    np.testing.assert_allclose(whole, merged, rtol=1e-12, atol=1e-12)


def test_action_all_video_padded_equals_self_only():
    B, n, H, D, T, F = 1, 4, 1, 8, 2, 3
    qa, ka, va = RNG.standard_normal((3, B, n, H, D))
    fk, fv = RNG.standard_normal((2, B, F * T, H, D))
    pad = np.ones((1, F), np.uint8)
    np.testing.assert_allclose(O.action_attention(qa, ka, va, fk, fv, pad, T),
                               O.action_attention(qa, ka, va, None, None, pad, T), rtol=1e-14)


# ----------------------------------------------------------------------------- chunk

def _tiny_inputs(B=1, L=4, S=2, H=2, D=4, T=2, Fh=2, Ff=2, n=3, Nv=2, Ne=3, C=3, A=2):
    r = np.random.default_rng(7)
    g = lambda *s: r.standard_normal(s)
    M = -(-L // S)
    inp = {
        "hist_q": [g(B, Fh * T, H, D) for _ in range(L)],
        "hist_k": [g(B, Fh * T, H, D) for _ in range(L)],
        "hist_v": [g(B, Fh * T, H, D) for _ in range(L)],
        "imag_q": [[g(B, Ff * T, H, D) for _ in range(L)] for _ in range(Nv)],
        "imag_k": [[g(B, Ff * T, H, D) for _ in range(L)] for _ in range(Nv)],
        "imag_v": [[g(B, Ff * T, H, D) for _ in range(L)] for _ in range(Nv)],
        "final_q": [g(B, Ff * T, H, D) for _ in range(L)],
        "final_k": [g(B, Ff * T, H, D) for _ in range(L)],
        "final_v": [g(B, Ff * T, H, D) for _ in range(L)],
        "fuse_weights": [O.fuse_weights(g(len(I))) for I in O.interval_partition(L, S)],
        "act_q": [[g(B, n, H, D) for _ in range(L)] for _ in range(Ne)],
        "act_k": [[g(B, n, H, D) for _ in range(L)] for _ in range(Ne)],
        "act_v": [[g(B, n, H, D) for _ in range(L)] for _ in range(Ne)],
        "x_future": g(B, Ff * T, C), "v_future": [g(B, Ff * T, C) for _ in range(Nv)],
        "x_act": g(B, n, A), "v_act": [g(B, n, A) for _ in range(Ne)],
    }
    kw = dict(L=L, S=S, T=T, F_h=Fh, F_f=Ff, n_video_steps=Nv, n_euler_steps=Ne, sigma_star=0.9)
    return inp, kw, M


def test_chunk_composes_the_stage_definitions():
    inp, kw, M = _tiny_inputs()
    pad = np.array([[1, 0, 0, 0]], np.uint8)
    out = O.chunk(inp, pad=pad, **kw)
    L, T, Fh, Ff = kw["L"], kw["T"], kw["F_h"], kw["F_f"]
    # Euler chains close in one sum of dsigma * v
    s_a = O.flow_schedule(kw["n_euler_steps"])
    want = inp["x_act"] + sum((s_a[i + 1] - s_a[i]) * inp["v_act"][i]
                              for i in range(kw["n_euler_steps"]))
    np.testing.assert_allclose(out["x_act"], want, atol=1e-13)
    s_v = O.flow_schedule(kw["n_video_steps"], 0.9)
    want = inp["x_future"] - 0.1 * sum(inp["v_future"]) / kw["n_video_steps"]
    np.testing.assert_allclose(out["x_future"], want, atol=1e-13)
    assert abs(s_v[-1] - s_v[0] + 0.1) < 1e-15
    # per-layer cache of valid frames = that layer's history / final-pass K
    for l in range(L):
        np.testing.assert_array_equal(out["k_cache"][l][:, T:Fh * T], inp["hist_k"][l][:, T:])
        np.testing.assert_array_equal(out["v_cache"][l][:, Fh * T:], inp["final_v"][l])
    # fused pair m = weighted sum of its interval's caches
    for m, I in enumerate(O.interval_partition(L, kw["S"])):
        fk = sum(w * out["k_cache"][j] for w, j in zip(inp["fuse_weights"][m], I))
        np.testing.assert_allclose(out["fused_k"][m], fk, atol=1e-14)
    # layers outside the interaction set never read video
    for i in range(kw["n_euler_steps"]):
        for l in range(L):
            if l in O.interaction_layers(L, kw["S"]):
                continue
            so = O.action_attention(inp["act_q"][i][l], inp["act_k"][i][l], inp["act_v"][i][l],
                                    None, None, pad, T)
            np.testing.assert_array_equal(out["act_o"][i][l], so)
    # imagination outputs read the history cache of their own layer
    l = 1
    whole_q = np.concatenate([inp["hist_q"][l], inp["imag_q"][0][l]], axis=1)
    whole_k = np.concatenate([inp["hist_k"][l], inp["imag_k"][0][l]], axis=1)
    whole_v = np.concatenate([inp["hist_v"][l], inp["imag_v"][0][l]], axis=1)
    one = O.video_prefill(whole_q, whole_k, whole_v, None, None, pad, None, T, 0, Fh + Ff)
    np.testing.assert_allclose(out["imag_o"][0][l], one[:, Fh * T:], atol=1e-13)


def _bf_attend(q, keys, vals):
    """softmax(q k^T / sqrt(D)) v for one query row, with plain loops and math.exp."""
    D = len(q)
    sc = [sum(q[d] * k[d] for d in range(D)) / math.sqrt(D) for k in keys]
    mx = max(sc)
    e = [math.exp(x - mx) for x in sc]
    z = sum(e)
    return [sum(e[j] * vals[j][d] for j in range(len(keys))) / z for d in range(len(vals[0]))]


def _bf_video(q, kn, vn, kc, vc, f0, f1, pad, T):
    """A video pass over query frames [f0, f1): a query of frame f reads every non-padded frame
    <= f (R2-R3), from the cache below f0 and from the call's own K/V from f0 on; padded query
    frames stay 0."""
    B, _, H, _ = np.shape(q)
    o = np.zeros(np.shape(q))
    for b in range(B):
        for f in range(f0, f1):
            if pad[b][f]:
                continue
            src = [(g, t) for g in range(f + 1) if not pad[b][g] for t in range(T)]
            for h in range(H):
                keys = [list(kc[b, g * T + t, h]) if g < f0 else list(kn[b, (g - f0) * T + t, h]) for g, t in src]
                vals = [list(vc[b, g * T + t, h]) if g < f0 else list(vn[b, (g - f0) * T + t, h]) for g, t in src]
                for t in range(T):
                    row = (f - f0) * T + t
                    o[b, row, h] = _bf_attend(list(q[b, row, h]), keys, vals)
    return o


def _bf_store(cache, new, f0, f1, pad, T):
    """The cache with frames [f0, f1) that are not padding taken from the call's K or V."""
    c = np.array(cache, dtype=np.float64)
    for b in range(c.shape[0]):
        for f in range(f0, f1):
            if not pad[b][f]:
                c[b, f * T:(f + 1) * T] = new[b, (f - f0) * T:(f - f0 + 1) * T]
    return c


def _bf_action(qa, ka, va, fk, fv, pad, T, F):
    """Action queries over the non-padded frames of a fused pair (when the layer reads one,
    R9) followed by the action keys."""
    B, n, H, _ = np.shape(qa)
    o = np.zeros(np.shape(qa))
    for b in range(B):
        for h in range(H):
            keys, vals = [], []
            if fk is not None:
                for g in range(F):
                    if not pad[b][g]:
                        keys += [list(fk[b, g * T + t, h]) for t in range(T)]
                        vals += [list(fv[b, g * T + t, h]) for t in range(T)]
            keys += [list(ka[b, j, h]) for j in range(n)]
            vals += [list(va[b, j, h]) for j in range(n)]
            for r in range(n):
                o[b, r, h] = _bf_attend(list(qa[b, r, h]), keys, vals)
    return o


def _bf_intervals(L, S):
    """I_m = {S m, .., min(S m + S, L) - 1}; the interaction layer of I_m is its last (R5)."""
    iv = [list(range(S * m, min(S * m + S, L))) for m in range(-(-L // S))]
    return iv, {I[-1]: m for m, I in enumerate(iv)}


def _bf_history(inp, pad, L, T, Fh, F):
    B, _, H, D = np.shape(inp["hist_q"][0])
    kc = [np.zeros((B, F * T, H, D)) for _ in range(L)]
    vc = [np.zeros((B, F * T, H, D)) for _ in range(L)]
    outs = []
    for l in range(L):
        outs.append(_bf_video(inp["hist_q"][l], inp["hist_k"][l], inp["hist_v"][l], kc[l], vc[l], 0, Fh, pad, T))
        kc[l], vc[l] = _bf_store(kc[l], inp["hist_k"][l], 0, Fh, pad, T), _bf_store(vc[l], inp["hist_v"][l], 0, Fh, pad, T)
    return outs, kc, vc


def _bf_chunk(inp, pad, L, S, T, Fh, Ff, Nv, Ne, sigma_star):
    """One chunk restated from the readings with loops and math.exp, calling nothing of the
    oracle: the history pass over frames [0, Fh), its K/V stored for non-padded frames; Nv
    imagination passes over the stored history and their own future K/V, each followed by an
    Euler step of -(1 - sigma*) / Nv on the future latents (R1, R7); the final pass, its K/V
    stored (R6); fused pair m = sum of w_m,j x cache_j over I_m (R5); Ne action steps where
    layer max(I_m) reads fused pair m and the other layers the action keys only, each followed
    by an Euler step of -1 / Ne."""
    F = Fh + Ff
    out = {"imag_o": [], "final_o": [], "act_o": []}
    out["hist_o"], kc, vc = _bf_history(inp, pad, L, T, Fh, F)
    x = np.array(inp["x_future"], dtype=np.float64)
    for s in range(Nv):
        out["imag_o"].append([_bf_video(inp["imag_q"][s][l], inp["imag_k"][s][l], inp["imag_v"][s][l],
                                        kc[l], vc[l], Fh, F, pad, T) for l in range(L)])
        x = x - (1.0 - sigma_star) / Nv * np.asarray(inp["v_future"][s])
    out["x_future"] = x
    for l in range(L):
        out["final_o"].append(_bf_video(inp["final_q"][l], inp["final_k"][l], inp["final_v"][l], kc[l], vc[l],
                                        Fh, F, pad, T))
        kc[l], vc[l] = _bf_store(kc[l], inp["final_k"][l], Fh, F, pad, T), _bf_store(vc[l], inp["final_v"][l], Fh, F, pad, T)
    out["k_cache"], out["v_cache"] = kc, vc
    iv, reader = _bf_intervals(L, S)
    out["fused_k"] = [sum(w * kc[j] for w, j in zip(inp["fuse_weights"][m], I)) for m, I in enumerate(iv)]
    out["fused_v"] = [sum(w * vc[j] for w, j in zip(inp["fuse_weights"][m], I)) for m, I in enumerate(iv)]
    xa = np.array(inp["x_act"], dtype=np.float64)
    for i in range(Ne):
        out["act_o"].append([_bf_action(inp["act_q"][i][l], inp["act_k"][i][l], inp["act_v"][i][l],
                                        out["fused_k"][reader[l]] if l in reader else None,
                                        out["fused_v"][reader[l]] if l in reader else None, pad, T, F)
                             for l in range(L)])
        xa = xa - 1.0 / Ne * np.asarray(inp["v_act"][i])
    out["x_act"] = xa
    return out


def _bf_chunk_joint(inp, pad, L, S, T, Fh, Ff, N):
    """The co-denoising chunk restated (R10): the history pass once; at joint step i every layer
    passes the future frames with that step's Q/K/V and stores their K/V, the fused pairs are
    formed from the caches, every action layer reads, and both latents take an Euler step of
    -1 / N."""
    F = Fh + Ff
    out = {"joint_o": [], "act_o": []}
    out["hist_o"], kc, vc = _bf_history(inp, pad, L, T, Fh, F)
    iv, reader = _bf_intervals(L, S)
    x = np.array(inp["x_future"], dtype=np.float64)
    xa = np.array(inp["x_act"], dtype=np.float64)
    for i in range(N):
        outs = []
        for l in range(L):
            outs.append(_bf_video(inp["joint_q"][i][l], inp["joint_k"][i][l], inp["joint_v"][i][l], kc[l], vc[l],
                                  Fh, F, pad, T))
            kc[l] = _bf_store(kc[l], inp["joint_k"][i][l], Fh, F, pad, T)
            vc[l] = _bf_store(vc[l], inp["joint_v"][i][l], Fh, F, pad, T)
        out["joint_o"].append(outs)
        fk = [sum(w * kc[j] for w, j in zip(inp["fuse_weights"][m], I)) for m, I in enumerate(iv)]
        fv = [sum(w * vc[j] for w, j in zip(inp["fuse_weights"][m], I)) for m, I in enumerate(iv)]
        out["act_o"].append([_bf_action(inp["act_q"][i][l], inp["act_k"][i][l], inp["act_v"][i][l],
                                        fk[reader[l]] if l in reader else None,
                                        fv[reader[l]] if l in reader else None, pad, T, F) for l in range(L)])
        x = x - 1.0 / N * np.asarray(inp["v_future"][i])
        xa = xa - 1.0 / N * np.asarray(inp["v_act"][i])
    out.update(k_cache=kc, v_cache=vc, fused_k=fk, fused_v=fv, x_future=x, x_act=xa)
    return out


def _assert_same_chunk(got, want, lists, nested):
    for key in lists:
        assert len(got[key]) == len(want[key])
        for a, b in zip(got[key], want[key]):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    for key in nested:
        assert len(got[key]) == len(want[key])
        for ra, rb in zip(got[key], want[key]):
            for a, b in zip(ra, rb):
                np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["x_future"], want["x_future"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(got["x_act"], want["x_act"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("pad_row", [[1, 0, 0, 0], [0, 0, 0, 0]])
def test_chunk_matches_a_brute_force_restatement(pad_row):
    inp, kw, M = _tiny_inputs()
    pad = np.array([pad_row], np.uint8)
    got = O.chunk(inp, pad=pad, **kw)
    want = _bf_chunk(inp, pad, kw["L"], kw["S"], kw["T"], kw["F_h"], kw["F_f"], kw["n_video_steps"],
                     kw["n_euler_steps"], kw["sigma_star"])
    _assert_same_chunk(got, want, ("hist_o", "final_o", "k_cache", "v_cache", "fused_k", "fused_v"),
                       ("imag_o", "act_o"))


def test_action_never_changes_video_outputs():
    inp, kw, _ = _tiny_inputs()
    pad = np.zeros((1, 4), np.uint8)
    a = O.chunk(inp, pad=pad, **kw)
    inp2 = dict(inp)
    inp2["act_k"] = [[x + 3.0 for x in row] for row in inp["act_k"]]
    inp2["act_v"] = [[x - 2.0 for x in row] for row in inp["act_v"]]
    b = O.chunk(inp2, pad=pad, **kw)
    for key in ("hist_o", "final_o"):
        for x, y in zip(a[key], b[key]):
            np.testing.assert_array_equal(x, y)
    for m in range(len(a["fused_k"])):
        np.testing.assert_array_equal(a["fused_k"][m], b["fused_k"][m])


# ----------------------------------------------------------------------------- co-denoising

def _joint_inputs(N=3, **kw):
    inp, ckw, M = _tiny_inputs(Nv=N, Ne=N, **kw)
    # the joint steps re-use the tiny imagination draws as their future Q/K/V
    inp["joint_q"], inp["joint_k"], inp["joint_v"] = inp["imag_q"], inp["imag_k"], inp["imag_v"]
    jkw = {k: ckw[k] for k in ("L", "S", "T", "F_h", "F_f")}
    return inp, jkw, N


@pytest.mark.parametrize("pad_row", [[1, 0, 0, 0], [0, 0, 0, 0]])
def test_joint_chunk_matches_a_brute_force_restatement(pad_row):
    inp, jkw, N = _joint_inputs(N=3)
    pad = np.array([pad_row], np.uint8)
    got = O.chunk_joint(inp, n_steps=N, pad=pad, **jkw)
    want = _bf_chunk_joint(inp, pad, jkw["L"], jkw["S"], jkw["T"], jkw["F_h"], jkw["F_f"], N)
    _assert_same_chunk(got, want, ("hist_o", "k_cache", "v_cache", "fused_k", "fused_v"), ("joint_o", "act_o"))


def test_joint_chunk_of_one_step_is_the_one_shot_chunk():
    # One joint step: the history pass, one future pass whose K/V fill the cache, the fused
    # pairs, one action step and one Euler step 1 -> 0 -- the IDM chunk with no imagination step
    # whose cache pass takes the same future Q/K/V.
    inp, jkw, _ = _joint_inputs(N=1)
    pad = np.array([[1, 0, 0, 0]], np.uint8)
    joint = O.chunk_joint(inp, n_steps=1, pad=pad, **jkw)
    idm_inp = dict(inp, final_q=inp["joint_q"][0], final_k=inp["joint_k"][0], final_v=inp["joint_v"][0])
    idm = O.chunk(idm_inp, n_video_steps=0, n_euler_steps=1, sigma_star=1.0, pad=pad, **jkw)
    for x, y in zip(joint["hist_o"], idm["hist_o"]):
        np.testing.assert_array_equal(x, y)
    for x, y in zip(joint["joint_o"][0], idm["final_o"]):
        np.testing.assert_array_equal(x, y)
    for key in ("k_cache", "v_cache", "fused_k", "fused_v"):
        for x, y in zip(joint[key], idm[key]):
            np.testing.assert_array_equal(x, y)
    for x, y in zip(joint["act_o"][0], idm["act_o"][0]):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(joint["x_act"], idm["x_act"])


def test_joint_chunk_steps_only_see_their_own_and_earlier_inputs():
    inp, jkw, N = _joint_inputs(N=3)
    pad = np.zeros((1, 4), np.uint8)
    a = O.chunk_joint(inp, n_steps=N, pad=pad, **jkw)
    inp2 = dict(inp)
    inp2["joint_k"] = inp["joint_k"][:2] + [[x + 5.0 for x in inp["joint_k"][2]]]
    inp2["joint_v"] = inp["joint_v"][:2] + [[x - 1.0 for x in inp["joint_v"][2]]]
    b = O.chunk_joint(inp2, n_steps=N, pad=pad, **jkw)
    for i in range(2):
        for key in ("joint_o", "act_o"):
            for x, y in zip(a[key][i], b[key][i]):
                np.testing.assert_array_equal(x, y)
    # the last step's future K/V are what the caches hold at the end
    T, Fh = jkw["T"], jkw["F_h"]
    for l in range(jkw["L"]):
        np.testing.assert_array_equal(b["k_cache"][l][:, Fh * T:], inp2["joint_k"][2][l])


def test_joint_chunk_euler_recovers_the_clean_latents():
    # With the true flow-matching velocity u = eps - x0 and the start x = eps, the shared
    # schedule 1 -> 0 brings both latents back to x0 (closed form of the path).
    inp, jkw, N = _joint_inputs(N=4)
    r = np.random.default_rng(3)
    x0f, epsf = r.standard_normal(inp["x_future"].shape), r.standard_normal(inp["x_future"].shape)
    x0a, epsa = r.standard_normal(inp["x_act"].shape), r.standard_normal(inp["x_act"].shape)
    inp = dict(inp, x_future=epsf, v_future=[epsf - x0f] * N, x_act=epsa, v_act=[epsa - x0a] * N)
    out = O.chunk_joint(inp, n_steps=N, pad=np.zeros((1, 4), np.uint8), **jkw)
    np.testing.assert_allclose(out["x_future"], x0f, atol=1e-13)
    np.testing.assert_allclose(out["x_act"], x0a, atol=1e-13)


# ----------------------------------------------------------------------------- streamed chunks

@pytest.mark.parametrize("p_prev,p_next", [(2, 1), (0, 0)], ids=["window_grows", "window_full"])
def test_streamed_chunk_equals_the_chunk_recomputed_over_the_slid_window(p_prev, p_next):
    # The previous chunk's caches shifted by one frame plus one pass of the newest frame give
    # exactly the chunk computed from scratch over the slid window (whose history inputs are
    # the previous ones moved one frame earlier, the oldest dropped, the newest appended).
    inp, kw, M = _tiny_inputs(Fh=4)
    L, T, Fh, Ff = kw["L"], kw["T"], kw["F_h"], kw["F_f"]
    F = Fh + Ff
    pad_prev = np.array([[1] * p_prev + [0] * (F - p_prev)], np.uint8)
    pad_next = np.array([[1] * p_next + [0] * (F - p_next)], np.uint8)
    prev = O.chunk(inp, pad=pad_prev, **kw)
    r = np.random.default_rng(11)
    new = {n: [r.standard_normal((1, T) + inp["hist_k"][0].shape[2:]) for _ in range(L)] for n in ("q", "k", "v")}
    step = dict(inp, new_q=new["q"], new_k=new["k"], new_v=new["v"])
    got = O.chunk_stream(prev, step, pad=pad_next, **kw)
    slid = dict(inp)
    for n in ("q", "k", "v"):
        slid["hist_" + n] = [np.concatenate([inp["hist_" + n][l][:, T:], new[n][l]], axis=1) for l in range(L)]
    want = O.chunk(slid, pad=pad_next, **kw)
    for l in range(L):
        np.testing.assert_allclose(got["hist_o"][l], want["hist_o"][l][:, (Fh - 1) * T:], atol=1e-13)
    for key in ("k_cache", "v_cache", "fused_k", "fused_v"):
        for x, y in zip(got[key], want[key]):
            np.testing.assert_allclose(x, y, atol=1e-13)
    for key in ("imag_o", "act_o"):
        for xs, ys in zip(got[key], want[key]):
            for x, y in zip(xs, ys):
                np.testing.assert_allclose(x, y, atol=1e-13)
    for x, y in zip(got["final_o"], want["final_o"]):
        np.testing.assert_allclose(x, y, atol=1e-13)
