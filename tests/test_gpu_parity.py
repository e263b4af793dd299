"""GPU parity: every C-ABI entry point against the fp64 oracle on the same seeded inputs.

Sizes span several tiles, frames and a ragged tail; the checks cover both kernel paths
(CUDA-core fp32/bf16 and tensor-core bf16), padding (prefix and scattered), grouped attention
blocks, the cache store, the fusion epilogue, the standalone fusion, the action read with and
without video, and the degenerate cases (one frame, one action token, all-but-one padded)."""

import numpy as np
import pytest
import torch

from oracle import wam_oracle as O
from cached_kv_attention_b200 import wam
from tests.gpu_util import assert_parity, dev_normal, to64, valid_rows

pytestmark = pytest.mark.gpu

SENTINEL = 12288.0  # exactly representable in bf16 and fp32


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    wam.device_error(clear=True)


# ----------------------------------------------------------------------------- Euler

@pytest.mark.parametrize("n", [1, 3, 4, 17, 1000, (1 << 20) + 3])
def test_euler_step(n):
    x = dev_normal((n,), 11, "x", n)
    v = dev_normal((n,), 11, "v", n)
    ref = O.euler_step(to64(x), to64(v), -0.1)
    wam.flow_euler_step(x, v, -0.1)
    assert_parity(to64(x), ref, "f32", "euler")


def test_euler_full_schedule_recovers_x0_on_gpu():
    x0 = dev_normal((4096,), 12, "x0")
    eps = dev_normal((4096,), 12, "eps")
    x, u = eps.clone(), eps - x0
    s = wam.flow_schedule(10, 0.0)
    for i in range(10):
        wam.flow_euler_step(x, u, float(s[i + 1] - s[i]))
    assert_parity(to64(x), to64(x0), "f32", "euler recovery")


# ----------------------------------------------------------------------------- masks

MASK_CASES = [
    # B, T, pad rows, blocks, calls
    (1, 2, [[1, 0, 0]], None, [(0, 3), (1, 3), (2, 3)]),
    (3, 3, [[0, 1, 0, 0, 1, 0], [1, 1, 0, 0, 0, 0], [0, 0, 0, 0, 0, 0]], None, [(0, 6), (2, 5)]),
    (2, 2, [[1, 0, 0, 0, 0], [0, 0, 1, 0, 0]], [0, 1, 2, 3, 3], [(0, 3), (3, 5), (0, 5)]),
    (1, 4, [[0, 0, 0, 0]], [0, 0, 1, 1], [(0, 2), (2, 4), (0, 4)]),
]


@pytest.mark.parametrize("B,T,pad,blocks,calls", MASK_CASES)
def test_video_mask_bit_exact(B, T, pad, blocks, calls):
    F = len(pad[0])
    lay = wam.VideoLayout(B, 1, 64, T, F, pad, blocks)
    for fb, fe in calls:
        got = wam.debug_video_mask(lay, fb, fe).cpu().numpy().astype(bool)
        want = O.video_allowed(np.array(pad, np.uint8), blocks, T, fb, fe)
        np.testing.assert_array_equal(got, want)


# ----------------------------------------------------------------------------- prefill

def _prefill_case(B, H, D, T, F, F_h, pad, blocks, dtype, std, seed, fuse=None):
    """History call [0, F_h) then future call [F_h, F) through the cache; returns GPU and
    oracle results."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    lay = wam.VideoLayout(B, H, D, T, F, pad, blocks)
    pad = np.array(pad, np.uint8)
    N = F * T
    g = lambda name, tok, *i: dev_normal((B, tok, H, D), seed, name, *i, std=std, dtype=tdt)
    qh, kh, vh = g("qh", F_h * T), g("kh", F_h * T), g("vh", F_h * T)
    qf, kf, vf = g("qf", (F - F_h) * T), g("kf", (F - F_h) * T), g("vf", (F - F_h) * T)
    kc = torch.full((B, N, H, D), SENTINEL, dtype=tdt, device="cuda")
    vc = torch.full((B, N, H, D), SENTINEL, dtype=tdt, device="cuda")
    oh = torch.full((B, F_h * T, H, D), SENTINEL, device="cuda")
    of = torch.full((B, (F - F_h) * T, H, D), SENTINEL, device="cuda")
    wam.video_prefill_kv(lay, 0, F_h, qh, kh, vh, kc, vc, oh, store_kv=True)
    wam.video_prefill_kv(lay, F_h, F, qf, kf, vf, kc, vc, of, store_kv=True)
    torch.cuda.synchronize()
    z = np.zeros((B, N, H, D))
    kc_ref = O.cache_store(z, to64(kh), pad, T, 0, F_h)
    vc_ref = O.cache_store(z, to64(vh), pad, T, 0, F_h)
    oh_ref = O.video_prefill(to64(qh), to64(kh), to64(vh), None, None, pad, blocks, T, 0, F_h)
    of_ref = O.video_prefill(to64(qf), to64(kf), to64(vf), kc_ref, vc_ref, pad, blocks, T, F_h, F)
    kc_ref = O.cache_store(kc_ref, to64(kf), pad, T, F_h, F)
    return dict(lay=lay, pad=pad, oh=oh, of=of, kc=kc, vc=vc, oh_ref=oh_ref, of_ref=of_ref,
                kc_ref=kc_ref, kh=kh, kf=kf)


def _check_prefill(r, T, F_h, F, dtype):
    pad = r["pad"]
    rows_h, rows_f = valid_rows(pad, T, 0, F_h), valid_rows(pad, T, F_h, F)
    oh, of = to64(r["oh"]), to64(r["of"])
    assert_parity(oh[rows_h], r["oh_ref"][rows_h], dtype, "history O")
    assert_parity(of[rows_f], r["of_ref"][rows_f], dtype, "future O")
    # rows of padding frames are not written
    assert np.all(oh[~rows_h] == SENTINEL) and np.all(of[~rows_f] == SENTINEL)
    # the cache holds the new K of every valid frame bit-exactly; padded frames untouched
    kc = to64(r["kc"])
    krow = valid_rows(pad, T, 0, F)
    np.testing.assert_array_equal(kc[krow], r["kc_ref"][krow])
    assert np.all(kc[~krow] == SENTINEL)


SIMT_CASES = [
    # B, H, D, T, F, F_h, pad, blocks, dtype, std
    (1, 2, 64, 16, 4, 2, [[0, 0, 0, 0]], None, "f32", 1.0),          # the tiny fp32 shape
    (2, 3, 128, 13, 5, 3, [[1, 0, 0, 0, 0], [0, 1, 0, 0, 0]], None, "f32", 1.0),
    (1, 2, 64, 7, 6, 4, [[1, 1, 1, 0, 0, 0]], [0, 1, 2, 3, 4, 4], "f32", 2.0),
    (2, 2, 128, 24, 4, 2, [[0, 0, 0, 0], [1, 0, 0, 0]], None, "bf16", 1.0),
    (1, 1, 64, 1, 3, 1, [[0, 0, 0]], None, "f32", 1.0),               # one token per frame
]


@pytest.mark.parametrize("B,H,D,T,F,F_h,pad,blocks,dtype,std", SIMT_CASES)
def test_prefill_cuda_core_path(B, H, D, T, F, F_h, pad, blocks, dtype, std):
    r = _prefill_case(B, H, D, T, F, F_h, pad, blocks, dtype, std, seed=21)
    _check_prefill(r, T, F_h, F, dtype)


TC_CASES = [
    # B, H, T, F, F_h, pad, blocks, std
    (1, 2, 128, 3, 2, [[0, 0, 0]], None, 1 / np.sqrt(128)),          # near-uniform softmax
    (2, 3, 128, 5, 3, [[1, 0, 0, 0, 0], [0, 0, 1, 0, 0]], None, 1.0),  # logit std ~ 1
    (2, 2, 256, 5, 3, [[1, 1, 0, 0, 0], [0, 0, 0, 0, 0]], [0, 1, 2, 3, 3], 2.0),  # peaky
    (1, 2, 768, 4, 2, [[0, 0, 0, 0]], None, 1 / np.sqrt(128)),         # 768 tokens per frame
    (1, 1, 128, 1, 1, [[0]], None, 1.0),                               # a single frame
]


@pytest.mark.parametrize("B,H,T,F,F_h,pad,blocks,std", TC_CASES)
def test_prefill_tensor_core_path(B, H, T, F, F_h, pad, blocks, std):
    if F_h == F:
        lay = wam.VideoLayout(B, H, 128, T, F, pad, blocks)
        q, k, v = (dev_normal((B, F * T, H, 128), 31, n, std=std, dtype=torch.bfloat16)
                   for n in "qkv")
        kc = torch.zeros_like(k)
        o = torch.zeros((B, F * T, H, 128), device="cuda")
        wam.video_prefill_kv(lay, 0, F, q, k, v, kc, kc.clone(), o)
        ref = O.video_prefill(to64(q), to64(k), to64(v), None, None, np.array(pad), blocks, T, 0, F)
        assert_parity(to64(o), ref, "bf16", "single frame")
        return
    r = _prefill_case(B, H, 128, T, F, F_h, pad, blocks, "bf16", std, seed=22)
    _check_prefill(r, T, F_h, F, "bf16")


@pytest.mark.parametrize("dtype,T", [("f32", 16), ("bf16", 128), ("bf16", 24)])
def test_fusion_epilogue_over_an_interval(dtype, T):
    B, H, D, F = 2, 2, 128, 3
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    pad = np.array([[1, 0, 0], [0, 0, 0]], np.uint8)
    lay = wam.VideoLayout(B, H, D, T, F, pad)
    N = F * T
    acc_k = torch.zeros((B, N, H, D), device="cuda")
    acc_v = torch.zeros_like(acc_k)
    fk = torch.full((B, N, H, D), SENTINEL, dtype=tdt, device="cuda")
    fv = torch.full_like(fk, SENTINEL)
    logits = np.array([0.3, -1.2, 0.8], np.float32)
    w = wam.fuse_weights(logits)
    ks, vs = [], []
    for j in range(3):
        q, k, v = (dev_normal((B, N, H, D), 41, n, j, dtype=tdt) for n in "qkv")
        kc, vc = torch.zeros_like(k), torch.zeros_like(v)
        o = torch.zeros((B, N, H, D), device="cuda")
        epi = wam.FuseEpilogue(w[j], j == 0, j == 2, acc_k, acc_v, fk, fv)
        wam.video_prefill_kv(lay, 0, F, q, k, v, kc, vc, o, fuse=epi)
        ks.append(to64(k)), vs.append(to64(v))
    torch.cuda.synchronize()
    w64 = O.fuse_weights(logits.astype(np.float64))
    rows = valid_rows(pad, T, 0, F)
    assert_parity(to64(fk)[rows], O.fuse_interval(ks, w64)[rows], dtype, "fused K")
    assert_parity(to64(fv)[rows], O.fuse_interval(vs, w64)[rows], dtype, "fused V")
    assert np.all(to64(fk)[~rows] == SENTINEL)


@pytest.mark.parametrize("T", [16, 128])
def test_fusion_epilogue_one_hot_is_exact(T):
    B, H, D, F = 1, 2, 128, 2
    lay = wam.VideoLayout(B, H, D, T, F)
    N = F * T
    acc = torch.zeros((B, N, H, D), device="cuda")
    acc2 = torch.zeros_like(acc)
    fk = torch.zeros((B, N, H, D), dtype=torch.bfloat16, device="cuda")
    fv = torch.zeros_like(fk)
    keep = None
    for j, wj in enumerate([0.0, 1.0, 0.0]):
        q, k, v = (dev_normal((B, N, H, D), 42, n, j, dtype=torch.bfloat16) for n in "qkv")
        o = torch.zeros((B, N, H, D), device="cuda")
        epi = wam.FuseEpilogue(wj, j == 0, j == 2, acc, acc2, fk, fv)
        wam.video_prefill_kv(lay, 0, F, q, k, v, torch.zeros_like(k), torch.zeros_like(v), o, fuse=epi)
        if j == 1:
            keep = (k.clone(), v.clone())
    torch.cuda.synchronize()
    assert torch.equal(fk, keep[0]) and torch.equal(fv, keep[1])


# ----------------------------------------------------------------------------- standalone fusion

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_standalone_fusion(dtype):
    B, H, D, T, F = 2, 3, 64, 8, 4
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    pad = np.array([[1, 0, 0, 0], [0, 0, 1, 0]], np.uint8)
    lay = wam.VideoLayout(B, H, D, T, F, pad)
    ks = [dev_normal((B, F * T, H, D), 51, "k", j, dtype=tdt) for j in range(4)]
    vs = [dev_normal((B, F * T, H, D), 51, "v", j, dtype=tdt) for j in range(4)]
    logits = np.array([0.1, 0.7, -0.4, 1.5], np.float32)
    w = wam.fuse_weights(logits)
    fk = torch.full_like(ks[0], SENTINEL)
    fv = torch.full_like(vs[0], SENTINEL)
    wam.fuse_interval_kv(lay, ks, vs, w, 0, F, fk, fv)
    w64 = O.fuse_weights(logits.astype(np.float64))
    rows = valid_rows(pad, T, 0, F)
    assert_parity(to64(fk)[rows], O.fuse_interval([to64(k) for k in ks], w64)[rows], dtype, "K")
    assert_parity(to64(fv)[rows], O.fuse_interval([to64(v) for v in vs], w64)[rows], dtype, "V")
    assert np.all(to64(fk)[~rows] == SENTINEL)
    # one-hot weights reproduce one layer bit-exactly
    wam.fuse_interval_kv(lay, ks, vs, [0.0, 0.0, 1.0, 0.0], 0, F, fk, fv)
    torch.cuda.synchronize()
    assert np.array_equal(to64(fk)[rows], to64(ks[2])[rows])


# ----------------------------------------------------------------------------- action read

ACTION_CASES = [
    # B, H, D, T, F, n_act, pad, dtype, std, video
    (1, 2, 64, 16, 4, 8, [[0, 0, 0, 0]], "f32", 1.0, True),      # the tiny fp32 shape
    (1, 2, 64, 16, 4, 8, [[0, 0, 0, 0]], "f32", 1.0, False),
    (2, 3, 128, 64, 5, 32, [[1, 1, 0, 0, 0], [0, 0, 1, 0, 0]], "bf16", 1 / np.sqrt(128), True),
    (2, 3, 128, 128, 5, 17, [[1, 0, 0, 0, 0], [0, 0, 0, 0, 0]], "bf16", 1.0, True),
    (1, 4, 128, 768, 7, 32, [[0] * 7], "bf16", 1 / np.sqrt(128), True),   # 16 splits
    (1, 24, 128, 768, 4, 32, [[1, 0, 0, 0]], "bf16", 2.0, True),          # peaky
    (2, 3, 128, 64, 3, 1, [[0, 0, 0], [1, 1, 0]], "bf16", 1.0, True),     # one action token
    (2, 3, 128, 64, 3, 32, [[0, 0, 0], [1, 1, 0]], "bf16", 1.0, False),   # self-only layer
    (1, 2, 128, 40, 3, 32, [[0, 1, 0]], "bf16", 1.0, True),               # T % 64 != 0
    (1, 2, 128, 64, 3, 48, [[0, 1, 0]], "bf16", 1.0, True),               # n_act > 32
    (4, 64, 128, 128, 1, 32, [[0]] * 4, "bf16", 1.0, True),               # whole (b, h) per CTA
]


@pytest.mark.parametrize("B,H,D,T,F,n_act,pad,dtype,std,video", ACTION_CASES)
def test_action_attention(B, H, D, T, F, n_act, pad, dtype, std, video):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    lay = wam.VideoLayout(B, H, D, T, F, pad)
    fk = dev_normal((B, F * T, H, D), 61, "fk", std=std, dtype=tdt) if video else None
    fv = dev_normal((B, F * T, H, D), 61, "fv", std=std, dtype=tdt) if video else None
    qa, ka, va = (dev_normal((B, n_act, H, D), 61, n, std=std, dtype=tdt) for n in ("qa", "ka", "va"))
    o = torch.full((B, n_act, H, D), SENTINEL, device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, o)
    ref = O.action_attention(to64(qa), to64(ka), to64(va), to64(fk) if video else None,
                             to64(fv) if video else None, np.array(pad), T)
    assert_parity(to64(o), ref, dtype, "action O")


# One case per cluster size of the 128-key read: the runtime co-schedules 15 clusters of 8 CTAs,
# 22 of 6, 26 of 5, 33 of 4, 45 of 3, 74 of 2 on a 148-SM B200 at this footprint, so these B x H
# give 8, 6, 5, 4, 3, 2 and 1 CTAs per (episode, head).  n_act below the cluster size leaves
# owners with no rows of the merge, and the first case (one valid 512-token frame: 5 tiles with
# the action tile, over 8 CTAs) leaves three slices with no tile at all.
MERGE_CASES = [
    # B, H, F, n_act, pad
    (1, 4, 2, 1, [[1, 0]]),
    (2, 8, 3, 5, [[0, 0, 0], [1, 0, 0]]),
    (1, 24, 3, 32, [[0, 1, 0]]),
    (1, 30, 3, 7, [[0, 0, 0]]),
    (2, 20, 3, 32, [[1, 0, 0], [0, 0, 0]]),
    (3, 20, 2, 3, [[0, 0], [0, 1], [0, 0]]),
    (4, 25, 2, 32, [[0, 0]] * 4),
]


@pytest.mark.parametrize("B,H,F,n_act,pad", MERGE_CASES)
def test_action_cluster_merge_every_split(B, H, F, n_act, pad):
    T = 512
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    fk, fv = (dev_normal((B, F * T, H, 128), 65, x, dtype=torch.bfloat16) for x in ("fk", "fv"))
    qa, ka, va = (dev_normal((B, n_act, H, 128), 65, x, dtype=torch.bfloat16) for x in ("qa", "ka", "va"))
    o = torch.full((B, n_act, H, 128), SENTINEL, device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, o)
    ref = O.action_attention(to64(qa), to64(ka), to64(va), to64(fk), to64(fv), np.array(pad), T)
    assert_parity(to64(o), ref, "bf16", f"action O, B x H = {B * H}")


@pytest.mark.parametrize("n_act", [32, 5])
def test_action_large_logit_jumps(n_act):
    # Later key frames score far above earlier ones, so each query's running reference has to
    # move in the middle of a CTA's run (and the accumulated output be rescaled) several times.
    B, H, T, F = 1, 6, 128, 8
    lay = wam.VideoLayout(B, H, 128, T, F)
    scale = torch.tensor([1.0 + 2.5 * f for f in range(F)], device="cuda").repeat_interleave(T)
    fk = dev_normal((B, F * T, H, 128), 64, "fk", dtype=torch.float32) * scale[None, :, None, None]
    fk = fk.to(torch.bfloat16)
    fv = dev_normal((B, F * T, H, 128), 64, "fv", dtype=torch.bfloat16)
    qa, ka, va = (dev_normal((B, n_act, H, 128), 64, x, dtype=torch.bfloat16) for x in ("qa", "ka", "va"))
    o = torch.full((B, n_act, H, 128), SENTINEL, device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, o)
    ref = O.action_attention(to64(qa), to64(ka), to64(va), to64(fk), to64(fv), np.zeros((1, F)), T)
    assert_parity(to64(o), ref, "bf16", "action logit jumps")


def test_action_output_in_bf16():
    B, H, T, F, n = 1, 2, 64, 3, 32
    lay = wam.VideoLayout(B, H, 128, T, F)
    fk, fv = (dev_normal((B, F * T, H, 128), 62, x, dtype=torch.bfloat16) for x in ("fk", "fv"))
    qa, ka, va = (dev_normal((B, n, H, 128), 62, x, dtype=torch.bfloat16) for x in ("qa", "ka", "va"))
    o = torch.zeros((B, n, H, 128), dtype=torch.bfloat16, device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, o)
    ref = O.action_attention(to64(qa), to64(ka), to64(va), to64(fk), to64(fv), np.zeros((1, F)), T)
    assert_parity(to64(o), ref, "bf16", "action O bf16")


# ----------------------------------------------------------------------------- invariances

def test_padded_keys_and_action_inputs_never_change_video_outputs():
    B, H, T, F, F_h = 1, 2, 128, 4, 2
    pad = [[1, 0, 0, 0]]
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    q, k, v = (dev_normal((B, F * T, H, 128), 71, n, dtype=torch.bfloat16) for n in "qkv")
    o1 = torch.zeros((B, F * T, H, 128), device="cuda")
    kc = torch.zeros_like(k)
    wam.video_prefill_kv(lay, 0, F, q, k, v, kc, kc.clone(), o1)
    k2, v2 = k.clone(), v.clone()
    k2[:, :T] = 100.0
    v2[:, :T] = -100.0
    o2 = torch.zeros_like(o1)
    wam.video_prefill_kv(lay, 0, F, q, k2, v2, kc, kc.clone(), o2)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, T:], o2[:, T:])
    # later frames never change earlier outputs
    k3 = k.clone()
    k3[:, 3 * T:] += 1.0
    o3 = torch.zeros_like(o1)
    wam.video_prefill_kv(lay, 0, F, q, k3, v, kc, kc.clone(), o3)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, T:3 * T], o3[:, T:3 * T])


def test_action_padded_frames_are_never_read():
    B, H, T, F, n = 1, 2, 64, 4, 32
    pad = [[1, 1, 0, 0]]
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    fk, fv = (dev_normal((B, F * T, H, 128), 72, x, dtype=torch.bfloat16) for x in ("fk", "fv"))
    qa, ka, va = (dev_normal((B, n, H, 128), 72, x, dtype=torch.bfloat16) for x in ("qa", "ka", "va"))
    o1 = torch.zeros((B, n, H, 128), device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, o1)
    fk[:, :2 * T] = float("nan")
    fv[:, :2 * T] = float("nan")
    o2 = torch.zeros_like(o1)
    wam.action_attn(lay, fk, fv, qa, ka, va, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_action_workspace_is_reused_and_checked():
    # 24 heads x 85 tiles over 148 CTAs: every (b, h) is split over several CTAs and merged
    # through the workspace; calling twice with one workspace must give identical outputs.
    B, H, T, F, n = 2, 24, 768, 7, 32
    pad = [[1, 0, 0, 0, 0, 0, 0], [0, 0, 1, 1, 0, 0, 0]]
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    fk, fv = (dev_normal((B, F * T, H, 128), 63, x, std=1 / np.sqrt(128), dtype=torch.bfloat16)
              for x in ("fk", "fv"))
    qa, ka, va = (dev_normal((B, n, H, 128), 63, x, std=1 / np.sqrt(128), dtype=torch.bfloat16)
                  for x in ("qa", "ka", "va"))
    need = wam.action_attn_workspace_size(lay, torch.bfloat16, n, True)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    o1 = torch.zeros((B, n, H, 128), device="cuda")
    o2 = torch.zeros_like(o1)
    wam.action_attn(lay, fk, fv, qa, ka, va, o1, workspace=ws)
    wam.action_attn(lay, fk, fv, qa, ka, va, o2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert int(ws[: B * H * 4].view(torch.int32).abs().sum()) == 0   # tickets back at zero
    ref = O.action_attention(to64(qa), to64(ka), to64(va), to64(fk), to64(fv), np.array(pad), T)
    assert_parity(to64(o1), ref, "bf16", "action split over CTAs")
    with pytest.raises(wam.WamError) as e:
        wam.action_attn(lay, fk, fv, qa, ka, va, o1, workspace=ws[: need // 2])
    assert e.value.status == 4


@pytest.mark.parametrize("big_frame", [0, 1, 2])
def test_prefill_tensor_core_large_logit_jumps(big_frame):
    # Keys of one frame scaled by 100: logits jump by ~100+ log2 units between key tiles, which
    # moves the softmax reference mid-row (O, l and the P already written are rescaled in TMEM)
    # when the big frame comes after others in the key order.
    B, H, T, F = 1, 2, 128, 3
    lay = wam.VideoLayout(B, H, 128, T, F)
    q, k, v = (dev_normal((B, F * T, H, 128), 33, n, dtype=torch.bfloat16) for n in "qkv")
    k[:, big_frame * T:(big_frame + 1) * T] *= 100.0
    o = torch.zeros((B, F * T, H, 128), device="cuda")
    wam.video_prefill_kv(lay, 0, F, q, k, v, torch.zeros_like(k), torch.zeros_like(v), o)
    ref = O.video_prefill(to64(q), to64(k), to64(v), None, None, np.zeros((1, F)), None, T, 0, F)
    assert_parity(to64(o), ref, "bf16", f"logit jumps, big frame {big_frame}")


# ----------------------------------------------------------------------------- frame copies

@pytest.mark.parametrize("tdt", [torch.bfloat16, torch.float32])
def test_copy_frames_moves_whole_frames_of_every_episode(tdt):
    B, H, D, T, F = 2, 3, 64, 16, 5
    lay = wam.VideoLayout(B, H, D, T, F)
    src = [dev_normal((B, F * T, H, D), 81, "src", j, dtype=tdt) for j in range(3)]
    dst = [torch.full_like(x, SENTINEL) for x in src]
    wam.copy_frames(lay, src, dst, 2, 1, 3)          # frames 2..4 -> 1..3
    torch.cuda.synchronize()
    for x, y in zip(src, dst):
        assert torch.equal(y[:, T:4 * T], x[:, 2 * T:5 * T])
        assert torch.all(y[:, :T] == SENTINEL) and torch.all(y[:, 4 * T:] == SENTINEL)
    wam.copy_frames(lay, src, dst, 0, 0, 0)          # nothing to copy
    torch.cuda.synchronize()
