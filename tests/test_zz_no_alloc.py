"""The prefill-with-fusion entry point that allocates nothing, for callers that cannot call
cudaMalloc (code running under CUDA graph capture, plug-ins confined to a host's memory pool,
runtimes that allocate only at start-up).  Its fusion accumulator lives inside the library.

The check: one fusion interval (first, middle, last layer) through the new entry point, twice
in a row, gives the same fused pair, outputs and cache as the entry point with a caller-owned
accumulator, within the bf16 tolerance the other parity tests use, and its fused pair matches
the oracle's weighted interval sum.  This file is collected last on purpose."""

import numpy as np
import pytest
import torch

from cached_kv_attention_b200 import wam
from oracle import wam_oracle as O
from tests.gpu_util import assert_parity, dev_normal, to64

pytestmark = pytest.mark.gpu


def _interval(lay, B, N, H, D, seed):
    g = lambda n, j: dev_normal((B, N, H, D), seed, n, j, std=1 / np.sqrt(128), dtype=torch.bfloat16)
    return [(g("q", j), g("k", j), g("v", j)) for j in range(3)]


def test_noalloc_fusion_matches_caller_owned_accumulator_twice():
    B, H, D, T, F = 1, 4, 128, 128, 5
    pad = np.array([[1, 0, 0, 0, 0]], np.uint8)
    lay = wam.VideoLayout(B, H, D, T, F, pad)
    N = F * T
    assert B * N * H * D <= wam.NOALLOC_FUSE_ACC_ELEMS
    w = wam.fuse_weights(np.array([0.4, -0.3, 1.1], np.float32))
    z = lambda dt=torch.bfloat16: torch.zeros((B, N, H, D), dtype=dt, device="cuda")

    # the existing entry point with a caller-owned accumulator
    acc_k, acc_v = z(torch.float32), z(torch.float32)
    ref_fk, ref_fv = z(), z()
    ref_o, ref_kc = [], []
    layers = _interval(lay, B, N, H, D, 91)
    for j, (q, k, v) in enumerate(layers):
        kc, vc, o = z(), z(), torch.zeros((B, N, H, D), device="cuda")
        epi = wam.FuseEpilogue(w[j], j == 0, j == 2, acc_k, acc_v, ref_fk, ref_fv)
        wam.video_prefill_kv(lay, 0, F, q, k, v, kc, vc, o, fuse=epi)
        ref_o.append(o), ref_kc.append(kc)
    torch.cuda.synchronize()

    rows = np.repeat(pad[0] == 0, T)
    for run in range(2):  # two calls of the interval in a row share the library's array
        fk, fv = z(), z()
        for j, (q, k, v) in enumerate(layers):
            kc, vc, o = z(), z(), torch.zeros((B, N, H, D), device="cuda")
            wam.video_prefill_kv_fuse_noalloc(lay, 0, F, q, k, v, kc, vc, o, w[j], j == 0, j == 2,
                                              fk, fv)
            torch.cuda.synchronize()
            assert_parity(to64(o)[0, rows], to64(ref_o[j])[0, rows], "bf16", f"noalloc O {run},{j}")
            assert torch.equal(kc, ref_kc[j])
        wam.device_error()
        assert_parity(to64(fk)[0, rows], to64(ref_fk)[0, rows], "bf16", f"noalloc fused K {run}")
        assert_parity(to64(fv)[0, rows], to64(ref_fv)[0, rows], "bf16", f"noalloc fused V {run}")
        # and against the oracle's weighted interval sum of the three layers' stored K/V
        wk = O.fuse_interval([to64(k) for _, k, _ in layers], w)
        wv = O.fuse_interval([to64(v) for _, _, v in layers], w)
        assert_parity(to64(fk)[0, rows], wk[0, rows], "bf16", f"noalloc fused K vs oracle {run}")
        assert_parity(to64(fv)[0, rows], wv[0, rows], "bf16", f"noalloc fused V vs oracle {run}")


def test_noalloc_rejects_layouts_beyond_its_array():
    # A call that uses the accumulator (not a one-layer interval) beyond the array's size is
    # rejected before anything is launched.
    big = wam.VideoLayout(1, 24, 128, 768, 26)  # 61 million elements
    x = torch.zeros(16, device="cuda")
    for first, last in ((True, False), (False, False), (False, True)):
        with pytest.raises(wam.WamError) as e:
            wam.video_prefill_kv_fuse_noalloc(big, 0, 26, x, x, x, x, x, x, 1.0, first, last, x, x)
        assert e.value.status == 2 and "WAM_NOALLOC_FUSE_ACC_ELEMS" in str(e.value)


def test_noalloc_one_layer_interval_beyond_the_array_is_accepted():
    # A one-layer interval (first and last) never touches the accumulator, so a layout larger
    # than the array is accepted and matches the entry point with a caller-owned accumulator.
    B, H, D, T, F = 1, 8, 128, 128, 33
    assert B * F * T * H * D > wam.NOALLOC_FUSE_ACC_ELEMS
    lay = wam.VideoLayout(B, H, D, T, F)
    N = F * T
    q, k, v = (dev_normal((B, N, H, D), 93, n, std=1 / np.sqrt(128), dtype=torch.bfloat16)
               for n in ("q", "k", "v"))
    z = lambda dt=torch.bfloat16: torch.zeros((B, N, H, D), dtype=dt, device="cuda")
    fk, fv, kc, vc, o = z(), z(), z(), z(), z(torch.float32)
    wam.video_prefill_kv_fuse_noalloc(lay, 0, F, q, k, v, kc, vc, o, 0.75, True, True, fk, fv)
    rfk, rfv, rkc, rvc, ro = z(), z(), z(), z(), z(torch.float32)
    epi = wam.FuseEpilogue(0.75, True, True, None, None, rfk, rfv)
    wam.video_prefill_kv(lay, 0, F, q, k, v, rkc, rvc, ro, fuse=epi)
    torch.cuda.synchronize()
    wam.device_error()
    assert torch.equal(fk, rfk) and torch.equal(fv, rfv)
    assert torch.equal(kc, rkc) and torch.equal(o, ro)
