"""The prefill-with-fusion entry point that allocates nothing, for callers that cannot call
cudaMalloc (code running under CUDA graph capture, plug-ins confined to a host's memory pool,
runtimes that allocate only at start-up).  Its fusion accumulator lives inside the library.

The check: one fusion interval (first, middle, last layer) through the new entry point, twice
in a row, gives the same fused pair, outputs and cache as the entry point with a caller-owned
accumulator, within the bf16 tolerance the other parity tests use.  This file is collected
last on purpose."""

import numpy as np
import pytest
import torch

from cached_kv_attention_b200 import wam
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


def test_noalloc_rejects_layouts_beyond_its_array():
    big = wam.VideoLayout(1, 24, 128, 768, 26)  # 61 million elements
    x = torch.zeros(16, device="cuda")
    with pytest.raises(wam.WamError) as e:
        wam.video_prefill_kv_fuse_noalloc(big, 0, 26, x, x, x, x, x, x, 1.0, True, True, x, x)
    assert e.value.status == 2 and "WAM_NOALLOC_FUSE_ACC_ELEMS" in str(e.value)
