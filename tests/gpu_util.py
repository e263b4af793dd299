"""Helpers shared by the GPU parity tests: seeded inputs on the CPU copied to the device, and
the tolerances the checks apply."""

import json
import os

import numpy as np
import torch

from cached_kv_attention_b200 import synth

# Tolerances of the parity bar: fp32 path max|err| <= 1e-5 max|ref|; bf16 paths (fp32
# accumulation) max|err| <= 1e-2 max|ref| and mean relative error sum|err| / sum|ref| <= 2e-3.
F32_MAX_REL = 1e-5
BF16_MAX_REL = 1e-2
BF16_MEAN_REL = 2e-3


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else \
        t.detach().cpu().double().numpy()


def dev_normal(shape, seed, name, *idx, std=1.0, dtype=torch.float32):
    """Seeded CPU draw (bit-reproducible), then copied to the GPU."""
    return synth.normal(tuple(shape), seed, name, *idx, std=std, dtype=dtype).cuda()


def assert_parity(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    scale = np.abs(ref).max()
    log = os.environ.get("WAM_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"what": what, "dtype": str(dtype), "n": int(err.size),
                                "max_rel": float(err.max() / max(scale, 1e-300)),
                                "mean_rel": float(err.sum() / max(np.abs(ref).sum(), 1e-300))}) + "\n")
    if dtype in ("f32", torch.float32):
        assert err.max() <= F32_MAX_REL * scale, f"{what}: max err {err.max():.3e} vs {scale:.3e}"
    else:
        assert err.max() <= BF16_MAX_REL * scale, f"{what}: max err {err.max():.3e} vs {scale:.3e}"
        mean_rel = err.sum() / max(np.abs(ref).sum(), 1e-300)
        assert mean_rel <= BF16_MEAN_REL, f"{what}: mean rel err {mean_rel:.3e}"
    return float(err.max() / max(scale, 1e-300))


def valid_rows(pad, T, f_begin, f_end):
    """Query-row mask [B, (f_end - f_begin) * T] of non-padding frames."""
    pad = np.asarray(pad).astype(bool)
    return np.repeat(~pad[:, f_begin:f_end], T, axis=1)
