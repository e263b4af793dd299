"""The bench's algorithmic work, which is the numerator of every roofline figure, counted a
second way on the CPU.

Prefill FLOPs are 4 D H per allowed (query token, key token) pair: Q K^T and P V each take D
multiply-adds per pair.  The pairs are counted from the oracle's block-causal padding mask at
T = 2 and scaled by (T / 2)^2, which is exact because the mask is constant over each
(query frame, key frame) block.  Action bytes are the valid video keys the oracle's action mask
admits, times H D, times K and V, times 2 bytes, for each interaction read."""

import pytest

import bench
from cached_kv_attention_b200 import synth
from oracle import wam_oracle as O

NAMES = [n for n, w in synth.WORKLOADS.items() if w.T % 2 == 0 and n != "tiny_f32"]


def allowed_pairs(w, pad, f0, f1, t=2):
    return int(O.video_allowed(pad, None, t, f0, f1).sum()) * (w.T // t) ** 2


@pytest.mark.parametrize("name", NAMES)
def test_prefill_flops_are_the_masks_allowed_pairs(name):
    w = synth.WORKLOADS[name]
    pad = synth.pad_mask(w).numpy()
    work = bench.algorithmic_work(w, pad)
    per_pair = 4 * w.D * w.H
    # history pass: every history frame, or only the newest one when the window is kept
    hist = allowed_pairs(w, pad, w.F_h - 1 if w.slide else 0, w.F_h)
    fut = allowed_pairs(w, pad, w.F_h, w.F)  # one pass of the future frames over all keys
    n_fut = w.n_euler_steps if w.joint else w.n_video_steps + 1  # imagination steps + cache pass
    assert work["imag_flops_per_launch"] == per_pair * fut
    assert work["prefill_flops"] == per_pair * w.L * (hist + n_fut * fut)
    assert work["prefill_launches"] == w.L * (1 + n_fut)


@pytest.mark.parametrize("name", NAMES)
def test_action_bytes_are_the_masks_valid_keys(name):
    w = synth.WORKLOADS[name]
    pad = synth.pad_mask(w).numpy()
    work = bench.algorithmic_work(w, pad)
    t = 2
    video_keys = int(O.action_key_allowed(pad, t, w.n_act)[:, : w.F * t].sum()) * (w.T // t)
    assert work["valid_keys"] == video_keys
    # one head's K or V row: bf16, or NVFP4's 4-bit codes plus one 8-bit scale per 16 elements
    row = w.D * 2 if w.kv_format == "bf16" else w.D * 4 // 8 + w.D // 16 * 1
    assert work["fused_read_bytes"] == video_keys * w.H * row * 2
    reads = len(O.interaction_layers(w.L, w.S)) * w.n_euler_steps
    assert work["action_reads"] == reads
    qkvo = w.B * w.n_act * w.H * w.D * (3 * 2 + 4)  # bf16 Q, K, V in; fp32 O out
    assert work["action_bytes"] == reads * work["fused_read_bytes"] + w.L * w.n_euler_steps * qkvo


def test_the_19_2s_figures_quoted_in_the_docs():
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    work = bench.algorithmic_work(w, synth.pad_mask(w).numpy())
    assert round(work["imag_flops_per_launch"] / 1e9, 1) == 94.2  # 13 visible frame pairs
    assert round(work["prefill_flops"] / 1e12, 2) == 17.39
    assert work["valid_keys"] == 5376 and round(work["fused_read_bytes"] / 1e6, 1) == 66.1
