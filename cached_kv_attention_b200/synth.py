"""Seeded synthetic inputs for the WAM attention stack.

This module holds the workload shapes and the random draws that both the CUDA path and its
checks consume.  It contains none of the method's arithmetic (no attention, fusion, schedule
or Euler step): only sizes, seeds and distributions.

Every tensor is drawn from its own ``torch.Generator`` whose seed is a stable hash of
(workload seed, tensor name, indices), so any single tensor of a chunk can be regenerated on
its own, in any order, on the CPU or on the GPU.  CPU draws are bit-identical across runs;
GPU draws use torch's CUDA generator and serve only timing runs.

Workload shapes follow the pages: 30 layers, 24 heads x 128 (Fast-WAM 精读, SECTION 04),
768 tokens per latent frame, 2 imagined frames and 4 video steps to sigma* = 0.9 (Long-WAM
源码精读 §04), fusion stride 4 (Faster-WAM详解 §3.2), 32 actions and 10 Euler steps
(Fast-WAM 精读, SECTION 07), padding of unavailable early history (Long-WAM Summary §3.3).
"""

from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "seed_for", "normal", "pad_mask", "layout_of"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str           # "f32" or "bf16": storage and input type of Q/K/V and caches
    B: int               # episodes
    L: int               # layers
    S: int               # fusion interval (stride of the interaction set)
    H: int               # heads
    D: int               # head dim
    T: int               # tokens per latent frame
    F_h: int             # history frames
    F_f: int             # imagined future frames
    n_act: int           # action tokens
    n_video_steps: int   # imagination steps to sigma*
    n_euler_steps: int   # action Euler steps
    sigma_star: float
    qkv_std: float       # Q/K/V ~ N(0, qkv_std^2)
    C: int               # channels of the future latent (placeholder, not on the pages)
    A: int               # action dim (RoboTwin: 14)
    pad_rule: str        # "none" | "prefix:<P>" | "prefix_frac:<pmax>" | "prefix_unif:<Pmax>"
    seed: int
    joint: bool = False  # co-denoising: the future frames are re-passed at every action step
    slide: bool = False  # history window kept across chunks: only the newest frame is passed
    kv_format: str = "bf16"  # fused pairs read by the action layers: "bf16", or "nvfp4" (encoded
                             # from the bf16 pairs once the final pass has completed them)

    @property
    def F(self) -> int:
        return self.F_h + self.F_f

    @property
    def N(self) -> int:
        return self.F * self.T

    @property
    def M(self) -> int:
        return -(-self.L // self.S)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_BF = dict(dtype="bf16", L=30, S=4, H=24, D=128, T=768, F_f=2, n_act=32, n_video_steps=4,
           n_euler_steps=10, sigma_star=0.9, qkv_std=1.0 / math.sqrt(128), C=64, A=14)

WORKLOADS = {
    # tiny fp32: all inputs N(0,1), seed 0
    "tiny_f32": Workload("tiny_f32", "f32", B=1, L=4, S=2, H=2, D=64, T=16, F_h=2, F_f=2,
                         n_act=8, n_video_steps=2, n_euler_steps=2, sigma_star=0.9,
                         qkv_std=1.0, C=8, A=14, pad_rule="none", seed=0),
    "ctx2.4s_bf16": Workload("ctx2.4s_bf16", B=1, F_h=3, pad_rule="none", seed=1, **_BF),
    # 80% of the 24 history frames are padding: the 19 earliest
    "ctx19.2s_bf16": Workload("ctx19.2s_bf16", B=1, F_h=24, pad_rule="prefix:19", seed=2, **_BF),
    # padding over a random 0-90% fraction of the 48 history frames
    "ctx38.4s_bf16": Workload("ctx38.4s_bf16", B=1, F_h=48, pad_rule="prefix_frac:0.9", seed=3,
                              **_BF),
    # 4 independent 19.2 s episodes, P_b ~ U{0..21}
    "batched4_bf16": Workload("batched4_bf16", B=4, F_h=24, pad_rule="prefix_unif:21", seed=4,
                              **_BF),
}
# Interaction-stride variants of the 19.2 s chunk ("世界模型之Faster-WAM详解" §4.3 ablates strides
# 1, 2, 4, 7, 14): every layer reads its own K/V (S = 1: one-layer intervals), S = 2, S = 7,
# S = 14 (intervals {0-13}, {14-27}, {28, 29}); and the one-shot variant (§3.1: one video pass
# at sigma* = 1, no imagination step).
for _s in (1, 2, 7, 14):
    WORKLOADS[f"stride{_s}_ctx19.2s_bf16"] = WORKLOADS["ctx19.2s_bf16"].replace(
        name=f"stride{_s}_ctx19.2s_bf16", S=_s)
WORKLOADS["oneshot_ctx19.2s_bf16"] = WORKLOADS["ctx19.2s_bf16"].replace(
    name="oneshot_ctx19.2s_bf16", n_video_steps=0, sigma_star=1.0)
# Co-denoising (CoD, "Long-WAM ... | Summary" App. F: V4/A4): video and actions denoised
# together in 4 joint steps; every step re-passes the future frames (cache store and fusion)
# before its action reads.
WORKLOADS["cod4_ctx19.2s_bf16"] = WORKLOADS["ctx19.2s_bf16"].replace(
    name="cod4_ctx19.2s_bf16", joint=True, n_video_steps=0, n_euler_steps=4, sigma_star=0.0)
# The 19.2 s chunk with the history window kept across chunks (steady state: each chunk one
# new frame in, the oldest of the 5 valid frames out).
WORKLOADS["slide_ctx19.2s_bf16"] = WORKLOADS["ctx19.2s_bf16"].replace(
    name="slide_ctx19.2s_bf16", slide=True)
# The 19.2 s chunk with a low-precision fused cache ("Long-WAM: 机器人操作模型的长历史..." §四: the
# LongLive-2.0 KV cache is NVFP4): the 8 fused pairs are encoded after the final pass and every
# interaction read decodes them.
WORKLOADS["nvfp4_ctx19.2s_bf16"] = WORKLOADS["ctx19.2s_bf16"].replace(
    name="nvfp4_ctx19.2s_bf16", kv_format="nvfp4")


def seed_for(seed: int, name: str, *idx: int) -> int:
    """Stable 63-bit seed of one named tensor."""
    key = f"{seed}/{name}/" + "/".join(str(int(i)) for i in idx)
    return int.from_bytes(hashlib.sha256(key.encode()).digest()[:8], "little") & ((1 << 63) - 1)


def normal(shape: Tuple[int, ...], seed: int, name: str, *idx: int, std: float = 1.0,
           dtype: torch.dtype = torch.float32, device: str = "cpu") -> torch.Tensor:
    """N(0, std^2) draw in fp32, then rounded once to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(seed, name, *idx))
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def pad_mask(w: Workload) -> torch.Tensor:
    """uint8 [B, F]: 1 marks a padding frame.  Padding is a prefix of the earliest history
    frames (unavailable early history); the imagined frames are never padding."""
    pad = torch.zeros((w.B, w.F), dtype=torch.uint8)
    g = torch.Generator().manual_seed(seed_for(w.seed, "pad"))
    rule = w.pad_rule
    for b in range(w.B):
        if rule == "none":
            P = 0
        elif rule.startswith("prefix:"):
            P = int(rule.split(":")[1])
        elif rule.startswith("prefix_frac:"):
            pmax = float(rule.split(":")[1])
            P = int(math.floor(float(torch.rand((), generator=g)) * pmax * w.F_h))
        elif rule.startswith("prefix_unif:"):
            P = int(torch.randint(0, int(rule.split(":")[1]) + 1, (), generator=g))
        else:
            raise ValueError(rule)
        P = min(P, w.F_h - 1)  # the current observation frame is never padding
        pad[b, :P] = 1
    return pad


def random_pad_mask(B: int, F: int, seed: int, p: float = 0.4,
                    keep_last: Optional[int] = 1) -> torch.Tensor:
    """uint8 [B, F] with frames padded independently with probability p (parity stress; not
    a pages workload).  The last ``keep_last`` frames stay valid."""
    g = torch.Generator().manual_seed(seed_for(seed, "random_pad", B, F))
    pad = (torch.rand((B, F), generator=g) < p).to(torch.uint8)
    if keep_last:
        pad[:, F - keep_last:] = 0
    return pad


def layout_of(w: Workload):
    """(B, H, D, T, F) of a workload."""
    return w.B, w.H, w.D, w.T, w.F


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32
