"""Plain fp64 CPU oracle of the world-action-model (WAM) attention stack.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  The
product path (the CUDA library and its Python binding) never imports, links or calls it,
and it imports nothing from the product path.

Every function is the direct definition of one step, in float64, written for a reader to
check against the pages by eye: masked softmax attention over an explicit boolean mask,
a weighted sum for the fusion, ``x + dsigma * v`` for Euler.  There is no online softmax, no
tiling and no reordering; ``numpy.matmul`` is the only library primitive used as a step.
Inputs are the exact values the GPU receives (bf16 or fp32), widened to float64.

Sources (page title, section):
  [LW-src]  "Long-WAM 源码精读" (yeyulingfeng.com), §03 method, §04 source reading
  [LW-tut]  "Long-WAM: 机器人操作模型的长历史..." (bloombook.cn), §三
  [FW]      "Fast-WAM 精读" (alicepotter4869.xyz), SECTION 04, 05, 07
  [LW-sum]  "Long-WAM: Scaling the Context of World-Action Models | Summary"
            (greeksharifa.github.io), §3.1-3.3, §4.2, App. B.2
  [FSW]     "世界模型之Faster-WAM详解" (171host.com), §3.1-3.4

Readings taken where the pages leave a step open:
  R1  schedule warp phi = identity (shift 1); the rescale that lands on sigma* is the affine
      map sigma = sigma* + (1 - sigma*) * phi(u), the only affine map pinning both ends.
  R2  one attention block = one latent frame unless ``frame_block`` groups frames.
  R3  padding marks whole frames; queries in padded frames produce no output (row = 0) and
      keys in padded frames are never read.
  R4  attention scale = 1/sqrt(D).
  R5  fusion weight W_fuse[m, j] is one scalar per (interval, layer), shared by K, V, all heads
      and tokens; interval I_m = {S*m, ..., min(S*m + S, L) - 1}; interaction layer j_m = max(I_m).
  R6  the per-layer cache holds the K/V of a separate pass at sigma* after the imagination
      steps; velocities, projections and RoPE need trained weights, so every pass takes fresh
      Q/K/V inputs and every Euler step a given velocity.

Parity unpinned: none of the functions below; the model semantics that need trained weights
(velocity field, projections, RoPE) and the schedule warp ``_phi`` of the real system are out
of reach, and only the identity choice and the schedule endpoints are pinned.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "time_shift", "flow_schedule", "euler_step",
    "block_ids", "video_allowed", "action_key_allowed",
    "masked_attention", "video_prefill", "cache_store",
    "interval_partition", "interaction_layers", "fuse_weights", "fuse_interval",
    "action_attention", "chunk", "chunk_joint", "chunk_stream",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------------------
# a2  flow-matching schedules      [LW-src] §04 (partial denoising to sigma*); [FSW] §3.4
# --------------------------------------------------------------------------------------

def time_shift(u, shift: float) -> np.ndarray:
    """phi(u) = s*u / (1 + (s-1)*u), the SD3 time shift (Esser et al., 2024).

    Not printed on the pages (they only name ``_phi(u, shift)``); offered as an option.
    shift = 1 gives the identity, the default reading R1.
    """
    u = _f64(u)
    if shift == 1.0:
        return u
    return shift * u / (1.0 + (shift - 1.0) * u)


def flow_schedule(n_steps: int, sigma_end: float = 0.0, shift: float = 1.0) -> np.ndarray:
    """Noise levels sigma_0 .. sigma_n of an n-step flow-matching sampler.

    [LW-src] §04 (对照一): u = linspace(1, 0, steps + 1), sigma_full = phi(u) runs 1 -> 0, then a
    rescale makes the start pure noise and the end land exactly on sigma* (0.9 with 4 video
    steps).  Reading R1: sigma_i = sigma_end + (1 - sigma_end) * phi(u_i).  The action sampler
    ([FSW] §3.4, 10 steps, [FW] SECTION 07) is the same with sigma_end = 0.
    """
    if n_steps < 1:
        raise ValueError("n_steps must be >= 1")
    u = np.array([(n_steps - i) / n_steps for i in range(n_steps + 1)], dtype=np.float64)
    return sigma_end + (1.0 - sigma_end) * time_shift(u, shift)


def euler_step(x, v, dsigma: float) -> np.ndarray:
    """One Euler step of the probability-flow ODE: x <- x + dsigma * v.

    Path x_sigma = (1 - sigma) x + sigma eps and target u = eps - x ([LW-src] §03; [FW] SECTION 05;
    [FSW] §3.4), so d x_sigma / d sigma = u and stepping sigma down by |dsigma| follows the path.
    """
    return _f64(x) + float(dsigma) * _f64(v)


# --------------------------------------------------------------------------------------
# a1  frames, padding and the two attention predicates
#     [LW-sum] §3.1-3.2 (block-causal video, video never reads actions), §3.3 (padding of
#     unavailable history); [LW-tut] §三 (asymmetric interface)
# --------------------------------------------------------------------------------------

def block_ids(frame_block: Optional[Sequence[int]], n_frames: int) -> np.ndarray:
    """Block id of each latent frame; default one block per frame (reading R2)."""
    if frame_block is None:
        return np.arange(n_frames, dtype=np.int64)
    blk = np.asarray(frame_block, dtype=np.int64)
    if blk.shape != (n_frames,) or np.any(np.diff(blk) < 0):
        raise ValueError("frame_block must be a nondecreasing [F] sequence")
    return blk


def video_allowed(pad, frame_block, T: int, f_begin: int, f_end: int,
                  rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Boolean [B, (f_end - f_begin) * T, f_end * T]: may video query q read video key k?

    A video query reads its own and earlier visual blocks and never an action token
    ([LW-sum] §3.2); keys of padded (unavailable) frames are never read and queries of padded
    frames produce nothing (reading R3).  Query tokens are the frames [f_begin, f_end) of the
    call; key tokens are all frames [0, f_end).  ``rows`` keeps only those query rows.
    """
    pad = np.asarray(pad).astype(bool)
    B, F = pad.shape
    blk = block_ids(frame_block, F)
    q_tok = np.arange(f_begin * T, f_end * T) if rows is None else f_begin * T + np.asarray(rows)
    q_frame = q_tok // T
    k_frame = np.arange(0, f_end * T) // T
    causal = blk[k_frame][None, :] <= blk[q_frame][:, None]            # [Q, K]
    key_ok = ~pad[:, k_frame]                                            # [B, K]
    query_ok = ~pad[:, q_frame]                                          # [B, Q]
    return causal[None, :, :] & key_ok[:, None, :] & query_ok[:, :, None]


def action_key_allowed(pad, T: int, n_act: int, with_video: bool = True) -> np.ndarray:
    """Boolean [B, (F*T if with_video) + n_act]: which keys an action query may read.

    Action queries read the observed history, the partially denoised future and the whole
    noisy action chunk ([LW-sum] §3.2; [LW-tut] §三); only padded video frames are excluded.
    The mask is the same for every action query (the chunk attends bidirectionally).
    """
    pad = np.asarray(pad).astype(bool)
    B, _ = pad.shape
    act = np.ones((B, n_act), dtype=bool)
    if not with_video:
        return act
    return np.concatenate([np.repeat(~pad, T, axis=1), act], axis=1)


# --------------------------------------------------------------------------------------
# attention by definition        [FW] SECTION 07 (K = [K_video; K_action], softmax read)
# --------------------------------------------------------------------------------------

def masked_attention(q, k, v, allowed, scale: float) -> np.ndarray:
    """O_i = sum_k softmax_k(scale * q_i . k_k) v_k over the keys allowed for row i.

    q [Lq, D], k [Lk, D], v [Lk, Dv], allowed bool [Lq, Lk].  A row with no allowed key is 0.
    Keys that no row may read are dropped before the product: they contribute nothing.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    allowed = np.asarray(allowed, dtype=bool)
    used = np.nonzero(allowed.any(axis=0))[0]
    out = np.zeros((q.shape[0], v.shape[1]), dtype=np.float64)
    if used.size == 0:
        return out
    k, v, allowed = k[used], v[used], allowed[:, used]
    s = scale * (q @ k.T)
    s = np.where(allowed, s, -np.inf)
    has = allowed.any(axis=1)
    m = np.where(has, s.max(axis=1), 0.0)
    p = np.where(allowed, np.exp(s - m[:, None]), 0.0)
    denom = p.sum(axis=1)
    out[has] = (p[has] @ v) / denom[has, None]
    return out


def _default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)  # reading R4


# --------------------------------------------------------------------------------------
# a3-a5  block-causal video prefill of the per-layer K/V cache
#        [LW-src] §04 (prefill_video_cache builds a per-layer {"k","v"} list after the
#        imagination); [LW-sum] §3.2, §4.2 (observed-video KV reused within a call)
# --------------------------------------------------------------------------------------

def video_prefill(q, k_new, v_new, k_cache, v_cache, pad, frame_block, T: int,
                  f_begin: int, f_end: int, scale: Optional[float] = None,
                  heads: Optional[Sequence[int]] = None,
                  rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Output O [B, Q, H, D] of one layer's video attention for query frames [f_begin, f_end).

    The key set is the cached K/V of frames [0, f_begin) followed by the new K/V of frames
    [f_begin, f_end); the mask is ``video_allowed``.  ``heads`` / ``rows`` restrict which
    outputs are computed (others are left 0) so that single outputs of a large call can be
    checked one by one.
    """
    q = _f64(q)
    B, Q, H, D = q.shape
    if Q != (f_end - f_begin) * T:
        raise ValueError("q must hold (f_end - f_begin) * T tokens")
    scale = _default_scale(D) if scale is None else scale
    n_old = f_begin * T
    if n_old:
        keys = np.concatenate([_f64(k_cache)[:, :n_old], _f64(k_new)], axis=1)
        vals = np.concatenate([_f64(v_cache)[:, :n_old], _f64(v_new)], axis=1)
    else:
        keys, vals = _f64(k_new), _f64(v_new)
    rows = np.arange(Q) if rows is None else np.asarray(rows)
    padb = np.asarray(pad).astype(bool)
    heads = range(H) if heads is None else heads
    o = np.zeros((B, Q, H, v_new.shape[-1]), dtype=np.float64)
    for b in range(B):
        # rows of padded query frames read nothing and stay 0 (reading R3): not computed
        rows_b = rows[~padb[b, f_begin + rows // T]]
        allowed = video_allowed(padb[b:b + 1], frame_block, T, f_begin, f_end, rows=rows_b)[0]
        for h in heads:
            o[b, rows_b, h] = masked_attention(q[b, rows_b, h], keys[b, :, h], vals[b, :, h],
                                               allowed, scale)
    return o


def cache_store(cache, new, pad, T: int, f_begin: int, f_end: int) -> np.ndarray:
    """The cache after a prefill call: frames [f_begin, f_end) that are not padding take the
    new K (or V); padded frames are neither stored nor read, so they keep what they held."""
    out = _f64(cache).copy()
    pad = np.asarray(pad).astype(bool)
    new = _f64(new)
    for b in range(out.shape[0]):
        for f in range(f_begin, f_end):
            if not pad[b, f]:
                out[b, f * T:(f + 1) * T] = new[b, (f - f_begin) * T:(f - f_begin + 1) * T]
    return out


# --------------------------------------------------------------------------------------
# a6  Interval KV-Fusion          [FSW] §3.2 (interaction set J, stride 4 -> M = 8), §3.3
# --------------------------------------------------------------------------------------

def interval_partition(L: int, S: int) -> List[List[int]]:
    """I_m = {S*m, ..., min(S*m + S, L) - 1} for m = 0 .. ceil(L/S) - 1 (reading R5)."""
    if L < 1 or S < 1:
        raise ValueError("L and S must be >= 1")
    return [list(range(S * m, min(S * m + S, L))) for m in range(-(-L // S))]


def interaction_layers(L: int, S: int) -> List[int]:
    """j_m = max(I_m): the interaction layer reads the depth interval that precedes it."""
    return [I[-1] for I in interval_partition(L, S)]


def fuse_weights(logits) -> np.ndarray:
    """W_fuse[m, :] = softmax over the layers j in I_m of the learned logits ([FSW] §3.3)."""
    x = _f64(logits)
    e = np.exp(x - x.max())
    return e / e.sum()


def fuse_interval(layers: Sequence, weights) -> np.ndarray:
    """(K_bar, V_bar)_{j_m} = sum_{j in I_m} W_fuse[m, j] (K_j, V_j)  ([FSW] §3.3).

    Applied to K and to V separately; the fused tensor has one layer's length.
    """
    w = _f64(weights)
    if len(layers) != w.shape[0]:
        raise ValueError("one weight per layer")
    acc = np.zeros(np.shape(layers[0]), dtype=np.float64)
    for wj, x in zip(w, layers):
        acc = acc + wj * _f64(x)
    return acc


# --------------------------------------------------------------------------------------
# a7  asymmetric action attention  [FW] SECTION 07 (K=[K_video;K_action], V=[V_video;V_action]);
#     [LW-sum] §3.2, §4.2 (one softmax over both buffers)
# --------------------------------------------------------------------------------------

def action_attention(qa, ka, va, fused_k, fused_v, pad, T: int,
                     scale: Optional[float] = None,
                     heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """O [B, n_act, H, D] of action queries over [fused video K/V (valid frames); action K/V].

    ``fused_k is None`` is a layer outside the interaction set: action self-attention only.
    """
    qa = _f64(qa)
    B, n, H, D = qa.shape
    scale = _default_scale(D) if scale is None else scale
    with_video = fused_k is not None
    if with_video:
        keys = np.concatenate([_f64(fused_k), _f64(ka)], axis=1)
        vals = np.concatenate([_f64(fused_v), _f64(va)], axis=1)
    else:
        keys, vals = _f64(ka), _f64(va)
    allowed = action_key_allowed(pad, T, n, with_video)
    heads = range(H) if heads is None else heads
    o = np.zeros((B, n, H, vals.shape[-1]), dtype=np.float64)
    for b in range(B):
        for h in heads:
            o[b, :, h] = masked_attention(qa[b, :, h], keys[b, :, h], vals[b, :, h],
                                          np.repeat(allowed[b][None, :], n, axis=0), scale)
    return o


# --------------------------------------------------------------------------------------
# a3 -> a8  one action chunk       [LW-src] §04 (imagine to sigma*, then prefill, then the
#           action loop reusing the cache); [FSW] §3.1-3.4 (fusion, sparse reads, 10 steps)
# --------------------------------------------------------------------------------------

def chunk(inp: Dict, *, L: int, S: int, T: int, F_h: int, F_f: int, n_video_steps: int,
          n_euler_steps: int, sigma_star: float, pad, frame_block=None,
          heads: Optional[Sequence[int]] = None) -> Dict:
    """All stages of one action chunk in the order a3 -> a8.

    ``inp`` holds per-pass inputs (arrays [B, tokens, H, D] unless noted):
      hist_q/k/v[l]            history pass, frames [0, F_h)
      imag_q/k/v[s][l]         imagination step s, future frames [F_h, F)
      final_q/k/v[l]           final pass at sigma*, future frames
      fuse_weights[m]          [|I_m|] softmax-normalised weights
      act_q/k/v[i][l]          action step i, [B, n_act, H, D]
      x_future, v_future[s]    future latents [B, F_f*T, C] and velocities
      x_act, v_act[i]          action latents [B, n_act, A] and velocities
    Returns every stage output, the per-layer caches and the fused caches (float64).
    """
    F = F_h + F_f
    kv = np.shape(inp["hist_k"][0])
    B, _, H, D = kv
    N = F * T
    zeros = np.zeros((B, N, H, D))
    out: Dict = {"hist_o": [], "imag_o": [], "final_o": [], "act_o": []}
    k_cache = [zeros.copy() for _ in range(L)]
    v_cache = [zeros.copy() for _ in range(L)]

    # a3: history prefill, one call per layer
    for l in range(L):
        out["hist_o"].append(video_prefill(inp["hist_q"][l], inp["hist_k"][l], inp["hist_v"][l],
                                           k_cache[l], v_cache[l], pad, frame_block, T, 0, F_h,
                                           heads=heads))
        k_cache[l] = cache_store(k_cache[l], inp["hist_k"][l], pad, T, 0, F_h)
        v_cache[l] = cache_store(v_cache[l], inp["hist_v"][l], pad, T, 0, F_h)

    rest = chunk_after_history(inp, k_cache, v_cache, L=L, S=S, T=T, F_h=F_h, F_f=F_f,
                               n_video_steps=n_video_steps, n_euler_steps=n_euler_steps,
                               sigma_star=sigma_star, pad=pad, frame_block=frame_block, heads=heads)
    rest["hist_o"] = out["hist_o"]
    return rest


def chunk_after_history(inp: Dict, k_cache, v_cache, *, L: int, S: int, T: int, F_h: int,
                        F_f: int, n_video_steps: int, n_euler_steps: int, sigma_star: float, pad,
                        frame_block=None, heads: Optional[Sequence[int]] = None) -> Dict:
    """Stages a4 -> a8 of ``chunk`` given the per-layer caches of the history frames (the
    lists are updated in place with the future frames)."""
    F = F_h + F_f
    out: Dict = {"imag_o": [], "final_o": [], "act_o": []}
    # a4: imagination passes and Euler steps on the future latents, sigma 1 -> sigma*.  With no
    # video step (the one-shot variant: one video pass at sigma* = 1, [FSW] §3.1) the cache pass
    # follows directly.
    sig_v = flow_schedule(n_video_steps, sigma_star) if n_video_steps > 0 else None
    x_future = _f64(inp["x_future"])
    for s in range(n_video_steps):
        outs = []
        for l in range(L):
            outs.append(video_prefill(inp["imag_q"][s][l], inp["imag_k"][s][l],
                                      inp["imag_v"][s][l], k_cache[l], v_cache[l], pad,
                                      frame_block, T, F_h, F, heads=heads))
        out["imag_o"].append(outs)
        x_future = euler_step(x_future, inp["v_future"][s], sig_v[s + 1] - sig_v[s])
    out["x_future"] = x_future

    # a5: final pass at sigma*, its future K/V go to the cache
    for l in range(L):
        out["final_o"].append(video_prefill(inp["final_q"][l], inp["final_k"][l],
                                            inp["final_v"][l], k_cache[l], v_cache[l], pad,
                                            frame_block, T, F_h, F, heads=heads))
        k_cache[l] = cache_store(k_cache[l], inp["final_k"][l], pad, T, F_h, F)
        v_cache[l] = cache_store(v_cache[l], inp["final_v"][l], pad, T, F_h, F)
    out["k_cache"], out["v_cache"] = k_cache, v_cache

    # a6: Interval KV-Fusion
    parts = interval_partition(L, S)
    out["fused_k"] = [fuse_interval([k_cache[j] for j in I], inp["fuse_weights"][m])
                      for m, I in enumerate(parts)]
    out["fused_v"] = [fuse_interval([v_cache[j] for j in I], inp["fuse_weights"][m])
                      for m, I in enumerate(parts)]

    # a7 + a8: action denoising; interaction layers read their fused pair
    reader = {j: m for m, j in enumerate(interaction_layers(L, S))}
    sig_a = flow_schedule(n_euler_steps, 0.0)
    x_act = _f64(inp["x_act"])
    for i in range(n_euler_steps):
        outs = []
        for l in range(L):
            m = reader.get(l)
            fk = out["fused_k"][m] if m is not None else None
            fv = out["fused_v"][m] if m is not None else None
            outs.append(action_attention(inp["act_q"][i][l], inp["act_k"][i][l],
                                         inp["act_v"][i][l], fk, fv, pad, T, heads=heads))
        out["act_o"].append(outs)
        x_act = euler_step(x_act, inp["v_act"][i], sig_a[i + 1] - sig_a[i])
    out["x_act"] = x_act
    return out


# --------------------------------------------------------------------------------------
# Co-denoising (CoD) chunk            [LW-sum] Fig. 2 and App. F (IDM versus co-denoising,
#                                     V4/A4); [FSW] §1-2 (Joint-WAM updates the future video
#                                     and the actions at every denoising step)
# --------------------------------------------------------------------------------------

def chunk_joint(inp: Dict, *, L: int, S: int, T: int, F_h: int, F_f: int, n_steps: int, pad,
                frame_block=None, heads: Optional[Sequence[int]] = None) -> Dict:
    """One chunk with video and actions denoised together in ``n_steps`` joint steps.

    Reading R10 (the pages give the idea and latencies, not the step order): the history pass
    runs once; at joint step i every layer first passes the future frames (queries over the
    cached history and the step's own future K/V), their K/V replace the future frames of the
    layer's cache, the fused pairs are formed again, then every action layer reads (interaction
    layers their fused pair), and both latents take one Euler step on one schedule 1 -> 0.

    ``inp`` holds hist_q/k/v[l], joint_q/k/v[i][l] (future frames at step i), fuse_weights[m],
    act_q/k/v[i][l], x_future, v_future[i], x_act, v_act[i].
    """
    F = F_h + F_f
    B, _, H, D = np.shape(inp["hist_k"][0])
    N = F * T
    zeros = np.zeros((B, N, H, D))
    out: Dict = {"hist_o": [], "joint_o": [], "act_o": []}
    k_cache = [zeros.copy() for _ in range(L)]
    v_cache = [zeros.copy() for _ in range(L)]
    for l in range(L):
        out["hist_o"].append(video_prefill(inp["hist_q"][l], inp["hist_k"][l], inp["hist_v"][l],
                                           k_cache[l], v_cache[l], pad, frame_block, T, 0, F_h,
                                           heads=heads))
        k_cache[l] = cache_store(k_cache[l], inp["hist_k"][l], pad, T, 0, F_h)
        v_cache[l] = cache_store(v_cache[l], inp["hist_v"][l], pad, T, 0, F_h)
    parts = interval_partition(L, S)
    reader = {j: m for m, j in enumerate(interaction_layers(L, S))}
    sig = flow_schedule(n_steps, 0.0)
    x_future, x_act = _f64(inp["x_future"]), _f64(inp["x_act"])
    for i in range(n_steps):
        outs = []
        for l in range(L):
            outs.append(video_prefill(inp["joint_q"][i][l], inp["joint_k"][i][l],
                                      inp["joint_v"][i][l], k_cache[l], v_cache[l], pad,
                                      frame_block, T, F_h, F, heads=heads))
            k_cache[l] = cache_store(k_cache[l], inp["joint_k"][i][l], pad, T, F_h, F)
            v_cache[l] = cache_store(v_cache[l], inp["joint_v"][i][l], pad, T, F_h, F)
        out["joint_o"].append(outs)
        fused_k = [fuse_interval([k_cache[j] for j in I], inp["fuse_weights"][m]) for m, I in enumerate(parts)]
        fused_v = [fuse_interval([v_cache[j] for j in I], inp["fuse_weights"][m]) for m, I in enumerate(parts)]
        outs = []
        for l in range(L):
            m = reader.get(l)
            outs.append(action_attention(inp["act_q"][i][l], inp["act_k"][i][l], inp["act_v"][i][l],
                                         fused_k[m] if m is not None else None,
                                         fused_v[m] if m is not None else None, pad, T, heads=heads))
        out["act_o"].append(outs)
        x_future = euler_step(x_future, inp["v_future"][i], sig[i + 1] - sig[i])
        x_act = euler_step(x_act, inp["v_act"][i], sig[i + 1] - sig[i])
    out.update(k_cache=k_cache, v_cache=v_cache, fused_k=fused_k, fused_v=fused_v,
               x_future=x_future, x_act=x_act)
    return out


# --------------------------------------------------------------------------------------
# Streamed chunk: the history window kept across chunks     [LW-sum] §4.2 and App. B.2
#                 (observed-video K/V computed once and reused; the conditions under which a
#                 reused cache stays valid); [LW-src] §05 (streaming encoding of new frames)
# --------------------------------------------------------------------------------------

def chunk_stream(prev: Dict, inp: Dict, *, L: int, S: int, T: int, F_h: int, F_f: int,
                 n_video_steps: int, n_euler_steps: int, sigma_star: float, pad,
                 frame_block=None, heads: Optional[Sequence[int]] = None) -> Dict:
    """The next chunk of an episode whose history window slid by one frame.

    Reading R11: between chunks one observation frame arrives; the window keeps F_h frames, so
    every cached frame moves one position earlier and the oldest leaves it (``pad`` is this
    chunk's padding: the frames the previous chunk held at f + 1 are the ones valid at f).  The
    per-layer caches and the fused pairs of the surviving frames are the previous chunk's,
    shifted; only the newest frame (F_h - 1) is passed through the layers (queries over the
    cached window and itself), stored and folded.  The imagination, cache and action stages
    then run as in ``chunk``.

    ``prev`` is a previous chunk's output (its k_cache and v_cache are used; the fused pairs of
    the surviving frames are sums over those caches, so forming them again from the shifted
    caches equals shifting them); ``inp`` holds new_q/k/v[l] ([B, T, H, D], the newest frame)
    and the imagination, final, fusion and action inputs of ``chunk``.  Returns the same keys as
    ``chunk`` with hist_o[l] the newest frame's output ([B, T, H, D]).
    """
    F = F_h + F_f
    pad = np.asarray(pad)
    shift = lambda x: np.concatenate([x[:, T:F_h * T], np.zeros_like(x[:, :T]), x[:, F_h * T:]], axis=1)
    keep = lambda x: np.where(_row_valid(pad, T, F)[:, :, None, None], x, 0.0)
    k_cache = [keep(shift(x)) for x in prev["k_cache"]]
    v_cache = [keep(shift(x)) for x in prev["v_cache"]]
    out: Dict = {"hist_o": [], "imag_o": [], "final_o": [], "act_o": []}
    for l in range(L):
        out["hist_o"].append(video_prefill(inp["new_q"][l], inp["new_k"][l], inp["new_v"][l],
                                           k_cache[l], v_cache[l], pad, frame_block, T, F_h - 1,
                                           F_h, heads=heads))
        k_cache[l] = cache_store(k_cache[l], inp["new_k"][l], pad, T, F_h - 1, F_h)
        v_cache[l] = cache_store(v_cache[l], inp["new_v"][l], pad, T, F_h - 1, F_h)
    rest = chunk_after_history(inp, k_cache, v_cache, L=L, S=S, T=T, F_h=F_h, F_f=F_f,
                               n_video_steps=n_video_steps, n_euler_steps=n_euler_steps,
                               sigma_star=sigma_star, pad=pad, frame_block=frame_block, heads=heads)
    rest["hist_o"] = out["hist_o"]
    return rest


def _row_valid(pad, T: int, F: int) -> np.ndarray:
    """[B, F*T] True on the rows of non-padding frames."""
    pad = np.asarray(pad)
    return np.repeat(pad[:, :F] == 0, T, axis=1)
