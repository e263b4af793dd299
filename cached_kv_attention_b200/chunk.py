"""One action chunk of the WAM attention stack, issued through the C ABI.

Stage order (one chunk):
  a3  history prefill, one call per layer, with the cache store and the fusion epilogue
  a4  N_v imagination passes (future queries over cached history + current future K/V),
      each followed by an Euler step of the future latents (sigma 1 -> sigma*)
  a5  final pass at sigma*, storing the future K/V and completing the fused pairs
  a6  Interval KV-Fusion (in the a3/a5 epilogues, or as standalone calls)
  a7  N_e Euler steps x L action layers: the M interaction layers read their fused pair,
      the others attend to the action chunk only
  a8  one Euler step of the action latents per step
("Long-WAM 源码精读" §04; "世界模型之Faster-WAM详解" §3.1-3.4; "Fast-WAM 精读" SECTION 07.)

Projections, MLPs and RoPE need trained weights, so every pass takes fresh seeded Q/K/V and
every Euler step a seeded velocity.  The chunk's arguments are marshalled once in
``prepare``; ``run`` then only issues the C calls on one stream, which also lets a CUDA graph
capture the whole chunk.
"""

from __future__ import annotations

import ctypes
from typing import Callable, Dict, List, Optional

import numpy as np
import torch

from . import synth
from . import wam
from .synth import Workload

__all__ = ["make_inputs", "ChunkRunner", "interval_partition", "interaction_layers"]


def interval_partition(L: int, S: int) -> List[List[int]]:
    """Layers of each fusion interval: {S*m, ..., min(S*m + S, L) - 1}."""
    return [list(range(S * m, min(S * m + S, L))) for m in range(-(-L // S))]


def interaction_layers(L: int, S: int) -> List[int]:
    """The action layer that reads interval m is the last layer of the interval."""
    return [I[-1] for I in interval_partition(L, S)]


def make_inputs(w: Workload, device: str = "cpu", post: Optional[Callable] = None) -> Dict:
    """Seeded inputs of one chunk (see ``synth``); drawn on ``device``.  ``post``, if given,
    is applied to each Q/K/V tensor as soon as it is drawn and its result is stored instead
    (for example a copy to the GPU, so a full-size chunk never holds every draw at once)."""
    dt = synth.torch_dtype(w)
    B, H, D, T = w.B, w.H, w.D, w.T
    hist, fut = w.F_h * T, w.F_f * T
    keep = post if post is not None else (lambda t: t)

    def qkv(name, tokens, *idx):
        return keep(synth.normal((B, tokens, H, D), w.seed, name, *idx, std=w.qkv_std, dtype=dt,
                                 device=device))

    inp = {
        "hist_q": [qkv("hist_q", hist, l) for l in range(w.L)],
        "hist_k": [qkv("hist_k", hist, l) for l in range(w.L)],
        "hist_v": [qkv("hist_v", hist, l) for l in range(w.L)],
        "imag_q": [[qkv("imag_q", fut, s, l) for l in range(w.L)] for s in range(w.n_video_steps)],
        "imag_k": [[qkv("imag_k", fut, s, l) for l in range(w.L)] for s in range(w.n_video_steps)],
        "imag_v": [[qkv("imag_v", fut, s, l) for l in range(w.L)] for s in range(w.n_video_steps)],
        "final_q": [qkv("final_q", fut, l) for l in range(w.L)] if not w.joint else [],
        "final_k": [qkv("final_k", fut, l) for l in range(w.L)] if not w.joint else [],
        "final_v": [qkv("final_v", fut, l) for l in range(w.L)] if not w.joint else [],
        # co-denoising: the future frames' Q/K/V at every joint step
        "joint_q": [[qkv("joint_q", fut, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)]
                   if w.joint else [],
        "joint_k": [[qkv("joint_k", fut, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)]
                   if w.joint else [],
        "joint_v": [[qkv("joint_v", fut, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)]
                   if w.joint else [],
        "fuse_logits": [synth.normal((len(I),), w.seed, "fuse_logits", m)
                        for m, I in enumerate(interval_partition(w.L, w.S))],
        "act_q": [[qkv("act_q", w.n_act, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)],
        "act_k": [[qkv("act_k", w.n_act, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)],
        "act_v": [[qkv("act_v", w.n_act, i, l) for l in range(w.L)] for i in range(w.n_euler_steps)],
        # sliding window: the newest history frame of a streamed chunk
        "new_q": [qkv("new_q", T, l) for l in range(w.L)] if w.slide else [],
        "new_k": [qkv("new_k", T, l) for l in range(w.L)] if w.slide else [],
        "new_v": [qkv("new_v", T, l) for l in range(w.L)] if w.slide else [],
        "x_future": synth.normal((B, fut, w.C), w.seed, "x_future", device=device),
        "v_future": [synth.normal((B, fut, w.C), w.seed, "v_future", s, device=device)
                     for s in range(w.n_euler_steps if w.joint else w.n_video_steps)],
        "x_act": synth.normal((B, w.n_act, w.A), w.seed, "x_act", device=device),
        "v_act": [synth.normal((B, w.n_act, w.A), w.seed, "v_act", i, device=device)
                  for i in range(w.n_euler_steps)],
    }
    return inp


def _vp(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class ChunkRunner:
    """Device buffers and the prepared C calls of one chunk.

    inputs        dict from ``make_inputs`` (tensors already on the device)
    distinct_out  keep one output buffer per pass (tests) or reuse one per pass kind (bench)
    fusion        "epilogue" (fold in the cache store) or "standalone" (wam_fuse_interval_kv)
    """

    def __init__(self, w: Workload, inputs: Dict, pad=None, frame_block=None,
                 distinct_out: bool = True, fusion: str = "epilogue", o_dtype=torch.float32,
                 device: str = "cuda"):
        self.w, self.inp, self.fusion = w, inputs, fusion
        dt = synth.torch_dtype(w)
        B, H, D, T, F, N = w.B, w.H, w.D, w.T, w.F, w.N
        pad = synth.pad_mask(w) if pad is None else pad
        self.pad = np.asarray(pad, dtype=np.uint8)
        self.layout = wam.VideoLayout(B, H, D, T, F, self.pad, frame_block)
        dev = torch.device(device)
        z = lambda *s, dtype=dt: torch.zeros(s, dtype=dtype, device=dev)
        # per-layer caches and fused pairs; the sliding-window mode keeps two sets used in turn
        self._sets = [([z(B, N, H, D) for _ in range(w.L)], [z(B, N, H, D) for _ in range(w.L)],
                       [z(B, N, H, D) for _ in range(w.M)], [z(B, N, H, D) for _ in range(w.M)])
                      for _ in range(2 if w.slide else 1)]
        self._use_set(0)
        self.chunks_per_run = 1
        if w.slide:
            if fusion != "epilogue":
                raise ValueError("the sliding-window mode folds the fusion into its passes (epilogue)")
            P = int(self.pad[0, :w.F_h].sum())
            if not (np.all(self.pad[:, :P] == 1) and np.all(self.pad[:, P:] == 0) and P < w.F_h):
                raise ValueError("the sliding-window mode needs the same padding prefix in every episode")
            self.slide_pad = P
        self.acc_k = z(B, N, H, D, dtype=torch.float32)
        self.acc_v = z(B, N, H, D, dtype=torch.float32)
        hist, fut = w.F_h * T, w.F_f * T
        n_h = w.L if distinct_out else 1
        n_i = w.L * w.n_video_steps if distinct_out else 1
        n_a = w.L * w.n_euler_steps if distinct_out else 1
        self.hist_o = [z(B, hist, H, D, dtype=o_dtype) for _ in range(n_h)]
        self.final_o = [z(B, fut, H, D, dtype=o_dtype) for _ in range(n_h)]
        self.imag_o = [z(B, fut, H, D, dtype=o_dtype) for _ in range(n_i)]
        self.act_o = [z(B, w.n_act, H, D, dtype=o_dtype) for _ in range(n_a)]
        self.new_o = [z(B, T, H, D, dtype=o_dtype) for _ in range(n_h if w.slide else 0)]
        if w.joint and fusion != "epilogue":
            raise ValueError("co-denoising chunks fold the fusion into the future passes (epilogue)")
        self.joint_o = [z(B, fut, H, D, dtype=o_dtype) for _ in range(n_a if w.joint else 0)]
        self.x_future = inputs["x_future"].clone()
        self.x_act = inputs["x_act"].clone()
        # one-shot variant (no video step): the cache pass runs at sigma* directly
        self.sig_v = (wam.flow_schedule(w.n_video_steps, w.sigma_star) if w.n_video_steps > 0
                      else [w.sigma_star])
        self.sig_a = wam.flow_schedule(w.n_euler_steps, 0.0)
        self.parts = interval_partition(w.L, w.S)
        self.fw = [wam.fuse_weights(lg.cpu().numpy()) for lg in inputs["fuse_logits"]]
        ws_bytes = wam.action_attn_workspace_size(self.layout, dt, w.n_act, True)
        self.workspace = torch.zeros(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        self.nvfp4 = None
        if w.kv_format == "nvfp4":
            if w.joint or w.slide or fusion != "epilogue" or w.dtype != "bf16":
                raise ValueError("the NVFP4 fused cache is built for the bf16 IDM chunk with the fusion epilogue")
            self.nvfp4 = wam.Nvfp4Cache(self.layout, 2 * w.M, device=dev.index)
        self.calls: List = []
        self._keep: List = []

    # ------------------------------------------------------------------ preparation
    def _epilogue(self, l: int):
        if self.fusion != "epilogue":
            return None
        m, j = l // self.w.S, l % self.w.S
        I = self.parts[m]
        e = wam.FuseEpilogue(self.fw[m][j], j == 0, l == I[-1], self.acc_k, self.acc_v,
                             self.fused_k[m], self.fused_v[m])
        self._keep.append(e)
        return e.ref

    def prepare(self, stream=None) -> "ChunkRunner":
        w = self.w
        s = ctypes.c_void_p(wam._stream(stream))
        lay = self.layout.ref
        dt = wam.BF16 if w.dtype == "bf16" else wam.F32
        o_dt = wam.F32 if self.hist_o[0].dtype == torch.float32 else dt

        def o_of(lst, idx):
            return _vp(lst[idx % len(lst)])

        if w.slide:
            return self._prepare_slide(lay, dt, o_dt, s, o_of)
        calls = []
        hist_end = self._history_calls(calls, lay, dt, o_dt, s, o_of)
        if w.joint:
            return self._prepare_joint(calls, hist_end, lay, dt, o_dt, s, o_of)
        imag_end, video_end = self._rest_calls(calls, lay, dt, o_dt, s, o_of)
        self.calls = calls
        # stage boundaries (call indices): the video stages a3 (history), a4 (imagination passes
        # and four small Euler steps), a5-a6 (final pass, standalone fusion), then the action
        # stages a7-a8
        self.stages = [("history", 0, hist_end), ("imagination", hist_end, imag_end),
                       ("final", imag_end, video_end)]
        if self.action_start > video_end:
            self.stages.append(("quantize", video_end, self.action_start))
        self.stages.append(("action", self.action_start, len(calls)))
        self.fused_read_call = self._first_fused_read(calls, video_end)
        return self

    @staticmethod
    def _first_fused_read(calls, start):
        return next(i for i in range(start, len(calls))
                    if calls[i][0] is wam.lib.wam_action_attn_nvfp4 or
                    (calls[i][0] is wam.lib.wam_action_attn_ex and calls[i][1][2] is not None))

    def _history_calls(self, calls, lay, dt, o_dt, s, o_of) -> int:
        """a3: history prefill with the cache store (+ fusion epilogue), all history frames."""
        w, L, inp = self.w, wam.lib, self.inp
        for l in range(w.L):
            calls.append((L.wam_video_prefill_kv,
                          (lay, dt, 0, w.F_h, _vp(inp["hist_q"][l]), _vp(inp["hist_k"][l]),
                           _vp(inp["hist_v"][l]), _vp(self.k_cache[l]), _vp(self.v_cache[l]), 1,
                           o_of(self.hist_o, l), o_dt, self._epilogue(l), s)))
        return len(calls)

    def _rest_calls(self, calls, lay, dt, o_dt, s, o_of):
        """a4-a8 on the current buffer set; returns the call indices where the final pass and
        the action stages start."""
        w, L, inp, F_h, F = self.w, wam.lib, self.inp, self.w.F_h, self.w.F
        # a4: imagination passes + Euler on the future latents
        nf = self.x_future.numel()
        for st in range(w.n_video_steps):
            for l in range(w.L):
                calls.append((L.wam_video_prefill_kv,
                              (lay, dt, F_h, F, _vp(inp["imag_q"][st][l]),
                               _vp(inp["imag_k"][st][l]), _vp(inp["imag_v"][st][l]),
                               _vp(self.k_cache[l]), _vp(self.v_cache[l]), 0,
                               o_of(self.imag_o, st * w.L + l), o_dt, None, s)))
            ds = float(self.sig_v[st + 1] - self.sig_v[st])
            calls.append((L.wam_flow_euler_step, (nf, _vp(self.x_future),
                                                  _vp(inp["v_future"][st]), ds, s)))
        imag_end = len(calls)
        # a5: final pass at sigma*, store future K/V (+ complete the fused pairs)
        for l in range(w.L):
            calls.append((L.wam_video_prefill_kv,
                          (lay, dt, F_h, F, _vp(inp["final_q"][l]), _vp(inp["final_k"][l]),
                           _vp(inp["final_v"][l]), _vp(self.k_cache[l]), _vp(self.v_cache[l]), 1,
                           o_of(self.final_o, l), o_dt, self._epilogue(l), s)))
        # a6 standalone: fuse each interval over all frames once the caches are complete
        if self.fusion == "standalone":
            for m, I in enumerate(self.parts):
                kp = (ctypes.c_void_p * len(I))(*[self.k_cache[j].data_ptr() for j in I])
                vp = (ctypes.c_void_p * len(I))(*[self.v_cache[j].data_ptr() for j in I])
                wt = (ctypes.c_float * len(I))(*[float(x) for x in self.fw[m]])
                self._keep += [kp, vp, wt]
                calls.append((L.wam_fuse_interval_kv,
                              (lay, dt, len(I), kp, vp, wt, 0, F, _vp(self.fused_k[m]),
                               _vp(self.fused_v[m]), s)))
        video_end = len(calls)
        # low-precision fused cache: every fused pair encoded once, after the final pass
        q = self.nvfp4
        if q is not None:
            tensors = [t for m in range(w.M) for t in (self.fused_k[m], self.fused_v[m])]
            arr = lambda ts: (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
            fp, cp, sp = arr(tensors), arr(q.codes), arr(q.scales)
            self._keep += [fp, cp, sp]
            calls.append((L.wam_fused_to_nvfp4, (lay, len(tensors), fp, cp, sp, _vp(q.s_g),
                                                 _vp(q.workspace), q.workspace.numel(), s)))
        self.action_start = len(calls)
        # a7 + a8: action denoising
        reader = {j: m for m, j in enumerate(interaction_layers(w.L, w.S))}
        na = self.x_act.numel()
        for i in range(w.n_euler_steps):
            for l in range(w.L):
                m = reader.get(l)
                qa_, ka_, va_ = (_vp(inp[k][i][l]) for k in ("act_q", "act_k", "act_v"))
                if q is not None and m is not None:
                    sg = q.s_g.data_ptr()
                    calls.append((L.wam_action_attn_nvfp4,
                                  (lay, _vp(q.codes[2 * m]), _vp(q.scales[2 * m]),
                                   ctypes.c_void_p(sg + 8 * m), _vp(q.codes[2 * m + 1]),
                                   _vp(q.scales[2 * m + 1]), ctypes.c_void_p(sg + 8 * m + 4), w.n_act,
                                   qa_, ka_, va_, o_of(self.act_o, i * w.L + l), o_dt,
                                   _vp(self.workspace), self.workspace.numel(),
                                   wam.ACTION_FUSED_READY, s)))
                    continue
                fk = _vp(self.fused_k[m]) if m is not None else None
                fv = _vp(self.fused_v[m]) if m is not None else None
                # the fused pairs are read-only in the action loop (completed by the video stage)
                calls.append((L.wam_action_attn_ex,
                              (lay, dt, fk, fv, w.n_act, qa_, ka_, va_,
                               o_of(self.act_o, i * w.L + l), o_dt, _vp(self.workspace),
                               self.workspace.numel(), wam.ACTION_FUSED_READY, s)))
            ds = float(self.sig_a[i + 1] - self.sig_a[i])
            calls.append((L.wam_flow_euler_step, (na, _vp(self.x_act), _vp(inp["v_act"][i]), ds, s)))
        return imag_end, video_end

    def _use_set(self, k: int) -> None:
        self.k_cache, self.v_cache, self.fused_k, self.fused_v = self._sets[k]

    def _prepare_slide(self, lay, dt, o_dt, s, o_of) -> "ChunkRunner":
        """History window kept across chunks: ``prime_calls`` fill buffer set 1 with a full chunk;
        one run is two streamed chunks (set 1 -> 0, then 0 -> 1), each moving the surviving
        frames' caches and fused pairs one frame earlier into the other set, passing only the
        newest frame through the layers, then the imagination, cache and action stages."""
        w, L, inp, F_h, P = self.w, wam.lib, self.inp, self.w.F_h, self.slide_pad
        self._use_set(1)
        prime = []
        self._history_calls(prime, lay, dt, o_dt, s, o_of)
        self._rest_calls(prime, lay, dt, o_dt, s, o_of)
        self.prime_calls = prime
        calls, stages = [], []
        for k in (0, 1):
            src, dst = self._sets[1 - k], self._sets[k]
            self._use_set(k)
            tensors = [(a, b) for sa, sb in zip(src, dst) for a, b in zip(sa, sb)]
            sp = (ctypes.c_void_p * len(tensors))(*[a.data_ptr() for a, _ in tensors])
            dp = (ctypes.c_void_p * len(tensors))(*[b.data_ptr() for _, b in tensors])
            self._keep += [sp, dp]
            c0 = len(calls)
            calls.append((L.wam_copy_frames, (lay, dt, len(tensors), sp, dp, P + 1, P, F_h - 1 - P, s)))
            h0 = len(calls)
            for l in range(w.L):
                calls.append((L.wam_video_prefill_kv,
                              (lay, dt, F_h - 1, F_h, _vp(inp["new_q"][l]), _vp(inp["new_k"][l]),
                               _vp(inp["new_v"][l]), _vp(self.k_cache[l]), _vp(self.v_cache[l]), 1,
                               o_of(self.new_o, l), o_dt, self._epilogue(l), s)))
            h1 = len(calls)
            imag_end, video_end = self._rest_calls(calls, lay, dt, o_dt, s, o_of)
            if k == 0:
                stages = [("copy", c0, h0), ("history", h0, h1), ("imagination", h1, imag_end),
                          ("final", imag_end, video_end), ("action", video_end, len(calls))]
                self.fused_read_call = self._first_fused_read(calls, video_end)
        self.calls, self.stages, self.chunks_per_run = calls, stages, 2
        return self

    def prime(self) -> None:
        """Sliding-window mode: fill buffer set 1 with one full chunk (the state the first
        streamed chunk continues from)."""
        for fn, args in self.prime_calls:
            st = fn(*args)
            if st:
                wam.check(st)

    def _prepare_joint(self, calls, hist_end, lay, dt, o_dt, s, o_of) -> "ChunkRunner":
        """Co-denoising: at every joint step i the future frames are passed through all layers
        (their K/V stored into the caches and folded into the fused pairs by the epilogue), then
        the action layers read, then both latents take one Euler step on the shared schedule."""
        w, L, inp, F_h, F = self.w, wam.lib, self.inp, self.w.F_h, self.w.F
        sig = wam.flow_schedule(w.n_euler_steps, 0.0)
        reader = {j: m for m, j in enumerate(interaction_layers(w.L, w.S))}
        nf, na = self.x_future.numel(), self.x_act.numel()
        self.stages = [("history", 0, hist_end)]
        for i in range(w.n_euler_steps):
            v0 = len(calls)
            for l in range(w.L):
                calls.append((L.wam_video_prefill_kv,
                              (lay, dt, F_h, F, _vp(inp["joint_q"][i][l]), _vp(inp["joint_k"][i][l]),
                               _vp(inp["joint_v"][i][l]), _vp(self.k_cache[l]), _vp(self.v_cache[l]),
                               1, o_of(self.joint_o, i * w.L + l), o_dt, self._epilogue(l), s)))
            a0 = len(calls)
            for l in range(w.L):
                m = reader.get(l)
                fk = _vp(self.fused_k[m]) if m is not None else None
                fv = _vp(self.fused_v[m]) if m is not None else None
                # the fused pairs were written by this step's video passes, several calls earlier
                calls.append((L.wam_action_attn_ex,
                              (lay, dt, fk, fv, w.n_act, _vp(inp["act_q"][i][l]),
                               _vp(inp["act_k"][i][l]), _vp(inp["act_v"][i][l]),
                               o_of(self.act_o, i * w.L + l), o_dt, _vp(self.workspace),
                               self.workspace.numel(), wam.ACTION_FUSED_READY, s)))
            ds = float(sig[i + 1] - sig[i])
            calls.append((L.wam_flow_euler_step, (nf, _vp(self.x_future), _vp(inp["v_future"][i]), ds, s)))
            calls.append((L.wam_flow_euler_step, (na, _vp(self.x_act), _vp(inp["v_act"][i]), ds, s)))
            self.stages += [(f"video{i}", v0, a0), (f"action{i}", a0, len(calls))]
        self.calls = calls
        self.fused_read_call = next(i for i in range(hist_end, len(calls))
                                    if calls[i][0] is L.wam_action_attn_ex and calls[i][1][2] is not None)
        return self

    def reset_latents(self) -> None:
        """Restore the Euler states to the chunk's initial noise (device copies)."""
        self.x_future.copy_(self.inp["x_future"])
        self.x_act.copy_(self.inp["x_act"])

    def run(self, events: Optional[Dict] = None, stream=None) -> None:
        """Issue the prepared calls (one chunk, or two in the sliding-window mode).  ``events``
        maps a stage name to (start, end) CUDA events that are recorded on ``stream`` around
        that stage (also inside a graph capture when the events are external)."""
        marks: Dict[int, List] = {}
        if events:
            stream = torch.cuda.current_stream() if stream is None else stream
            for name, i0, i1 in self.stages:
                ev = events.get(name)
                if ev:
                    marks.setdefault(i0, []).append(ev[0])
                    marks.setdefault(i1, []).append(ev[1])
        for i, (fn, args) in enumerate(self.calls):
            for e in marks.get(i, ()):
                e.record(stream)
            st = fn(*args)
            if st:
                wam.check(st)
        for e in marks.get(len(self.calls), ()):
            e.record(stream)

    # ------------------------------------------------------------------ counts
    def launches_per_chunk(self) -> int:
        """Kernels this chunk launches (the library launches one kernel per call, except the
        CUDA-core prefill path, which adds a store kernel)."""
        return len(self.calls)
