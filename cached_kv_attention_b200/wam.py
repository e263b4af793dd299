"""Thin Python binding of libwam.so: the same entry points as include/wam.h, with torch
tensors for device memory and streams.  Every wrapper only marshals arguments; all work runs
in the library's CUDA kernels.  Importing this module fails loudly if the library is missing.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = [
    "WamError", "F32", "BF16", "VideoLayout", "FuseEpilogue", "lib",
    "video_prefill_kv", "fuse_interval_kv", "action_attn", "flow_euler_step",
    "flow_schedule", "fuse_weights", "debug_video_mask", "device_error", "exported_names",
    "video_prefill_kv_fuse_noalloc", "NOALLOC_FUSE_ACC_ELEMS", "action_attn_workspace_size",
    "action_workspace", "debug_prefill_order", "debug_wait_timeout",
    "nvfp4_workspace_size", "fused_to_nvfp4", "Nvfp4Cache", "action_attn_nvfp4",
    "debug_action_plan", "ACTION_FUSED_READY",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwam.so")

F32, BF16 = 0, 1
_STATUS = {0: "WAM_OK", 1: "WAM_ERR_INVALID_ARGUMENT", 2: "WAM_ERR_UNSUPPORTED",
           3: "WAM_ERR_CUDA", 4: "WAM_ERR_WORKSPACE", 5: "WAM_ERR_TIMEOUT"}


class WamError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class _Layout(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("T", ctypes.c_int32), ("F", ctypes.c_int32),
                ("frame_pad", ctypes.c_void_p), ("frame_block", ctypes.c_void_p)]


class _Fuse(ctypes.Structure):
    _fields_ = [("weight", ctypes.c_float), ("first_in_interval", ctypes.c_int32),
                ("last_in_interval", ctypes.c_int32), ("acc_k", ctypes.c_void_p),
                ("acc_v", ctypes.c_void_p), ("fused_k", ctypes.c_void_p),
                ("fused_v", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m cached_kv_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, \
        ctypes.c_double
    lay = ctypes.POINTER(_Layout)
    sigs = {
        "wam_video_prefill_kv": [lay, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, i32,
                                 ctypes.POINTER(_Fuse), vp],
        "wam_fuse_interval_kv": [lay, i32, i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                 ctypes.POINTER(f32), i32, i32, vp, vp, vp],
        "wam_action_attn": [lay, i32, vp, vp, i32, vp, vp, vp, vp, i32, vp, ctypes.c_size_t, vp],
        "wam_action_attn_ex": [lay, i32, vp, vp, i32, vp, vp, vp, vp, i32, vp, ctypes.c_size_t,
                               ctypes.c_uint32, vp],
        "wam_action_attn_workspace_size": [lay, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)],
        "wam_flow_euler_step": [i64, vp, vp, f32, vp],
        "wam_copy_frames": [lay, i32, i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp],
        "wam_flow_schedule": [i32, f64, f64, ctypes.POINTER(f64)],
        "wam_fuse_weights": [i32, ctypes.POINTER(f32), ctypes.POINTER(f32)],
        "wam_debug_video_mask": [lay, i32, i32, vp, vp],
        "wam_debug_prefill_order": [lay, i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                    ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "wam_device_error": [i32],
        "wam_debug_wait_timeout": [i32, vp],
        "wam_debug_action_plan": [lay, i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                  ctypes.POINTER(i32)],
        "wam_nvfp4_workspace_size": [i32, ctypes.POINTER(ctypes.c_size_t)],
        "wam_fused_to_nvfp4": [lay, i32, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                               vp, vp, ctypes.c_size_t, vp],
        "wam_action_attn_nvfp4": [lay, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, i32, vp,
                                  ctypes.c_size_t, ctypes.c_uint32, vp],
        "wam_video_prefill_kv_fuse_noalloc": [lay, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp,
                                              i32, f32, i32, i32, vp, vp, vp],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.wam_last_error.argtypes = []
    L.wam_last_error.restype = ctypes.c_char_p
    L.wam_version.argtypes = []
    L.wam_version.restype = ctypes.c_int32
    return L


lib = _load()


def exported_names() -> list:
    """Names of the C entry points this binding declares (all must be exported)."""
    return ["wam_video_prefill_kv", "wam_fuse_interval_kv", "wam_action_attn",
            "wam_flow_euler_step", "wam_flow_schedule", "wam_fuse_weights",
            "wam_debug_video_mask", "wam_device_error", "wam_last_error", "wam_version",
            "wam_video_prefill_kv_fuse_noalloc", "wam_action_attn_workspace_size",
            "wam_copy_frames", "wam_debug_prefill_order", "wam_debug_wait_timeout",
            "wam_nvfp4_workspace_size", "wam_fused_to_nvfp4", "wam_action_attn_nvfp4",
            "wam_action_attn_ex", "wam_debug_action_plan"]


def check(status: int) -> None:
    if status != 0:
        raise WamError(status, lib.wam_last_error().decode())


class VideoLayout:
    """Geometry of one call: B episodes, H heads, D head dim, T tokens per frame, F frames,
    an optional host padding mask [B, F] and optional attention-block ids [F]."""

    def __init__(self, B: int, H: int, D: int, T: int, F: int,
                 frame_pad=None, frame_block: Optional[Sequence[int]] = None):
        self.B, self.H, self.D, self.T, self.F = B, H, D, T, F
        self.pad = None if frame_pad is None else \
            np.ascontiguousarray(np.asarray(frame_pad, dtype=np.uint8).reshape(B, F))
        self.block = None if frame_block is None else \
            np.ascontiguousarray(np.asarray(frame_block, dtype=np.int32))
        self.c = _Layout(B, H, D, T, F,
                         None if self.pad is None else self.pad.ctypes.data,
                         None if self.block is None else self.block.ctypes.data)
        self.ref = ctypes.byref(self.c)

    @property
    def N(self) -> int:
        return self.F * self.T


class FuseEpilogue:
    """Interval KV-Fusion folded into one layer's cache store."""

    def __init__(self, weight: float, first: bool, last: bool, acc_k=None, acc_v=None,
                 fused_k=None, fused_v=None):
        self.c = _Fuse(float(weight), int(first), int(last), _ptr(acc_k), _ptr(acc_v),
                       _ptr(fused_k), _ptr(fused_v))
        self.ref = ctypes.byref(self.c)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def video_prefill_kv(layout: VideoLayout, f_begin: int, f_end: int, q, k_new, v_new,
                     k_cache, v_cache, o, store_kv: bool = True,
                     fuse: Optional[FuseEpilogue] = None, stream=None) -> None:
    check(lib.wam_video_prefill_kv(layout.ref, _dtype(q), f_begin, f_end, _ptr(q), _ptr(k_new),
                                   _ptr(v_new), _ptr(k_cache), _ptr(v_cache), int(store_kv),
                                   _ptr(o), _dtype(o), None if fuse is None else fuse.ref,
                                   _stream(stream)))


NOALLOC_FUSE_ACC_ELEMS = 4 * 1024 * 1024


def video_prefill_kv_fuse_noalloc(layout: VideoLayout, f_begin: int, f_end: int, q, k_new, v_new,
                                  k_cache, v_cache, o, weight: float, first: bool, last: bool,
                                  fused_k=None, fused_v=None, store_kv: bool = True,
                                  stream=None) -> None:
    """The prefill with the fusion epilogue whose fp32 accumulator lives inside the library
    (for callers that cannot allocate device memory); B*F*T*H*D <= NOALLOC_FUSE_ACC_ELEMS."""
    check(lib.wam_video_prefill_kv_fuse_noalloc(
        layout.ref, _dtype(q), f_begin, f_end, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
        _ptr(v_cache), int(store_kv), _ptr(o), _dtype(o), float(weight), int(first), int(last),
        _ptr(fused_k), _ptr(fused_v), _stream(stream)))


def fuse_interval_kv(layout: VideoLayout, k_layers, v_layers, weights, f_begin: int,
                     f_end: int, fused_k, fused_v, stream=None) -> None:
    n = len(k_layers)
    kp = (ctypes.c_void_p * n)(*[_ptr(t) for t in k_layers])
    vp = (ctypes.c_void_p * n)(*[_ptr(t) for t in v_layers])
    w = (ctypes.c_float * n)(*[float(x) for x in weights])
    check(lib.wam_fuse_interval_kv(layout.ref, _dtype(fused_k), n, kp, vp, w, f_begin, f_end,
                                   _ptr(fused_k), _ptr(fused_v), _stream(stream)))


def copy_frames(layout: VideoLayout, src, dst, f_src: int, f_dst: int, n_frames: int,
                stream=None) -> None:
    """Frames [f_src, f_src + n_frames) of every src tensor to [f_dst, ...) of its dst."""
    n = len(src)
    sp = (ctypes.c_void_p * n)(*[_ptr(t) for t in src])
    dp = (ctypes.c_void_p * n)(*[_ptr(t) for t in dst])
    check(lib.wam_copy_frames(layout.ref, _dtype(src[0]), n, sp, dp, f_src, f_dst, n_frames,
                              _stream(stream)))


def action_attn_workspace_size(layout: VideoLayout, dtype: torch.dtype, n_act: int,
                               with_video: bool = True) -> int:
    """Bytes of workspace wam_action_attn needs for this layout on the current device."""
    out = ctypes.c_size_t(0)
    dt = BF16 if dtype == torch.bfloat16 else F32
    check(lib.wam_action_attn_workspace_size(layout.ref, dt, n_act, int(with_video),
                                             ctypes.byref(out)))
    return out.value


_workspaces = {}


def action_workspace(nbytes: int, device=None) -> Optional[torch.Tensor]:
    """A zero-filled device workspace of at least nbytes, cached per device.  The library
    leaves it ready for the next call; calls sharing it must not overlap on the GPU."""
    if nbytes == 0:
        return None
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    ws = _workspaces.get(dev)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        _workspaces[dev] = ws
    return ws


ACTION_FUSED_READY = 1


def action_attn(layout: VideoLayout, fused_k, fused_v, qa, ka, va, o, workspace=None,
                stream=None, flags: int = 0) -> None:
    """flags: ACTION_FUSED_READY when the fused pair is not written by the call issued right
    before this one on the stream (see wam_action_attn_ex)."""
    n_act = qa.shape[1]
    if workspace is None:
        need = action_attn_workspace_size(layout, qa.dtype, n_act, fused_k is not None)
        workspace = action_workspace(need, qa.device.index)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib.wam_action_attn_ex(layout.ref, _dtype(qa), _ptr(fused_k), _ptr(fused_v), n_act,
                                 _ptr(qa), _ptr(ka), _ptr(va), _ptr(o), _dtype(o), _ptr(workspace),
                                 ws_bytes, int(flags), _stream(stream)))


def flow_euler_step(x, v, dsigma: float, stream=None) -> None:
    if x.dtype != torch.float32 or v.dtype != torch.float32 or x.numel() != v.numel():
        raise ValueError("x and v must be fp32 tensors of the same size")
    check(lib.wam_flow_euler_step(x.numel(), _ptr(x), _ptr(v), float(dsigma), _stream(stream)))


def flow_schedule(n_steps: int, sigma_end: float = 0.0, shift: float = 1.0) -> np.ndarray:
    out = np.zeros(n_steps + 1, dtype=np.float64) if n_steps >= 0 else np.zeros(1)
    check(lib.wam_flow_schedule(n_steps, sigma_end, shift,
                                out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return out


def fuse_weights(logits) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(logits, dtype=np.float32))
    out = np.zeros_like(x)
    check(lib.wam_fuse_weights(x.size, x.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                               out.ctypes.data_as(ctypes.POINTER(ctypes.c_float))))
    return out


def debug_video_mask(layout: VideoLayout, f_begin: int, f_end: int, stream=None) -> torch.Tensor:
    T = layout.T
    mask = torch.empty((layout.B, (f_end - f_begin) * T, f_end * T), dtype=torch.uint8,
                       device="cuda")
    check(lib.wam_debug_video_mask(layout.ref, f_begin, f_end, _ptr(mask), _stream(stream)))
    return mask


def debug_prefill_order(layout: VideoLayout, f_begin: int, f_end: int, n_sms: int,
                        with_pairing: bool = False):
    """Work items of a tensor-core prefill call over [f_begin, f_end) in launch order for a
    device of n_sms SMs (host only): int32 arrays (episode, frame, n_key_frames), and with
    with_pairing also whether items (2i, 2i + 1) share CTAs."""
    cap = max(layout.B * (f_end - f_begin), 1)
    ep, fr, nk = (np.zeros(cap, dtype=np.int32) for _ in range(3))
    n = ctypes.c_int32(0)
    paired = ctypes.c_int32(0)
    P = ctypes.POINTER(ctypes.c_int32)
    check(lib.wam_debug_prefill_order(layout.ref, f_begin, f_end, n_sms, ep.ctypes.data_as(P),
                                      fr.ctypes.data_as(P), nk.ctypes.data_as(P), ctypes.byref(n),
                                      ctypes.byref(paired)))
    out = ep[:n.value], fr[:n.value], nk[:n.value]
    return out + (bool(paired.value),) if with_pairing else out


def nvfp4_workspace_size(n: int) -> int:
    out = ctypes.c_size_t(0)
    check(lib.wam_nvfp4_workspace_size(int(n), ctypes.byref(out)))
    return out.value


class Nvfp4Cache:
    """Device buffers of NVFP4-encoded fused tensors of one layout: per tensor the codes
    [B, H, N, D / 2] and E4M3 block scales [B, H, N, D / 16] (uint8, head-major), and one fp32
    tensor scale each in ``s_g`` [n]."""

    def __init__(self, layout: VideoLayout, n: int, device=None):
        B, H, N, D = layout.B, layout.H, layout.N, layout.D
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.codes = [torch.zeros((B, H, N, D // 2), dtype=torch.uint8, device=dev) for _ in range(n)]
        self.scales = [torch.zeros((B, H, N, D // 16), dtype=torch.uint8, device=dev) for _ in range(n)]
        self.s_g = torch.zeros(n, dtype=torch.float32, device=dev)
        self.workspace = torch.zeros(nvfp4_workspace_size(n), dtype=torch.uint8, device=dev)


def fused_to_nvfp4(layout: VideoLayout, fused, cache: Nvfp4Cache, stream=None) -> None:
    """NVFP4-encode the bf16 fused tensors ``fused`` (a list) into ``cache``."""
    n = len(fused)
    fp = (ctypes.c_void_p * n)(*[_ptr(t) for t in fused])
    cp = (ctypes.c_void_p * n)(*[_ptr(t) for t in cache.codes[:n]])
    sp = (ctypes.c_void_p * n)(*[_ptr(t) for t in cache.scales[:n]])
    check(lib.wam_fused_to_nvfp4(layout.ref, n, fp, cp, sp, _ptr(cache.s_g), _ptr(cache.workspace),
                                 cache.workspace.numel(), _stream(stream)))


def action_attn_nvfp4(layout: VideoLayout, cache: Nvfp4Cache, k_index: int, v_index: int, qa, ka,
                      va, o, workspace=None, stream=None, flags: int = 0) -> None:
    """The action read over the NVFP4 fused pair held in ``cache`` at tensors k_index / v_index."""
    n_act = qa.shape[1]
    if workspace is None:
        need = action_attn_workspace_size(layout, torch.bfloat16, n_act, True)
        workspace = action_workspace(need, qa.device.index)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    sg = cache.s_g.data_ptr()
    check(lib.wam_action_attn_nvfp4(layout.ref, _ptr(cache.codes[k_index]), _ptr(cache.scales[k_index]),
                                    sg + 4 * k_index, _ptr(cache.codes[v_index]),
                                    _ptr(cache.scales[v_index]), sg + 4 * v_index, n_act, _ptr(qa),
                                    _ptr(ka), _ptr(va), _ptr(o), _dtype(o), _ptr(workspace), ws_bytes,
                                    int(flags), _stream(stream)))


def debug_wait_timeout(polls: int = 10000, stream=None) -> None:
    """Launch a wait that gives up after ``polls`` polls and records WAM_ERR_TIMEOUT in the
    device error word (read it with ``device_error``)."""
    check(lib.wam_debug_wait_timeout(int(polls), _stream(stream)))


def debug_action_plan(layout: VideoLayout, n_sms: int):
    """The NVFP4 read's work split on a device of n_sms SMs (host only): (kparts [B] int32,
    CTAs launched, largest part count)."""
    k = np.zeros(layout.B, dtype=np.int32)
    n, mx = ctypes.c_int32(0), ctypes.c_int32(0)
    check(lib.wam_debug_action_plan(layout.ref, int(n_sms), k.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                    ctypes.byref(n), ctypes.byref(mx)))
    return k, n.value, mx.value


def device_error(clear: bool = True) -> None:
    """Synchronise and raise WamError if a kernel's bounded wait gave up."""
    check(lib.wam_device_error(int(clear)))
