"""The C-ABI library on the host: it loads, exports every symbol include/wam.h declares, its
host helpers agree with the oracle, and bad arguments are rejected with a status and a
message before anything reaches the GPU.  No compute call is made (CPU only)."""

import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import wam_oracle as O
from cached_kv_attention_b200 import wam

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L = wam.lib
FAKE = 0x7F0000000000  # 16-byte aligned stand-in address; never dereferenced by these tests


def declared_functions():
    src = open(os.path.join(ROOT, "include", "wam.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wam_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"libwam.so does not export {n}"
    assert set(wam.exported_names()) <= set(names)
    assert L.wam_version() >= 100


def test_flow_schedule_matches_oracle():
    for n, end, shift in ((4, 0.9, 1.0), (10, 0.0, 1.0), (2, 0.9, 1.0), (7, 0.3, 3.0)):
        got = wam.flow_schedule(n, end, shift)
        want = O.flow_schedule(n, end, shift)
        assert got[0] == 1.0 and got[-1] == end          # endpoints bit-exact
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_fuse_weights_match_oracle():
    rng = np.random.default_rng(3)
    for n in (1, 2, 4, 16):
        x = rng.standard_normal(n).astype(np.float32)
        got = wam.fuse_weights(x)
        np.testing.assert_allclose(got, O.fuse_weights(x.astype(np.float64)), rtol=2e-7, atol=1e-8)
        assert abs(float(got.astype(np.float64).sum()) - 1.0) < 1e-6
    onehot = wam.fuse_weights([0.0, -np.inf, -np.inf])
    assert onehot.tolist() == [1.0, 0.0, 0.0]


def _lay(B=1, H=2, D=64, T=16, F=4, pad=None, block=None):
    return wam.VideoLayout(B, H, D, T, F, pad, block)


def _prefill(lay, f_begin=0, f_end=2, q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, store=1, o=FAKE,
             dt=wam.F32, o_dt=wam.F32, fuse=None):
    return L.wam_video_prefill_kv(lay.ref if lay is not None else None, dt, f_begin, f_end, q, k,
                                  v, kc, vc, store, o, o_dt, fuse, None)


def _msg():
    return L.wam_last_error().decode()


@pytest.mark.parametrize("kw,status,needle", [
    (dict(f_begin=2, f_end=2), 1, "frame range"),
    (dict(f_begin=-1, f_end=2), 1, "frame range"),
    (dict(f_begin=0, f_end=5), 1, "frame range"),
    (dict(q=0), 1, "q is NULL"),
    (dict(q=FAKE + 8), 1, "16-byte"),
    (dict(o=0), 1, "o is NULL"),
    (dict(kc=0, f_begin=2, f_end=4), 1, "k_cache"),
    (dict(dt=7), 1, "dtype"),
    (dict(dt=wam.F32, o_dt=wam.BF16), 2, "o_dt"),
])
def test_prefill_rejects_bad_arguments(kw, status, needle):
    assert _prefill(_lay(), **kw) == status
    assert needle in _msg()


def test_prefill_rejects_bad_layouts():
    assert _prefill(None) == 1 and "layout" in _msg()
    assert _prefill(_lay(D=96)) == 2 and "head dim" in _msg()
    assert _prefill(_lay(F=300)) == 2 and "WAM_MAX_FRAMES" in _msg()
    assert _prefill(_lay(B=8, F=200)) == 2 and "WAM_MAX_EPISODE_FRAMES" in _msg()
    assert _prefill(_lay(pad=[[0, 2, 0, 0]])) == 1 and "frame_pad" in _msg()
    assert _prefill(_lay(block=[0, 2, 1, 3])) == 1 and "nondecreasing" in _msg()
    # a call may not split an attention block
    assert _prefill(_lay(block=[0, 1, 1, 2]), 0, 2) == 1 and "splits" in _msg()
    assert _prefill(_lay(block=[0, 0, 1, 2]), 1, 3) == 1 and "splits" in _msg()


def test_prefill_rejects_bad_fusion_epilogue():
    e = wam._Fuse(0.5, 0, 0, None, FAKE, FAKE, FAKE)
    assert _prefill(_lay(), fuse=ctypes.byref(e)) == 1 and "acc_k" in _msg()
    e = wam._Fuse(0.5, 0, 1, FAKE, FAKE, None, FAKE)
    assert _prefill(_lay(), fuse=ctypes.byref(e)) == 1 and "fused_k" in _msg()
    e = wam._Fuse(float("nan"), 1, 1, None, None, FAKE, FAKE)
    assert _prefill(_lay(), fuse=ctypes.byref(e)) == 1 and "weight" in _msg()


def test_action_rejects_bad_arguments():
    lay = _lay()
    call = lambda **kw: L.wam_action_attn(lay.ref, kw.get("dt", wam.F32), kw.get("fk", FAKE),
                                          kw.get("fv", FAKE), kw.get("n", 8), kw.get("qa", FAKE),
                                          FAKE, FAKE, FAKE, wam.F32, None, 0, None)
    assert call(n=0) == 1 and "n_act" in _msg()
    assert call(n=129) == 1 and "n_act" in _msg()
    assert call(fv=0) == 1 and "both" in _msg()
    assert call(qa=FAKE + 4) == 1 and "aligned" in _msg()


def test_fusion_and_euler_reject_bad_arguments():
    lay = _lay()
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    w = (ctypes.c_float * 2)(0.5, 0.5)
    assert L.wam_fuse_interval_kv(lay.ref, wam.F32, 0, arr, arr, w, 0, 4, FAKE, FAKE, None) == 1
    assert L.wam_fuse_interval_kv(lay.ref, wam.F32, 17, arr, arr, w, 0, 4, FAKE, FAKE, None) == 1
    assert L.wam_fuse_interval_kv(lay.ref, wam.F32, 2, arr, arr, w, 3, 3, FAKE, FAKE, None) == 1
    bad = (ctypes.c_void_p * 2)(FAKE, 0)
    assert L.wam_fuse_interval_kv(lay.ref, wam.F32, 2, bad, arr, w, 0, 4, FAKE, FAKE, None) == 1
    assert "layer 1" in _msg()
    assert L.wam_flow_euler_step(-1, FAKE, FAKE, 0.1, None) == 1
    assert L.wam_flow_euler_step(0, None, None, 0.1, None) == 0   # empty: nothing to do
    assert L.wam_flow_euler_step(4, FAKE, FAKE, float("inf"), None) == 1
    assert L.wam_flow_euler_step(4, FAKE + 4, FAKE, 0.1, None) == 1


def test_host_helpers_reject_bad_arguments():
    out = (ctypes.c_double * 3)()
    assert L.wam_flow_schedule(0, 0.9, 1.0, out) == 1
    assert L.wam_flow_schedule(2, 1.0, 1.0, out) == 1
    assert L.wam_flow_schedule(2, 0.9, 0.0, out) == 1
    x = (ctypes.c_float * 2)(-math.inf, -math.inf)
    y = (ctypes.c_float * 2)()
    assert L.wam_fuse_weights(2, x, y) == 1 and "-inf" in _msg()
    assert L.wam_fuse_weights(0, x, y) == 1


def test_error_message_is_thread_local_and_cleared():
    assert _prefill(None) == 1 and _msg()
    out = (ctypes.c_double * 3)()
    assert L.wam_flow_schedule(2, 0.5, 1.0, out) == 0
    assert _msg() == ""


def test_copy_frames_rejects_bad_arguments():
    lay = _lay(B=1, H=2, D=64, T=16, F=4)
    nbytes = 4 * 16 * 2 * 64 * 4          # one fp32 tensor [1, F*T, H, D]
    a, b = FAKE, FAKE + 4 * nbytes
    pair = lambda x: (ctypes.c_void_p * 1)(x)
    call = lambda n=1, s=pair(a), d=pair(b), fs=1, fd=0, nf=3: L.wam_copy_frames(
        lay.ref, wam.F32, n, s, d, fs, fd, nf, None)
    assert call(n=0) == 1 and "n must be" in _msg()
    assert call(n=129) == 1 and "n must be" in _msg()
    assert call(fs=2, nf=3) == 1 and "outside" in _msg()
    assert call(fd=-1) == 1 and "outside" in _msg()
    assert call(nf=-1) == 1 and "outside" in _msg()
    assert call(d=pair(a + nbytes // 2)) == 1 and "overlap" in _msg()
    assert call(d=pair(b + 4)) == 1 and "aligned" in _msg()
    assert call(s=pair(0)) == 1 and "NULL" in _msg()
    assert call(nf=0) == 0                   # nothing to copy: valid, launches nothing


def test_debug_prefill_order_rejects_bad_arguments():
    lay = _lay(B=1, H=2, D=128, T=256, F=4)
    out = [(ctypes.c_int32 * 8)() for _ in range(3)]
    n = ctypes.c_int32(-1)
    paired = ctypes.c_int32(-1)
    call = lambda f0=0, f1=4, ep=out[0], fr=out[1], nk=out[2], cnt=ctypes.byref(n), pr=None: \
        L.wam_debug_prefill_order(lay.ref, f0, f1, 148, ep, fr, nk, cnt, pr)
    assert call(f0=2, f1=2) == 1 and "frame range" in _msg()
    assert call(ep=None) == 1 and "NULL" in _msg()
    assert call(cnt=None) == 1 and "NULL" in _msg()
    bad_t = _lay(B=1, H=2, D=128, T=64, F=4)
    assert L.wam_debug_prefill_order(bad_t.ref, 0, 4, 148, out[0], out[1], out[2],
                                     ctypes.byref(n), None) == 1 and "multiple of 128" in _msg()
    # host only: valid without a GPU.  8 CTAs on 148 SMs, 2 query tiles per frame, 4 items of
    # 4, 3, 2 and 1 key frames: paired, most with fewest
    assert call(pr=ctypes.byref(paired)) == 0 and n.value == 4 and paired.value == 1
    assert list(out[2])[:4] == [4, 1, 3, 2] and list(out[1])[:4] == [3, 0, 2, 1]
    assert call() == 0 and n.value == 4             # the pairing flag is optional
