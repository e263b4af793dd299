"""Host entry points called from several threads at once.

The library keeps small per-device host caches (SM count, the cluster split of the action
read) and a thread-local error message.  ctypes releases the GIL for the duration of a foreign
call, so these threads really do enter the library together."""

import threading

import numpy as np
import pytest
import torch

from cached_kv_attention_b200 import synth, wam
from tests.gpu_util import dev_normal

N_THREADS = 8


def _run_threads(fn):
    barrier = threading.Barrier(N_THREADS)
    out = [None] * N_THREADS

    def body(i):
        barrier.wait()
        try:
            out[i] = ("ok", fn(i))
        except Exception as e:  # noqa: BLE001 - reported per thread below
            out[i] = ("err", e)

    ts = [threading.Thread(target=body, args=(i,)) for i in range(N_THREADS)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    return out


def test_prefill_order_from_many_threads_matches_one_thread():
    w = synth.WORKLOADS["batched4_bf16"]
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    want = wam.debug_prefill_order(lay, 0, w.F_h, 148)
    # each thread alternates between two work lists, so the per-thread memo is both hit and missed
    def fn(i):
        res = []
        for r in range(20):
            f_begin, f_end = ((0, w.F_h), (w.F_h, w.F))[(i + r) % 2]
            res.append(((f_begin, f_end), wam.debug_prefill_order(lay, f_begin, f_end, 148)))
        return res
    other = wam.debug_prefill_order(lay, w.F_h, w.F, 148)
    for status, res in _run_threads(fn):
        assert status == "ok", res
        for (f_begin, _), got in res:
            ref = want if f_begin == 0 else other
            for g, r in zip(got, ref):
                np.testing.assert_array_equal(g, r)


def test_workspace_size_from_many_threads_is_consistent():
    # With a GPU every thread gets the same size; without one every thread gets the same
    # error, and each thread's message is its own (thread-local).
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, synth.pad_mask(w).numpy())

    def fn(i):
        vals = []
        for _ in range(50):
            try:
                vals.append(("size", wam.action_attn_workspace_size(lay, torch.bfloat16, 32, True)))
            except wam.WamError as e:
                vals.append(("status", e.status))
        return vals

    results = _run_threads(fn)
    first = results[0][1][0]
    for status, vals in results:
        assert status == "ok"
        assert all(v == first for v in vals), vals[:4]


@pytest.mark.gpu
def test_action_reads_from_many_threads_match_one_thread():
    # Eight host threads launch fused reads at once, each on its own stream; every output
    # equals the single-thread result bit for bit.
    w = synth.WORKLOADS["ctx2.4s_bf16"]
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    B, H, D, N = w.B, w.H, w.D, w.N
    g = lambda n, tok: dev_normal((B, tok, H, D), 41, n, std=w.qkv_std, dtype=torch.bfloat16)
    fk, fv = g("fk", N), g("fv", N)
    qa, ka, va = g("qa", 32), g("ka", 32), g("va", 32)
    ref = torch.zeros((B, 32, H, D), device="cuda")
    wam.action_attn(lay, fk, fv, qa, ka, va, ref)
    torch.cuda.synchronize()
    outs = [torch.zeros_like(ref) for _ in range(N_THREADS)]
    streams = [torch.cuda.Stream() for _ in range(N_THREADS)]
    nbytes = wam.action_attn_workspace_size(lay, torch.bfloat16, 32, True)
    wss = [torch.zeros(max(nbytes, 16), dtype=torch.uint8, device="cuda") for _ in range(N_THREADS)]

    def fn(i):
        torch.cuda.set_device(0)
        for _ in range(10):
            wam.action_attn(lay, fk, fv, qa, ka, va, outs[i], workspace=wss[i] if nbytes else None,
                            stream=streams[i])
        return True

    for status, res in _run_threads(fn):
        assert status == "ok", res
    torch.cuda.synchronize()
    wam.device_error()
    for o in outs:
        assert torch.equal(o, ref)
