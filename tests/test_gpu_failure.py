"""Failure detection without a GPU fault.

Every mbarrier wait in the attention kernels is bounded: a wait that gives up records
WAM_ERR_TIMEOUT in the library's device error word, the kernel skips its remaining work and
returns, and wam_device_error() reports the status on the host.  wam_debug_wait_timeout runs
one such wait on a barrier that nothing arrives on, with a short poll limit and nothing else
in flight, so the path can be exercised without a fault, a trap or a hang."""

import time

import numpy as np
import pytest

from cached_kv_attention_b200 import chunk as C
from cached_kv_attention_b200 import synth, wam
from oracle import wam_oracle as O
from tests.gpu_util import assert_parity, to64


def test_debug_wait_rejects_bad_poll_limits():
    # rejected before any CUDA call (no GPU needed): the raw entry point with a null stream
    for polls in (0, -3, (1 << 24) + 1):
        assert wam.lib.wam_debug_wait_timeout(polls, None) == 1
        assert b"polls" in wam.lib.wam_last_error()


def _tree(x, fn):
    return [_tree(y, fn) for y in x] if isinstance(x, list) else fn(x)


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_the_device_stays_usable():
    wam.device_error(clear=True)  # start from a clear word
    t0 = time.perf_counter()
    wam.debug_wait_timeout(10000)
    with pytest.raises(wam.WamError) as e:
        wam.device_error(clear=False)
    elapsed = time.perf_counter() - t0
    assert e.value.status == 5 and "bounded wait" in str(e.value)
    assert elapsed < 60.0
    # not cleared by a read without `clear`; cleared by one with it
    with pytest.raises(wam.WamError) as e:
        wam.device_error(clear=True)
    assert e.value.status == 5
    wam.device_error()

    # the next smoke-sized chunk runs and matches the oracle
    w = synth.WORKLOADS["tiny_f32"]
    inp_cpu = C.make_inputs(w, "cpu")
    inp = {k: _tree(v, lambda t: t.cuda()) for k, v in inp_cpu.items()}
    r = C.ChunkRunner(w, inp, distinct_out=True).prepare()
    r.run()
    wam.device_error()
    inp64 = {k: _tree(v, to64) for k, v in inp_cpu.items()}
    inp64["fuse_weights"] = [O.fuse_weights(x) for x in inp64.pop("fuse_logits")]
    ref = O.chunk(inp64, L=w.L, S=w.S, T=w.T, F_h=w.F_h, F_f=w.F_f,
                  n_video_steps=w.n_video_steps, n_euler_steps=w.n_euler_steps,
                  sigma_star=w.sigma_star, pad=synth.pad_mask(w).numpy())
    assert_parity(to64(r.x_act), ref["x_act"], "f32", "x_act after a timeout")
    for l in range(w.L):
        assert_parity(to64(r.act_o[l]), ref["act_o"][0][l], "f32", f"action {l} after a timeout")
    assert np.isfinite(to64(r.x_future)).all()
