"""End-to-end parity of one action chunk, and stage parity at the full workload sizes in the
launch configuration the benchmark times (sampled outputs the oracle computes one by one)."""

import numpy as np
import pytest
import torch

from oracle import wam_oracle as O
from cached_kv_attention_b200 import chunk as C
from cached_kv_attention_b200 import synth, wam
from tests.gpu_util import assert_parity, dev_normal, to64, valid_rows

pytestmark = pytest.mark.gpu


def _tree(x, fn):
    if isinstance(x, list):
        return [_tree(y, fn) for y in x]
    return fn(x)


def _run_chunk(w, fusion="epilogue", frame_block=None):
    inp_cpu = C.make_inputs(w, "cpu")
    inp = {k: _tree(v, lambda t: t.cuda()) for k, v in inp_cpu.items()}
    r = C.ChunkRunner(w, inp, frame_block=frame_block, distinct_out=True, fusion=fusion).prepare()
    r.run()
    wam.device_error()
    inp64 = {k: _tree(v, to64) for k, v in inp_cpu.items()}
    inp64["fuse_weights"] = [O.fuse_weights(lg) for lg in inp64.pop("fuse_logits")]
    return r, inp64


def _oracle_chunk(w, inp64, pad, heads=None, frame_block=None):
    return O.chunk(inp64, L=w.L, S=w.S, T=w.T, F_h=w.F_h, F_f=w.F_f,
                   n_video_steps=w.n_video_steps, n_euler_steps=w.n_euler_steps,
                   sigma_star=w.sigma_star, pad=pad, frame_block=frame_block, heads=heads)


def _compare_chunk(w, r, ref, pad, heads, dtype):
    hs = list(range(w.H)) if heads is None else list(heads)
    T, F_h, F = w.T, w.F_h, w.F
    rows_h, rows_f = valid_rows(pad, T, 0, F_h), valid_rows(pad, T, F_h, F)
    for l in range(w.L):
        assert_parity(to64(r.hist_o[l])[:, :, hs][rows_h], ref["hist_o"][l][:, :, hs][rows_h], dtype, f"hist {l}")
        assert_parity(to64(r.final_o[l])[:, :, hs][rows_f], ref["final_o"][l][:, :, hs][rows_f], dtype, f"final {l}")
        for s in range(w.n_video_steps):
            got = to64(r.imag_o[s * w.L + l])[:, :, hs][rows_f]
            assert_parity(got, ref["imag_o"][s][l][:, :, hs][rows_f], dtype, f"imag {s},{l}")
    rows = valid_rows(pad, T, 0, F)
    for l in range(w.L):
        np.testing.assert_array_equal(to64(r.k_cache[l])[rows], ref["k_cache"][l][rows])
        np.testing.assert_array_equal(to64(r.v_cache[l])[rows], ref["v_cache"][l][rows])
    for m in range(w.M):
        assert_parity(to64(r.fused_k[m])[rows], ref["fused_k"][m][rows], dtype, f"fused K {m}")
        assert_parity(to64(r.fused_v[m])[rows], ref["fused_v"][m][rows], dtype, f"fused V {m}")
    for i in range(w.n_euler_steps):
        for l in range(w.L):
            assert_parity(to64(r.act_o[i * w.L + l])[:, :, hs], ref["act_o"][i][l][:, :, hs], dtype,
                          f"action {i},{l}")
    assert_parity(to64(r.x_future), ref["x_future"], "f32", "x_future")
    assert_parity(to64(r.x_act), ref["x_act"], "f32", "x_act")


@pytest.mark.parametrize("fusion", ["epilogue", "standalone"])
def test_tiny_fp32_chunk_end_to_end(fusion):
    w = synth.WORKLOADS["tiny_f32"]
    r, inp64 = _run_chunk(w, fusion)
    pad = synth.pad_mask(w).numpy()
    ref = _oracle_chunk(w, inp64, pad)
    _compare_chunk(w, r, ref, pad, None, "f32")


@pytest.mark.parametrize("variant", [dict(S=1), dict(S=3), dict(L=16, S=14),
                                     dict(n_video_steps=0, sigma_star=1.0)],
                         ids=["stride1", "stride3", "stride14_L16", "one_shot"])
def test_tiny_fp32_chunk_variants(variant):
    # The interaction-stride and one-shot variants run the same calls with other S / video steps.
    w = synth.WORKLOADS["tiny_f32"].replace(seed=8, **variant)
    r, inp64 = _run_chunk(w)
    pad = synth.pad_mask(w).numpy()
    ref = _oracle_chunk(w, inp64, pad)
    _compare_chunk(w, r, ref, pad, None, "f32")


def test_bf16_chunk_stride1_768_token_frames():
    # Every layer reads its own-layer K/V (S = 1) at the 768-token frame shape, two heads checked.
    w = synth.WORKLOADS["ctx2.4s_bf16"].replace(L=3, S=1, n_video_steps=1, n_euler_steps=2,
                                                pad_rule="prefix:1", seed=9)
    r, inp64 = _run_chunk(w)
    pad = synth.pad_mask(w).numpy()
    heads = [3, 20]
    ref = _oracle_chunk(w, inp64, pad, heads=heads)
    _compare_chunk(w, r, ref, pad, heads, "bf16")


def test_tiny_fp32_chunk_padded_and_grouped_future():
    w = synth.WORKLOADS["tiny_f32"].replace(F_h=3, pad_rule="prefix:1", seed=5)
    blocks = [0, 1, 2, 3, 3]
    r, inp64 = _run_chunk(w, "epilogue", frame_block=blocks)
    pad = synth.pad_mask(w).numpy()
    ref = _oracle_chunk(w, inp64, pad, frame_block=blocks)
    _compare_chunk(w, r, ref, pad, None, "f32")


@pytest.mark.slow
def test_bf16_chunk_768_token_frames_sampled_heads():
    # The 2.4 s chunk shape (24 heads x 128, 768 tokens per frame, 3 + 2 frames, 4 video steps)
    # with 8 layers (two fusion intervals) and 3 Euler steps; the oracle runs two heads.
    w = synth.WORKLOADS["ctx2.4s_bf16"].replace(L=8, n_euler_steps=3, pad_rule="prefix:1", seed=6)
    r, inp64 = _run_chunk(w)
    pad = synth.pad_mask(w).numpy()
    heads = [0, 17]
    ref = _oracle_chunk(w, inp64, pad, heads=heads)
    _compare_chunk(w, r, ref, pad, heads, "bf16")


# ----------------------------------------------------------------------------- full sizes

def _sample_rows(pad_b, T, f_begin, f_end, per_frame, rng):
    rows = []
    for f in range(f_begin, f_end):
        if not pad_b[f]:
            rows += list((f - f_begin) * T + rng.choice(T, per_frame, replace=False))
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["ctx19.2s_bf16", "ctx38.4s_bf16", "batched4_bf16"])
def test_full_size_stages_sampled(name):
    """One history layer, one imagination call and one fused action read at the workload's
    full size, launched exactly as the chunk launches them; the oracle computes sampled
    query rows of three heads one by one."""
    w = synth.WORKLOADS[name]
    rng = np.random.default_rng(0)
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    B, H, D, T, N = w.B, w.H, w.D, w.T, w.N
    bf = torch.bfloat16
    g = lambda n, tok: dev_normal((B, tok, H, D), w.seed, "full_" + n, std=w.qkv_std, dtype=bf)
    qh, kh, vh = g("qh", w.F_h * T), g("kh", w.F_h * T), g("vh", w.F_h * T)
    qf, kf, vf = g("qf", w.F_f * T), g("kf", w.F_f * T), g("vf", w.F_f * T)
    kc, vc = torch.zeros((B, N, H, D), dtype=bf, device="cuda"), torch.zeros((B, N, H, D), dtype=bf, device="cuda")
    oh = torch.zeros((B, w.F_h * T, H, D), device="cuda")
    of = torch.zeros((B, w.F_f * T, H, D), device="cuda")
    wam.video_prefill_kv(lay, 0, w.F_h, qh, kh, vh, kc, vc, oh, store_kv=True)
    wam.video_prefill_kv(lay, w.F_h, w.F, qf, kf, vf, kc, vc, of, store_kv=False)
    qa, ka, va = (g(n, w.n_act) for n in ("qa", "ka", "va"))
    oa = torch.zeros((B, w.n_act, H, D), device="cuda")
    wam.action_attn(lay, kc, vc, qa, ka, va, oa)   # the cache stands in for a fused pair
    torch.cuda.synchronize()
    wam.device_error()
    heads = [0, H // 2, H - 1]
    kc64, vc64 = to64(kc), to64(vc)
    for b in range(B):
        pb = pad[b:b + 1]
        # history rows
        rows = _sample_rows(pad[b], T, 0, w.F_h, 6, rng)
        ref = O.video_prefill(to64(qh[b:b + 1]), to64(kh[b:b + 1]), to64(vh[b:b + 1]), None, None,
                              pb, None, T, 0, w.F_h, heads=heads, rows=rows)
        assert_parity(to64(oh[b:b + 1])[:, rows][:, :, heads], ref[:, rows][:, :, heads], "bf16", f"{name} hist b{b}")
        # imagination rows read the stored history cache
        rows = _sample_rows(pad[b], T, w.F_h, w.F, 12, rng)
        ref = O.video_prefill(to64(qf[b:b + 1]), to64(kf[b:b + 1]), to64(vf[b:b + 1]), kc64[b:b + 1],
                              vc64[b:b + 1], pb, None, T, w.F_h, w.F, heads=heads, rows=rows)
        assert_parity(to64(of[b:b + 1])[:, rows][:, :, heads], ref[:, rows][:, :, heads], "bf16", f"{name} imag b{b}")
        # the cache holds the new history K of valid frames bit-exactly
        krows = valid_rows(pb, T, 0, w.F_h)[0]
        np.testing.assert_array_equal(kc64[b, :w.F_h * T][krows], to64(kh[b])[krows])
        # action read over the full cache
        ref = O.action_attention(to64(qa[b:b + 1]), to64(ka[b:b + 1]), to64(va[b:b + 1]),
                                 kc64[b:b + 1], vc64[b:b + 1], pb, T, heads=heads)
        assert_parity(to64(oa[b:b + 1])[:, :, heads], ref[:, :, heads], "bf16", f"{name} action b{b}")


# ----------------------------------------------------------------------------- co-denoising

@pytest.mark.parametrize("name,dtype", [("tiny_f32", "f32"), ("ctx2.4s_bf16", "bf16")])
def test_joint_chunk(name, dtype):
    # Co-denoising: every joint step re-passes the future frames (cache store + fusion
    # epilogue) before its action reads; compared step by step with the oracle's joint chunk.
    base = synth.WORKLOADS[name]
    if dtype == "f32":
        w = base.replace(seed=12, joint=True, n_video_steps=0, n_euler_steps=3)
        heads = None
    else:
        w = base.replace(L=3, S=2, joint=True, n_video_steps=0, n_euler_steps=2,
                         pad_rule="prefix:1", seed=13)
        heads = [5, 19]
    r, inp64 = _run_chunk(w)
    pad = synth.pad_mask(w).numpy()
    ref = O.chunk_joint(inp64, L=w.L, S=w.S, T=w.T, F_h=w.F_h, F_f=w.F_f,
                        n_steps=w.n_euler_steps, pad=pad, heads=heads)
    hs = list(range(w.H)) if heads is None else heads
    T, F_h, F = w.T, w.F_h, w.F
    rows_h, rows_f, rows = valid_rows(pad, T, 0, F_h), valid_rows(pad, T, F_h, F), valid_rows(pad, T, 0, F)
    for l in range(w.L):
        assert_parity(to64(r.hist_o[l])[:, :, hs][rows_h], ref["hist_o"][l][:, :, hs][rows_h], dtype, f"hist {l}")
    for i in range(w.n_euler_steps):
        for l in range(w.L):
            assert_parity(to64(r.joint_o[i * w.L + l])[:, :, hs][rows_f], ref["joint_o"][i][l][:, :, hs][rows_f],
                          dtype, f"joint {i},{l}")
            assert_parity(to64(r.act_o[i * w.L + l])[:, :, hs], ref["act_o"][i][l][:, :, hs], dtype,
                          f"joint action {i},{l}")
    for l in range(w.L):
        np.testing.assert_array_equal(to64(r.k_cache[l])[rows], ref["k_cache"][l][rows])
    for m in range(w.M):
        assert_parity(to64(r.fused_k[m])[rows], ref["fused_k"][m][rows], dtype, f"joint fused K {m}")
        assert_parity(to64(r.fused_v[m])[rows], ref["fused_v"][m][rows], dtype, f"joint fused V {m}")
    assert_parity(to64(r.x_future), ref["x_future"], "f32", "joint x_future")
    assert_parity(to64(r.x_act), ref["x_act"], "f32", "joint x_act")


# ----------------------------------------------------------------------------- sliding window

@pytest.mark.parametrize("name,dtype", [("tiny_f32", "f32"), ("ctx2.4s_bf16", "bf16")])
def test_sliding_window_chunks(name, dtype):
    # A full chunk primes buffer set 1; one run streams two chunks (set 1 -> 0, then 0 -> 1),
    # each moving the kept frames one position earlier (wam_copy_frames) and passing only the
    # newest frame.  Compared with the oracle's streamed chunks continuing from its full chunk.
    base = synth.WORKLOADS[name]
    if dtype == "f32":
        w = base.replace(F_h=3, pad_rule="prefix:1", slide=True, seed=14)
        heads = None
    else:
        w = base.replace(F_h=4, L=3, S=2, n_video_steps=1, n_euler_steps=2, pad_rule="prefix:1",
                         slide=True, seed=15)
        heads = [2, 21]
    inp_cpu = C.make_inputs(w, "cpu")
    inp = {k: _tree(v, lambda t: t.cuda()) for k, v in inp_cpu.items()}
    r = C.ChunkRunner(w, inp, distinct_out=True).prepare()
    r.prime()
    r.run()
    wam.device_error()
    inp64 = {k: _tree(v, to64) for k, v in inp_cpu.items()}
    inp64["fuse_weights"] = [O.fuse_weights(lg) for lg in inp64.pop("fuse_logits")]
    pad = synth.pad_mask(w).numpy()
    kw = dict(L=w.L, S=w.S, T=w.T, F_h=w.F_h, F_f=w.F_f, n_video_steps=w.n_video_steps,
              n_euler_steps=w.n_euler_steps, sigma_star=w.sigma_star, pad=pad, heads=heads)
    prime = O.chunk(inp64, **kw)
    first = O.chunk_stream(prime, inp64, **kw)
    second = O.chunk_stream(first, inp64, **kw)
    hs = list(range(w.H)) if heads is None else heads
    rows = valid_rows(pad, w.T, 0, w.F)
    rows_f = valid_rows(pad, w.T, w.F_h, w.F)
    for k_set, ref in ((0, first), (1, second)):
        kc, vc, fk, fv = r._sets[k_set]
        for l in range(w.L):
            np.testing.assert_array_equal(to64(kc[l])[rows], ref["k_cache"][l][rows])
            np.testing.assert_array_equal(to64(vc[l])[rows], ref["v_cache"][l][rows])
        for m in range(w.M):
            assert_parity(to64(fk[m])[rows], ref["fused_k"][m][rows], dtype, f"slide fused K {k_set},{m}")
            assert_parity(to64(fv[m])[rows], ref["fused_v"][m][rows], dtype, f"slide fused V {k_set},{m}")
    for l in range(w.L):   # the outputs hold the second streamed chunk's
        assert_parity(to64(r.new_o[l])[:, :, hs], second["hist_o"][l][:, :, hs], dtype, f"slide newest {l}")
        assert_parity(to64(r.final_o[l])[:, :, hs][rows_f], second["final_o"][l][:, :, hs][rows_f], dtype,
                      f"slide final {l}")
        for i in range(w.n_euler_steps):
            assert_parity(to64(r.act_o[i * w.L + l])[:, :, hs], second["act_o"][i][l][:, :, hs], dtype,
                          f"slide action {i},{l}")


# ----------------------------------------------------------------------------- bench config

@pytest.mark.slow
def test_bench_config_chunk_end_to_end_sampled_heads():
    """The whole ctx19.2s_bf16 chunk the benchmark times: 30 layers, history prefill with the
    fusion epilogue, 4 imagination passes, the final cache pass folding 8 intervals (the last
    one {28, 29}), 80 fused reads of 5376 keys and 220 self-only reads, both Euler chains.
    Every stage output, cache and fused pair is compared with the oracle's chunk on two heads
    (attention and fusion are independent per head, so the oracle runs on those heads alone);
    the Euler states depend on no head and are compared whole."""
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    heads = [4, 19]
    pad = synth.pad_mask(w).numpy()

    def both(t):  # the device copy, and the sampled heads widened for the oracle
        return t.cuda(), to64(t[:, :, heads])

    pairs = C.make_inputs(w, "cpu", post=both)
    inp = {k: _tree(v, lambda p: p[0] if isinstance(p, tuple) else p.cuda()) for k, v in pairs.items()}
    inp64 = {k: _tree(v, lambda p: p[1] if isinstance(p, tuple) else to64(p)) for k, v in pairs.items()}
    del pairs
    inp64["fuse_weights"] = [O.fuse_weights(lg) for lg in inp64.pop("fuse_logits")]
    r = C.ChunkRunner(w, inp, distinct_out=True).prepare()
    r.run()
    wam.device_error()
    ref = _oracle_chunk(w, inp64, pad)

    T, F_h, F = w.T, w.F_h, w.F
    rows_h, rows_f, rows = valid_rows(pad, T, 0, F_h), valid_rows(pad, T, F_h, F), valid_rows(pad, T, 0, F)
    worst = {}

    def check(got, want, what, stage):
        e = assert_parity(got, want, "bf16", what)
        d = np.abs(np.asarray(got) - want)
        mean_rel = float(d.sum() / np.abs(want).sum())
        m = worst.setdefault(stage, [0.0, 0.0])
        m[0], m[1] = max(m[0], e), max(m[1], mean_rel)

    g = lambda t: to64(t)[:, :, heads]
    for l in range(w.L):
        check(g(r.hist_o[l])[rows_h], ref["hist_o"][l][rows_h], f"hist {l}", "history")
        check(g(r.final_o[l])[rows_f], ref["final_o"][l][rows_f], f"final {l}", "final")
        for s in range(w.n_video_steps):
            check(g(r.imag_o[s * w.L + l])[rows_f], ref["imag_o"][s][l][rows_f], f"imag {s},{l}", "imagination")
        np.testing.assert_array_equal(g(r.k_cache[l])[rows], ref["k_cache"][l][rows])
        np.testing.assert_array_equal(g(r.v_cache[l])[rows], ref["v_cache"][l][rows])
    for m in range(w.M):
        check(g(r.fused_k[m])[rows], ref["fused_k"][m][rows], f"fused K {m}", "fused pairs")
        check(g(r.fused_v[m])[rows], ref["fused_v"][m][rows], f"fused V {m}", "fused pairs")
    reader = set(C.interaction_layers(w.L, w.S))
    for i in range(w.n_euler_steps):
        for l in range(w.L):
            check(g(r.act_o[i * w.L + l]), ref["act_o"][i][l], f"action {i},{l}",
                  "fused read" if l in reader else "self-only read")
    assert_parity(to64(r.x_future), ref["x_future"], "f32", "x_future")
    assert_parity(to64(r.x_act), ref["x_act"], "f32", "x_act")
    for stage, (mx, mean) in worst.items():  # margins against the bf16 bounds (1e-2, 2e-3)
        print(f"bench-config parity {stage}: worst max|err|/max|ref| {mx:.2e}, worst mean rel {mean:.2e}")
