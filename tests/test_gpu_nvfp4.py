"""The low-precision (NVFP4) fused cache: the encoder against the oracle's codes.

The oracle (``oracle/nvfp4.py``) fixes every code decision in fp32; the library must produce
the same E2M1 codes, the same E4M3 block scales and the same fp32 tensor scale, bit for bit,
on the non-padding frames."""

import numpy as np
import pytest
import torch

from cached_kv_attention_b200 import synth, wam
from oracle import nvfp4 as Q
from tests.gpu_util import assert_parity, dev_normal, to64

pytestmark = pytest.mark.gpu


def _unpack(codes, scales):
    """Head-major packed device codes [B, H, N, D/2] and scales [B, H, N, D/16] to the oracle's
    layout: one code per element [B, N, H, D] and scales [B, N, H, D/16]."""
    c = codes.cpu().numpy()
    lo, hi = c & 0x0F, c >> 4
    el = np.stack([lo, hi], axis=-1).reshape(c.shape[:-1] + (c.shape[-1] * 2,))
    return el.transpose(0, 2, 1, 3), scales.cpu().numpy().transpose(0, 2, 1, 3)


def _check(lay, pad, tensors):
    cache = wam.Nvfp4Cache(lay, len(tensors))
    wam.fused_to_nvfp4(lay, tensors, cache)
    torch.cuda.synchronize()
    wam.device_error()
    rows = ~np.repeat(np.asarray(pad).astype(bool), lay.T, axis=1)  # [B, N] valid rows
    for j, t in enumerate(tensors):
        want_c, want_s, want_g = Q.quantize_cache(to64(t).astype(np.float32), pad, lay.T)
        got_c, got_s = _unpack(cache.codes[j], cache.scales[j])
        got_g = np.float32(cache.s_g[j].item())
        assert got_g.view(np.uint32) == np.float32(want_g).view(np.uint32), (got_g, want_g)
        np.testing.assert_array_equal(got_s[rows], want_s[rows])
        np.testing.assert_array_equal(got_c[rows], want_c[rows])
    return cache


def test_nvfp4_encoder_matches_oracle_codes_bit_exact():
    B, H, D, T, F = 2, 3, 128, 128, 5
    pad = np.array([[1, 1, 0, 0, 0], [0, 0, 0, 1, 0]], np.uint8)
    lay = wam.VideoLayout(B, H, D, T, F, pad)
    N = F * T
    x = dev_normal((B, N, H, D), 51, "nvfp4_x", std=1 / np.sqrt(128), dtype=torch.bfloat16)
    y = dev_normal((B, N, H, D), 52, "nvfp4_y", std=3.0, dtype=torch.bfloat16)
    # heavy tails: a few large values per tensor, and blocks of tiny values
    y[0, 300, 1, 5] = 900.0
    y[1, 10, 2, :16] = 1e-6
    _check(lay, pad, [x, y])


def test_nvfp4_encoder_ties_saturation_and_zeros():
    # amax = 2688 makes s_g = 1 exactly; a block whose amax is 6 gets scale 1, so its elements
    # are encoded as themselves: midpoints between E2M1 values must round to the even code.
    B, H, D, T, F = 1, 2, 128, 128, 2
    lay = wam.VideoLayout(B, H, D, T, F)
    x = torch.zeros((B, F * T, H, D), dtype=torch.bfloat16)
    x[0, 0, 0, 0] = 2688.0
    ties = [6.0, 2.5, 0.25, 0.75, 1.25, 1.75, 3.5, 5.0, -2.5, -0.25, -5.0, 0.1, -0.1, 4.5, 2.75, 0.0]
    x[0, 1, 0, :16] = torch.tensor(ties)
    x[0, 2, 1, :16] = torch.tensor([v * 4 for v in ties])     # scale 4: the same ties
    # amax 6.1875 rounds its block scale down to 1 (6.1875 / 6 = 1.03): 6.1875 saturates to 6
    x[0, 3, 1, 16:32] = torch.tensor([6.1875] + [1.0] * 15)
    z = torch.zeros((B, F * T, H, D), dtype=torch.bfloat16)  # all zero: s_g = 0, every code 0
    cache = _check(lay, np.zeros((B, F), np.uint8), [x.cuda(), z.cuda()])
    assert cache.s_g[0].item() == 1.0 and cache.s_g[1].item() == 0.0
    codes, scales = _unpack(cache.codes[0], cache.scales[0])
    assert list(Q.e2m1_decode(codes[0, 1, 0, :16])) == \
        [6.0, 2.0, 0.0, 1.0, 1.0, 2.0, 4.0, 4.0, -2.0, 0.0, -4.0, 0.0, 0.0, 4.0, 3.0, 0.0]
    assert Q.e4m3_decode(scales[0, 3, 1, 1]) == 1.0 and Q.e2m1_decode(codes[0, 3, 1, 16]) == 6.0


def test_nvfp4_encoder_on_a_fused_pair_of_the_bench_layout():
    # the 19.2 s layout: 7 valid frames of 768 tokens, 24 heads (16.5 M elements per tensor)
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    t = dev_normal((w.B, w.N, w.H, w.D), 53, "nvfp4_fused", std=w.qkv_std, dtype=torch.bfloat16)
    _check(lay, pad, [t])


def test_nvfp4_rejects_bad_arguments():
    lay = wam.VideoLayout(1, 2, 128, 128, 2)
    x = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    cache = wam.Nvfp4Cache(lay, 1)
    with pytest.raises(wam.WamError) as e:
        cache.workspace = cache.workspace[:16]
        wam.fused_to_nvfp4(lay, [x], cache)
    assert e.value.status == 4


# ---------------------------------------------------------------------------- the NVFP4 read

READ_CASES = [
    # B, H, T, F, pad, n_act, std
    (1, 2, 128, 3, [[0, 0, 0]], 32, 1 / np.sqrt(128)),
    (2, 3, 128, 5, [[1, 1, 0, 0, 0], [0, 1, 0, 0, 0]], 17, 1 / np.sqrt(128)),
    (2, 3, 128, 5, [[1, 0, 0, 1, 0], [0, 0, 0, 0, 0]], 32, 1.0),   # logit std ~1: reference moves
    (1, 4, 256, 4, [[1, 0, 0, 0]], 1, 2.0),                         # peaky, one action token
    (3, 24, 128, 6, [[1, 1, 1, 0, 0, 0], [0] * 6, [1, 0, 0, 0, 0, 0]], 32, 1 / np.sqrt(128)),
    (1, 24, 768, 4, [[1, 0, 0, 0]], 32, 1 / np.sqrt(128)),          # 768-token frames, 19 tiles
    (1, 8, 128, 12, [[0] * 12], 32, 1 / np.sqrt(128)),              # long runs: the rings wrap
]


def _report_non_finite(o, what):
    bad = ~np.isfinite(o)
    if bad.any():
        idx = np.nonzero(bad)
        print(f"{what}: {int(bad.sum())} non-finite outputs; episodes {np.unique(idx[0])}, "
              f"queries {np.unique(idx[1])}, heads {np.unique(idx[2])}")


@pytest.mark.parametrize("B,H,T,F,pad,n_act,std", READ_CASES)
def test_nvfp4_read_matches_oracle(B, H, T, F, pad, n_act, std):
    pad = np.array(pad, np.uint8)
    lay = wam.VideoLayout(B, H, 128, T, F, pad)
    N = F * T
    g = lambda n, tok: dev_normal((B, tok, H, 128), 61, "nvread_" + n, B, H, T, F, std=std, dtype=torch.bfloat16)
    fk, fv = g("fk", N), g("fv", N)
    qa, ka, va = g("qa", n_act), g("ka", n_act), g("va", n_act)
    cache = wam.Nvfp4Cache(lay, 2)
    wam.fused_to_nvfp4(lay, [fk, fv], cache)
    o = torch.zeros((B, n_act, H, 128), device="cuda")
    wam.action_attn_nvfp4(lay, cache, 0, 1, qa, ka, va, o)
    torch.cuda.synchronize()
    wam.device_error()
    qk = Q.quantize_cache(to64(fk).astype(np.float32), pad, T)
    qv = Q.quantize_cache(to64(fv).astype(np.float32), pad, T)
    ref = Q.action_attention_nvfp4(to64(qa), to64(ka), to64(va), qk, qv, pad, T)
    _report_non_finite(to64(o), "nvfp4 read")
    assert_parity(to64(o), ref, "bf16", "nvfp4 read")


def test_nvfp4_read_at_the_bench_layout_sampled_heads():
    # the 19.2 s layout (5376 valid keys, 24 heads) in the launch configuration the chunk uses
    w = synth.WORKLOADS["ctx19.2s_bf16"]
    pad = synth.pad_mask(w).numpy()
    lay = wam.VideoLayout(w.B, w.H, w.D, w.T, w.F, pad)
    g = lambda n, tok: dev_normal((w.B, tok, w.H, w.D), 62, "nvbench_" + n, std=w.qkv_std, dtype=torch.bfloat16)
    fk, fv = g("fk", w.N), g("fv", w.N)
    qa, ka, va = g("qa", w.n_act), g("ka", w.n_act), g("va", w.n_act)
    cache = wam.Nvfp4Cache(lay, 2)
    wam.fused_to_nvfp4(lay, [fk, fv], cache)
    o = torch.zeros((w.B, w.n_act, w.H, w.D), device="cuda")
    for _ in range(2):  # twice: the workspace tickets are left ready for the next call
        wam.action_attn_nvfp4(lay, cache, 0, 1, qa, ka, va, o)
    torch.cuda.synchronize()
    wam.device_error()
    heads = [0, 11, 23]
    # the tensor scale is taken over all heads, so the oracle encodes whole tensors and the
    # sampled heads are cut from its codes
    full_k = Q.quantize_cache(to64(fk).astype(np.float32), pad, w.T)
    full_v = Q.quantize_cache(to64(fv).astype(np.float32), pad, w.T)
    qk = (full_k[0][:, :, heads], full_k[1][:, :, heads], full_k[2])
    qv = (full_v[0][:, :, heads], full_v[1][:, :, heads], full_v[2])
    ref = Q.action_attention_nvfp4(to64(qa[:, :, heads]), to64(ka[:, :, heads]), to64(va[:, :, heads]),
                                   qk, qv, pad, w.T)
    _report_non_finite(to64(o), "nvfp4 read, bench layout")
    assert_parity(to64(o)[:, :, heads], ref, "bf16", "nvfp4 read, bench layout")


def test_nvfp4_chunk_action_reads_match_oracle():
    """A whole chunk with the NVFP4 fused cache (768-token frames, 8 layers, two fusion
    intervals, 3 Euler steps): every interaction read against the oracle's read over the oracle's
    own encoding of its fused pairs, rounded to bf16 as the library stores them
    ("Long-WAM ... | Summary" §4.2: fused KV kept in BF16 before any lower precision)."""
    from cached_kv_attention_b200 import chunk as C
    from oracle import wam_oracle as O
    w = synth.WORKLOADS["ctx2.4s_bf16"].replace(L=8, n_euler_steps=3, pad_rule="prefix:1", seed=21,
                                                kv_format="nvfp4")
    pad = synth.pad_mask(w).numpy()
    tree = lambda x, fn: [tree(y, fn) for y in x] if isinstance(x, list) else fn(x)
    inp_cpu = C.make_inputs(w, "cpu")
    inp = {k: tree(v, lambda t: t.cuda()) for k, v in inp_cpu.items()}
    r = C.ChunkRunner(w, inp, distinct_out=True).prepare()
    r.run()
    wam.device_error()
    heads = [2, 13]
    inp64 = {k: tree(v, to64) for k, v in inp_cpu.items()}
    inp64["fuse_weights"] = [O.fuse_weights(lg) for lg in inp64.pop("fuse_logits")]
    ref = O.chunk(inp64, L=w.L, S=w.S, T=w.T, F_h=w.F_h, F_f=w.F_f, n_video_steps=w.n_video_steps,
                  n_euler_steps=w.n_euler_steps, sigma_star=w.sigma_star, pad=pad, heads=heads)
    bf16 = lambda x: torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    enc = [(Q.quantize_cache(bf16(ref["fused_k"][m]), pad, w.T), Q.quantize_cache(bf16(ref["fused_v"][m]), pad, w.T))
           for m in range(w.M)]
    reader = {j: m for m, j in enumerate(C.interaction_layers(w.L, w.S))}
    for i in range(w.n_euler_steps):
        for l, m in reader.items():
            want = Q.action_attention_nvfp4(inp64["act_q"][i][l], inp64["act_k"][i][l], inp64["act_v"][i][l],
                                            enc[m][0], enc[m][1], pad, w.T, heads=heads)
            got = to64(r.act_o[i * w.L + l])
            assert_parity(got[:, :, heads], want[:, :, heads], "bf16", f"nvfp4 chunk read {i},{l}")
