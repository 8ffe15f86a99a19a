"""Fused RoPE and single-token append (the decode step's write side) against
the oracle.

TurboESM page, "Resumo tecnico" section 2: keys are RoPE'd first and rotated
after.  The library applies RoPE in fp32 from a cos/sin cache and then encodes
the result exactly; the oracle applies RoPE in double.  The two inputs differ
by a few fp32 roundings, so codes and signs may differ only at boundary ties
(oracle margin below 1e-6, counted by compare_compressed), and the norm gets
5 more fp32 units of tolerance: each RoPE'd element carries at most
3u (|x_i| + |x_{i+d/2}|) of error (cache value, product and fused add), which
moves ||x'|| by at most 3 sqrt(2) u ||x|| < 5u ||x||.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_util import ATTEND_RTOL, attend_errors, compare_compressed

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")
DEV = torch.device("cuda", 0)
THETA = 10000.0


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _raw_keys(w, b, h, t0, t1):
    """Keys of the prefill workload before RoPE (the generator's draw with its
    RoPE switched off), [t1 - t0, d] in the workload's dtype."""
    return synth.kv_slab(dataclasses.replace(w, rope=False), "K", b, h, t0, t1)


def test_rope_cache_values():
    cs = tq.tq_rope_cache(THETA, 64, 4096).cpu().numpy().astype(np.float64)
    pos = np.arange(4096)[:, None]
    ang = pos * THETA ** (-2.0 * np.arange(32) / 64)[None, :]
    assert np.abs(cs[:, :32] - np.cos(ang)).max() <= 2.0 ** -24
    assert np.abs(cs[:, 32:] - np.sin(ang)).max() <= 2.0 ** -24


@pytest.mark.parametrize("case", [("esm_k_bf16", 64, (2,), 64, torch.bfloat16),
                                  ("llama_k_bf16", 128, (3,), 128, torch.bfloat16),
                                  ("d64_f32_m0", 64, (4,), 0, torch.float32)])
def test_quantize_rope_matches_oracle(case):
    name, d, bits, m, dtype = case
    w = synth.WORKLOADS["esm_prefill"]
    # 3 slabs of the prefill workload's keys, ragged: 4099 rows over positions
    parts, pos = [], []
    for (b, h, t0, t1) in [(0, 0, 0, 2048), (1, 7, 2048, 4096), (3, 19, 1000, 1003)]:
        x = _raw_keys(w, b, h, t0, t1)
        if d == 128:
            x = torch.cat([x, x.flip(1)], dim=1)   # a 128-wide row from the same draw
        parts.append(x.to(dtype))
        pos.append(np.arange(t0, t1))
    x = torch.cat(parts)
    pos = np.concatenate(pos)
    n = x.shape[0]
    codec = tq.Codec(d, bits, m, 3)
    oc = O.make_codec(d, bits, m, 3)
    cs = tq.tq_rope_cache(THETA, d, 4096)
    out = tq.Compressed.empty(codec, n)
    tq.tq_quantize_rope(codec, x.to(DEV), cs, torch.from_numpy(pos.astype(np.int32)).to(DEV), out)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(codec) == 0
    o = O.quantize(O.rope_rotate_half(x.to(torch.float64).numpy(), pos, THETA), oc)
    st = compare_compressed(out, o, oc, nu_extra_ulp=5.0)
    print(name, st)
    # without RoPE the same rows would give other codes: the rotation is applied
    plain = tq.Compressed.empty(codec, n)
    tq.tq_quantize(codec, x.to(DEV), plain)
    torch.cuda.synchronize()
    assert not torch.equal(plain.codes, out.codes)


def test_rope_position_outside_the_cache_is_reported():
    codec = tq.Codec(64, (2,), 64, 0)
    cs = tq.tq_rope_cache(THETA, 64, 100)
    x = synth.gaussian_rows(3, 10, 64).to(DEV)
    pos = torch.arange(10, dtype=torch.int32, device=DEV)
    pos[4] = 100                                   # one past the cache
    out = tq.Compressed.empty(codec, 10)
    tq.tq_quantize_rope(codec, x, cs, pos, out)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(codec) == 3
    assert tq.tq_codec_device_error(codec) == 0     # read and cleared
    # the host refuses an append position beyond the cache
    cache = tq.Compressed.empty(codec, 4 * 200)
    with pytest.raises(tq.TQError):
        tq.tq_append(codec, x[:4].contiguous(), 150, 200, cache, cs)


def test_append_then_attend_matches_oracle():
    # A decode step on a small GQA layer: the cache holds T tokens per (b, h)
    # sequence-head; tokens 0..T-2 were compressed by a prefill (RoPE'd keys),
    # the step appends token T-1 (key with RoPE at position T-1, value plain)
    # into its fixed slot and attends over all T.
    B, Hq, Hkv, T, d = 2, 8, 2, 300, 128
    kc, vc = tq.Codec(d, (3,), 128, 5), tq.Codec(d, (4,), 0, 6)
    okc, ovc = O.make_codec(d, (3,), 128, 5), O.make_codec(d, (4,), 0, 6)
    kx = synth.heavy_rows(21, B * Hkv * T, d, n_out=2).reshape(B * Hkv, T, d)
    vx = synth.heavy_rows(22, B * Hkv * T, d, n_out=2).reshape(B * Hkv, T, d)
    q = synth.gaussian_rows(23, B * Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d)
    cs = tq.tq_rope_cache(THETA, d, 4096)
    n = B * Hkv * T
    K, V = tq.Compressed.empty(kc, n), tq.Compressed.empty(vc, n)
    # prefill of tokens 0..T-2, row (r, t) at r * T + t
    pos = torch.arange(T, dtype=torch.int32).repeat(B * Hkv)
    pre = torch.arange(n) % T != T - 1
    kflat, vflat = kx.reshape(n, d), vx.reshape(n, d)
    tq.tq_quantize_rope(kc, kflat.to(DEV), cs, pos.to(DEV), K)
    tq.tq_quantize(vc, vflat.to(DEV), V)
    torch.cuda.synchronize()
    before = [t.clone() for t in (K.codes, K.signs, K.norms, K.rnorms, V.codes, V.norms)]
    # overwrite the last slot with garbage, then append the new token there
    last = torch.arange(B * Hkv) * T + (T - 1)
    for t in (K.codes, K.signs, V.codes):
        t[last] = -1
    K.norms[last] = -7.0
    V.norms[last] = -7.0
    tq.tq_append(kc, kx[:, T - 1].contiguous().to(DEV), T - 1, T, K, cs)
    tq.tq_append(vc, vx[:, T - 1].contiguous().to(DEV), T - 1, T, V)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0 and tq.tq_codec_device_error(vc) == 0
    # the append rewrote exactly the last slots, identically to the prefill
    for a, b in zip((K.codes, K.signs, K.norms, K.rnorms, V.codes, V.norms), before):
        assert torch.equal(a, b)
    # and those rows against the oracle
    okx = O.rope_rotate_half(kx[:, T - 1].to(torch.float64).numpy(), np.full(B * Hkv, T - 1), THETA)
    Ko_new = O.quantize(okx, okc)
    sub = tq.Compressed(K.codes[last], K.signs[last], K.norms[last], K.rnorms[last])
    print("appended keys", compare_compressed(sub, Ko_new, okc, nu_extra_ulp=5.0))
    # attention over the whole cache against the oracle on the same keys/values
    out = torch.empty((B, Hq, d), device=DEV)
    ws = tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV)
    qg = q.to(DEV).contiguous()
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, K, V, out, ws)
    torch.cuda.synchronize()
    Ko = O.quantize(O.rope_rotate_half(kflat.to(torch.float64).numpy(), pos.numpy(), THETA), okc)
    Vo = O.quantize(vflat.to(torch.float64).numpy(), ovc)
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T)
    err = attend_errors(out.cpu().numpy().astype(np.float64), oo)
    assert err.max() <= ATTEND_RTOL, err.max()
