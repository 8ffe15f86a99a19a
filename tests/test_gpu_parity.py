"""CUDA path (through the C ABI) against the oracle, element by element.

Small cases span several tiles with ragged tails; the full-size cases run the
launch configuration the benchmark times and compare sampled outputs, which
the oracle computes one by one from the same seeded inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_util import (ATTEND_RTOL, LOGIT_RTOL, attend_errors, compare_compressed, logit_errors)

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def gpu_quantize(codec, x_cpu: torch.Tensor, ld_pad: int = 0):
    n, d = x_cpu.shape
    if ld_pad:
        buf = torch.zeros((n, d + ld_pad), dtype=x_cpu.dtype)
        buf[:, :d] = x_cpu
        xg = buf.to(DEV)[:, :d]
    else:
        xg = x_cpu.to(DEV)
    out = tq.Compressed.empty(codec, n)
    tq.tq_quantize(codec, xg, out)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(codec) == 0
    return out


def o_codec(d, bits, m, seed=0):
    return O.make_codec(d, bits, m, seed)


def oracle_compressed_to_gpu(oc: O.Compressed, m: int):
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    return tq.Compressed(g(oc.codes), g(oc.signs) if m else None,
                         torch.from_numpy(oc.norms).to(DEV), torch.from_numpy(oc.rnorms).to(DEV) if m else None)


# ------------------------------------------------------------------ quantise
QUANT_CASES = [
    # name, d, bits, m, dtype, n, generator
    ("tiny_fp32", 128, (2,), 128, torch.float32, 4096, "tiny"),
    ("k3_bf16", 128, (3,), 128, torch.bfloat16, 3001, "heavy"),
    ("seg23_bf16", 128, (2, 3), 64, torch.bfloat16, 2049, "heavy"),
    ("v4_bf16_m0", 128, (4,), 0, torch.bfloat16, 1537, "heavy"),
    ("d64_rope_bf16", 64, (2,), 64, torch.bfloat16, 4099, "rope"),
    ("d256_fp16", 256, (1,), 32, torch.float16, 515, "gauss"),
    ("d512_b4", 512, (4,), 96, torch.float32, 257, "heavy32"),
    ("d1536_fp32", 1536, (3,), 256, torch.float32, 300, "mixture"),
]


def make_rows(kind, n, d, dtype):
    if kind == "tiny":
        w = synth.WORKLOADS["tiny"]
        return synth.kv_slab(w, "K", 0, 0, 0, n)
    if kind == "heavy":
        return synth.heavy_rows(n + d, n, d, n_out=2, dtype=dtype)
    if kind == "heavy32":
        return synth.heavy_rows(n + d, n, d, n_out=3, dtype=torch.float32)
    if kind == "rope":
        w = synth.WORKLOADS["esm_prefill"]
        return synth.kv_slab(w, "K", 1, 3, 0, n)
    if kind == "gauss":
        return synth.gaussian_rows(n, n, d, dtype=dtype)
    if kind == "mixture":
        return synth.search_rows(synth.VSEARCH, 0, n)
    raise ValueError(kind)


@pytest.mark.parametrize("case", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
def test_quantize_matches_oracle(case):
    name, d, bits, m, dtype, n, kind = case
    x = make_rows(kind, n, d, dtype)
    codec = tq.Codec(d, bits, m, 0)
    oc = o_codec(d, bits, m)
    g = gpu_quantize(codec, x)
    o = O.quantize(x.to(torch.float64).numpy(), oc)
    st = compare_compressed(g, o, oc)
    print(name, st)


def test_quantize_padded_rows_and_edge_rows():
    d, bits, m = 128, (3,), 128
    rng = np.random.default_rng(5)
    x = rng.standard_normal((40, d)).astype(np.float32)
    x[0] = 0.0                                  # zero vector
    x[1] = 1e-30 * x[1]                         # tiny values
    x[2] = 1e30 * x[2]                          # huge values (fp32 range)
    x[3] = 0.0
    x[3, 77] = -3.0                             # single spike
    x[4] = 1.0                                  # constant row
    x[5, :64] = 0.0                             # half zero
    xt = torch.from_numpy(x)
    codec = tq.Codec(d, bits, m, 7)
    oc = o_codec(d, bits, m, seed=7)
    g = gpu_quantize(codec, xt, ld_pad=4)
    o = O.quantize(x.astype(np.float64), oc)
    print(compare_compressed(g, o, oc))
    assert g.norms[0].item() == 0.0
    # n = 0 is a no-op
    tq.tq_quantize(codec, torch.empty((0, d), device=DEV), tq.Compressed.empty(codec, 0))


def test_quantize_rejects_bad_arguments():
    codec = tq.Codec(128, (2,), 64, 0)
    out = tq.Compressed.empty(codec, 8)
    x = torch.zeros((8, 128), device=DEV, dtype=torch.bfloat16)
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize(codec, x[:, 1:], out)      # misaligned base
    assert e.value.status == 1
    bad = tq.Compressed(out.codes, None, out.norms, out.rnorms)
    with pytest.raises(tq.TQError):
        tq.tq_quantize(codec, x, bad)             # signs missing with m > 0


# -------------------------------------------------------------------- scores
SCORE_CASES = [
    # name, B, Hq, Hkv, T, d, bits, m, dtype
    ("tiny", 1, 16, 1, 4096, 128, (2,), 128, torch.float32),
    ("gqa_k3", 2, 8, 2, 1000, 128, (3,), 128, torch.bfloat16),
    ("seg23", 1, 4, 1, 777, 128, (2, 3), 64, torch.bfloat16),
    ("mse_only", 1, 2, 2, 300, 128, (4,), 0, torch.bfloat16),
    ("g32", 1, 32, 1, 129, 64, (2,), 64, torch.bfloat16),
    ("g3", 2, 6, 2, 2050, 64, (3,), 32, torch.float16),
]


def _score_inputs(B, Hq, Hkv, T, d, dtype, seed):
    if (B, Hq, Hkv, T, d) == (1, 16, 1, 4096, 128):
        w = synth.WORKLOADS["tiny"]
        return synth.kv_slab(w, "K", 0, 0).reshape(1, 1, T, d), synth.queries(w)
    k = synth.heavy_rows(seed, B * Hkv * T, d, n_out=2, dtype=dtype).reshape(B, Hkv, T, d)
    q = synth.gaussian_rows(seed + 1, B * Hq, d, dtype=dtype).reshape(B, Hq, d)
    return k, q


@pytest.mark.parametrize("case", SCORE_CASES, ids=[c[0] for c in SCORE_CASES])
def test_scores_match_oracle(case):
    name, B, Hq, Hkv, T, d, bits, m, dtype = case
    k, q = _score_inputs(B, Hq, Hkv, T, d, dtype, seed=T)
    kc = tq.Codec(d, bits, m, 0)
    oc = o_codec(d, bits, m)
    # end to end: each side quantises and scores on its own
    K = gpu_quantize(kc, k.reshape(-1, d))
    qg = q.to(DEV).contiguous()
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), DEV)
    logits = torch.empty((B, Hq, T), device=DEV)
    tq.tq_scores(kc, qg, B, Hq, Hkv, T, K, logits, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    Ko = O.quantize(k.reshape(-1, d).to(torch.float64).numpy(), oc)
    st = compare_compressed(K, Ko, oc)
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Ko, oc, B, Hq, Hkv, T)
    nu = Ko.norms.astype(np.float64).reshape(B, Hkv, T).repeat(Hq // Hkv, axis=1)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, nu, qn, d)
    assert st["code_mismatch"] == 0 and st["sign_mismatch"] == 0, st
    assert err.max() <= LOGIT_RTOL, err.max()
    # the scorer alone, fed the oracle's compressed arrays
    Kg = oracle_compressed_to_gpu(Ko, m)
    logits2 = torch.empty_like(logits)
    tq.tq_scores(kc, qg, B, Hq, Hkv, T, Kg, logits2, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    err2 = logit_errors(logits2.cpu().numpy().astype(np.float64), lo, nu, qn, d)
    assert err2.max() <= LOGIT_RTOL, err2.max()
    print(name, st, "max err", err.max(), err2.max())


# ------------------------------------------------------------------- attend
ATTEND_CASES = [
    # name, B, Hq, Hkv, T, d, kbits, km, vbits, scale, vm (value sketch rows:
    # > 0 makes tq_attend use the QJL-corrected values)
    ("gqa", 2, 8, 2, 3000, 128, (3,), 128, (4,), 0.0, 0),
    ("t1", 1, 4, 1, 1, 128, (3,), 128, (4,), 0.0, 0),
    ("t5_scale", 1, 2, 2, 5, 128, (2,), 64, (3,), 0.3, 0),
    ("d64_g1", 3, 4, 4, 1111, 64, (2,), 64, (2,), 0.0, 0),
    ("g16_long", 1, 16, 1, 9000, 128, (2, 3), 64, (4,), 0.0, 0),
    ("vqjl_gqa", 2, 8, 2, 2500, 128, (3,), 128, (2,), 0.0, 128),
    ("vqjl_t1", 1, 4, 1, 1, 128, (3,), 64, (3,), 0.0, 32),
    ("vqjl_g8_long", 1, 8, 1, 5000, 64, (2,), 64, (2,), 0.0, 64),
]


@pytest.mark.parametrize("case", ATTEND_CASES, ids=[c[0] for c in ATTEND_CASES])
def test_attend_matches_oracle(case):
    name, B, Hq, Hkv, T, d, kb, km, vb, scale, vm = case
    dtype = torch.bfloat16
    k = synth.heavy_rows(T + 1, B * Hkv * T, d, n_out=2, dtype=dtype)
    v = synth.heavy_rows(T + 2, B * Hkv * T, d, n_out=2, dtype=dtype)
    q = synth.gaussian_rows(T + 3, B * Hq, d, dtype=dtype).reshape(B, Hq, d) * 2.0
    kc, vc = tq.Codec(d, kb, km, 0), tq.Codec(d, vb, vm, 1)
    okc, ovc = o_codec(d, kb, km, 0), o_codec(d, vb, vm, 1)
    K, V = gpu_quantize(kc, k), gpu_quantize(vc, v)
    ws = tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV)
    out = torch.empty((B, Hq, d), device=DEV)
    qg = q.to(DEV).contiguous()
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, K, V, out, ws, scale=scale)
    torch.cuda.synchronize()
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    sk = compare_compressed(K, Ko, okc)
    sv = compare_compressed(V, Vo, ovc)
    assert sk["code_mismatch"] == sk["sign_mismatch"] == sv["code_mismatch"] == sv["sign_mismatch"] == 0, (sk, sv)
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T, scale=scale or None)
    err = attend_errors(out.cpu().numpy().astype(np.float64), oo)
    assert err.max() <= ATTEND_RTOL, err.max()
    # isolated: oracle-compressed keys and values
    out2 = torch.empty_like(out)
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, oracle_compressed_to_gpu(Ko, km), oracle_compressed_to_gpu(Vo, vm),
                 out2, ws, scale=scale)
    torch.cuda.synchronize()
    err2 = attend_errors(out2.cpu().numpy().astype(np.float64), oo)
    assert err2.max() <= ATTEND_RTOL, err2.max()
    print(name, "max rel err", err.max(), err2.max())


def test_attend_qjl_values_on_the_prefill_shape():
    # the ESM-2-shaped prefill config's keys (after RoPE) and values, both
    # 2 bits + QJL m = 64: one full (batch, head) slab of 4096 tokens attended
    # by its query head with QJL-corrected values, against the oracle
    w = synth.WORKLOADS["esm_prefill"]
    d, T = w.d, w.T
    kc, vc = tq.Codec(d, w.k_bits, w.k_m, w.codec_seed), tq.Codec(d, w.v_bits, w.v_m, w.codec_seed + 1)
    okc, ovc = o_codec(d, w.k_bits, w.k_m, w.codec_seed), o_codec(d, w.v_bits, w.v_m, w.codec_seed + 1)
    k = synth.kv_slab(w, "K", 2, 11)
    v = synth.kv_slab(w, "V", 2, 11)
    q = synth.gaussian_rows(77, 1, d, dtype=torch.bfloat16).reshape(1, 1, d) * 2.0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    ws = tq.workspace(tq.tq_attend_workspace_size(kc, vc, 1, 1, 1, T), DEV)
    out = torch.empty((1, 1, d), device=DEV)
    tq.tq_attend(kc, vc, q.to(DEV).contiguous(), 1, 1, 1, T, oracle_compressed_to_gpu(Ko, w.k_m),
                 oracle_compressed_to_gpu(Vo, w.v_m), out, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, 1, 1, 1, T)
    err = attend_errors(out.cpu().numpy().astype(np.float64), oo)
    assert err.max() <= ATTEND_RTOL, err.max()
    # the correction is really applied: the MSE-only output is far from it
    plain = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, o_codec(d, w.v_bits, 0, w.codec_seed + 1),
                     1, 1, 1, T)
    assert attend_errors(plain, oo).max() > 10 * ATTEND_RTOL


# ------------------------------------------------------- full-size (sampled)
def _full_kv(w, which):
    return synth.kv_full(w, which)


def _sample_rows_oracle(w, which, codec_o, rows):
    """Oracle compression of selected rows (b, h, t) of a workload tensor."""
    out = []
    for r in rows:
        b, rem = divmod(int(r), w.Hkv * w.T)
        h, t = divmod(rem, w.T)
        out.append(synth.kv_slab(w, which, b, h, t, t + 1))
    x = torch.cat(out).to(torch.float64).numpy()
    return O.quantize(x, codec_o)


def _subset(c, rows):
    rows_t = torch.as_tensor(rows, device=DEV, dtype=torch.long)
    pick = lambda t: None if t is None else t.index_select(0, rows_t)
    return tq.Compressed(pick(c.codes), pick(c.signs), pick(c.norms), pick(c.rnorms))


@pytest.mark.parametrize("wname", ["llama8b_decode", "longctx", "esm_prefill"])
def test_full_size_sampled(wname):
    w = synth.WORKLOADS[wname]
    d = w.d
    kc = tq.Codec(d, w.k_bits, w.k_m, w.codec_seed)
    okc = o_codec(d, w.k_bits, w.k_m, w.codec_seed)
    kx = _full_kv(w, "K").to(DEV).reshape(-1, d)
    K = tq.Compressed.empty(kc, w.n_keys)
    tq.tq_quantize(kc, kx, K)
    torch.cuda.synchronize()
    rows = synth.sample_indices(7, w.n_keys, 2048)
    Ko = _sample_rows_oracle(w, "K", okc, rows)
    print(wname, "K", compare_compressed(_subset(K, rows), Ko, okc))
    if w.v_bits:
        vc = tq.Codec(d, w.v_bits, w.v_m, w.codec_seed + 1)
        ovc = o_codec(d, w.v_bits, w.v_m, w.codec_seed + 1)
        vx = _full_kv(w, "V").to(DEV).reshape(-1, d)
        V = tq.Compressed.empty(vc, w.n_keys)
        tq.tq_quantize(vc, vx, V)
        torch.cuda.synchronize()
        del vx
        Vo = _sample_rows_oracle(w, "V", ovc, rows)
        print(wname, "V", compare_compressed(_subset(V, rows), Vo, ovc))
    del kx
    if wname == "esm_prefill":
        return
    q = synth.queries(w)
    qg = q.to(DEV).contiguous()
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, w.B, w.Hq, w.Hkv), DEV)
    logits = torch.empty((w.B, w.Hq, w.T), device=DEV)
    tq.tq_scores(kc, qg, w.B, w.Hq, w.Hkv, w.T, K, logits, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    # repeated calls in the benchmark's launch configuration: the same logits
    # bit for bit, and no wait of the pipeline ever gives up
    again = torch.empty_like(logits)
    for _ in range(20):
        tq.tq_scores(kc, qg, w.B, w.Hq, w.Hkv, w.T, K, again, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    assert torch.equal(again, logits)
    del again
    # sampled logits: key row r against each of its G query heads
    qo = q.to(torch.float64).numpy()
    lg = logits.cpu().numpy()
    errs = []
    for j, r in enumerate(rows[:512]):
        b, rem = divmod(int(r), w.Hkv * w.T)
        h, t = divmod(rem, w.T)
        one = O.Compressed(Ko.codes[j:j + 1], Ko.signs[j:j + 1], Ko.norms[j:j + 1], Ko.rnorms[j:j + 1])
        for g in range(w.G):
            hq = h * w.G + g
            lo = O.estimate_scores(qo[b, hq][None, None], one, okc, 1, 1, 1, 1)[0, 0, 0]
            e = logit_errors(np.array([lg[b, hq, t]], np.float64), np.array([lo]), Ko.nu64[j],
                             np.linalg.norm(qo[b, hq]), d)
            errs.append(e[0])
    assert max(errs) <= LOGIT_RTOL, max(errs)
    print(wname, "sampled logits max err", max(errs))
    if wname == "llama8b_decode":
        out = torch.empty((w.B, w.Hq, d), device=DEV)
        ws2 = tq.workspace(tq.tq_attend_workspace_size(kc, vc, w.B, w.Hq, w.Hkv, w.T), DEV)
        tq.tq_attend(kc, vc, qg, w.B, w.Hq, w.Hkv, w.T, K, V, out, ws2)
        torch.cuda.synchronize()
        assert tq.tq_codec_device_error(kc) == 0 and tq.tq_codec_device_error(vc) == 0
        for (b, hq) in [(0, 0), (5, 17)]:
            h = hq // w.G
            Kb = O.quantize(synth.kv_slab(w, "K", b, h).to(torch.float64).numpy(), okc)
            Vb = O.quantize(synth.kv_slab(w, "V", b, h).to(torch.float64).numpy(), ovc)
            oo = O.attend(qo[b, hq][None, None], Kb, Vb, okc, ovc, 1, 1, 1, w.T)
            err = attend_errors(out[b, hq].cpu().numpy().astype(np.float64)[None, None], oo)
            assert err.max() <= ATTEND_RTOL, (b, hq, err.max())
            print(wname, "attend", (b, hq), err.max())
