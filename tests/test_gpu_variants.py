"""Codec variants against the oracle: TurboESM's per-element residual sign,
the dense Haar rotation and FibQuant's k = 2 vector codes.

TurboESM page, "Resumo tecnico" section 2, "Correcao de Residuo QJL de 1
Bit": one sign bit per element of the quantisation residual, and a
first-order correction by the residual's mean magnitude mu.  The library
runs it as the QJL stage with S = I (m = d) and the constant mu sqrt(2d/pi)
in the per-row residual scale; the oracle evaluates
nu (<q', c_hat> + mu <q', sign(r)>) / sqrt(d) and nu (c_hat + mu sign(r)) /
sqrt(d) directly, with mu from its own quadrature.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_util import (ATTEND_RTOL, LOGIT_RTOL, attend_errors, compare_compressed, logit_errors)

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")
DEV = torch.device("cuda", 0)
SIGN = 1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _up(oc, m):
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    return tq.Compressed(g(oc.codes), g(oc.signs), torch.from_numpy(oc.norms).to(DEV),
                         torch.from_numpy(oc.rnorms).to(DEV))


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 2)])
def test_sign_residual_quantize_and_scores(d, bits):
    B, Hq, Hkv, T = 2, 8, 2, 1500
    kc = tq.Codec(d, (bits,), d, 4, residual=SIGN)
    okc = O.make_codec(d, (bits,), d, 4, residual="sign")
    k = synth.heavy_rows(41, B * Hkv * T, d, n_out=2)
    q = synth.gaussian_rows(42, B * Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d)
    K = tq.Compressed.empty(kc, B * Hkv * T)
    tq.tq_quantize(kc, k.to(DEV), K)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    print("quantize", compare_compressed(K, Ko, okc))
    # the stored residual scale is the format's constant, equal to the oracle's
    rn = K.rnorms.cpu().numpy()
    assert np.all(rn == rn[0])
    assert abs(float(rn[0]) - float(Ko.rnorms[0])) <= 2 * np.spacing(np.float32(Ko.rnorms[0]))
    # scores, end to end and on the oracle's compressed keys
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), DEV)
    qg = q.to(DEV).contiguous()
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Ko, okc, B, Hq, Hkv, T)
    nu = Ko.nu64.reshape(B, Hkv, 1, T).repeat(Hq // Hkv, axis=2).reshape(B, Hq, T)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    for KK in (K, _up(Ko, d)):
        logits = torch.empty((B, Hq, T), device=DEV)
        tq.tq_scores(kc, qg, B, Hq, Hkv, T, KK, logits, ws)
        torch.cuda.synchronize()
        err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, nu, qn, d)
        assert err.max() <= LOGIT_RTOL, err.max()


def test_sign_residual_values_in_attend():
    B, Hq, Hkv, T, d = 1, 4, 1, 2000, 128
    kc, vc = tq.Codec(d, (3,), 128, 0), tq.Codec(d, (3,), d, 1, residual=SIGN)
    okc, ovc = O.make_codec(d, (3,), 128, 0), O.make_codec(d, (3,), d, 1, residual="sign")
    k = synth.heavy_rows(51, T, d, n_out=2)
    v = synth.heavy_rows(52, T, d, n_out=2)
    q = synth.gaussian_rows(53, Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d) * 2.0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    out = torch.empty((B, Hq, d), device=DEV)
    ws = tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV)
    tq.tq_attend(kc, vc, q.to(DEV).contiguous(), B, Hq, Hkv, T, _up(Ko, 128), _up(Vo, d), out, ws)
    torch.cuda.synchronize()
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T)
    err = attend_errors(out.cpu().numpy().astype(np.float64), oo)
    assert err.max() <= ATTEND_RTOL, err.max()


# ------------------------------------------------------------ Haar rotation
# FibQuant page, section 1, step 2: a shared random orthogonal rotation,
# Haar.  The library applies the fp32 rounding of the dense Pi; the oracle its
# fp64 Pi from numpy's QR, so z differs by at most sqrt(d) 2^-24: only codes
# and signs within 1e-6 of a decision (ties, counted) may differ.
HAAR = 1


@pytest.mark.parametrize("d,bits,m", [(128, 3, 128), (64, 2, 64)])
def test_haar_quantize_scores_attend(d, bits, m):
    B, Hq, Hkv, T = 1, 8, 2, 1200
    kc = tq.Codec(d, (bits,), m, 9, rotation=HAAR)
    vc = tq.Codec(d, (4,), 0, 10, rotation=HAAR)
    okc = O.make_codec(d, (bits,), m, 9, rotation="haar")
    ovc = O.make_codec(d, (4,), 0, 10, rotation="haar")
    k = synth.heavy_rows(61, B * Hkv * T, d, n_out=2)
    v = synth.heavy_rows(62, B * Hkv * T, d, n_out=2)
    q = synth.gaussian_rows(63, B * Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d) * 2.0
    K, V = tq.Compressed.empty(kc, B * Hkv * T), tq.Compressed.empty(vc, B * Hkv * T)
    tq.tq_quantize(kc, k.to(DEV), K)
    tq.tq_quantize(vc, v.to(DEV), V)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0 and tq.tq_codec_device_error(vc) == 0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    print("haar K", compare_compressed(K, Ko, okc), "V", compare_compressed(V, Vo, ovc))
    qg = q.to(DEV).contiguous()
    # scores on the oracle's compressed keys
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), DEV)
    logits = torch.empty((B, Hq, T), device=DEV)
    tq.tq_scores(kc, qg, B, Hq, Hkv, T, _up(Ko, m), logits, ws)
    torch.cuda.synchronize()
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Ko, okc, B, Hq, Hkv, T)
    nu = Ko.nu64.reshape(B, Hkv, 1, T).repeat(Hq // Hkv, axis=2).reshape(B, Hq, T)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, nu, qn, d)
    assert err.max() <= LOGIT_RTOL, err.max()
    # attention (inverse rotation of the output by Pi^T)
    out = torch.empty((B, Hq, d), device=DEV)
    wsa = tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV)
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    Vg = tq.Compressed(g(Vo.codes), None, torch.from_numpy(Vo.norms).to(DEV), None)
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, _up(Ko, m), Vg, out, wsa)
    torch.cuda.synchronize()
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T)
    err = attend_errors(out.cpu().numpy().astype(np.float64), oo)
    assert err.max() <= ATTEND_RTOL, err.max()


# ------------------------------------------------------------ FibQuant, k = 2
# FibQuant page, sections 2.2-2.3: blocks of two rotated coordinates take the
# nearest of 2^vq_bits shared codewords.  The library's codebook is checked
# against the oracle's on the host; here the encoder (fp32 with a certified
# nearest-codeword decision, fp64 for the uncertain rows), the CUDA-core
# scorer and the attention kernel against the oracle.
@pytest.mark.parametrize("d,vq_bits,m,dtype", [(128, 5, 128, torch.bfloat16), (64, 4, 64, torch.float32),
                                               (128, 3, 0, torch.bfloat16), (256, 6, 0, torch.float32)])
def test_fibquant_quantize_scores_attend(d, vq_bits, m, dtype):
    B, Hq, Hkv, T = 1, 8, 2, 1100
    kc = tq.Codec(d, (1,), m, 11, vq_bits=vq_bits)
    vc = tq.Codec(d, (1,), 0, 12, vq_bits=vq_bits)
    okc = O.make_codec(d, (1,), m, 11, vq_bits=vq_bits)
    ovc = O.make_codec(d, (1,), 0, 12, vq_bits=vq_bits)
    k = synth.heavy_rows(71, B * Hkv * T, d, n_out=2).to(dtype)
    k[3] = 0
    v = synth.heavy_rows(72, B * Hkv * T, d, n_out=2).to(dtype)
    q = synth.gaussian_rows(73, B * Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d) * 2.0
    K, V = tq.Compressed.empty(kc, B * Hkv * T), tq.Compressed.empty(vc, B * Hkv * T)
    tq.tq_quantize(kc, k.to(DEV), K)
    tq.tq_quantize(vc, v.to(DEV), V)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0 and tq.tq_codec_device_error(vc) == 0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    print("fibquant K", compare_compressed(K, Ko, okc), "V", compare_compressed(V, Vo, ovc))
    qg = q.to(DEV).contiguous()
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), DEV)
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Ko, okc, B, Hq, Hkv, T)
    nu = Ko.nu64.reshape(B, Hkv, 1, T).repeat(Hq // Hkv, axis=2).reshape(B, Hq, T)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    logits = torch.empty((B, Hq, T), device=DEV)
    tq.tq_scores(kc, qg, B, Hq, Hkv, T, _up(Ko, m), logits, ws)
    torch.cuda.synchronize()
    err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, nu, qn, d)
    assert err.max() <= LOGIT_RTOL, err.max()
    # attention: FibQuant keys and values, and FibQuant values under scalar keys
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    Vg = tq.Compressed(g(Vo.codes), None, torch.from_numpy(Vo.norms).to(DEV), None)
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T)
    out = torch.empty((B, Hq, d), device=DEV)
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, _up(Ko, m), Vg, out,
                 tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV))
    torch.cuda.synchronize()
    assert attend_errors(out.cpu().numpy().astype(np.float64), oo).max() <= ATTEND_RTOL
    sc, osc = tq.Codec(d, (3,), 64, 13), O.make_codec(d, (3,), 64, 13)
    So = O.quantize(k.to(torch.float64).numpy(), osc)
    tq.tq_attend(sc, vc, qg, B, Hq, Hkv, T, _up(So, 64), Vg, out,
                 tq.workspace(tq.tq_attend_workspace_size(sc, vc, B, Hq, Hkv, T), DEV))
    torch.cuda.synchronize()
    oo = O.attend(q.to(torch.float64).numpy(), So, Vo, osc, ovc, B, Hq, Hkv, T)
    assert attend_errors(out.cpu().numpy().astype(np.float64), oo).max() <= ATTEND_RTOL


def test_fibquant_unsupported_paths_are_refused():
    # the top-k search and the fused RoPE encoder take scalar codes only, and
    # FibQuant values with a sketch have no attention kernel
    d = 128
    c = tq.Codec(d, (1,), 64, 0, vq_bits=4)
    x = synth.gaussian_rows(1, 64, d, dtype=torch.bfloat16).to(DEV)
    X = tq.Compressed.empty(c, 64)
    tq.tq_quantize(c, x, X)
    ws = tq.workspace(1 << 20, DEV)
    idx = torch.empty((4, 4), dtype=torch.int32, device=DEV)
    sc = torch.empty((4, 4), dtype=torch.float32, device=DEV)
    with pytest.raises(tq.TQError) as e:
        tq.tq_search_topk(c, x[:4].contiguous(), X, 64, 4, idx, sc, ws)
    assert e.value.status == 2
    cs = tq.tq_rope_cache(10000.0, d, 16)
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_rope(c, x, cs, torch.zeros(64, dtype=torch.int32, device=DEV), X)
    assert e.value.status == 2
    q = x[:4].reshape(1, 4, d).contiguous()
    out = torch.empty((1, 4, d), device=DEV)
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend(c, c, q, 1, 4, 1, 64, X, X, out, tq.workspace(tq.tq_attend_workspace_size(c, c, 1, 4, 1, 64), DEV))
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(c) == 0


@pytest.mark.parametrize("d,vq_bits,m,dtype,n", [(64, 1, 0, torch.float16, 777), (512, 8, 32, torch.bfloat16, 300)])
def test_fibquant_smallest_and_largest_codebooks(d, vq_bits, m, dtype, n):
    # N = 2 (0.5 bits per coordinate, two antipodal codewords) with fp16 rows,
    # and N = 256 (4 bits per coordinate) at d = 512 (eight words per plane,
    # one sign word per row)
    c = tq.Codec(d, (1,), m, 21, vq_bits=vq_bits)
    oc = O.make_codec(d, (1,), m, 21, vq_bits=vq_bits)
    assert np.array_equal(c.vq_codebook(), oc.vq_cb)
    x = synth.heavy_rows(81, n, d, n_out=2).to(dtype)
    x[5] = 0
    X = tq.Compressed.empty(c, n)
    tq.tq_quantize(c, x.to(DEV), X)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(c) == 0
    Xo = O.quantize(x.to(torch.float64).numpy(), oc)
    print("fibquant N =", 1 << vq_bits, compare_compressed(X, Xo, oc))
    B, Hq, Hkv = 1, 4, 1
    q = synth.gaussian_rows(82, Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d)
    logits = torch.empty((B, Hq, n), device=DEV)
    tq.tq_scores(c, q.to(DEV).contiguous(), B, Hq, Hkv, n, _up(Xo, m), logits,
                 tq.workspace(tq.tq_scores_workspace_size(c, B, Hq, Hkv), DEV))
    torch.cuda.synchronize()
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Xo, oc, B, Hq, Hkv, n)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, Xo.nu64[None, None, :], qn, d)
    assert err.max() <= LOGIT_RTOL, err.max()


def test_fibquant_append_writes_its_slots():
    # single-token append of FibQuant keys into slot t of every (b, h) row
    # block: the slots equal the oracle's codes of those rows, every other
    # cache row is untouched
    d, vq_bits, m, rows, T, t = 128, 5, 64, 6, 50, 37
    c = tq.Codec(d, (1,), m, 5, vq_bits=vq_bits)
    oc = O.make_codec(d, (1,), m, 5, vq_bits=vq_bits)
    x = synth.heavy_rows(91, rows, d, n_out=2).to(torch.bfloat16)
    cache = tq.Compressed.empty(c, rows * T)
    for a in (cache.codes, cache.signs):
        a.fill_(-1)
    cache.norms.fill_(-1.0)
    cache.rnorms.fill_(-1.0)
    tq.tq_append(c, x.to(DEV), t, T, cache)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(c) == 0
    slots = [r * T + t for r in range(rows)]
    Xo = O.quantize(x.to(torch.float64).numpy(), oc)
    print("fibquant append", compare_compressed(cache, Xo, oc, rows=slots))
    others = np.setdiff1d(np.arange(rows * T), slots)
    assert np.all(cache.codes.cpu().numpy()[others] == -1)
    assert np.all(cache.norms.cpu().numpy()[others] == -1.0)


def test_haar_with_fibquant_codes():
    # the FibQuant page's own pipeline: norm, shared Haar rotation, k = 2
    # vector codes (plus the QJL stage here); values Haar + FibQuant, m = 0
    d, vq_bits, m = 128, 4, 64
    B, Hq, Hkv, T = 1, 4, 1, 900
    kc = tq.Codec(d, (1,), m, 31, rotation=HAAR, vq_bits=vq_bits)
    vc = tq.Codec(d, (1,), 0, 32, rotation=HAAR, vq_bits=vq_bits)
    okc = O.make_codec(d, (1,), m, 31, rotation="haar", vq_bits=vq_bits)
    ovc = O.make_codec(d, (1,), 0, 32, rotation="haar", vq_bits=vq_bits)
    k = synth.heavy_rows(101, T, d, n_out=2).to(torch.bfloat16)
    v = synth.heavy_rows(102, T, d, n_out=2).to(torch.bfloat16)
    q = synth.gaussian_rows(103, Hq, d, dtype=torch.bfloat16).reshape(B, Hq, d) * 2.0
    K, V = tq.Compressed.empty(kc, T), tq.Compressed.empty(vc, T)
    tq.tq_quantize(kc, k.to(DEV), K)
    tq.tq_quantize(vc, v.to(DEV), V)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(kc) == 0 and tq.tq_codec_device_error(vc) == 0
    Ko = O.quantize(k.to(torch.float64).numpy(), okc)
    Vo = O.quantize(v.to(torch.float64).numpy(), ovc)
    print("haar + fibquant K", compare_compressed(K, Ko, okc), "V", compare_compressed(V, Vo, ovc))
    qg = q.to(DEV).contiguous()
    logits = torch.empty((B, Hq, T), device=DEV)
    tq.tq_scores(kc, qg, B, Hq, Hkv, T, _up(Ko, m), logits, tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), DEV))
    torch.cuda.synchronize()
    lo = O.estimate_scores(q.to(torch.float64).numpy(), Ko, okc, B, Hq, Hkv, T)
    qn = np.linalg.norm(q.to(torch.float64).numpy(), axis=-1)[:, :, None]
    err = logit_errors(logits.cpu().numpy().astype(np.float64), lo, Ko.nu64[None, None, :], qn, d)
    assert err.max() <= LOGIT_RTOL, err.max()
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    Vg = tq.Compressed(g(Vo.codes), None, torch.from_numpy(Vo.norms).to(DEV), None)
    out = torch.empty((B, Hq, d), device=DEV)
    tq.tq_attend(kc, vc, qg, B, Hq, Hkv, T, _up(Ko, m), Vg, out,
                 tq.workspace(tq.tq_attend_workspace_size(kc, vc, B, Hq, Hkv, T), DEV))
    torch.cuda.synchronize()
    oo = O.attend(q.to(torch.float64).numpy(), Ko, Vo, okc, ovc, B, Hq, Hkv, T)
    assert attend_errors(out.cpu().numpy().astype(np.float64), oo).max() <= ATTEND_RTOL
