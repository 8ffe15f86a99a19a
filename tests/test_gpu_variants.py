"""Codec variants against the oracle: TurboESM's per-element residual sign.

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
