"""libtq on the host (no GPU): exported symbols, the host Lloyd-Max solver and
the codec's random draws against the oracle, and argument checking.

The library and the oracle share no code; these tests compare two independent
implementations of the same definitions (splitmix64 + Box-Muller draws, and a
Lloyd-Max solver in theta-space with Gauss-Legendre quadrature and a
closed-form first moment against the oracle's adaptive quadrature in z).
"""
import ctypes
import os
import re

import numpy as np
import pytest

import kv_cache_vector_09_b200 as tq
import oracle as O
from conftest import ROOT


def _header_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]*?\b(tq_\w+)\s*\(", src)))


def test_library_exports_every_header_symbol():
    syms = _header_symbols()
    assert len(syms) >= 12, syms
    lib = ctypes.CDLL(tq.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s


@pytest.mark.parametrize("bits,d", [(1, 64), (2, 64), (2, 128), (3, 128), (4, 128), (3, 1536), (2, 256), (4, 64)])
def test_host_codebook_matches_oracle(bits, d):
    cen, bnd = tq.tq_make_codebook(bits, d)
    oc, ob = O.published_codebook(bits, d)
    assert np.array_equal(cen, oc), (cen, oc)
    assert np.array_equal(bnd, ob), (bnd, ob)


@pytest.mark.parametrize("d,bits,m,seed", [(128, (2,), 128, 0), (128, (3,), 128, 0), (128, (2, 3), 64, 0),
                                           (64, (2,), 64, 0), (128, (4,), 0, 0), (1536, (3,), 256, 0),
                                           (256, (1,), 32, 12345)])
def test_host_codec_draws_match_oracle(d, bits, m, seed):
    c = tq.Codec(d, bits, m, seed, device=-1)
    S, ds, cen, bnd = c.export()
    oc = O.make_codec(d, bits, m, seed)
    neg = np.array([(ds[i // 32] >> (i % 32)) & 1 for i in range(d)], dtype=bool)
    assert np.array_equal(np.where(neg, -1.0, 1.0), oc.D)
    if m:
        assert np.array_equal(S, oc.S), np.abs(S - oc.S).max()
    for s in range(len(bits)):
        assert np.array_equal(cen[s], oc.cen[s]) and np.array_equal(bnd[s], oc.bnd[s])
    W = sum(b * (d // len(bits)) // 32 for b in bits)
    assert c.code_words == W and c.sign_words == m // 32
    assert c.code_words == oc.words


def test_invalid_arguments_are_rejected_on_the_host():
    lib = tq.c_api()
    with pytest.raises(tq.TQError) as e:
        tq.tq_make_codebook(5, 128)
    assert e.value.status == 1
    with pytest.raises(tq.TQError) as e:
        tq.Codec(96, (2,), 64, 0, device=-1)
    assert e.value.status == 2
    for bad in [dict(d=128, seg_bits=(0,), m=32), dict(d=128, seg_bits=(2,), m=40),
                dict(d=128, seg_bits=(2, 2, 2), m=32), dict(d=128, seg_bits=(2,), m=2048)]:
        with pytest.raises(tq.TQError) as e:
            tq.Codec(bad["d"], bad["seg_bits"][:3], bad["m"], 0, device=-1) if len(bad["seg_bits"]) <= 2 else \
                _raw_spec(lib, bad)
        assert e.value.status == 1
    # compute calls on a host-only codec fail before touching a GPU
    c = tq.Codec(128, (2,), 64, 0, device=-1)
    comp = tq.tq_compressed()
    st = lib.tq_quantize(c.handle, None, 1, 1, 128, ctypes.byref(comp), None)
    assert st == 1 and "host-only" in tq.tq_last_error_string()
    v = ctypes.c_size_t()
    assert lib.tq_scores_workspace_size(c.handle, 8, 32, 8, ctypes.byref(v)) == 0 and v.value >= 8 * 32 * (128 + 64) * 4
    assert lib.tq_codec_destroy(None) == 0
    c.close()
    c.close()
    assert tq.tq_status_string(6) == "Lloyd-Max did not converge"


def _raw_spec(lib, bad):
    spec = tq.tq_spec(bad["d"], 3, (ctypes.c_int32 * 2)(2, 2), bad["m"], 0)
    h = ctypes.c_void_p()
    st = lib.tq_codec_create(ctypes.byref(spec), -1, ctypes.byref(h))
    raise tq.TQError(st, "tq_codec_create", tq.tq_last_error_string())


def test_not_converged_is_reported():
    cen = np.zeros(8, np.float32)
    bnd = np.zeros(7, np.float32)
    lib = tq.c_api()
    st = lib.tq_make_codebook(3, 128, 1e-15, 3, cen.ctypes.data, bnd.ctypes.data)
    assert st == 6 and np.all(cen == 0)


def test_search_arguments_are_checked_on_the_host():
    lib = tq.c_api()
    c = tq.Codec(1536, (3,), 256, 0, device=-1)
    assert tq.tq_search_workspace_size(c, 1024, 10) > 0
    for nq, k in [(4, 0), (4, 33), (-1, 10)]:
        with pytest.raises(tq.TQError) as e:
            tq.tq_search_workspace_size(c, nq, k)
        assert e.value.status == 1
    seg = tq.Codec(128, (2, 3), 64, 0, device=-1)
    with pytest.raises(tq.TQError) as e:
        tq.tq_search_workspace_size(seg, 4, 10)
    assert e.value.status == 2
    # a compute call on a host-only codec fails before touching a GPU
    xs = tq.tq_compressed()
    st = lib.tq_search_topk(c.handle, None, 0, 4, ctypes.byref(xs), 100, 10, None, None, None, 0, None)
    assert st == 1 and "host-only" in tq.tq_last_error_string()


def test_bench_search_batches_follow_the_library_rule():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    # 64 KB of top-k lists (8k + 4 bytes per query), multiples of 256, at least 256
    assert b.search_batches(1024, 10) == 2
    assert b.search_batches(768, 10) == 1
    assert b.search_batches(300, 32) == 2
    assert b.search_batches(1, 1) == 1


def test_bench_traffic_is_reported_only_for_the_measured_sources(monkeypatch):
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod2", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    stages = sorted(b.STAGE_SOURCES)
    assert stages == sorted(b.TRAFFIC)
    # every stage's digest covers its own kernel file and the shared sources
    for st in stages:
        for n in b.STAGE_SOURCES[st] + b.STEP_SHARED_SOURCES:
            assert os.path.exists(os.path.join(ROOT, "kv_cache_vector_09_b200", "csrc", n)), n
    # a figure recorded against the current sources is reported, one recorded
    # against other sources is not, and one stage's digest does not gate another
    cur = {st: b.stage_sources_digest(st) for st in stages}
    monkeypatch.setattr(b, "TRAFFIC", {st: (1000 + i, cur[st]) for i, st in enumerate(stages)})
    assert [b.measured_traffic(st) for st in stages] == [1000 + i for i in range(len(stages))]
    stale = dict(b.TRAFFIC)
    stale["tq_scores"] = (7, "0" * 64)
    monkeypatch.setattr(b, "TRAFFIC", stale)
    assert b.measured_traffic("tq_scores") is None
    assert b.measured_traffic("tq_attend") == stale["tq_attend"][0]
    assert b.measured_traffic("no_such_stage") is None
    assert cur["tq_scores"] != cur["tq_attend"]


def test_sign_residual_codec_checks_and_tables():
    # TurboESM's per-element residual sign: one segment, m = d, S = I; the
    # codec's mu equals the oracle's (independent quadratures)
    import oracle as O
    with pytest.raises(tq.TQError):
        tq.Codec(128, (2, 3), 128, 0, device=-1, residual=tq.TQ_RESIDUAL_SIGN)
    with pytest.raises(tq.TQError):
        tq.Codec(128, (3,), 64, 0, device=-1, residual=tq.TQ_RESIDUAL_SIGN)
    c = tq.Codec(128, (3,), 128, 0, device=-1, residual=tq.TQ_RESIDUAL_SIGN)
    S, _, _, _ = c.export()
    assert np.array_equal(S, np.eye(128, dtype=np.float32))


def test_haar_rotation_matches_the_oracle():
    # independent draws and factorisations (fp64 Gram-Schmidt in the library,
    # numpy QR in the oracle) of the same Haar rotation
    for d, seed in ((64, 5), (128, 1)):
        c = tq.Codec(d, (3,), 0, seed, device=-1, rotation=tq.TQ_ROTATION_HAAR)
        Pi = c.rotation_matrix().astype(np.float64)
        assert np.abs(Pi - O.haar_rotation(seed, d)).max() < 1e-6
    # the Hadamard codec's dense form equals the oracle's
    c = tq.Codec(128, (3,), 0, 7, device=-1)
    assert np.abs(c.rotation_matrix() - O.rotation_matrix(O.rademacher_signs(7, 128))).max() < 1e-7
    with pytest.raises(tq.TQError):
        tq.Codec(512, (3,), 0, 0, device=-1, rotation=tq.TQ_ROTATION_HAAR)


@pytest.mark.parametrize("vq_bits,d", [(1, 64), (3, 128), (5, 128), (4, 256), (6, 64)])
def test_fibquant_codebook_matches_the_oracle(vq_bits, d):
    # the library's FibQuant construction (C++) against the oracle's (numpy):
    # both run the same fp64 spiral + Lloyd steps in the same order, so the
    # fp32 codewords agree to within one rounding
    c = tq.Codec(d, (1,), 64, 0, device=-1, vq_bits=vq_bits)
    cb = c.vq_codebook()
    ob = O.fibquant_codebook(vq_bits, d)
    assert cb.shape == ob.shape == (1 << vq_bits, 2)
    assert np.all(np.abs(cb - ob) <= np.spacing(np.abs(ob))), np.abs(cb - ob).max()
    assert c.code_words == vq_bits * d // 64


def test_fibquant_codec_checks():
    for kw in (dict(vq_bits=9), dict(vq_bits=-1)):
        with pytest.raises(tq.TQError) as e:
            tq.Codec(128, (1,), 0, 0, device=-1, **kw)
        assert e.value.status == 1  # TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError) as e:
        tq.Codec(128, (2, 3), 0, 0, device=-1, vq_bits=4)
    assert e.value.status == 2  # TQ_ERR_UNSUPPORTED
    with pytest.raises(tq.TQError) as e:
        tq.Codec(128, (1,), 128, 0, device=-1, vq_bits=4, residual=tq.TQ_RESIDUAL_SIGN)
    assert e.value.status == 2  # TQ_ERR_UNSUPPORTED
    # a scalar codec has no vector codebook; the search takes scalar codes only
    with pytest.raises(tq.TQError):
        tq.Codec(128, (3,), 0, 0, device=-1).vq_codebook()
    with pytest.raises(tq.TQError) as e:
        tq.tq_search_workspace_size(tq.Codec(128, (1,), 0, 0, device=-1, vq_bits=4), 8, 4)
    assert e.value.status == 2  # TQ_ERR_UNSUPPORTED
