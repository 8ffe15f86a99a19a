"""tq_scores_noalloc: logits for callers that cannot allocate device memory.

Some callers cannot allocate device memory at all: code under a fixed memory
budget handed out once, plug-ins whose host framework owns every allocation,
or bindings without access to CUDA's allocator.  For them libtq has
tq_scores_noalloc, which runs tq_scores on a 2 MiB scratch array compiled into
the library instead of a caller workspace.  This test calls it through the C
ABI twice in a row, on different shapes so that the second call runs on what
the first left in the shared scratch.  Each time its logits must match those of
tq_scores with a caller workspace.  It also checks that an oversized request is
refused without writing anything.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from parity_util import LOGIT_RTOL

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _case(B, Hq, Hkv, T, d, bits, m, dtype, seed):
    dev = torch.device("cuda", 0)
    kc = tq.Codec(d, bits, m, seed)
    k = synth.heavy_rows(seed, B * Hkv * T, d, n_out=2, dtype=dtype).to(dev)
    q = synth.gaussian_rows(seed + 1, B * Hq, d, dtype=dtype).reshape(B, Hq, d).to(dev).contiguous()
    K = tq.Compressed.empty(kc, B * Hkv * T)
    tq.tq_quantize(kc, k, K)
    ref = torch.empty((B, Hq, T), device=dev)
    ws = tq.workspace(tq.tq_scores_workspace_size(kc, B, Hq, Hkv), dev)
    tq.tq_scores(kc, q, B, Hq, Hkv, T, K, ref, ws)
    return kc, q, K, ref


def _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out):
    lib = tq.c_api()
    st = K.struct()
    dt = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}[q.dtype]
    status = lib.tq_scores_noalloc(kc.handle, q.data_ptr(), dt, B, Hq, Hkv, T, ctypes.byref(st), out.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    return status


def _assert_close(out, ref):
    o, r = out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
    scale = np.maximum(np.abs(r), np.abs(r).mean())
    err = np.abs(o - r) / scale
    assert err.max() <= LOGIT_RTOL, err.max()


def test_noalloc_scores_match_workspace_scores_twice():
    cases = [
        (1, 16, 1, 4096, 128, (2,), 128, torch.float32, 11),
        (2, 8, 2, 1000, 128, (3,), 128, torch.bfloat16, 12),
    ]
    for (B, Hq, Hkv, T, d, bits, m, dtype, seed) in cases:
        kc, q, K, ref = _case(B, Hq, Hkv, T, d, bits, m, dtype, seed)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out) == 0, tq.tq_last_error_string()
        torch.cuda.synchronize()
        _assert_close(out, ref)


def test_noalloc_rejects_requests_above_its_scratch():
    d, m = 128, 128
    kc = tq.Codec(d, (2,), m, 0)
    B, Hq, Hkv, T = 64, 64, 64, 4           # 4096 queries x (d + m) floats = 4 MiB of scratch
    assert tq.tq_scores_workspace_size(kc, B, Hq, Hkv) > (2 << 20)
    dev = torch.device("cuda", 0)
    q = torch.zeros((B, Hq, d), device=dev)
    K = tq.Compressed.empty(kc, B * Hkv * T)
    out = torch.full((B, Hq, T), 7.0, device=dev)
    status = _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out)
    torch.cuda.synchronize()
    assert status == 2 and "scratch" in tq.tq_last_error_string()
    assert bool((out == 7.0).all())
