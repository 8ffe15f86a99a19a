"""tq_scores_noalloc: logits for callers that cannot allocate device memory.

Some callers cannot allocate device memory at all: code under a fixed memory
budget handed out once, plug-ins whose host framework owns every allocation,
or bindings without access to CUDA's allocator.  For them libtq has
tq_scores_noalloc, which runs tq_scores on a 2 MiB scratch array compiled into
the library instead of a caller workspace.

The test calls it through the C ABI on two shapes, in the order small, large,
small, where "large" needs more scratch bytes (tq_scores_workspace_size) than
"small": the third call runs on a scratch that a bigger call has just filled,
so a read of a stale byte would show.  Every call's logits are compared with
the oracle's estimator on the same compressed keys (the oracle compresses
them and its arrays are uploaded), within the logit tolerance of the other
parity tests.  It also checks that an oversized request is refused without
writing anything.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_util import LOGIT_RTOL, logit_errors

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _case(B, Hq, Hkv, T, d, bits, m, dtype, seed):
    """Keys compressed by the oracle and uploaded; the oracle's logits."""
    kc = tq.Codec(d, bits, m, seed)
    oc = O.make_codec(d, bits, m, seed)
    k = synth.heavy_rows(seed, B * Hkv * T, d, n_out=2, dtype=dtype)
    q = synth.gaussian_rows(seed + 1, B * Hq, d, dtype=dtype).reshape(B, Hq, d)
    ok = O.quantize(k.to(torch.float64).numpy(), oc)
    q64 = q.to(torch.float64).numpy()
    want = O.estimate_scores(q64, ok, oc, B, Hq, Hkv, T)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    K = tq.Compressed(up(ok.codes), up(ok.signs) if m else None, torch.from_numpy(ok.norms).to(DEV),
                      torch.from_numpy(ok.rnorms).to(DEV) if m else None)
    # logit floor nu ||q|| / sqrt(d) per (b, h, t)
    G = Hq // Hkv
    nu = ok.nu64.reshape(B, Hkv, 1, T).repeat(G, axis=2).reshape(B, Hq, T)
    qn = np.linalg.norm(q64, axis=-1)[:, :, None]
    return kc, q.to(DEV).contiguous(), K, want, nu, qn, tq.tq_scores_workspace_size(kc, B, Hq, Hkv)


def _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out):
    lib = tq.c_api()
    st = K.struct()
    dt = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}[q.dtype]
    return lib.tq_scores_noalloc(kc.handle, q.data_ptr(), dt, B, Hq, Hkv, T, ctypes.byref(st), out.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)


def test_noalloc_scores_match_oracle_small_large_small():
    shapes = [
        (1, 16, 1, 4096, 128, (2,), 128, torch.float32, 11),
        (2, 8, 2, 1000, 128, (3,), 128, torch.bfloat16, 12),
    ]
    cases = [(s, _case(*s)) for s in shapes]
    cases.sort(key=lambda c: c[1][-1])           # by scratch bytes needed
    (s_small, c_small), (s_large, c_large) = cases
    assert c_large[-1] > c_small[-1]
    for (B, Hq, Hkv, T, d, *_), (kc, q, K, want, nu, qn, _need) in ((s_small, c_small), (s_large, c_large),
                                                                      (s_small, c_small)):
        out = torch.full((B, Hq, T), float("nan"), device=DEV)
        assert _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out) == 0, tq.tq_last_error_string()
        torch.cuda.synchronize()
        err = logit_errors(out.cpu().numpy().astype(np.float64), want, nu, qn, d)
        assert err.max() <= LOGIT_RTOL, err.max()


def test_noalloc_rejects_requests_above_its_scratch():
    d, m = 128, 128
    kc = tq.Codec(d, (2,), m, 0)
    B, Hq, Hkv, T = 64, 64, 64, 4           # 4096 queries x (d + m) floats = 4 MiB of scratch
    assert tq.tq_scores_workspace_size(kc, B, Hq, Hkv) > (2 << 20)
    q = torch.zeros((B, Hq, d), device=DEV)
    K = tq.Compressed.empty(kc, B * Hkv * T)
    out = torch.full((B, Hq, T), 7.0, device=DEV)
    status = _noalloc_raw(kc, q, B, Hq, Hkv, T, K, out)
    torch.cuda.synchronize()
    assert status == 2 and "scratch" in tq.tq_last_error_string()
    assert bool((out == 7.0).all())
