"""tq_search_topk on the GPU against the oracle's top-k (same compressed index).

The oracle evaluates the estimator in double on the GPU's compressed arrays
(stage-wise comparison, so a tie-decided code cannot cascade) and returns the
top-k by a full sort, ties to the lower row.  The GPU result must hold the
same rows except where the oracle's scores lie within 1e-5 nu ||q|| of the
k-th score (rows that close may swap), report each row's score to within that
tolerance, and list the scores in non-increasing order.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_09_b200")
DEV = torch.device("cuda", 0)
TIE = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _to_oracle(comp, m):
    h = lambda t: t.cpu().numpy().view(np.uint32) if t is not None else None
    return O.Compressed(codes=h(comp.codes), signs=h(comp.signs) if m else np.zeros((comp.codes.shape[0], 0), np.uint32),
                        norms=comp.norms.cpu().numpy(), rnorms=comp.rnorms.cpu().numpy() if m else
                        np.zeros(comp.codes.shape[0], np.float32))


def _gpu_search(codec, q, X, n, k):
    nq = q.shape[0]
    idx = torch.full((nq, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((nq, k), float("nan"), dtype=torch.float32, device=DEV)
    ws = tq.workspace(tq.tq_search_workspace_size(codec, nq, k), DEV)
    tq.tq_search_topk(codec, q.to(DEV).contiguous(), X, n, k, idx, sc, ws)
    torch.cuda.synchronize()
    assert tq.tq_codec_device_error(codec) == 0
    return idx.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64)


def check_topk(gi, gs, oi, os_, full_scores, tol):
    """gi/gs: GPU rows/scores; oi/os_: oracle top-k; full_scores(q, rows) ->
    oracle scores of arbitrary rows; tol[q]: tie band."""
    nq, k = gi.shape
    for i in range(nq):
        assert np.all(np.diff(gs[i]) <= tol[i] * 1e-3 + 0.0), (i, gs[i])
        assert len(set(gi[i].tolist())) == k, (i, gi[i])
        ref = full_scores(i, gi[i])
        assert np.all(np.abs(ref - gs[i]) <= tol[i]), (i, np.abs(ref - gs[i]).max(), tol[i])
        kth = os_[i, -1]
        must = set(oi[i][os_[i] > kth + tol[i]].tolist())
        assert must <= set(gi[i].tolist()), (i, must - set(gi[i].tolist()))
        assert np.all(ref >= kth - tol[i]), (i, ref.min(), kth)


SEARCH_CASES = [
    # name, d, bits, m, n, nq, k, query dtype, rows
    ("vsearch_small", 1536, (3,), 256, 6000, 40, 10, torch.float32, "mixture"),
    ("d128_b2_m64_k1", 128, (2,), 64, 1000, 300, 1, torch.float32, "gauss"),
    ("d128_b4_m0_k32", 128, (4,), 0, 777, 17, 32, torch.bfloat16, "gauss"),
    ("d64_b1_m32_nk", 64, (1,), 32, 5, 3, 5, torch.float16, "gauss"),
    ("d256_b3_m128_tail", 256, (3,), 128, 4099, 257, 7, torch.float32, "gauss"),
]


def _rows(kind, n, d, seed):
    if kind == "mixture":
        return synth.search_rows(synth.VSEARCH, 0, n)
    return synth.gaussian_rows(seed, n, d, dtype=torch.float32)


@pytest.mark.parametrize("case", SEARCH_CASES, ids=[c[0] for c in SEARCH_CASES])
def test_search_topk_matches_oracle(case):
    name, d, bits, m, n, nq, k, qdt, kind = case
    x = _rows(kind, n, d, 17 + d)
    if kind == "mixture":
        q = synth.search_queries(synth.VSEARCH)[:nq]
    else:
        q = synth.gaussian_rows(23 + d, nq, d, dtype=torch.float32)
    q = q.to(qdt)
    codec = tq.Codec(d, bits, m, 0)
    X = tq.Compressed.empty(codec, n)
    tq.tq_quantize(codec, x.to(DEV), X)
    torch.cuda.synchronize()
    gi, gs = _gpu_search(codec, q, X, n, k)
    oc = O.make_codec(d, bits, m, 0)
    Xo = _to_oracle(X, m)
    q64 = q.to(torch.float64).numpy()
    oi, os_ = O.search_topk(q64, Xo, oc, k)
    numax = float(Xo.norms.max())
    tol = TIE * numax * np.linalg.norm(q64, axis=1)

    def full_scores(i, rows):
        sub = O.Compressed(codes=Xo.codes[rows], signs=Xo.signs[rows], norms=Xo.norms[rows], rnorms=Xo.rnorms[rows])
        return O.estimate_scores(q64[i:i + 1], sub, oc, 1, 1, 1, len(rows))[0, 0]

    check_topk(gi, gs, oi, os_, full_scores, tol)
    print(name, "max |score err| / tol ok;", "kth", os_[:, -1][:3])


def test_search_rejects_bad_arguments():
    codec = tq.Codec(128, (2,), 64, 0)
    n = 300
    X = tq.Compressed.empty(codec, n)
    q = torch.zeros((4, 128), device=DEV)
    idx = torch.zeros((4, 33), dtype=torch.int32, device=DEV)
    sc = torch.zeros((4, 33), dtype=torch.float32, device=DEV)
    ws = tq.workspace(tq.tq_search_workspace_size(codec, 4, 32), DEV)
    for k, nn in [(0, n), (33, n), (10, 5)]:
        with pytest.raises(tq.TQError) as e:
            tq.tq_search_topk(codec, q, X, nn, k, idx, sc, ws)
        assert e.value.status == 1
    small = tq.workspace(16, DEV)
    with pytest.raises(tq.TQError) as e:
        tq.tq_search_topk(codec, q, X, n, 10, idx[:, :10].contiguous(), sc[:, :10].contiguous(), small)
    assert e.value.status == 1
    c2 = tq.Codec(128, (2, 3), 64, 0)
    with pytest.raises(tq.TQError) as e:
        tq.tq_search_workspace_size(c2, 4, 10)
    assert e.value.status == 2


def test_search_full_size_sampled():
    """The bench's launch: 1M-row index (d = 1536, b = 3, m = 256), all 1024
    queries, top-10.  Two sampled queries are checked against the oracle's
    scores of every index row (evaluated in blocks on the GPU's compressed
    index)."""
    w = synth.VSEARCH
    codec = tq.Codec(w.d, w.bits, w.m, w.codec_seed)
    X = tq.Compressed.empty(codec, w.n)
    for r0 in range(0, w.n, w.row_block):
        r1 = min(w.n, r0 + w.row_block)
        tq.tq_quantize(codec, synth.search_rows(w, r0, r1).to(DEV), X.rows(r0, r1))
    torch.cuda.synchronize()
    q = synth.search_queries(w)
    gi, gs = _gpu_search(codec, q, X, w.n, w.k)
    oc = O.make_codec(w.d, w.bits, w.m, w.codec_seed)
    Xo = _to_oracle(X, w.m)
    picks = synth.sample_indices(91, w.nq, 2)
    q64 = q[picks].to(torch.float64).numpy()
    # oracle top-k over all rows, block by block, then merged by a full sort
    blk = 32768
    cand_i, cand_s = [], []
    for r0 in range(0, w.n, blk):
        r1 = min(w.n, r0 + blk)
        sub = O.Compressed(codes=Xo.codes[r0:r1], signs=Xo.signs[r0:r1], norms=Xo.norms[r0:r1],
                           rnorms=Xo.rnorms[r0:r1])
        ii, ss = O.search_topk(q64, sub, oc, w.k, row_offset=r0)
        cand_i.append(ii)
        cand_s.append(ss)
    ci, cs = np.concatenate(cand_i, axis=1), np.concatenate(cand_s, axis=1)
    oi = np.empty((len(picks), w.k), np.int64)
    os_ = np.empty((len(picks), w.k))
    for t in range(len(picks)):
        order = np.lexsort((ci[t], -cs[t]))[:w.k]
        oi[t], os_[t] = ci[t, order], cs[t, order]
    tol = TIE * float(Xo.norms.max()) * np.linalg.norm(q64, axis=1)

    def full_scores(t, rows):
        sub = O.Compressed(codes=Xo.codes[rows], signs=Xo.signs[rows], norms=Xo.norms[rows], rnorms=Xo.rnorms[rows])
        return O.estimate_scores(q64[t:t + 1], sub, oc, 1, 1, 1, len(rows))[0, 0]

    check_topk(gi[picks], gs[picks], oi, os_, full_scores, tol)
    print("full-size search, queries", picks.tolist(), "kth", os_[:, -1])
