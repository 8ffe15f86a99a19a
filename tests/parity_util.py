"""Comparators between the CUDA path (through the C ABI) and the oracle.

Data flows only from the seeded generators to both sides; nothing the CUDA
path produces is fed to the oracle.
"""
import math

import numpy as np
import torch

import oracle as O

CODE_TIE = 1e-6     # |z - boundary| below this (oracle, z units) is a tie
SIGN_TIE = 1e-6     # |(S r)_j| / ||r|| below this (oracle) is a tie
LOGIT_RTOL = 1e-3   # |dl| <= 1e-3 * max(|l|, nu ||q|| / sqrt(d))
ATTEND_RTOL = 2e-3  # ||do|| / ||o|| per (b, h)


def to_np_u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def compare_compressed(g, o: O.Compressed, codec: O.Codec, rows=None, nu_extra_ulp: float = 0.0):
    """g: kv_cache_vector_09_b200.Compressed (device) for the same rows as o.
    Returns counts; raises AssertionError on any mismatch that is not a tie.
    nu_extra_ulp widens the norm tolerance by that many fp32 units for paths
    whose input is itself an fp32 evaluation (the fused RoPE)."""
    sel = slice(None) if rows is None else rows
    gc = to_np_u32(g.codes)[sel]
    stats = dict(rows=int(gc.shape[0]), code_mismatch=0, code_ties=0, sign_mismatch=0, sign_ties=0)
    bad_rows = np.zeros(gc.shape[0], dtype=bool)
    if not np.array_equal(gc, o.codes):
        gi = O.unpack_codes(gc, codec)
        diff = gi != o.code_idx
        stats["code_mismatch"] = int(diff.sum())
        ties = diff & (o.code_margin < CODE_TIE)
        stats["code_ties"] = int(ties.sum())
        assert np.array_equal(diff, ties), (
            f"code mismatch away from a boundary: {int((diff & ~ties).sum())} coordinates, "
            f"min margin {o.code_margin[diff & ~ties].min():.3e}")
        bad_rows = diff.any(axis=1)
    nu_g = g.norms.detach().cpu().numpy()[sel]
    # fp32 norm: 8 partial sums of squares + sqrt, relative error <= (d/16 + 3) 2^-24
    nu_tol = ((codec.d / 16 + 3) * 2.0 ** -24 + 2.0 ** -24) + nu_extra_ulp * 2.0 ** -24
    assert np.all(np.abs(nu_g.astype(np.float64) - o.nu64) <= nu_tol * o.nu64 + 1e-38), "norms"
    if codec.m > 0:
        gs = to_np_u32(g.signs)[sel]
        if not np.array_equal(gs[~bad_rows], o.signs[~bad_rows]):
            gb = O.unpack_bits(gs, codec.m)
            ob = O.unpack_bits(o.signs, codec.m)
            diff = (gb != ob) & ~bad_rows[:, None]
            rel = np.abs(o.t) / np.maximum(o.gamma64[:, None], 1e-300)
            ties = diff & (rel < SIGN_TIE)
            stats["sign_mismatch"] = int(diff.sum())
            stats["sign_ties"] = int(ties.sum())
            assert np.array_equal(diff, ties), (
                f"sign mismatch away from zero: {int((diff & ~ties).sum())} bits, "
                f"min |t|/gamma {rel[diff & ~ties].min():.3e}")
        gg = g.rnorms.detach().cpu().numpy()[sel].astype(np.float64)
        ok = ~bad_rows
        if getattr(codec, "residual", "qjl") == "sign":
            # per-element residual sign: the stored scale is the codec's
            # constant mu sqrt(2d/pi) (independent quadratures: 2 fp32 units)
            want = o.rnorms.astype(np.float64)
            assert np.all(np.abs(gg - want) <= 2 * np.spacing(np.float32(want[0]))), "rnorms constant"
        else:
            assert np.all(np.abs(gg[ok] - o.gamma64[ok]) <= 1e-5 * np.maximum(o.gamma64[ok], 1e-30)), "rnorms"
    return stats


def logit_errors(l_gpu: np.ndarray, l_orc: np.ndarray, nu: np.ndarray, qn: np.ndarray, d: int):
    """Normalised error |dl| / max(|l|, nu ||q|| / sqrt(d)); nu, qn broadcast to l."""
    floor = nu * qn / math.sqrt(d)
    return np.abs(l_gpu - l_orc) / np.maximum(np.abs(l_orc), np.maximum(floor, 1e-30))


def attend_errors(o_gpu: np.ndarray, o_orc: np.ndarray):
    num = np.linalg.norm(o_gpu - o_orc, axis=-1)
    den = np.maximum(np.linalg.norm(o_orc, axis=-1), 1e-30)
    return num / den
