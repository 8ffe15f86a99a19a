"""B200-native TurboQuant-style KV-cache compression: Python binding of libtq.

This module only marshals arguments for the C ABI declared in ``include/tq.h``
(same function names); every step of the codec runs in the CUDA kernels of
``libtq.so``.  PyTorch supplies device memory and streams.  There is no CPU
fallback: importing this package fails loudly if ``libtq.so`` is missing
(build it with ``python kv_cache_vector_09_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK = 0
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_NO_MEMORY",
                4: "TQ_ERR_CUDA", 5: "TQ_ERR_DEVICE_ASSERT", 6: "TQ_ERR_NOT_CONVERGED"}
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
_DTYPES = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}


class TQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


TQ_RESIDUAL_QJL, TQ_RESIDUAL_SIGN = 0, 1
TQ_ROTATION_RHT, TQ_ROTATION_HAAR = 0, 1


class tq_spec(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("nseg", ctypes.c_int32), ("seg_bits", ctypes.c_int32 * 2),
                ("m", ctypes.c_int32), ("seed", ctypes.c_uint64), ("residual", ctypes.c_int32),
                ("rotation", ctypes.c_int32), ("vq_bits", ctypes.c_int32)]


class tq_compressed(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("norms", ctypes.c_void_p),
                ("rnorms", ctypes.c_void_p)]


class tq_rope(ctypes.Structure):
    _fields_ = [("cos_sin", ctypes.c_void_p), ("max_pos", ctypes.c_int32), ("positions", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python kv_cache_vector_09_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "tq_make_codebook": [I, I, ctypes.c_double, I, P, P],
        "tq_codec_create": [P, I, ctypes.POINTER(P)],
        "tq_codec_destroy": [P],
        "tq_codec_export": [P, P, P, P, P],
        "tq_codec_layout": [P, ctypes.POINTER(I), ctypes.POINTER(I)],
        "tq_codec_rotation": [P, P],
        "tq_codec_vq_codebook": [P, P],
        "tq_quantize": [P, P, I, I64, I64, P, P],
        "tq_rope_cache": [ctypes.c_double, I, I, P, P],
        "tq_quantize_rope": [P, P, I, I64, I64, P, P, P],
        "tq_append": [P, P, I, I64, I64, P, I64, I64, P, P],
        "tq_scores_workspace_size": [P, I, I, I, ctypes.POINTER(SZ)],
        "tq_scores": [P, P, I, I, I, I, I64, P, P, P, SZ, P],
        "tq_scores_noalloc": [P, P, I, I, I, I, I64, P, P, P],
        "tq_attend_workspace_size": [P, P, I, I, I, I64, ctypes.POINTER(SZ)],
        "tq_attend": [P, P, P, I, I, I, I, I64, ctypes.c_float, P, P, P, SZ, P, P],
        "tq_search_workspace_size": [P, I, I, ctypes.POINTER(SZ)],
        "tq_search_topk": [P, P, I, I, P, I64, I, P, P, P, SZ, P],
        "tq_codec_device_error": [P, P, ctypes.POINTER(ctypes.c_uint32)],
        "tq_codec_exact_rows": [P, P, I, ctypes.POINTER(ctypes.c_uint64)],
    }
    for name, args in sig.items():
        try:
            fn = getattr(lib, name)
        except AttributeError as e:
            raise ImportError(f"{LIB_PATH} lacks {name}: rebuild it with `python kv_cache_vector_09_b200/build.py`") from e
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.tq_status_string.argtypes = [ctypes.c_int]
    lib.tq_status_string.restype = ctypes.c_char_p
    lib.tq_last_error_string.argtypes = []
    lib.tq_last_error_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def _check(status: int, where: str) -> None:
    if status != TQ_OK:
        raise TQError(status, where, _lib.tq_last_error_string().decode())


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(status).decode()


def tq_last_error_string() -> str:
    return _lib.tq_last_error_string().decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------------- calls
def tq_make_codebook(bits: int, d: int, tol: float = 0.0, max_iter: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Host Lloyd-Max codebook: (centroids [2^bits], boundaries [2^bits - 1]) fp32."""
    cen = np.zeros(1 << bits, dtype=np.float32)
    bnd = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check(_lib.tq_make_codebook(bits, d, tol, max_iter, cen.ctypes.data, bnd.ctypes.data), "tq_make_codebook")
    return cen, bnd


class Codec:
    """A tq_codec handle (freed with the object)."""

    def __init__(self, d: int, seg_bits: Sequence[int], m: int, seed: int = 0, device: int = 0,
                 residual: int = TQ_RESIDUAL_QJL, rotation: int = TQ_ROTATION_RHT, vq_bits: int = 0):
        seg_bits = tuple(int(b) for b in seg_bits)
        self.d, self.seg_bits, self.m, self.seed, self.device = d, seg_bits, m, seed, device
        self.residual, self.rotation, self.vq_bits = residual, rotation, vq_bits
        spec = tq_spec(d, len(seg_bits), (ctypes.c_int32 * 2)(*(seg_bits + (0,) * (2 - len(seg_bits)))), m, seed,
                       residual, rotation, vq_bits)
        h = ctypes.c_void_p()
        _check(_lib.tq_codec_create(ctypes.byref(spec), device, ctypes.byref(h)), "tq_codec_create")
        self._h = h
        cw, sw = ctypes.c_int(), ctypes.c_int()
        _check(_lib.tq_codec_layout(h, ctypes.byref(cw), ctypes.byref(sw)), "tq_codec_layout")
        self.code_words, self.sign_words = cw.value, sw.value

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def export(self):
        """(S [m, d] fp32, dsigns [ceil(d/32)] uint32, cen list, bnd list) host copies."""
        S = np.zeros((self.m, self.d), dtype=np.float32)
        ds = np.zeros((self.d + 31) // 32, dtype=np.uint32)
        nc = sum(1 << b for b in self.seg_bits)
        cen = np.zeros(nc, dtype=np.float32)
        bnd = np.zeros(nc - len(self.seg_bits), dtype=np.float32)
        _check(_lib.tq_codec_export(self._h, S.ctypes.data if self.m else None, ds.ctypes.data, cen.ctypes.data,
                                    bnd.ctypes.data), "tq_codec_export")
        cl, bl, oc, ob = [], [], 0, 0
        for b in self.seg_bits:
            cl.append(cen[oc:oc + (1 << b)])
            bl.append(bnd[ob:ob + (1 << b) - 1])
            oc += 1 << b
            ob += (1 << b) - 1
        return S, ds, cl, bl

    def vq_codebook(self) -> np.ndarray:
        """FibQuant codewords [2^vq_bits, 2] fp32 (z units), host copy."""
        cb = np.zeros((1 << self.vq_bits, 2), dtype=np.float32)
        _check(_lib.tq_codec_vq_codebook(self._h, cb.ctypes.data), "tq_codec_vq_codebook")
        return cb

    def rotation_matrix(self) -> np.ndarray:
        """The codec's rotation Pi [d, d] (y = Pi u), host copy."""
        Pi = np.zeros((self.d, self.d), dtype=np.float32)
        _check(_lib.tq_codec_rotation(self._h, Pi.ctypes.data), "tq_codec_rotation")
        return Pi

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            _check(_lib.tq_codec_destroy(self._h), "tq_codec_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tq_codec_create(d: int, seg_bits: Sequence[int], m: int, seed: int = 0, device: int = 0) -> Codec:
    return Codec(d, seg_bits, m, seed, device)


class Compressed:
    """Caller-owned compressed rows (device tensors): codes [n, W] uint32 (held
    as int32), signs [n, m/32], norms [n] fp32, rnorms [n] fp32."""

    def __init__(self, codes: torch.Tensor, signs: Optional[torch.Tensor], norms: torch.Tensor,
                 rnorms: Optional[torch.Tensor]):
        self.codes, self.signs, self.norms, self.rnorms = codes, signs, norms, rnorms

    @classmethod
    def empty(cls, codec: Codec, n: int, device=None) -> "Compressed":
        device = device if device is not None else torch.device("cuda", codec.device)
        codes = torch.empty((n, codec.code_words), dtype=torch.int32, device=device)
        signs = torch.empty((n, codec.sign_words), dtype=torch.int32, device=device) if codec.m else None
        norms = torch.empty((n,), dtype=torch.float32, device=device)
        rnorms = torch.empty((n,), dtype=torch.float32, device=device) if codec.m else None
        return cls(codes, signs, norms, rnorms)

    def struct(self) -> tq_compressed:
        return tq_compressed(_ptr(self.codes), _ptr(self.signs), _ptr(self.norms), _ptr(self.rnorms))

    def rows(self, r0: int, r1: int) -> "Compressed":
        sl = lambda t: None if t is None else t[r0:r1]
        return Compressed(sl(self.codes), sl(self.signs), sl(self.norms), sl(self.rnorms))


def tq_quantize(codec: Codec, x: torch.Tensor, out: Compressed, stream=None) -> Compressed:
    """Compress the rows of x ([n, ld >= d] with unit column stride)."""
    assert x.dim() == 2 and x.stride(1) == 1, "x must be [n, ld] with contiguous rows"
    st = out.struct()
    _check(_lib.tq_quantize(codec.handle, x.data_ptr(), _DTYPES[x.dtype], x.shape[0], x.stride(0),
                            ctypes.byref(st), _stream(stream)), "tq_quantize")
    return out


def tq_rope_cache(theta: float, d: int, max_pos: int, device=None, stream=None) -> torch.Tensor:
    """RoPE cos/sin cache [max_pos, d] fp32 on the device (cos(pos theta_i) in
    columns i < d/2, sin(pos theta_i) in columns d/2 + i)."""
    device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    cs = torch.empty((max_pos, d), dtype=torch.float32, device=device)
    _check(_lib.tq_rope_cache(float(theta), d, max_pos, cs.data_ptr(), _stream(stream)), "tq_rope_cache")
    return cs


def _rope_struct(cos_sin: torch.Tensor, positions: Optional[torch.Tensor]) -> tq_rope:
    assert cos_sin.dtype == torch.float32 and cos_sin.is_contiguous()
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.is_contiguous()
    return tq_rope(cos_sin.data_ptr(), cos_sin.shape[0], _ptr(positions))


def tq_quantize_rope(codec: Codec, x: torch.Tensor, cos_sin: torch.Tensor, positions: torch.Tensor,
                     out: Compressed, stream=None) -> Compressed:
    """Compress the rows of x after rotate-half RoPE at positions[i] (int32)."""
    assert x.dim() == 2 and x.stride(1) == 1, "x must be [n, ld] with contiguous rows"
    st = out.struct()
    rp = _rope_struct(cos_sin, positions)
    _check(_lib.tq_quantize_rope(codec.handle, x.data_ptr(), _DTYPES[x.dtype], x.shape[0], x.stride(0),
                                 ctypes.byref(rp), ctypes.byref(st), _stream(stream)), "tq_quantize_rope")
    return out


def tq_append(codec: Codec, x: torch.Tensor, t: int, T: int, cache: Compressed, cos_sin: Optional[torch.Tensor] = None,
              stream=None) -> Compressed:
    """Compress row r of x ([rows, ld]) into cache row r * T + t, after RoPE at
    position t when cos_sin is given."""
    assert x.dim() == 2 and x.stride(1) == 1, "x must be [rows, ld] with contiguous rows"
    st = cache.struct()
    rp = _rope_struct(cos_sin, None) if cos_sin is not None else None
    _check(_lib.tq_append(codec.handle, x.data_ptr(), _DTYPES[x.dtype], x.shape[0], x.stride(0),
                          ctypes.byref(rp) if rp is not None else None, t, T, ctypes.byref(st), _stream(stream)),
           "tq_append")
    return cache


def tq_scores_workspace_size(kc: Codec, B: int, Hq: int, Hkv: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.tq_scores_workspace_size(kc.handle, B, Hq, Hkv, ctypes.byref(v)), "tq_scores_workspace_size")
    return v.value


def tq_scores(kc: Codec, q: torch.Tensor, B: int, Hq: int, Hkv: int, T: int, K: Compressed,
              logits: torch.Tensor, workspace: torch.Tensor, stream=None) -> torch.Tensor:
    assert q.is_contiguous() and logits.is_contiguous() and logits.dtype == torch.float32
    st = K.struct()
    _check(_lib.tq_scores(kc.handle, q.data_ptr(), _DTYPES[q.dtype], B, Hq, Hkv, T, ctypes.byref(st),
                          logits.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          _stream(stream)), "tq_scores")
    return logits


def tq_scores_noalloc(kc: Codec, q: torch.Tensor, B: int, Hq: int, Hkv: int, T: int, K: Compressed,
                      logits: torch.Tensor, stream=None) -> torch.Tensor:
    """tq_scores without a workspace, for callers that cannot allocate device
    memory: the library's built-in 2 MiB scratch is used instead.  Calls share
    that scratch, so calls that may overlap on the GPU must be serialised."""
    assert q.is_contiguous() and logits.is_contiguous() and logits.dtype == torch.float32
    st = K.struct()
    _check(_lib.tq_scores_noalloc(kc.handle, q.data_ptr(), _DTYPES[q.dtype], B, Hq, Hkv, T, ctypes.byref(st),
                                  logits.data_ptr(), _stream(stream)), "tq_scores_noalloc")
    return logits


def tq_attend_workspace_size(kc: Codec, vc: Codec, B: int, Hq: int, Hkv: int, T: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.tq_attend_workspace_size(kc.handle, vc.handle, B, Hq, Hkv, T, ctypes.byref(v)),
           "tq_attend_workspace_size")
    return v.value


def tq_attend(kc: Codec, vc: Codec, q: torch.Tensor, B: int, Hq: int, Hkv: int, T: int, K: Compressed,
              V: Compressed, out: torch.Tensor, workspace: torch.Tensor, scale: float = 0.0,
              stream=None) -> torch.Tensor:
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    ks, vs = K.struct(), V.struct()
    _check(_lib.tq_attend(kc.handle, vc.handle, q.data_ptr(), _DTYPES[q.dtype], B, Hq, Hkv, T, scale,
                          ctypes.byref(ks), ctypes.byref(vs), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size(), out.data_ptr(), _stream(stream)),
           "tq_attend")
    return out


def tq_search_workspace_size(codec: Codec, nq: int, k: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.tq_search_workspace_size(codec.handle, nq, k, ctypes.byref(v)), "tq_search_workspace_size")
    return v.value


def tq_search_topk(codec: Codec, q: torch.Tensor, index: Compressed, n: int, k: int, idx: torch.Tensor,
                   score: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Top-k index rows per query (idx int32 [nq, k], score fp32 [nq, k])."""
    assert q.is_contiguous() and q.dim() == 2
    assert idx.dtype == torch.int32 and score.dtype == torch.float32 and idx.is_contiguous() and score.is_contiguous()
    xs = index.struct()
    _check(_lib.tq_search_topk(codec.handle, q.data_ptr(), _DTYPES[q.dtype], q.shape[0], ctypes.byref(xs), n, k,
                               idx.data_ptr(), score.data_ptr(), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "tq_search_topk")
    return idx, score


def tq_codec_device_error(codec: Codec, stream=None) -> int:
    """Synchronise, read and clear the codec's device error word (0 = healthy)."""
    v = ctypes.c_uint32()
    st = _lib.tq_codec_device_error(codec.handle, _stream(stream), ctypes.byref(v))
    if st not in (TQ_OK, 5):
        _check(st, "tq_codec_device_error")
    return v.value


def tq_codec_exact_rows(codec: Codec, reset: bool = False, stream=None) -> int:
    """Rows tq_quantize re-evaluated in fp64 with this codec (synchronises)."""
    v = ctypes.c_uint64()
    _check(_lib.tq_codec_exact_rows(codec.handle, _stream(stream), int(reset), ctypes.byref(v)), "tq_codec_exact_rows")
    return v.value


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device byte buffer for the *_workspace_size calls."""
    return torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=device)


def c_api():
    """The loaded ctypes library (for tests of the raw C ABI)."""
    return _lib
