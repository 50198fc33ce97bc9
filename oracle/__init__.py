"""fp64 CPU oracle for masked softmax attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over (b, h)); this
module only compiles it with gcc, marshals numpy arrays through ctypes and
converts the BSH layout to BNSD by a transpose (data movement, no arithmetic).

Definitions followed (see the header of ``oracle.c`` for the full statement):

* "FlashAttentionScore fusion operator replacement guide", sec. 2 -- the
  attention formula Softmax(Q K^T / sqrt(d_k)) V; sec. 3.2 -- the call's
  parameters (layout BSH/BNSD, optional pse, atten_mask, scale, keep_prob);
  sec. 4 step 1 -- the unfused steps (matmul * scale, + mask, softmax,
  matmul with V), which is the order used here.
* Multimodal FlashAttention page, layer 2 -- the bool mask polarity
  (True = may attend) and the cross-modal rule built from modality ids.
* CogVLM page, "attention mask mechanism" -- the causal (tril) mask.
* Retrieval page, layer 2 -- the key-side document padding mask.

Every function here is pinned by the ``-m "not gpu"`` tests against closed
forms, library routines and finite differences (tests/test_oracle_*.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _Mask(ctypes.Structure):
    _fields_ = [
        ("causal", ctypes.c_int),
        ("kv_len", ctypes.c_void_p),
        ("mask", ctypes.c_void_p),
        ("msb", ctypes.c_int64),
        ("msh", ctypes.c_int64),
        ("msq", ctypes.c_int64),
        ("ids", ctypes.c_void_p),
        ("allow00", ctypes.c_int),
        ("allow01", ctypes.c_int),
        ("allow10", ctypes.c_int),
        ("allow11", ctypes.c_int),
        ("allow_diag", ctypes.c_int),
        ("add", ctypes.c_void_p),
        ("asb", ctypes.c_int64),
        ("ash", ctypes.c_int64),
        ("asq", ctypes.c_int64),
        ("dropout", ctypes.c_int),
        ("keep_prob", ctypes.c_double),
        ("seed", ctypes.c_uint64),
        ("offset", ctypes.c_uint64),
    ]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP).  Returns the path."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB_PATH + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                   "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_fwd.argtypes = [i, i, i, i, i, dp, dp, dp, dp,
                                   ctypes.POINTER(_Mask), ctypes.c_double, dp, dp]
        lib.oracle_fwd.restype = ctypes.c_int
        lib.oracle_bwd.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp,
                                   ctypes.POINTER(_Mask), ctypes.c_double, dp, dp, dp]
        lib.oracle_bwd.restype = ctypes.c_int
        lib.oracle_probs.argtypes = [i, i, i, i, i, i, i, dp, dp, dp,
                                     ctypes.POINTER(_Mask), ctypes.c_double, dp, dp]
        lib.oracle_probs.restype = ctypes.c_int
        lib.oracle_philox4x32.argtypes = [dp, dp, dp]
        lib.oracle_philox4x32.restype = None
        lib.oracle_dropout_mask.argtypes = [i, i, i, i, ctypes.POINTER(_Mask), dp]
        lib.oracle_dropout_mask.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [i]
        lib.oracle_get_threads.restype = i
        _lib = lib
    return _lib


class use_library:
    """Context manager that points this module at another build of the
    oracle (used by the mutation tests to check that the pins catch planted
    mistakes)."""

    def __init__(self, so_path: str):
        self.so_path = so_path
        self.saved = None

    def __enter__(self):
        global _lib
        self.saved = _lib
        _load()  # make sure the argtypes template exists
        lib = ctypes.CDLL(self.so_path)
        for name in ("oracle_fwd", "oracle_bwd", "oracle_probs", "oracle_philox4x32",
                     "oracle_dropout_mask"):
            ref = getattr(self.saved or _lib, name)
            getattr(lib, name).argtypes = ref.argtypes
            getattr(lib, name).restype = ref.restype
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_get_threads.restype = ctypes.c_int
        _lib = lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def set_threads(n: int) -> None:
    """Number of OpenMP threads the oracle uses (0 = OpenMP default)."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _to_bnsd(x: np.ndarray, layout: str, n_heads: int) -> np.ndarray:
    if layout == "BNSD":
        return np.ascontiguousarray(x)
    if layout == "BSH":
        b, s, hid = x.shape
        return np.ascontiguousarray(
            x.reshape(b, s, n_heads, hid // n_heads).transpose(0, 2, 1, 3))
    raise ValueError(f"unknown layout {layout}")


def _from_bnsd(x: np.ndarray, layout: str) -> np.ndarray:
    if layout == "BNSD":
        return x
    b, n, s, d = x.shape
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(b, s, n * d))


class _MaskHolder:
    """Keeps the numpy buffers a _Mask points to alive."""

    def __init__(self, B, N, Sq, Sk, causal, kv_len, mask, modality_ids,
                 allow, allow_diag, bias=None, dropout=None):
        self.m = _Mask()
        self.m.causal = 1 if causal else 0
        self.keep = []
        if kv_len is not None:
            kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32).reshape(B))
            self.keep.append(kl)
            self.m.kv_len = kl.ctypes.data
        if mask is not None:
            mk = np.asarray(mask)
            if hasattr(mask, "detach"):
                mk = mask.detach().cpu().numpy()
            mk = (mk != 0).astype(np.uint8)
            # broadcast to [B, N, Sq, Sk] without materialising a copy's strides
            mk4 = np.ascontiguousarray(np.broadcast_to(
                mk.reshape((1,) * (4 - mk.ndim) + mk.shape), (B, N, Sq, Sk)))
            self.keep.append(mk4)
            self.m.mask = mk4.ctypes.data
            self.m.msb = N * Sq * Sk
            self.m.msh = Sq * Sk
            self.m.msq = Sk
        if modality_ids is not None:
            if Sq != Sk:
                raise ValueError("modality mask needs Sq == Sk")
            ids = modality_ids
            if hasattr(ids, "detach"):
                ids = ids.detach().cpu().numpy()
            ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32).reshape(B, Sk))
            self.keep.append(ids)
            self.m.ids = ids.ctypes.data
            a = np.asarray(allow, dtype=np.int32).reshape(2, 2)
            self.m.allow00, self.m.allow01 = int(a[0, 0]), int(a[0, 1])
            self.m.allow10, self.m.allow11 = int(a[1, 0]), int(a[1, 1])
            self.m.allow_diag = 1 if allow_diag else 0
        if bias is not None:
            a = _f64(bias)
            a4 = np.ascontiguousarray(np.broadcast_to(
                a.reshape((1,) * (4 - a.ndim) + a.shape), (B, N, Sq, Sk)))
            self.keep.append(a4)
            self.m.add = a4.ctypes.data
            self.m.asb, self.m.ash, self.m.asq = N * Sq * Sk, Sq * Sk, Sk
        if dropout is not None:
            keep_prob, seed, offset = dropout
            if not (0.0 < keep_prob <= 1.0):
                raise ValueError("keep_prob must be in (0, 1]")
            self.m.dropout = 1
            self.m.keep_prob = float(keep_prob)
            self.m.seed = int(seed) & ((1 << 64) - 1)
            self.m.offset = int(offset) & ((1 << 64) - 1)


def _prep(q, k, v, n_heads, layout):
    q = _to_bnsd(_f64(q), layout, n_heads)
    k = _to_bnsd(_f64(k), layout, n_heads)
    v = _to_bnsd(_f64(v), layout, n_heads)
    B, N, Sq, D = q.shape
    Sk = k.shape[2]
    if k.shape != (B, N, Sk, D) or v.shape != (B, N, Sk, D):
        raise ValueError("q/k/v shapes disagree")
    return q, k, v, B, N, Sq, Sk, D


def fwd(q, k, v, scale, *, n_heads=None, layout="BNSD", causal=False,
        kv_len=None, mask=None, modality_ids=None, allow=((1, 1), (0, 1)),
        allow_diag=False, slopes=None, bias=None, dropout=None):
    """Attention forward in fp64.  Returns (out, lse) as numpy arrays.

    ``out`` has the layout of ``q``; ``lse`` is [B, N, Sq] (natural log,
    -inf for rows with no allowed key).  ``mask`` is a bool/uint8 array
    broadcastable to [B, N, Sq, Sk] with 1 = may attend.  ``bias`` is a float
    array broadcastable to [B, N, Sq, Sk] added to the scores (a dense pse or
    a float atten_mask; -inf entries mask their pair).  ``dropout`` is
    ``(keep_prob, seed, offset)`` or None (the generator and mask layout are
    in the header of oracle.c)."""
    if layout == "BSH" and n_heads is None:
        raise ValueError("BSH layout needs n_heads")
    q, k, v, B, N, Sq, Sk, D = _prep(q, k, v, n_heads, layout)
    mh = _MaskHolder(B, N, Sq, Sk, causal, kv_len, mask, modality_ids, allow,
                     allow_diag, bias, dropout)
    sl = None
    if slopes is not None:
        sl = np.ascontiguousarray(_f64(slopes).reshape(N))
    out = np.zeros((B, N, Sq, D), dtype=np.float64)
    lse = np.zeros((B, N, Sq), dtype=np.float64)
    rc = _load().oracle_fwd(B, N, Sq, Sk, D, q.ctypes.data, k.ctypes.data,
                            v.ctypes.data, None if sl is None else sl.ctypes.data,
                            ctypes.byref(mh.m), float(scale), out.ctypes.data,
                            lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_fwd failed ({rc})")
    return _from_bnsd(out, layout), lse


def bwd(q, k, v, dout, scale, *, n_heads=None, layout="BNSD", causal=False,
        kv_len=None, mask=None, modality_ids=None, allow=((1, 1), (0, 1)),
        allow_diag=False, slopes=None, bias=None, dropout=None):
    """Gradients (dq, dk, dv) of sum(dout * out) in fp64, layouts as the inputs."""
    if layout == "BSH" and n_heads is None:
        raise ValueError("BSH layout needs n_heads")
    q, k, v, B, N, Sq, Sk, D = _prep(q, k, v, n_heads, layout)
    do = _to_bnsd(_f64(dout), layout, n_heads)
    mh = _MaskHolder(B, N, Sq, Sk, causal, kv_len, mask, modality_ids, allow,
                     allow_diag, bias, dropout)
    sl = None
    if slopes is not None:
        sl = np.ascontiguousarray(_f64(slopes).reshape(N))
    dq = np.zeros((B, N, Sq, D), dtype=np.float64)
    dk = np.zeros((B, N, Sk, D), dtype=np.float64)
    dv = np.zeros((B, N, Sk, D), dtype=np.float64)
    rc = _load().oracle_bwd(B, N, Sq, Sk, D, q.ctypes.data, k.ctypes.data,
                            v.ctypes.data, do.ctypes.data,
                            None if sl is None else sl.ctypes.data,
                            ctypes.byref(mh.m), float(scale), dq.ctypes.data,
                            dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_bwd failed ({rc})")
    return _from_bnsd(dq, layout), _from_bnsd(dk, layout), _from_bnsd(dv, layout)


def probs(q, k, scale, b, h, *, n_heads=None, layout="BNSD", causal=False,
          kv_len=None, mask=None, modality_ids=None, allow=((1, 1), (0, 1)),
          allow_diag=False, slopes=None, bias=None, dropout=None):
    """Explicit probability matrix P [Sq, Sk] and lse [Sq] of one (b, h)."""
    q = _to_bnsd(_f64(q), layout, n_heads)
    k = _to_bnsd(_f64(k), layout, n_heads)
    B, N, Sq, D = q.shape
    Sk = k.shape[2]
    mh = _MaskHolder(B, N, Sq, Sk, causal, kv_len, mask, modality_ids, allow,
                     allow_diag, bias, dropout)
    sl = None
    if slopes is not None:
        sl = np.ascontiguousarray(_f64(slopes).reshape(N))
    p = np.zeros((Sq, Sk), dtype=np.float64)
    lse = np.zeros((Sq,), dtype=np.float64)
    rc = _load().oracle_probs(B, N, Sq, Sk, D, int(b), int(h), q.ctypes.data,
                              k.ctypes.data, None if sl is None else sl.ctypes.data,
                              ctypes.byref(mh.m), float(scale), p.ctypes.data,
                              lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_probs failed ({rc})")
    return p, lse


def philox4x32(counter, key):
    """Philox-4x32-10 of one 4-word counter and 2-word key (uint32 words)."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint32).reshape(4))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32).reshape(2))
    out = np.zeros(4, dtype=np.uint32)
    _load().oracle_philox4x32(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def dropout_keep_mask(B, N, Sq, Sk, keep_prob, seed, offset):
    """The dropout keep mask [B, N, Sq, Sk] (uint8, 1 = kept)."""
    mh = _MaskHolder(B, N, Sq, Sk, False, None, None, None, ((1, 1), (1, 1)), False,
                     None, (keep_prob, seed, offset))
    keep = np.zeros((B, N, Sq, Sk), dtype=np.uint8)
    rc = _load().oracle_dropout_mask(B, N, Sq, Sk, ctypes.byref(mh.m), keep.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_dropout_mask failed ({rc})")
    return keep
