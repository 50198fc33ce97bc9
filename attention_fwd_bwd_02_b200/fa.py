"""Thin ctypes binding over libfa_b200.so (include/fa.h).

Argument marshalling only: tensors are passed as device pointers with the
current PyTorch stream; every step of the computation runs in the library's
CUDA kernels.  PyTorch provides device memory (outputs, workspace) and
streams.  There is no fallback: if the library is missing or a call fails,
an exception is raised.

The Python signature mirrors the fusion-attention call of the
FlashAttentionScore guide (sec. 3.1): query, key, value, head_num,
input_layout, pse, padding mask, atten_mask, scale, keep_prob.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "fa.h")
TESTING_HEADER = os.path.join(os.path.dirname(_HERE), "include", "fa_testing.h")

(FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT,
 FA_ERR_CONCURRENT) = range(6)
FA_LAYOUT_BNSD, FA_LAYOUT_BSH = 0, 1
FA_F32, FA_BF16, FA_F16, FA_E4M3 = 0, 1, 2, 3
FA_MASK_CAUSAL, FA_MASK_KV_PADDING, FA_MASK_BOOL, FA_MASK_MODALITY = 1, 2, 4, 8
FA_PSE_NONE, FA_PSE_ALIBI, FA_PSE_DENSE = 0, 1, 2
FA_TILE_M = FA_TILE_N = 128


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        name = _status_name(status)
        super().__init__(f"{what}: {name} ({status})" if what else f"{name} ({status})")


class FaDropout(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64)]


class FaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("Sq", ctypes.c_int),
                ("Sk", ctypes.c_int), ("D", ctypes.c_int), ("layout", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class FaMask(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32),
                ("kv_len", ctypes.c_void_p),
                ("mask", ctypes.c_void_p),
                ("mask_stride_b", ctypes.c_int64),
                ("mask_stride_h", ctypes.c_int64),
                ("mask_stride_q", ctypes.c_int64),
                ("tile_map", ctypes.c_void_p),
                ("modality_ids", ctypes.c_void_p),
                ("allow", (ctypes.c_uint8 * 2) * 2),
                ("allow_diag", ctypes.c_uint8)]


class FaPse(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("slopes", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bias_stride_b", ctypes.c_int64),
                ("bias_stride_h", ctypes.c_int64), ("bias_stride_q", ctypes.c_int64)]


_lib = None


def _status_name(s):
    names = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
             3: "FA_ERR_CUDA", 4: "FA_ERR_TIMEOUT", 5: "FA_ERR_CONCURRENT"}
    return names.get(int(s), "FA_ERR_UNKNOWN")


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m attention_fwd_bwd_02_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        S, M, P = ctypes.POINTER(FaShape), ctypes.POINTER(FaMask), ctypes.POINTER(FaPse)
        R = ctypes.POINTER(FaDropout)
        L.fa_fwd.argtypes = [S, vp, vp, vp, P, M, ctypes.c_float, ctypes.c_float, R,
                             vp, vp, vp]
        L.fa_bwd.argtypes = [S, vp, vp, vp, vp, vp, vp, P, M, ctypes.c_float,
                             ctypes.c_float, R, vp, vp, vp, vp, sz, vp]
        L.fa_bwd_noalloc.argtypes = [S, vp, vp, vp, vp, vp, vp, P, M, ctypes.c_float,
                                     ctypes.c_float, R, vp, vp, vp, vp]
        L.fa_testing_fwd_withhold_q.argtypes = L.fa_fwd.argtypes
        L.fa_bwd_workspace_size.argtypes = [S]
        L.fa_bwd_workspace_size.restype = sz
        L.fa_mask_tile_map_size.argtypes = [S, M]
        L.fa_mask_tile_map_size.restype = sz
        L.fa_build_mask_tile_map.argtypes = [S, M, vp, vp]
        L.fa_build_modality_mask.argtypes = [ctypes.c_int, ctypes.c_int, vp,
                                             ctypes.POINTER((ctypes.c_uint8 * 2) * 2),
                                             ctypes.c_int, vp, vp]
        L.fa_sync_status.argtypes = [vp]
        L.fa_status_string.argtypes = [ctypes.c_int]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_version.restype = ctypes.c_char_p
        L.fa_last_cuda_error.restype = ctypes.c_char_p
        for fn in (L.fa_fwd, L.fa_testing_fwd_withhold_q, L.fa_bwd, L.fa_bwd_noalloc,
                   L.fa_build_mask_tile_map,
                   L.fa_build_modality_mask, L.fa_sync_status):
            fn.restype = ctypes.c_int
        _lib = L
    return _lib


def declared_functions(header: str = HEADER):
    """Names of the functions a header of include/ declares."""
    txt = open(header).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", txt)))


def _check(status, what):
    if status != FA_OK:
        if status == FA_ERR_CUDA:
            what = f"{what} [{lib().fa_last_cuda_error().decode()}]"
        raise FaError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


_NULL_CTX = contextlib.nullcontext()


def _on_device(dev):
    """Makes `dev` current for the call (no-op when it already is)."""
    dev = torch.device(dev)
    if dev.index is None or dev.index == torch.cuda.current_device():
        return _NULL_CTX
    return torch.cuda.device(dev)


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return FA_BF16
    if dt == torch.float16:
        return FA_F16
    if dt == torch.float32:
        return FA_F32
    if dt == torch.float8_e4m3fn:
        return FA_E4M3
    raise FaError(FA_ERR_UNSUPPORTED, f"dtype {dt}")


def out_dtype(dt):
    """dtype of the forward's output for operands of dtype dt (bf16 for e4m3)."""
    return torch.bfloat16 if dt == torch.float8_e4m3fn else dt


def make_shape(q, k, head_num, input_layout) -> FaShape:
    layout = {"BNSD": FA_LAYOUT_BNSD, "BSH": FA_LAYOUT_BSH}.get(input_layout)
    if layout is None:
        raise FaError(FA_ERR_INVALID_ARG, f"input_layout {input_layout!r}")
    if layout == FA_LAYOUT_BNSD:
        if q.dim() != 4 or k.dim() != 4:
            raise FaError(FA_ERR_INVALID_ARG, "BNSD tensors must be 4-D")
        B, N, Sq, D = q.shape
        Sk = k.shape[2]
        if head_num is not None and head_num != N:
            raise FaError(FA_ERR_INVALID_ARG, "head_num disagrees with q.shape[1]")
    else:
        if q.dim() != 3 or k.dim() != 3:
            raise FaError(FA_ERR_INVALID_ARG, "BSH tensors must be 3-D")
        B, Sq, H = q.shape
        Sk = k.shape[1]
        if head_num is None or head_num <= 0 or H % head_num:
            raise FaError(FA_ERR_INVALID_ARG, "head_num must divide the hidden size")
        N, D = head_num, H // head_num
    return FaShape(int(B), int(N), int(Sq), int(Sk), int(D), layout, _dtype_code(q.dtype))


def _check_operand(t, shape, name, like=None):
    if t is None:
        raise FaError(FA_ERR_INVALID_ARG, f"{name} is required")
    if not t.is_cuda:
        raise FaError(FA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise FaError(FA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if like is not None and (t.dtype != like.dtype or t.device != like.device):
        raise FaError(FA_ERR_INVALID_ARG, f"{name} dtype/device differ from q")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise FaError(FA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}, want {tuple(shape)}")


def _check_lse(lse, shape, like):
    if lse is None or not lse.is_cuda or lse.dtype != torch.float32 or \
            not lse.is_contiguous() or lse.device != like.device or \
            tuple(lse.shape) != (shape.B, shape.N, shape.Sq):
        raise FaError(FA_ERR_INVALID_ARG,
                      f"lse must be a contiguous fp32 [B, N, Sq] tensor on q's device")


def check_side_inputs(device, **tensors):
    """Every tensor the kernels read through a pointer (masks, lengths, ids,
    tile map, slopes, dense term) must live on the operands' device: a host
    or another GPU's pointer would be read by the kernel itself."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda or t.device != torch.device(device):
            raise FaError(FA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor on {device}")


class _Keep:
    """Holds tensors that a ctypes struct points to."""

    def __init__(self):
        self.items = []


def make_mask(shape: FaShape, *, causal=False, atten_mask=None, padding_kv_len=None,
              modality_ids=None, allow=((1, 1), (0, 1)), allow_diag=False,
              tile_map=None, keep: Optional[_Keep] = None) -> Optional[FaMask]:
    flags = 0
    m = FaMask()
    keep = keep or _Keep()
    if causal:
        flags |= FA_MASK_CAUSAL
    if padding_kv_len is not None:
        kl = padding_kv_len.to(torch.int32).contiguous()
        keep.items.append(kl)
        m.kv_len = kl.data_ptr()
        flags |= FA_MASK_KV_PADDING
    if atten_mask is not None:
        am = atten_mask
        if am.dtype == torch.bool:
            am = am.view(torch.uint8) if am.is_contiguous() else am.to(torch.uint8)
        if am.dtype != torch.uint8:
            raise FaError(FA_ERR_INVALID_ARG, "atten_mask must be bool or uint8 (1 = attend)")
        while am.dim() < 4:
            am = am.unsqueeze(0)
        if am.shape[-2:] != (shape.Sq, shape.Sk) or am.stride(-1) != 1:
            am = am.expand(am.shape[0], am.shape[1], shape.Sq, shape.Sk).contiguous()
        keep.items.append(am)
        sb = 0 if am.shape[0] == 1 else am.stride(0)
        sh = 0 if am.shape[1] == 1 else am.stride(1)
        m.mask = am.data_ptr()
        m.mask_stride_b, m.mask_stride_h, m.mask_stride_q = sb, sh, am.stride(2)
        flags |= FA_MASK_BOOL
        if tile_map is not None:
            keep.items.append(tile_map)
            m.tile_map = tile_map.data_ptr()
    if modality_ids is not None:
        ids = modality_ids.to(torch.int32).contiguous()
        keep.items.append(ids)
        m.modality_ids = ids.data_ptr()
        for a in range(2):
            for c in range(2):
                m.allow[a][c] = 1 if allow[a][c] else 0
        m.allow_diag = 1 if allow_diag else 0
        flags |= FA_MASK_MODALITY
    m.flags = flags
    return m if flags else None


def make_dropout(keep_prob, seed, offset) -> Optional[FaDropout]:
    """The Philox seed and block offset of the dropout mask (include/fa.h,
    fa_dropout); None when keep_prob == 1.  keep_prob < 1 needs an explicit
    seed."""
    if not (0.0 < float(keep_prob) <= 1.0):
        raise FaError(FA_ERR_INVALID_ARG, f"keep_prob {keep_prob} outside (0, 1]")
    if float(keep_prob) == 1.0:
        return None
    if seed is None:
        raise FaError(FA_ERR_INVALID_ARG, "keep_prob < 1 needs a dropout seed")
    return FaDropout(int(seed) & (2**64 - 1), int(offset) & (2**64 - 1))


def split_atten_mask(atten_mask):
    """(bool mask, additive term): a bool/uint8 atten_mask selects pairs
    (1 = may attend); a floating one is added to the scaled scores (the
    guide's unfused steps, sec. 4 step 1)."""
    if atten_mask is not None and atten_mask.is_floating_point():
        return None, atten_mask
    return atten_mask, None


def _dense_term(t: torch.Tensor, shape: FaShape, keep: _Keep):
    """Device fp32 view of a dense additive term broadcastable to
    [B, N, Sq, Sk] (leading dims 1 or full); returns (ptr, sb, sh, sq)."""
    if not t.is_cuda:
        raise FaError(FA_ERR_INVALID_ARG, "the dense pse / float mask must be a CUDA tensor")
    a = t if t.dtype == torch.float32 else t.to(torch.float32)
    while a.dim() < 4:
        a = a.unsqueeze(0)
    if a.dim() != 4 or tuple(a.shape[-2:]) != (shape.Sq, shape.Sk) or \
            a.shape[0] not in (1, shape.B) or a.shape[1] not in (1, shape.N):
        raise FaError(FA_ERR_INVALID_ARG,
                      f"dense pse / float mask of shape {tuple(t.shape)} does not broadcast "
                      f"to [{shape.B}, {shape.N}, {shape.Sq}, {shape.Sk}]")
    if a.stride(-1) != 1 or a.stride(-2) < shape.Sk:
        a = a.contiguous()
    keep.items.append(a)
    # a size-1 or expanded (stride 0) batch / head dimension is a broadcast
    sb = 0 if a.shape[0] == 1 else a.stride(0)
    sh = 0 if a.shape[1] == 1 else a.stride(1)
    return a.data_ptr(), sb, sh, a.stride(2)


def make_pse(pse: Optional[torch.Tensor], keep: _Keep, shape: Optional[FaShape] = None,
             add: Optional[torch.Tensor] = None) -> Optional[FaPse]:
    """pse: an ALiBi slope vector [N] or a dense term broadcastable to
    [B, N, Sq, Sk]; add: a float atten_mask (another dense term).  Only one
    dense term is taken."""
    ps = FaPse()
    if pse is not None and pse.dim() == 1:
        s = pse.to(torch.float32).contiguous()
        keep.items.append(s)
        ps.kind |= FA_PSE_ALIBI
        ps.slopes = s.data_ptr()
    elif pse is not None:
        if add is not None:
            raise FaError(FA_ERR_UNSUPPORTED,
                          "a dense pse and a float atten_mask: pass their sum as one of them")
        add = pse
    if add is not None:
        if shape is None:
            raise FaError(FA_ERR_INVALID_ARG, "a dense term needs the problem shape")
        ps.bias, ps.bias_stride_b, ps.bias_stride_h, ps.bias_stride_q = _dense_term(add, shape, keep)
        ps.kind |= FA_PSE_DENSE
    return ps if ps.kind else None


def fwd(query, key, value, head_num=None, input_layout="BNSD", pse=None,
        padding_kv_len=None, atten_mask=None, scale=None, keep_prob=1.0, *,
        causal=False, modality_ids=None, allow=((1, 1), (0, 1)), allow_diag=False,
        tile_map=None, out=None, lse=None, seed=None, offset=0,
        _withhold_q=False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused attention forward.  Returns (out, lse).

    pse: ALiBi slope vector [N] (fp32), a dense term broadcastable to
    [B, N, Sq, Sk] added to the scaled scores, or None.  atten_mask:
    bool/uint8 tensor broadcastable to [B, N, Sq, Sk], 1 = may attend, or a
    floating tensor of that shape added to the scaled scores (finite or
    -inf; -inf masks the pair).  causal: the
    lower-triangular rule.  padding_kv_len: int [B] valid keys per batch.
    modality_ids [B, S] with the 2x2 ``allow`` table and ``allow_diag``.
    keep_prob < 1: dropout with the Philox mask of seed and offset
    (include/fa.h, fa_dropout; offset counts 128-bit blocks, so a fresh
    mask needs offset advanced by ceil(Sk / 8)); pass the same values to bwd.
    float8_e4m3fn q/k/v (D = 128): the fp8 forward; out is bf16, and the
    caller folds the dequantisation factors of q and k into scale and
    multiplies out by that of v.
    scale has no default (pass 1/sqrt(D) explicitly)."""
    if scale is None:
        raise FaError(FA_ERR_INVALID_ARG, "scale must be given explicitly")
    shape = make_shape(query, key, head_num, input_layout)
    _check_operand(query, None, "query")
    _check_operand(key, None, "key", query)
    _check_operand(value, key.shape, "value", query)
    keep = _Keep()
    check_side_inputs(query.device, pse=pse, atten_mask=atten_mask, padding_kv_len=padding_kv_len,
                      modality_ids=modality_ids, tile_map=tile_map)
    atten_mask, add = split_atten_mask(atten_mask)
    m = make_mask(shape, causal=causal, atten_mask=atten_mask,
                  padding_kv_len=padding_kv_len, modality_ids=modality_ids,
                  allow=allow, allow_diag=allow_diag, tile_map=tile_map, keep=keep)
    ps = make_pse(pse, keep, shape, add)
    dr = make_dropout(keep_prob, seed, offset)
    if out is None:
        out = torch.empty(query.shape, dtype=out_dtype(query.dtype), device=query.device)
    if lse is None:
        lse = torch.empty((shape.B, shape.N, shape.Sq), dtype=torch.float32,
                          device=query.device)
    _check_operand(out, query.shape, "out")
    if out.dtype != out_dtype(query.dtype) or out.device != query.device:
        raise FaError(FA_ERR_INVALID_ARG, f"out must be {out_dtype(query.dtype)} on q's device")
    _check_lse(lse, shape, query)
    entry = lib().fa_testing_fwd_withhold_q if _withhold_q else lib().fa_fwd
    with _on_device(query.device):
        st = entry(ctypes.byref(shape), _ptr(query), _ptr(key), _ptr(value),
                   None if ps is None else ctypes.byref(ps),
                   None if m is None else ctypes.byref(m),
                   float(scale), float(keep_prob),
                   None if dr is None else ctypes.byref(dr), _ptr(out), _ptr(lse),
                   _stream(query))
    _check(st, "fa_fwd")
    return out, lse


def testing_fwd_withhold_q(query, key, value, head_num=None, input_layout="BNSD",
                           scale=None, **kw):
    """Test only (include/fa_testing.h): the forward with its query tiles
    withheld, so that its bounded waits expire.  The next sync_status()
    raises FaError(FA_ERR_TIMEOUT)."""
    return fwd(query, key, value, head_num, input_layout, scale=scale,
               _withhold_q=True, **kw)


def bwd_workspace_size(shape: FaShape) -> int:
    return int(lib().fa_bwd_workspace_size(ctypes.byref(shape)))


def bwd(query, key, value, out, dout, lse, head_num=None, input_layout="BNSD",
        pse=None, padding_kv_len=None, atten_mask=None, scale=None, keep_prob=1.0, *,
        causal=False, modality_ids=None, allow=((1, 1), (0, 1)), allow_diag=False,
        tile_map=None, workspace=None, dq=None, dk=None, dv=None, seed=None, offset=0):
    """Gradients (dq, dk, dv) of sum(dout * out), recomputing P from lse."""
    if scale is None:
        raise FaError(FA_ERR_INVALID_ARG, "scale must be given explicitly")
    if query.dtype == torch.float8_e4m3fn:
        raise FaError(FA_ERR_UNSUPPORTED, "the e4m3 path is forward only")
    shape = make_shape(query, key, head_num, input_layout)
    for t, n in ((query, "query"), (key, "key"), (value, "value"), (out, "out"),
                 (dout, "dout")):
        _check_operand(t, None, n, query)
    keep = _Keep()
    check_side_inputs(query.device, pse=pse, atten_mask=atten_mask, padding_kv_len=padding_kv_len,
                      modality_ids=modality_ids, tile_map=tile_map)
    atten_mask, add = split_atten_mask(atten_mask)
    m = make_mask(shape, causal=causal, atten_mask=atten_mask,
                  padding_kv_len=padding_kv_len, modality_ids=modality_ids,
                  allow=allow, allow_diag=allow_diag, tile_map=tile_map, keep=keep)
    ps = make_pse(pse, keep, shape, add)
    dr = make_dropout(keep_prob, seed, offset)
    need = bwd_workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=query.device)
    dq = torch.empty_like(query) if dq is None else dq
    dk = torch.empty_like(key) if dk is None else dk
    dv = torch.empty_like(value) if dv is None else dv
    for t, like, n in ((dq, query, "dq"), (dk, key, "dk"), (dv, value, "dv")):
        _check_operand(t, like.shape, n, query)
    _check_lse(lse, shape, query)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or \
            workspace.device != query.device:
        raise FaError(FA_ERR_INVALID_ARG, "workspace must be a contiguous uint8 tensor on q's device")
    with _on_device(query.device):
        st = lib().fa_bwd(ctypes.byref(shape), _ptr(query), _ptr(key), _ptr(value),
                          _ptr(out), _ptr(dout), _ptr(lse),
                          None if ps is None else ctypes.byref(ps),
                          None if m is None else ctypes.byref(m),
                          float(scale), float(keep_prob),
                          None if dr is None else ctypes.byref(dr),
                          _ptr(dq), _ptr(dk), _ptr(dv),
                          _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                          _stream(query))
    _check(st, "fa_bwd")
    return dq, dk, dv


NOALLOC_SCRATCH_BYTES = 32 << 20   # FA_NOALLOC_SCRATCH_BYTES of include/fa.h


def bwd_noalloc(query, key, value, out, dout, lse, head_num=None, input_layout="BNSD",
                pse=None, padding_kv_len=None, atten_mask=None, scale=None, keep_prob=1.0,
                *, causal=False, modality_ids=None, allow=((1, 1), (0, 1)),
                allow_diag=False, tile_map=None, dq=None, dk=None, dv=None, seed=None,
                offset=0):
    """Backward through fa_bwd_noalloc: the library's fixed scratch array
    replaces the workspace, so the call allocates no scratch (the outputs
    dq, dk, dv are still the caller's).  Shapes whose workspace would exceed
    NOALLOC_SCRATCH_BYTES raise FA_ERR_UNSUPPORTED."""
    if scale is None:
        raise FaError(FA_ERR_INVALID_ARG, "scale must be given explicitly")
    if query.dtype == torch.float8_e4m3fn:
        raise FaError(FA_ERR_UNSUPPORTED, "the e4m3 path is forward only")
    shape = make_shape(query, key, head_num, input_layout)
    for t, n in ((query, "query"), (key, "key"), (value, "value"), (out, "out"),
                 (dout, "dout")):
        _check_operand(t, None, n, query)
    keep = _Keep()
    check_side_inputs(query.device, pse=pse, atten_mask=atten_mask, padding_kv_len=padding_kv_len,
                      modality_ids=modality_ids, tile_map=tile_map)
    atten_mask, add = split_atten_mask(atten_mask)
    m = make_mask(shape, causal=causal, atten_mask=atten_mask,
                  padding_kv_len=padding_kv_len, modality_ids=modality_ids,
                  allow=allow, allow_diag=allow_diag, tile_map=tile_map, keep=keep)
    ps = make_pse(pse, keep, shape, add)
    dr = make_dropout(keep_prob, seed, offset)
    dq = torch.empty_like(query) if dq is None else dq
    dk = torch.empty_like(key) if dk is None else dk
    dv = torch.empty_like(value) if dv is None else dv
    for t, like, n in ((dq, query, "dq"), (dk, key, "dk"), (dv, value, "dv")):
        _check_operand(t, like.shape, n, query)
    _check_lse(lse, shape, query)
    with _on_device(query.device):
        st = lib().fa_bwd_noalloc(ctypes.byref(shape), _ptr(query), _ptr(key), _ptr(value),
                                  _ptr(out), _ptr(dout), _ptr(lse),
                                  None if ps is None else ctypes.byref(ps),
                                  None if m is None else ctypes.byref(m),
                                  float(scale), float(keep_prob),
                                  None if dr is None else ctypes.byref(dr), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _stream(query))
    _check(st, "fa_bwd_noalloc")
    return dq, dk, dv


def build_tile_map(atten_mask, query, key, head_num=None, input_layout="BNSD"):
    """Tile classification of a bool mask (one byte per 128 x 128 tile)."""
    shape = make_shape(query, key, head_num, input_layout)
    check_side_inputs(query.device, query=query, atten_mask=atten_mask)
    keep = _Keep()
    m = make_mask(shape, atten_mask=atten_mask, keep=keep)
    n = int(lib().fa_mask_tile_map_size(ctypes.byref(shape), ctypes.byref(m)))
    tm = torch.empty(max(n, 1), dtype=torch.uint8, device=query.device)
    with _on_device(query.device):
        st = lib().fa_build_mask_tile_map(ctypes.byref(shape), ctypes.byref(m),
                                          _ptr(tm), _stream(query))
    _check(st, "fa_build_mask_tile_map")
    return tm


def build_modality_mask(modality_ids, allow=((1, 1), (0, 1)), allow_diag=False):
    """Explicit cross-modal bool mask [B, S, S] (uint8, 1 = may attend)."""
    check_side_inputs(modality_ids.device, modality_ids=modality_ids)
    ids = modality_ids.to(torch.int32).contiguous()
    B, S = ids.shape
    mask = torch.empty((B, S, S), dtype=torch.uint8, device=ids.device)
    tab = ((ctypes.c_uint8 * 2) * 2)()
    for a in range(2):
        for c in range(2):
            tab[a][c] = 1 if allow[a][c] else 0
    with _on_device(ids.device):
        st = lib().fa_build_modality_mask(int(B), int(S), _ptr(ids), ctypes.byref(tab),
                                          1 if allow_diag else 0, _ptr(mask), _stream(ids))
    _check(st, "fa_build_modality_mask")
    return mask


def sync_status(device=None):
    """Synchronise the current stream and raise if a kernel timed out."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with _on_device(dev):
        st = lib().fa_sync_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    _check(st, "fa_sync_status")
