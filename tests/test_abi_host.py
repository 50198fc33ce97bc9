"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/fa.h declares, and
reject malformed arguments with the documented status codes before it
touches the GPU (argument validation runs first, on the host)."""
import ctypes

import pytest

from attention_fwd_bwd_02_b200 import build as fa_build
from attention_fwd_bwd_02_b200 import fa


@pytest.fixture(scope="module")
def L():
    fa_build.build()
    return fa.lib()


def test_exports_every_declared_function(L):
    names = fa.declared_functions()
    assert "fa_fwd" in names and "fa_bwd" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in fa.h but not exported"
    testing = fa.declared_functions(fa.TESTING_HEADER)
    assert testing == ["fa_testing_fwd_withhold_q"]
    for n in testing:
        assert hasattr(L, n), f"{n} declared in fa_testing.h but not exported"


def test_testing_entry_validates_like_fwd(L):
    # Same validation as fa_fwd, before any device work; fp32 has no hook.
    args = lambda shape: (ctypes.byref(shape), FAKE, FAKE, FAKE, None, None,
                          0.125, 1.0, None, FAKE, FAKE, None)
    assert L.fa_testing_fwd_withhold_q(*args(_shape(D=96))) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_testing_fwd_withhold_q(*args(_shape(B=-1))) == fa.FA_ERR_INVALID_ARG
    assert L.fa_testing_fwd_withhold_q(*args(_shape(dtype=fa.FA_F32))) == fa.FA_ERR_UNSUPPORTED


def test_status_strings_and_version(L):
    assert L.fa_status_string(0) == b"FA_OK"
    assert L.fa_status_string(4) == b"FA_ERR_TIMEOUT"
    assert L.fa_status_string(99) == b"FA_ERR_UNKNOWN"
    assert b"sm_100a" in L.fa_version()


def _shape(**kw):
    d = dict(B=2, N=4, Sq=256, Sk=256, D=128, layout=fa.FA_LAYOUT_BNSD, dtype=fa.FA_BF16)
    d.update(kw)
    return fa.FaShape(d["B"], d["N"], d["Sq"], d["Sk"], d["D"], d["layout"], d["dtype"])


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: validation fails first


def _fwd(L, shape, pse=None, mask=None, scale=0.125, keep_prob=1.0, ptr=FAKE, drop=None):
    return L.fa_fwd(ctypes.byref(shape), ptr, ptr, ptr,
                    None if pse is None else ctypes.byref(pse),
                    None if mask is None else ctypes.byref(mask),
                    scale, keep_prob, None if drop is None else ctypes.byref(drop),
                    ptr, ptr, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), fa.FA_ERR_UNSUPPORTED),          # bf16 head dim not 64/128
    (dict(D=96, dtype=fa.FA_F16), fa.FA_ERR_UNSUPPORTED),  # fp16 likewise
    (dict(D=256, dtype=fa.FA_F32), fa.FA_ERR_UNSUPPORTED),
    (dict(D=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(layout=7), fa.FA_ERR_INVALID_ARG),
    (dict(dtype=5), fa.FA_ERR_INVALID_ARG),
    (dict(N=70000), fa.FA_ERR_UNSUPPORTED),
    (dict(D=64, dtype=fa.FA_E4M3), fa.FA_ERR_UNSUPPORTED),  # e4m3 is D = 128 only
    (dict(dtype=4), fa.FA_ERR_INVALID_ARG),
])
def test_shape_validation(L, kw, code):
    assert _fwd(L, _shape(**kw)) == code


def test_keep_prob_and_scale(L):
    assert _fwd(L, _shape(), keep_prob=0.9) == fa.FA_ERR_INVALID_ARG   # no fa_dropout
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert _fwd(L, _shape(), keep_prob=bad, drop=fa.FaDropout(1, 2)) == fa.FA_ERR_INVALID_ARG
    # a valid dropout set-up passes validation (an empty problem then returns FA_OK)
    assert _fwd(L, _shape(B=0), keep_prob=0.9, drop=fa.FaDropout(1, 2)) == fa.FA_OK
    assert _fwd(L, _shape(), scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, _shape(), scale=float("inf")) == fa.FA_ERR_INVALID_ARG


def test_mask_validation(L):
    m = fa.FaMask()
    m.flags = 64                                    # unknown bit
    assert _fwd(L, _shape(), mask=m) == fa.FA_ERR_INVALID_ARG
    m = fa.FaMask(); m.flags = fa.FA_MASK_KV_PADDING  # kv_len missing
    assert _fwd(L, _shape(), mask=m) == fa.FA_ERR_INVALID_ARG
    m = fa.FaMask(); m.flags = fa.FA_MASK_BOOL        # mask pointer missing
    assert _fwd(L, _shape(), mask=m) == fa.FA_ERR_INVALID_ARG
    m = fa.FaMask(); m.flags = fa.FA_MASK_BOOL; m.mask = 0x10000; m.mask_stride_q = -1
    assert _fwd(L, _shape(), mask=m) == fa.FA_ERR_INVALID_ARG
    m = fa.FaMask(); m.flags = fa.FA_MASK_MODALITY; m.modality_ids = 0x10000
    assert _fwd(L, _shape(Sq=32, Sk=256), mask=m) == fa.FA_ERR_INVALID_ARG  # Sq != Sk
    m = fa.FaMask(); m.flags = fa.FA_MASK_MODALITY
    assert _fwd(L, _shape(), mask=m) == fa.FA_ERR_INVALID_ARG  # ids missing
    m = fa.FaMask(); m.flags = fa.FA_MASK_MODALITY; m.modality_ids = 0x10000
    assert _fwd(L, _shape(Sq=40000, Sk=40000), mask=m) == fa.FA_ERR_UNSUPPORTED


def test_pse_validation(L):
    assert _fwd(L, _shape(), pse=fa.FaPse(fa.FA_PSE_ALIBI, None)) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, _shape(), pse=fa.FaPse(3, 0x10000)) == fa.FA_ERR_INVALID_ARG  # no dense array
    assert _fwd(L, _shape(), pse=fa.FaPse(4, 0x10000)) == fa.FA_ERR_INVALID_ARG  # unknown kind
    S = _shape()
    ok = dict(bias=0x10000, bias_stride_b=0, bias_stride_h=0, bias_stride_q=S.Sk)
    for bad in (dict(bias=0x10002), dict(bias_stride_q=S.Sk - 1), dict(bias_stride_b=-1),
                dict(bias_stride_h=-4)):
        kw = dict(ok, **bad)
        ps = fa.FaPse(fa.FA_PSE_DENSE, None, kw["bias"], kw["bias_stride_b"],
                      kw["bias_stride_h"], kw["bias_stride_q"])
        assert _fwd(L, S, pse=ps) == fa.FA_ERR_INVALID_ARG, bad


def test_empty_problems_are_ok_without_launch(L):
    assert _fwd(L, _shape(B=0)) == fa.FA_OK
    assert _fwd(L, _shape(Sq=0)) == fa.FA_OK
    assert _fwd(L, _shape(N=0)) == fa.FA_OK


def test_bwd_validation(L):
    s = _shape()
    ws = L.fa_bwd_workspace_size(ctypes.byref(s))
    rows = 2 * 4 * 256
    assert ws >= rows * 128 * 4 + rows * 4
    assert L.fa_bwd_workspace_size(ctypes.byref(_shape(D=96))) == 0
    p = FAKE
    rc = L.fa_bwd(ctypes.byref(s), p, p, p, p, p, p, None, None, 0.1, 0.5, None, p, p, p,
                  p, ctypes.c_size_t(ws), None)
    assert rc == fa.FA_ERR_INVALID_ARG                  # keep_prob < 1 without fa_dropout
    rc = L.fa_bwd(ctypes.byref(s), p, p, p, p, p, p, None, None, 0.1, 1.0, None, p, p, p,
                  None, ctypes.c_size_t(ws), None)
    assert rc == fa.FA_ERR_INVALID_ARG                  # workspace missing
    rc = L.fa_bwd(ctypes.byref(s), p, p, p, p, p, p, None, None, 0.1, 1.0, None, p, p, p,
                  p, ctypes.c_size_t(ws - 16), None)
    assert rc == fa.FA_ERR_INVALID_ARG                  # workspace too small
    odd = ctypes.c_void_p(0x10008)
    rc = L.fa_bwd(ctypes.byref(s), odd, p, p, p, p, p, None, None, 0.1, 1.0, None, p, p, p,
                  p, ctypes.c_size_t(ws), None)
    assert rc == fa.FA_ERR_INVALID_ARG                  # misaligned tensor


def test_e4m3_backward_is_unsupported(L):
    s = _shape(dtype=fa.FA_E4M3)
    p = FAKE
    rc = L.fa_bwd(ctypes.byref(s), p, p, p, p, p, p, None, None, 0.1, 1.0, None, p, p, p,
                  p, ctypes.c_size_t(1 << 30), None)
    assert rc == fa.FA_ERR_UNSUPPORTED


def test_misaligned_forward_pointer(L):
    odd = ctypes.c_void_p(0x10008)
    s = _shape()
    rc = L.fa_fwd(ctypes.byref(s), odd, FAKE, FAKE, None, None, 0.1, 1.0, None, FAKE, FAKE, None)
    # Either the device lookup fails first on a machine without a GPU
    # (FA_ERR_CUDA) or the alignment check rejects it; never FA_OK.
    assert rc in (fa.FA_ERR_INVALID_ARG, fa.FA_ERR_CUDA)


def test_tile_map_size(L):
    m = fa.FaMask(); m.flags = fa.FA_MASK_BOOL; m.mask = 0x10000
    m.mask_stride_b, m.mask_stride_h, m.mask_stride_q = 300 * 300, 0, 300
    s = _shape(B=3, N=5, Sq=300, Sk=300)
    assert L.fa_mask_tile_map_size(ctypes.byref(s), ctypes.byref(m)) == 3 * 1 * 3 * 3
    m.mask_stride_h = 1
    assert L.fa_mask_tile_map_size(ctypes.byref(s), ctypes.byref(m)) == 3 * 5 * 3 * 3


def test_modality_mask_validation(L):
    tab = ((ctypes.c_uint8 * 2) * 2)()
    assert L.fa_build_modality_mask(-1, 4, FAKE, ctypes.byref(tab), 0, FAKE, None) == \
        fa.FA_ERR_INVALID_ARG
    assert L.fa_build_modality_mask(2, 4, None, ctypes.byref(tab), 0, FAKE, None) == \
        fa.FA_ERR_INVALID_ARG
    assert L.fa_build_modality_mask(0, 4, None, ctypes.byref(tab), 0, None, None) == fa.FA_OK


def test_python_binding_rejects_bad_layout():
    import torch
    q = torch.zeros(2, 3, 4)
    with pytest.raises(fa.FaError):
        fa.make_shape(q, q, 3, "BHSD")
    with pytest.raises(fa.FaError):
        fa.make_shape(q, q, 5, "BSH")     # 5 does not divide 4
