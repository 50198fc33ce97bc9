"""Host-side logic of the Python binding that needs no GPU: argument
splitting and validation for the dense additive term (pse tensor / float
atten_mask), dropout and the fp8 output type.  Nothing here launches a
kernel; errors must be raised before any device work."""
import pytest
import torch

from attention_fwd_bwd_02_b200 import fa


def test_float_masks_become_the_additive_term():
    b = torch.zeros(2, 3, dtype=torch.bool)
    u = torch.zeros(2, 3, dtype=torch.uint8)
    f = torch.zeros(2, 3, dtype=torch.float32)
    h = torch.zeros(2, 3, dtype=torch.bfloat16)
    assert fa.split_atten_mask(b) == (b, None)
    assert fa.split_atten_mask(u) == (u, None)
    m, a = fa.split_atten_mask(f)
    assert m is None and a is f
    m, a = fa.split_atten_mask(h)
    assert m is None and a is h
    assert fa.split_atten_mask(None) == (None, None)


def test_dropout_arguments():
    assert fa.make_dropout(1.0, None, 0) is None          # no dropout, no seed needed
    d = fa.make_dropout(0.9, 7, 3)
    assert (d.seed, d.offset) == (7, 3)
    d = fa.make_dropout(0.5, -1, -2)                      # wrapped to uint64
    assert (d.seed, d.offset) == (2**64 - 1, 2**64 - 2)
    for bad in (0.0, -0.1, 1.01, float("nan")):
        with pytest.raises(fa.FaError) as e:
            fa.make_dropout(bad, 1, 0)
        assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FaError) as e:
        fa.make_dropout(0.8, None, 0)                     # keep_prob < 1 needs a seed
    assert e.value.status == fa.FA_ERR_INVALID_ARG


def _shape(B=2, N=3, Sq=5, Sk=7, D=64):
    return fa.FaShape(B, N, Sq, Sk, D, fa.FA_LAYOUT_BNSD, fa.FA_BF16)


def test_pse_kinds():
    keep = fa._Keep()
    assert fa.make_pse(None, keep) is None
    ps = fa.make_pse(torch.tensor([0.5, 0.25, 0.125]), keep, _shape())
    assert ps.kind == fa.FA_PSE_ALIBI and ps.slopes != 0 and not ps.bias
    # a dense pse and a float mask at once: one term only
    with pytest.raises(fa.FaError) as e:
        fa.make_pse(torch.zeros(1, 3, 5, 7), keep, _shape(), add=torch.zeros(1, 3, 5, 7))
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_dense_term_must_be_on_the_device_and_broadcast():
    keep = fa._Keep()
    with pytest.raises(fa.FaError) as e:            # a CPU tensor is refused
        fa.make_pse(None, keep, _shape(), add=torch.zeros(5, 7))
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FaError):                 # no problem shape to check against
        fa.make_pse(torch.zeros(2, 3, 5, 7), keep, None)


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs CUDA tensors")
def test_dense_term_shapes_on_device():  # pragma: no cover - needs CUDA tensors
    keep = fa._Keep()
    ok = [(5, 7), (1, 3, 5, 7), (2, 1, 5, 7), (2, 3, 5, 7)]
    for shp in ok:
        ps = fa.make_pse(None, keep, _shape(), add=torch.zeros(shp, device="cuda"))
        assert ps.kind == fa.FA_PSE_DENSE and ps.bias_stride_q >= 7
    for shp in [(5, 6), (3, 3, 5, 7), (2, 2, 5, 7), (4, 5)]:
        with pytest.raises(fa.FaError):
            fa.make_pse(None, keep, _shape(), add=torch.zeros(shp, device="cuda"))


def test_e4m3_output_type_and_forward_only():
    assert fa.out_dtype(torch.float8_e4m3fn) == torch.bfloat16
    assert fa.out_dtype(torch.bfloat16) == torch.bfloat16
    assert fa.out_dtype(torch.float16) == torch.float16
    assert fa._dtype_code(torch.float8_e4m3fn) == fa.FA_E4M3
    q = torch.zeros(1, 1, 8, 128, dtype=torch.float8_e4m3fn)
    with pytest.raises(fa.FaError) as e:
        fa.bwd(q, q, q, q, q, torch.zeros(1, 1, 8), 1, scale=0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_side_inputs_must_be_on_the_device():
    # host tensors would reach the kernels as host pointers: refused up front
    t = torch.zeros(3)
    for name in ("pse", "atten_mask", "padding_kv_len", "modality_ids", "tile_map"):
        with pytest.raises(fa.FaError) as e:
            fa.check_side_inputs("cuda:0", **{name: t})
        assert e.value.status == fa.FA_ERR_INVALID_ARG
    fa.check_side_inputs("cuda:0", pse=None)          # absent inputs are fine
    with pytest.raises(fa.FaError):
        fa.build_modality_mask(torch.zeros(2, 4, dtype=torch.int32))


def test_bool_mask_views_pass_through_with_their_strides():
    # The forward reads aligned mask rows 16 bytes at a time and anything
    # else byte by byte: the binding must hand both kinds of view over as
    # they are (pointer and strides), copying only what the kernel cannot
    # index (a non-unit last stride or a shape to broadcast).
    shp = fa.FaShape(2, 3, 5, 32, 64, fa.FA_LAYOUT_BNSD, fa.FA_BF16)
    wide = torch.zeros(2, 1, 5, 48, dtype=torch.uint8)
    view = wide[..., 1:33]
    keep = fa._Keep()
    m = fa.make_mask(shp, atten_mask=view, keep=keep)
    assert m.mask == view.data_ptr() == wide.data_ptr() + 1
    assert (m.mask_stride_b, m.mask_stride_h, m.mask_stride_q) == (5 * 48, 0, 48)
    full = torch.ones(2, 3, 5, 32, dtype=torch.bool)
    m = fa.make_mask(shp, atten_mask=full, keep=keep)
    assert m.mask == full.data_ptr()
    assert (m.mask_stride_b, m.mask_stride_h, m.mask_stride_q) == (3 * 5 * 32, 5 * 32, 32)
    # a transposed view (last stride != 1) is copied into a contiguous mask
    t = torch.ones(2, 3, 32, 5, dtype=torch.uint8).transpose(-1, -2)
    m = fa.make_mask(shp, atten_mask=t, keep=keep)
    assert m.mask != t.data_ptr() and m.mask_stride_q == 32
