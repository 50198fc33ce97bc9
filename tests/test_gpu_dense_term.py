"""Forward and backward parity with a dense additive term -- the general
`pse` tensor of the FlashAttentionScore guide (sec. 3.2) or a float
`atten_mask` added to the scaled scores (sec. 4 step 1) -- against the fp64
oracle.  Covers broadcast shapes ([1|B, 1|N, Sq, Sk]), the vectorised and the
scalar loads (Sk a multiple of 4 or not), -inf entries and rows left with no
finite score, the combination with the causal rule, padding and ALiBi, both
layouts, fp16 and the fp32 path.  Needs a B200 (sm_100a)."""
import numpy as np
import pytest
import torch

import oracle
from attention_fwd_bwd_02_b200 import fa
from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def _term(shape, seed, scale=1.5, neginf_frac=0.0, empty_row=None):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(shape, generator=g, dtype=torch.float32) * scale
    if neginf_frac:
        drop = torch.rand(shape, generator=g) < neginf_frac
        a = a.masked_fill(drop, float("-inf"))
    if empty_row is not None:
        a[empty_row] = float("-inf")
    return a


def _run(c, term, as_mask=False, check_bwd=True):
    dev = P.to_dev(c)
    kw = P.mask_kwargs(c, dev)
    t = term.cuda()
    extra = dict(atten_mask=t) if as_mask else dict(pse=t)
    pse_alibi = dev["slopes"]
    if pse_alibi is not None and not as_mask:
        raise ValueError("ALiBi with a dense pse: pass the dense term as atten_mask")
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, c.layout, scale=c.scale,
                      **({"pse": pse_alibi} if pse_alibi is not None else {}), **extra, **kw)
    fa.sync_status()
    okw = P.oracle_kwargs(c)
    q, k, v, do = (P._bnsd(getattr(c, n), c) for n in ("q", "k", "v", "dout"))
    ref_o, ref_l = oracle.fwd(q, k, v, c.scale, bias=term.double().numpy(), **okw)
    got_o, got_l = P.gpu_heads(out, c), P.gpu_heads(lse, c, is_lse=True)
    P.assert_close(got_o, ref_o, c.dtype, f"{c.name} out")
    P.assert_close(got_l, ref_l, c.dtype, f"{c.name} lse")
    assert np.all(got_o[np.isneginf(ref_l)] == 0.0)
    if check_bwd:
        dq, dk, dv = fa.bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, c.N, c.layout,
                            scale=c.scale,
                            **({"pse": pse_alibi} if pse_alibi is not None else {}),
                            **extra, **kw)
        fa.sync_status()
        rq, rk, rv = oracle.bwd(q, k, v, do, c.scale, bias=term.double().numpy(), **okw)
        for got, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
            P.assert_close(P.gpu_heads(got, c), ref, c.dtype, f"{c.name} {what}")
    return out, lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("sq,sk,bshape", [(200, 333, "1N"), (256, 256, "BN"), (130, 260, "B1"),
                                          (77, 128, "11")])
def test_dense_pse(D, sq, sk, bshape):
    B, N = 2, 3
    c = I.make_case(f"dense_D{D}_{sq}x{sk}_{bshape}", B, N, sq, sk, D, seed=140)
    shape = ((B if bshape[0] == "B" else 1), (N if bshape[1] == "N" else 1), sq, sk)
    _run(c, _term(shape, 141))


@pytest.mark.parametrize("D", [64, 128])
def test_float_mask_with_neginf_and_empty_rows(D):
    c = I.make_case(f"fmask_D{D}", 2, 2, 190, 300, D, seed=142, kv_len_range=(100, 300))
    term = _term((2, 2, 190, 300), 143, neginf_frac=0.3, empty_row=(1, 0, 7))
    _run(c, term, as_mask=True)


@pytest.mark.parametrize("D", [64, 128])
def test_causal_alibi_and_dense_mask(D):
    c = I.make_case(f"calibi_dense_D{D}", 1, 4, 300, 300, D, seed=144, causal=True, alibi=True)
    _run(c, _term((1, 4, 300, 300), 145, scale=0.7), as_mask=True)


def test_zero_neginf_float_mask_matches_the_bool_mask():
    c = I.make_case("fmask_vs_bool", 2, 3, 160, 250, 64, seed=146)
    g = torch.Generator().manual_seed(147)
    keep = torch.rand(2, 3, 160, 250, generator=g) < 0.6
    term = torch.zeros(2, 3, 160, 250).masked_fill(~keep, float("-inf"))
    out_f, lse_f = _run(c, term, as_mask=True)
    out_b, lse_b = P.gpu_fwd(c, atten_mask=keep.cuda())
    P.assert_close(P.gpu_heads(out_f, c), P.gpu_heads(out_b, c), c.dtype, "float vs bool out")
    P.assert_close(P.gpu_heads(lse_f, c, is_lse=True), P.gpu_heads(lse_b, c, is_lse=True),
                   c.dtype, "float vs bool lse")


def test_bsh_layout_dense_pse():
    c = I.make_case("dense_bsh", 2, 4, 150, 150, 64, layout="BSH", seed=148,
                    modality=(60, 90))
    _run(c, _term((1, 4, 150, 150), 149))


def test_fp16_dense_pse():
    c = I.make_case("dense_fp16", 1, 2, 140, 270, 128, seed=150, dtype=torch.float16)
    _run(c, _term((1, 2, 140, 270), 151))


def test_fp32_path_dense_pse():
    c = I.make_case("dense_fp32", 1, 2, 70, 90, 64, seed=152, dtype=torch.float32)
    _run(c, _term((1, 2, 70, 90), 153, neginf_frac=0.2))


def test_constant_shift_moves_only_the_lse():
    c = I.make_case("dense_shift", 1, 2, 256, 256, 128, seed=154, causal=True)
    term = _term((1, 2, 256, 256), 155)
    o1, l1 = _run(c, term, check_bwd=False)
    o2, l2 = _run(c, term + 2.5, check_bwd=False)
    P.assert_close(P.gpu_heads(o2, c), P.gpu_heads(o1, c), c.dtype, "shifted out")
    np.testing.assert_allclose(l2.cpu().numpy(), l1.cpu().numpy() + 2.5, atol=2e-2)


def test_both_dense_terms_are_rejected():
    c = I.make_case("dense_both", 1, 1, 64, 64, 64, seed=156)
    dev = P.to_dev(c)
    t = torch.zeros(1, 1, 64, 64, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fwd(dev["q"], dev["k"], dev["v"], 1, "BNSD", scale=c.scale, pse=t, atten_mask=t)


def test_expanded_term_equals_its_copy():
    """An expanded (stride-0) batch dimension is passed as a broadcast: the
    result equals that of the materialised copy bit for bit."""
    c = I.make_case("dense_expand", 3, 2, 130, 200, 64, seed=157)
    dev = P.to_dev(c)
    base = _term((1, 2, 130, 200), 158).cuda()
    expanded = base.expand(3, 2, 130, 200)
    assert expanded.stride(0) == 0
    o1, l1 = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, pse=expanded)
    o2, l2 = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, pse=expanded.contiguous())
    fa.sync_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
