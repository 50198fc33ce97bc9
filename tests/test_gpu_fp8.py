"""The e4m3 (fp8) forward (the multimodal page's experimental "pure fp8"):
parity with the fp64 oracle, which reads the same e4m3-rounded inputs.
Needs a B200 (sm_100a).

Tolerance: the kernel rounds P to e4m3 (3 mantissa bits, a relative half-ulp
of 2^-4) before P V, so |d| <= 2^-4 max|V| / keep_prob (the worst case, all
rounding errors of one sign; plus 1e-2 for the bf16 output) bounds every
element, and mean |d| <= 0.01 / keep_prob bounds the typical error, where
the rounding errors largely cancel.  Measured without dropout: worst 0.056,
mean 0.004; with a dense term and dropout (peaked rows): worst 0.135, mean
0.006.  LSE is computed in fp32 from the exact e4m3 products and keeps the
16-bit bound."""
import numpy as np
import pytest
import torch

import oracle
from attention_fwd_bwd_02_b200 import fa
from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu
F8 = torch.float8_e4m3fn


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def _tol(c, keep_prob=1.0):
    vmax = float(c.v.float().abs().max())
    return dict(max_tol=(2.0 ** -4 * vmax + 1e-2) / keep_prob, mean_tol=1e-2 / keep_prob)


def _check(c, out, lse, ref_o, ref_l):
    assert out.dtype == torch.bfloat16
    P.assert_close(P.gpu_heads(out, c), ref_o, torch.bfloat16, f"{c.name} out", **_tol(c))
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, torch.bfloat16, f"{c.name} lse")


CASES = [
    ("nomask_200x333", dict(B=2, N=3, Sq=200, Sk=333)),
    ("causal_300", dict(B=2, N=3, Sq=300, Sk=300, causal=True)),
    ("causal_alibi_300", dict(B=2, N=4, Sq=300, Sk=300, causal=True, alibi=True)),
    ("padding_64x400", dict(B=3, N=2, Sq=64, Sk=400, kv_len_range=(0, 400))),
    ("bsh_modality_150", dict(B=2, N=4, Sq=150, Sk=150, layout="BSH", modality=(60, 90))),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[x[0] for x in CASES])
def test_fp8_forward_parity(name, kw):
    kw = dict(kw)
    B, N, Sq, Sk = (kw.pop(x) for x in ("B", "N", "Sq", "Sk"))
    c = I.make_case(f"fp8_{name}", B, N, Sq, Sk, 128, seed=310, dtype=F8, **kw)
    out, lse = P.gpu_fwd(c)
    ref_o, ref_l = P.oracle_fwd(c)
    _check(c, out, lse, ref_o, ref_l)


def test_fp8_dense_term_and_dropout():
    c = I.make_case("fp8_ext", 2, 2, 256, 256, 128, seed=311, dtype=F8, causal=True)
    dev = P.to_dev(c)
    g = torch.Generator().manual_seed(312)
    term = torch.randn(1, 2, 256, 256, generator=g)
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, causal=True,
                      atten_mask=term.cuda(), keep_prob=0.75, seed=9, offset=1)
    fa.sync_status()
    q, k, v = (P._bnsd(getattr(c, n), c) for n in ("q", "k", "v"))
    ref_o, ref_l = oracle.fwd(q, k, v, c.scale, causal=True, bias=term.double().numpy(),
                              dropout=(0.75, 9, 1))
    # dropout scales the kept P by 1/keep_prob: the bound grows with it
    P.assert_close(P.gpu_heads(out, c), ref_o, torch.bfloat16, "fp8 ext out", **_tol(c, 0.75))
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, torch.bfloat16, "fp8 ext lse")


def test_fp8_config2_shape_sampled():
    """Causal B=4 N=32 S=2048 D=128 in e4m3, three heads against the oracle."""
    c = I.make_case("fp8_cfg2", 4, 32, 2048, 2048, 128, seed=1002, dtype=F8, causal=True,
                    with_dout=False)
    out, lse = P.gpu_fwd(c)
    heads = [(0, 0), (1, 17), (3, 31)]
    ref_o, ref_l = P.oracle_fwd(c, heads)
    P.assert_close(P.gpu_heads(out, c, heads), ref_o, torch.bfloat16, "fp8 cfg2 out", **_tol(c))
    P.assert_close(P.gpu_heads(lse, c, heads, is_lse=True), ref_l, torch.bfloat16, "fp8 cfg2 lse")


def test_fp8_empty_keys_and_limits():
    c = I.make_case("fp8_empty", 1, 2, 64, 1, 128, seed=313, dtype=F8)
    dev = P.to_dev(c)
    k0, v0 = dev["k"][:, :, :0], dev["v"][:, :, :0]
    out, lse = fa.fwd(dev["q"], k0.contiguous(), v0.contiguous(), 2, scale=c.scale)
    fa.sync_status()
    assert out.dtype == torch.bfloat16 and torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))
    # the fp8 path is forward only, and D = 128 only
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], 2, scale=c.scale)
    with pytest.raises(fa.FaError) as e:
        fa.bwd(dev["q"], dev["k"], dev["v"], out, out, lse, 2, scale=c.scale)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    c64 = I.make_case("fp8_d64", 1, 1, 64, 64, 64, seed=314, dtype=F8)
    d64 = P.to_dev(c64)
    with pytest.raises(fa.FaError) as e:
        fa.fwd(d64["q"], d64["k"], d64["v"], 1, scale=c64.scale)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
