"""Dropout (keep_prob < 1, the FlashAttentionScore guide's keep_prob) on the
GPU against the fp64 oracle: the same Philox-4x32-10 mask (include/fa.h,
fa_dropout) must come out of the forward and the backward kernels, bit for
bit, and the outputs and gradients must match the oracle's.  Needs a B200
(sm_100a).

Tolerance (16-bit types): per element |d| <= (2e-2 + 4e-3 |ref|) / keep_prob
and mean |d| <= 2e-3 / keep_prob.  Kept probabilities are P / keep_prob, so
the 16-bit rounding of P, dP and dS in the kernels grows by that factor; and
dropout makes some gradient entries large (|dV| up to ~10 here), where the
16-bit output itself is rounded to 8 significant bits (half an ulp is
2^-9 |x|), which an absolute bound alone cannot allow for."""
import numpy as np
import pytest
import torch

import oracle
from attention_fwd_bwd_02_b200 import fa
from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu

SEED, OFFSET = 0x5EED_0123_4567_89AB, 42


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def _run(c, keep_prob, term=None, check_bwd=True, seed=SEED, offset=OFFSET):
    dev = P.to_dev(c)
    kw = P.mask_kwargs(c, dev)
    extra = {} if term is None else dict(atten_mask=term.cuda())
    drop = dict(keep_prob=keep_prob, seed=seed, offset=offset)
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, c.layout, pse=dev["slopes"],
                      scale=c.scale, **drop, **extra, **kw)
    fa.sync_status()
    okw = P.oracle_kwargs(c)
    if term is not None:
        okw["bias"] = term.double().numpy()
    q, k, v, do = (P._bnsd(getattr(c, n), c) for n in ("q", "k", "v", "dout"))
    od = (keep_prob, seed, offset)
    ref_o, ref_l = oracle.fwd(q, k, v, c.scale, dropout=od, **okw)
    _close(P.gpu_heads(out, c), ref_o, c.dtype, keep_prob, f"{c.name} out")
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, c.dtype, f"{c.name} lse")
    if check_bwd:
        dq, dk, dv = fa.bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, c.N, c.layout,
                            pse=dev["slopes"], scale=c.scale, **drop, **extra, **kw)
        fa.sync_status()
        rq, rk, rv = oracle.bwd(q, k, v, do, c.scale, dropout=od, **okw)
        for got, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
            _close(P.gpu_heads(got, c), ref, c.dtype, keep_prob, f"{c.name} {what}")
    return out, lse


def _close(got, ref, dtype, keep_prob, what):
    if dtype == torch.float32:
        P.assert_close(got, ref, dtype, what)
        return
    d = np.abs(np.asarray(got, np.float64) - ref)
    assert np.all(np.isfinite(d)), f"{what}: non-finite values"
    lim = (2e-2 + 4e-3 * np.abs(ref)) / keep_prob
    assert np.all(d <= lim), f"{what}: worst |d| - bound {float((d - lim).max()):.3e}"
    assert d.mean() <= 2e-3 / keep_prob, f"{what}: mean |d| {d.mean():.3e}"


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("sq,sk", [(256, 256), (200, 333)])
@pytest.mark.parametrize("keep_prob", [0.75, 0.5])
def test_dropout_parity(D, sq, sk, keep_prob):
    c = I.make_case(f"drop_D{D}_{sq}x{sk}_{keep_prob}", 2, 3, sq, sk, D, seed=200)
    _run(c, keep_prob)


@pytest.mark.parametrize("D", [64, 128])
def test_dropout_causal_alibi(D):
    c = I.make_case(f"drop_ca_D{D}", 2, 4, 300, 300, D, seed=201, causal=True, alibi=True)
    _run(c, 0.875)


@pytest.mark.parametrize("D", [64, 128])
def test_dropout_padding(D):
    c = I.make_case(f"drop_pad_D{D}", 3, 2, 200, 330, D, seed=208, kv_len_range=(0, 330))
    _run(c, 0.75)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("keep_prob", [1.0, 0.875])
def test_heavily_attended_keys_mixed_bound(D, keep_prob):
    """Causal + steep ALiBi + short documents: every query past a document's
    end puts almost all its probability on the document's last keys, so the
    dV of those keys sums P dO over up to ~250 queries and grows large; the
    same per-element bound as above, with and without dropout."""
    c = I.make_case(f"heavy_D{D}", 2, 4, 300, 300, D, seed=201, causal=True, alibi=True,
                    kv_len_range=(50, 300))
    dev = P.to_dev(c)
    kw = P.mask_kwargs(c, dev)
    drop = dict(keep_prob=keep_prob, seed=SEED, offset=OFFSET)
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, c.layout, pse=dev["slopes"],
                      scale=c.scale, **drop, **kw)
    dq, dk, dv = fa.bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, c.N, c.layout,
                        pse=dev["slopes"], scale=c.scale, **drop, **kw)
    fa.sync_status()
    okw = P.oracle_kwargs(c)
    q, k, v, do = (P._bnsd(getattr(c, n), c) for n in ("q", "k", "v", "dout"))
    od = (keep_prob, SEED, OFFSET) if keep_prob < 1 else None
    ro, rl = oracle.fwd(q, k, v, c.scale, dropout=od, **okw)
    _close(P.gpu_heads(out, c), ro, c.dtype, keep_prob, "heavy out")
    grads = oracle.bwd(q, k, v, do, c.scale, dropout=od, **okw)
    for got, ref, what in zip((dq, dk, dv), grads, ("dq", "dk", "dv")):
        _close(P.gpu_heads(got, c), ref, c.dtype, keep_prob, f"heavy {what}")


def test_dropout_bsh_modality_and_dense_term():
    c = I.make_case("drop_bsh", 2, 4, 150, 150, 64, layout="BSH", seed=202, modality=(60, 90))
    g = torch.Generator().manual_seed(203)
    _run(c, 0.625, term=torch.randn(1, 4, 150, 150, generator=g))


def test_dropout_fp16_and_fp32_path():
    _run(I.make_case("drop_fp16", 1, 2, 140, 270, 128, seed=204, dtype=torch.float16), 0.75)
    _run(I.make_case("drop_fp32", 1, 2, 70, 90, 64, seed=205, dtype=torch.float32), 0.75)


def _mask_probe(keep_prob, S, seed, offset):
    """Q = 0 gives p = 1/S for every pair.  With V = I the forward's O_ij is
    keep_ij / (S keep_prob); with dO = I the backward's dV_ji is the same
    value: both reveal the kernels' keep mask element by element."""
    B, N, D = 1, 2, 64
    assert S == D
    q = torch.zeros(B, N, S, D, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, N, S, D, dtype=torch.bfloat16, device="cuda")
    eye = torch.eye(S, D, dtype=torch.bfloat16, device="cuda").expand(B, N, S, D).contiguous()
    drop = dict(keep_prob=keep_prob, seed=seed, offset=offset)
    out, lse = fa.fwd(q, k, eye, N, "BNSD", scale=0.125, **drop)
    dq, dk, dv = fa.bwd(q, k, eye, out, eye, lse, N, "BNSD", scale=0.125, **drop)
    fa.sync_status()
    fwd_keep = (out.float().cpu().numpy() != 0)
    bwd_keep = (dv.float().cpu().numpy().transpose(0, 1, 3, 2) != 0)
    return fwd_keep, bwd_keep


@pytest.mark.parametrize("keep_prob,offset", [(0.5, 0), (0.875, 9)])
def test_kernel_masks_equal_the_oracle_mask(keep_prob, offset):
    S = 64
    fwd_keep, bwd_keep = _mask_probe(keep_prob, S, SEED, offset)
    want = oracle.dropout_keep_mask(1, 2, S, S, keep_prob, SEED, offset).astype(bool)
    np.testing.assert_array_equal(fwd_keep, want)
    np.testing.assert_array_equal(bwd_keep, want)


def test_keep_prob_one_and_lse_unchanged():
    c = I.make_case("drop_lse", 1, 2, 256, 256, 128, seed=206, causal=True)
    dev = P.to_dev(c)
    o1, l1 = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, causal=True)
    o2, l2 = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, causal=True,
                    keep_prob=1.0, seed=SEED)
    o3, l3 = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, scale=c.scale, causal=True,
                    keep_prob=0.5, seed=SEED)
    fa.sync_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(l1, l3)            # LSE is that of P before dropout
    assert not torch.equal(o1, o3)


def test_dropout_needs_a_seed():
    c = I.make_case("drop_noseed", 1, 1, 64, 64, 64, seed=207)
    dev = P.to_dev(c)
    with pytest.raises(fa.FaError):
        fa.fwd(dev["q"], dev["k"], dev["v"], 1, scale=c.scale, keep_prob=0.9)
