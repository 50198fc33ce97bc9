"""Abnormal and degenerate inputs on the GPU, after the evaluation page's
abnormal-input checks ("NPU evaluation" page, zero-valued inputs):

* outputs written through views into sentinel-filled buffers: the kernels
  write nothing outside out/lse (forward) and dq/dk/dv and the workspace
  (backward), on ragged shapes of both layouts and every mask kind;
* Q = 0: every allowed key gets the same weight, so O_i is the mean of the
  allowed V rows and LSE_i = ln(#allowed keys) -- checked against the
  oracle and against that closed form;
* constant V (the same row for every key): O_i equals that row for every
  row with a visible key, and dS = P o (dP - Delta) vanishes, so dQ = dK = 0.
Needs a B200 (sm_100a)."""
import math

import numpy as np
import pytest
import torch

from attention_fwd_bwd_02_b200 import fa
from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu

PAD = 64            # elements of margin on each side (128 B for 16-bit: keeps 16-byte alignment)
SENT16 = 0x7E5A     # 16-bit sentinel pattern
SENT32 = 0x7F51A5ED  # 32-bit sentinel pattern (a NaN: never a valid output)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def _bits_dtype(dtype):
    return torch.int16 if dtype in (torch.bfloat16, torch.float16) else torch.int32


def fenced(shape, dtype):
    """(buffer, view): `view` of `shape` sits in the middle of a buffer whose
    PAD-element margins hold a sentinel bit pattern."""
    n = math.prod(shape)
    buf = torch.empty(n + 2 * PAD, dtype=dtype, device="cuda")
    bits = buf.view(_bits_dtype(dtype))
    bits.fill_(SENT16 if bits.dtype == torch.int16 else SENT32)
    return buf, buf[PAD:PAD + n].view(shape)


def margins_intact(buf, n):
    bits = buf.view(_bits_dtype(buf.dtype))
    want = SENT16 if bits.dtype == torch.int16 else SENT32
    head, tail = bits[:PAD], bits[PAD + n:]
    return bool(torch.all(head == want)) and bool(torch.all(tail == want))


RAGGED = [
    ("nomask_77x333_D64", dict(B=2, N=3, Sq=77, Sk=333, D=64)),
    ("causal_alibi_300_D128", dict(B=1, N=2, Sq=300, Sk=300, D=128, causal=True, alibi=True)),
    ("padding_33x260_D64", dict(B=3, N=2, Sq=33, Sk=260, D=64, kv_len_range=(0, 260))),
    ("bsh_modality_130_D64", dict(B=2, N=4, Sq=130, Sk=130, D=64, layout="BSH",
                                  modality=(50, 80))),
    ("fp16_causal_129_D128", dict(B=1, N=3, Sq=129, Sk=129, D=128, causal=True,
                                  dtype=torch.float16)),
    ("fp32_ragged_70x90_D64", dict(B=1, N=2, Sq=70, Sk=90, D=64, dtype=torch.float32)),
]


def _case(name, kw, seed=71):
    kw = dict(kw)
    B, N, Sq, Sk, D = (kw.pop(x) for x in ("B", "N", "Sq", "Sk", "D"))
    return I.make_case(name, B, N, Sq, Sk, D, seed=seed, with_dout=True, **kw)


@pytest.mark.parametrize("name,kw", RAGGED, ids=[r[0] for r in RAGGED])
def test_outputs_stay_inside_their_views(name, kw):
    c = _case(name, kw)
    dev = P.to_dev(c)
    mk = P.mask_kwargs(c, dev)
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["dout"]
    ob, out = fenced(tuple(q.shape), q.dtype)
    lb, lse = fenced((c.B, c.N, c.Sq), torch.float32)
    fa.fwd(q, k, v, c.N, c.layout, pse=dev["slopes"], scale=c.scale, out=out, lse=lse, **mk)
    fa.sync_status()
    assert margins_intact(ob, out.numel()), "forward wrote outside out"
    assert margins_intact(lb, lse.numel()), "forward wrote outside lse"
    ref_o, ref_l = P.oracle_fwd(c)
    P.assert_close(P.gpu_heads(out, c), ref_o, c.dtype, f"{name} out")
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, c.dtype, f"{name} lse")

    qb, dq = fenced(tuple(q.shape), q.dtype)
    kb, dk = fenced(tuple(k.shape), k.dtype)
    vb, dv = fenced(tuple(v.shape), v.dtype)
    ws_n = fa.bwd_workspace_size(fa.make_shape(q, k, c.N, c.layout))
    wb = torch.empty(ws_n + 4096, dtype=torch.uint8, device="cuda")
    wb.fill_(0xA5)
    fa.bwd(q, k, v, out, do, lse, c.N, c.layout, pse=dev["slopes"], scale=c.scale,
           workspace=wb[:ws_n], dq=dq, dk=dk, dv=dv, **mk)
    fa.sync_status()
    for buf, t, what in ((qb, dq, "dq"), (kb, dk, "dk"), (vb, dv, "dv")):
        assert margins_intact(buf, t.numel()), f"backward wrote outside {what}"
    assert bool(torch.all(wb[ws_n:] == 0xA5)), "backward wrote past its workspace"
    # the forward's outputs are inputs here: unchanged
    assert margins_intact(ob, out.numel()) and margins_intact(lb, lse.numel())
    rq, rk, rv = P.oracle_bwd(c)
    for got, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        P.assert_close(P.gpu_heads(got, c), ref, c.dtype, f"{name} {what}")


def _zero_q(c):
    c.q = torch.zeros_like(c.q)
    return c


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_is_uniform_attention(D, causal):
    c = _zero_q(I.make_case(f"zeroq_D{D}_c{int(causal)}", 2, 3, 200, 333 if not causal else 200,
                            D, seed=72, causal=causal, with_dout=True))
    out, lse = P.gpu_fwd(c)
    ref_o, ref_l = P.oracle_fwd(c)
    got_o, got_l = P.gpu_heads(out, c), P.gpu_heads(lse, c, is_lse=True)
    P.assert_close(got_o, ref_o, c.dtype, "Q=0 out")
    P.assert_close(got_l, ref_l, c.dtype, "Q=0 lse")
    # closed form: the mean of the allowed V rows, LSE = ln(count)
    v = c.v.double().numpy()
    i = np.arange(c.Sq)
    cnt = (i + 1) if causal else np.full(c.Sq, c.Sk)
    if causal:
        mean = np.cumsum(v, axis=2) / cnt[None, None, :, None]
    else:
        mean = np.broadcast_to(v.mean(axis=2, keepdims=True), got_o.shape)
    P.assert_close(got_o, mean, c.dtype, "Q=0 out vs mean of V")
    np.testing.assert_allclose(got_l, np.broadcast_to(np.log(cnt), got_l.shape), atol=1e-5)
    dq, dk, dv = P.gpu_bwd(c, out, lse)
    rq, rk, rv = P.oracle_bwd(c)
    for got, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        P.assert_close(P.gpu_heads(got, c), ref, c.dtype, f"Q=0 {what}")


@pytest.mark.parametrize("D", [64, 128])
def test_constant_value_rows(D):
    c = I.make_case(f"constv_D{D}", 2, 2, 300, 300, D, seed=73, causal=True, alibi=True,
                    with_dout=True, kv_len_range=(0, 300))
    row = c.v[:, :, :1, :]
    c.v = row.expand_as(c.v).contiguous()
    out, lse = P.gpu_fwd(c)
    ref_o, ref_l = P.oracle_fwd(c)
    got_o = P.gpu_heads(out, c)
    P.assert_close(got_o, ref_o, c.dtype, "const V out")
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, c.dtype, "const V lse")
    # closed form: every row with a visible key equals the V row
    empty = np.isneginf(ref_l)
    want = np.broadcast_to(row.double().numpy(), got_o.shape).copy()
    want[empty] = 0.0
    P.assert_close(got_o, want, c.dtype, "const V out vs the row")
    dq, dk, dv = P.gpu_bwd(c, out, lse)
    rq, rk, rv = P.oracle_bwd(c)
    for got, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        P.assert_close(P.gpu_heads(got, c), ref, c.dtype, f"const V {what}")
    # dS = 0 up to the rounding of P and dP
    assert np.abs(P.gpu_heads(dq, c)).max() <= 2e-2
    assert np.abs(P.gpu_heads(dk, c)).max() <= 2e-2
