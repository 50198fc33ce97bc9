"""fp16 operands (Q, K, V, dO and the outputs in fp16; LSE fp32): forward and
backward parity of the CUDA path against the fp64 oracle on the same seeded
inputs, with the bounds of the 16-bit path.  The tensor-core kernels are the
bf16 ones with fp16 operand types (tcgen05 kind::f16 takes either).  Needs a
B200 (sm_100a)."""
import numpy as np
import pytest
import torch

from attention_fwd_bwd_02_b200 import fa
from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu
F16 = torch.float16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def check_fwd(case, mask_mode="modality"):
    out, lse = P.gpu_fwd(case, mask_mode)
    assert out.dtype == F16 and lse.dtype == torch.float32
    ref_o, ref_l = P.oracle_fwd(case)
    got_o = P.gpu_heads(out, case)
    P.assert_close(got_o, ref_o, case.dtype, f"{case.name} out")
    P.assert_close(P.gpu_heads(lse, case, is_lse=True), ref_l, case.dtype, f"{case.name} lse")
    assert np.all(got_o[np.isneginf(ref_l)] == 0.0)
    return out, lse


def check_bwd(case, mask_mode="modality"):
    out, lse = P.gpu_fwd(case, mask_mode)
    grads = P.gpu_bwd(case, out, lse, mask_mode)
    ref = P.oracle_bwd(case)
    for name, got, r in zip(("dq", "dk", "dv"), grads, ref):
        assert got.dtype == F16
        P.assert_close(P.gpu_heads(got, case), r, case.dtype, f"{case.name} {name}")
    return grads


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("sq,sk", [(300, 300), (77, 333), (1, 129)])
def test_f16_fwd_no_mask(D, sq, sk):
    check_fwd(I.make_case(f"f16_nomask_D{D}_{sq}x{sk}", 2, 3, sq, sk, D, dtype=F16, seed=61))


@pytest.mark.parametrize("D", [64, 128])
def test_f16_fwd_causal_alibi(D):
    check_fwd(I.make_case(f"f16_ca_D{D}", 2, 4, 333, 333, D, dtype=F16, seed=62, causal=True,
                          alibi=True))


def test_f16_fwd_padding_and_bsh_masks():
    c = I.make_case("f16_pad", 3, 2, 40, 300, 128, dtype=F16, seed=63, kv_len_range=(0, 300))
    c.kv_len[0] = 0
    check_fwd(c)
    m = I.make_case("f16_mm", 2, 12, 320, 320, 64, dtype=F16, layout="BSH", seed=64,
                    modality=(64, 256))
    check_fwd(m, mask_mode="bool+tilemap")


def test_f16_fwd_causal_full_size_sampled():
    # the causal decoder workload's shape (B=4, N=32, S=2048, D=128) in fp16;
    # the oracle checks a sample of heads
    c = I.make_case("f16_config2", 4, 32, 2048, 2048, 128, dtype=F16, seed=65, causal=True)
    out, lse = P.gpu_fwd(c)
    heads = [(0, 0), (1, 7), (3, 31)]
    ref_o, ref_l = P.oracle_fwd(c, heads)
    P.assert_close(P.gpu_heads(out, c, heads), ref_o, c.dtype, "f16 config2 out")
    P.assert_close(P.gpu_heads(lse, c, heads, is_lse=True), ref_l, c.dtype, "f16 config2 lse")


@pytest.mark.parametrize("D", [64, 128])
def test_f16_bwd_no_mask_and_causal_alibi(D):
    check_bwd(I.make_case(f"f16_bwd_D{D}", 2, 2, 200, 300, D, dtype=F16, seed=66))
    check_bwd(I.make_case(f"f16_bwd_ca_D{D}", 2, 3, 300, 300, D, dtype=F16, seed=67,
                          causal=True, alibi=True))


def test_f16_bwd_padding_and_bsh_modality():
    c = I.make_case("f16_bwd_pad", 4, 2, 32, 300, 64, dtype=F16, seed=68, kv_len_range=(0, 300))
    c.kv_len[0] = 0
    dq, dk, dv = check_bwd(c)
    assert torch.all(dq[0] == 0) and torch.all(dk[0] == 0) and torch.all(dv[0] == 0)
    m = I.make_case("f16_bwd_mm", 2, 12, 320, 320, 64, dtype=F16, layout="BSH", seed=69,
                    modality=(64, 256))
    check_bwd(m)


def test_mixed_dtypes_rejected():
    q = torch.zeros(1, 1, 8, 64, dtype=F16, device="cuda")
    k = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fwd(q, k, k, 1, "BNSD", scale=0.125)
