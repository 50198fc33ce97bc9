"""Backward parity of the CUDA path (through the C ABI) against the fp64
oracle on the same seeded inputs.  Needs a B200 (sm_100a)."""
import numpy as np
import pytest
import torch

from attention_fwd_bwd_02_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_fwd_bwd_02_b200 import build
    build.build()


def check_bwd(case, heads=None, mask_mode="modality", atten_mask=None, tile_map=None,
              max_tol=None, mean_tol=None):
    out, lse = P.gpu_fwd(case, mask_mode, atten_mask, tile_map)
    dq, dk, dv = P.gpu_bwd(case, out, lse, mask_mode, atten_mask, tile_map)
    ref = P.oracle_bwd(case, heads, atten_mask)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = P.gpu_heads(got, case, heads)
        P.assert_close(g, r, case.dtype, f"{case.name} {name}", max_tol, mean_tol)
    return dq, dk, dv


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("sq,sk", [(256, 256), (200, 300), (64, 130), (1, 70)])
def test_bf16_no_mask(D, sq, sk):
    c = I.make_case(f"bwd_D{D}_{sq}x{sk}", 2, 2, sq, sk, D, seed=31)
    check_bwd(c)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [128, 300])
def test_bf16_causal_alibi(D, S):
    c = I.make_case(f"bwd_ca_D{D}_S{S}", 2, 3, S, S, D, seed=32, causal=True, alibi=True)
    check_bwd(c)


@pytest.mark.parametrize("D,sq,sk", [(64, 200, 130), (128, 300, 420)])
def test_bf16_alibi_no_causal(D, sq, sk):
    # |i - j| changes sign inside the diagonal tiles: per-element bias there
    c = I.make_case(f"bwd_anc_D{D}_{sq}x{sk}", 1, 3, sq, sk, D, seed=39, alibi=True)
    check_bwd(c)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [128, 300])
def test_bf16_causal_no_alibi(D, S):
    # The causal rule alone: full tiles take the unmasked branch of the
    # softmax, the diagonal tiles the masked one, with no bias term.
    c = I.make_case(f"bwd_c_D{D}_S{S}", 2, 3, S, S, D, seed=38, causal=True)
    check_bwd(c)


def test_bf16_padding_with_empty_batch():
    c = I.make_case("bwd_pad", 4, 2, 32, 300, 64, seed=33, kv_len_range=(0, 300))
    c.kv_len[0] = 0
    dq, dk, dv = check_bwd(c)
    assert torch.all(dq[0] == 0) and torch.all(dk[0] == 0) and torch.all(dv[0] == 0)
    for b in range(c.B):   # keys nobody attends get exactly zero gradients
        n = int(c.kv_len[b])
        assert torch.all(dk[b, :, n:] == 0) and torch.all(dv[b, :, n:] == 0)


@pytest.mark.parametrize("mode", ["modality", "bool", "bool+tilemap"])
def test_bf16_multimodal_bsh(mode):
    c = I.make_case(f"bwd_mm_{mode}", 2, 12, 320, 320, 64, layout="BSH", seed=34,
                    modality=(64, 256))
    check_bwd(c, mask_mode=mode)


def test_bf16_bool_mask_empty_rows():
    c = I.make_case("bwd_bool", 2, 2, 200, 260, 128, seed=35)
    g = torch.Generator().manual_seed(6)
    m = (torch.rand(2, 2, 200, 260, generator=g) < 0.4)
    m[:, :, 7, :] = False
    mg = m.to(torch.uint8).cuda()
    dq, dk, dv = check_bwd(c, atten_mask=mg)
    assert torch.all(dq[:, :, 7] == 0)


@pytest.mark.parametrize("D", [16, 64, 100])
def test_fp32_path(D):
    c = I.make_case(f"bwd_f32_D{D}", 2, 2, 50, 70, D, dtype=torch.float32, seed=36,
                    kv_len_range=(1, 70), alibi=True)
    check_bwd(c)
    c2 = I.make_case(f"bwd_f32c_D{D}", 1, 2, 60, 60, D, dtype=torch.float32, seed=37,
                     causal=True, modality=(20, 40))
    check_bwd(c2)


def test_fp32_config1_bwd():
    check_bwd(I.config1())


def test_empty_query_and_key_sets():
    from attention_fwd_bwd_02_b200 import fa
    q = torch.randn(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(1, 2, 9, 64, dtype=torch.bfloat16, device="cuda")
    out, lse = fa.fwd(q, k, k, 2, "BNSD", scale=0.125)
    dq, dk, dv = fa.bwd(q, k, k, out, q, lse, 2, "BNSD", scale=0.125)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)
    q2 = torch.randn(1, 2, 5, 64, dtype=torch.bfloat16, device="cuda")
    k2 = torch.randn(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    out, lse = fa.fwd(q2, k2, k2, 2, "BNSD", scale=0.125)
    dq, dk, dv = fa.bwd(q2, k2, k2, out, q2, lse, 2, "BNSD", scale=0.125)
    torch.cuda.synchronize()
    assert torch.all(dq == 0)


# ------------------------------------------------------------ full workloads

def test_config2_causal_bwd_full_size_sampled():
    # The causal B=4 N=32 S=2048 D=128 workload, no bias, exactly as timed.
    c = I.config2(with_dout=True)
    heads = [(0, 0), (1, 17), (3, 31)]
    check_bwd(c, heads=heads)


@pytest.mark.parametrize("S,D", I.CONFIG5_SWEEP)
def test_config5_fwd_bwd_full_size_sampled(S, D):
    c = I.config5(S, D)
    heads = [(0, 0), (c.B - 1, 15)]
    check_bwd(c, heads=heads)
