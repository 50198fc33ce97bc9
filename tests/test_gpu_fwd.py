"""Forward parity of the CUDA path (through the C ABI) against the fp64
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


def check_fwd(case, heads=None, mask_mode="modality", atten_mask=None, tile_map=None):
    out, lse = P.gpu_fwd(case, mask_mode, atten_mask, tile_map)
    ref_o, ref_l = P.oracle_fwd(case, heads, atten_mask)
    got_o = P.gpu_heads(out, case, heads)
    got_l = P.gpu_heads(lse, case, heads, is_lse=True)
    P.assert_close(got_o, ref_o, case.dtype, f"{case.name} out")
    P.assert_close(got_l, ref_l, case.dtype, f"{case.name} lse")
    # rows with no visible key: exactly zero output
    empty = np.isneginf(ref_l)
    assert np.all(got_o[empty] == 0.0)
    return out, lse


# ------------------------------------------------------------ small sweeps

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("sq,sk", [(384, 384), (300, 300), (77, 333), (1, 129), (130, 1)])
def test_bf16_no_mask(D, sq, sk):
    c = I.make_case(f"nomask_D{D}_{sq}x{sk}", 2, 3, sq, sk, D, seed=11)
    check_fwd(c)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [128, 300, 520])
def test_bf16_causal(D, S):
    c = I.make_case(f"causal_D{D}_S{S}", 2, 2, S, S, D, seed=12, causal=True)
    check_fwd(c)


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_causal_alibi(D):
    c = I.make_case(f"alibi_D{D}", 2, 4, 333, 333, D, seed=13, causal=True, alibi=True)
    check_fwd(c)


@pytest.mark.parametrize("D,sq,sk", [(64, 200, 260), (128, 700, 650), (64, 300, 900)])
def test_bf16_alibi_no_causal(D, sq, sk):
    # key tiles on both sides of the diagonal, visited from it outward
    c = I.make_case(f"alibi_nc_D{D}_{sq}x{sk}", 1, 4, sq, sk, D, seed=14, alibi=True)
    check_fwd(c)


@pytest.mark.parametrize("sk", [256, 512, 300])
def test_bf16_padding(sk):
    c = I.make_case(f"pad_{sk}", 6, 3, 32, sk, 64, seed=15, kv_len_range=(0, sk))
    c.kv_len[0] = 0          # a batch with no visible key at all
    c.kv_len[1] = sk         # and one fully visible
    check_fwd(c)


@pytest.mark.parametrize("S", [24, 320])
@pytest.mark.parametrize("mode", ["modality", "bool", "bool+tilemap"])
def test_bf16_multimodal_bsh(S, mode):
    n_text = 8 if S == 24 else 64
    c = I.make_case(f"mm_S{S}_{mode}", 4, 12, S, S, 64, layout="BSH", seed=16,
                    modality=(n_text, S - n_text))
    check_fwd(c, mask_mode=mode)


def test_bf16_cross_modal_page_rule():
    # The multimodal page's own rule: attend only the other modality, plus self.
    c = I.make_case("mm_cross", 2, 2, 200, 200, 128, seed=17, modality=(70, 130),
                    allow=I.ALLOW_CROSS_ONLY, allow_diag=True)
    check_fwd(c)
    check_fwd(c, mask_mode="bool+tilemap")


@pytest.mark.parametrize("per_head", [False, True])
def test_bf16_bool_mask_with_empty_rows(per_head):
    c = I.make_case("boolmask", 2, 3, 260, 300, 128, seed=18)
    g = torch.Generator().manual_seed(5)
    shape = (2, 3 if per_head else 1, 260, 300)
    m = (torch.rand(shape, generator=g) < 0.5)
    m[:, :, 5, :] = False            # empty rows
    m[:, :, 130:, 128:256] = False   # a fully masked tile region
    m[0, :, 0:128, 0:128] = True     # a fully visible tile
    mg = m.to(torch.uint8).cuda()
    check_fwd(c, atten_mask=mg)
    from attention_fwd_bwd_02_b200 import fa
    tm = fa.build_tile_map(mg, c.q.cuda(), c.k.cuda(), c.N, c.layout)
    check_fwd(c, atten_mask=mg, tile_map=tm)


@pytest.mark.parametrize("D", [64, 128])
def test_bool_mask_row_reads_vector_and_byte(D):
    """The forward reads a 16-byte aligned mask row 16 bytes at a time in
    full key tiles and byte by byte in the ragged last tile or when the rows
    are not aligned.  Sk = 400 (rows of 400 bytes, aligned) takes both paths;
    the same mask as a view one byte into a wider buffer (unaligned rows)
    takes the byte path everywhere and must give the same result bit for bit.
    Nonzero bytes other than 1 (2, 0x80, 0xff) mean attend as 1 does."""
    B, N, Sq, Sk = 2, 3, 200, 400
    c = I.make_case(f"boolvec_D{D}", B, N, Sq, Sk, D, seed=21)
    g = torch.Generator().manual_seed(22)
    vals = torch.tensor([0, 1, 2, 0x80, 0xFF], dtype=torch.uint8)
    m = vals[torch.randint(0, 5, (B, 1, Sq, Sk), generator=g)]
    m[:, :, 7, :] = 0                      # a row with no visible key
    m[1, :, :, 128:256] = 0                # a fully masked tile column
    aligned = m.cuda()
    wide = torch.zeros(B, 1, Sq, Sk + 16, dtype=torch.uint8, device="cuda")
    wide[..., 1:Sk + 1] = aligned
    unaligned = wide[..., 1:Sk + 1]
    assert unaligned.data_ptr() % 16 == 1 and unaligned.stride(-1) == 1
    o1, l1 = check_fwd(c, atten_mask=aligned)
    o2, l2 = P.gpu_fwd(c, atten_mask=unaligned)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp32_config1():
    c = I.config1()
    check_fwd(c)


@pytest.mark.parametrize("D", [16, 40, 128])
def test_fp32_masks(D):
    c = I.make_case(f"f32_D{D}", 2, 2, 70, 90, D, dtype=torch.float32, seed=19,
                    kv_len_range=(0, 90), alibi=True)
    check_fwd(c)
    c2 = I.make_case(f"f32c_D{D}", 1, 2, 65, 65, D, dtype=torch.float32, seed=20,
                     causal=True, modality=(20, 45))
    check_fwd(c2)


def test_empty_keys_gives_zero_and_minus_inf():
    from attention_fwd_bwd_02_b200 import fa
    q = torch.randn(1, 2, 5, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    out, lse = fa.fwd(q, k, k.clone(), 2, "BNSD", scale=0.125)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(lse == float("-inf"))


# ------------------------------------------------------------ exact rules

def test_padded_keys_poisoned_bitwise_identical():
    c = I.make_case("poison", 4, 2, 64, 300, 128, seed=21, kv_len_range=(1, 299))
    out, lse = P.gpu_fwd(c)
    for b in range(c.B):
        n = int(c.kv_len[b])
        c.k[b, :, n:] = 1e30
        c.v[b, :, n:] = -1e30
    out2, lse2 = P.gpu_fwd(c)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_tile_skipping_is_bitwise_neutral():
    c = I.make_case("skip", 2, 2, 384, 384, 64, seed=22)
    m = torch.ones(2, 1, 384, 384, dtype=torch.uint8)
    m[:, :, :, 128:256] = 0
    m[:, :, 256:, :128] = 0
    mg = m.cuda()
    from attention_fwd_bwd_02_b200 import fa
    tm = fa.build_tile_map(mg, c.q.cuda(), c.k.cuda(), c.N, c.layout)
    assert tm.view(2, 3, 3).cpu().tolist()[0] == [[2, 0, 2], [2, 0, 2], [0, 0, 2]]
    o1, l1 = P.gpu_fwd(c, atten_mask=mg)
    o2, l2 = P.gpu_fwd(c, atten_mask=mg, tile_map=tm)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_modality_mode_equals_explicit_mask():
    c = I.config3(320)
    c = I.make_case("mm_eq", 8, 12, 320, 320, 64, layout="BSH", seed=23, modality=(64, 256))
    o1, l1 = P.gpu_fwd(c, "modality")
    o2, l2 = P.gpu_fwd(c, "bool")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_modality_mask_builder_matches_rule():
    from attention_fwd_bwd_02_b200 import fa
    ids = torch.tensor([[0, 0, 1, 1, 1], [1, 0, 1, 0, 0]], dtype=torch.int32)
    m = fa.build_modality_mask(ids.cuda(), ((1, 1), (0, 1)), False).cpu()
    for b in range(2):
        for i in range(5):
            for j in range(5):
                a, c = int(ids[b, i]), int(ids[b, j])
                assert m[b, i, j] == (1 if (a, c) != (1, 0) else 0)


# ------------------------------------------------------------ full workloads

def test_config2_causal_full_size_sampled():
    c = I.config2(with_dout=False)
    heads = [(0, 0), (1, 17), (3, 31)]
    check_fwd(c, heads=heads)


@pytest.mark.parametrize("S", [24, 320])
def test_config3_multimodal_full_size(S):
    c = I.config3(S)
    heads = None if S == 24 else [(0, 0), (17, 5), (63, 11)]
    check_fwd(c, heads=heads)


@pytest.mark.parametrize("sk", [256, 512])
def test_config4_retrieval_full_size_sampled(sk):
    c = I.config4(sk)
    heads = [(b, h) for b in (0, 7, 100, 255) for h in (0, 11)]
    check_fwd(c, heads=heads)


@pytest.mark.parametrize("S,D", I.CONFIG5_SWEEP)
def test_config5_fwd_full_size_sampled(S, D):
    c = I.config5(S, D)
    heads = [(0, 0), (c.B - 1, 15)]
    check_fwd(c, heads=heads)
