"""Pins for the fp64 oracle: it is checked against things other than itself.

* a hand-derived worked example (tests/golden/hand_two_keys.json);
* closed forms: Q = 0 gives the mean of the allowed V rows and
  LSE = ln(#allowed); V constant gives that constant; causal row 0 gives V_0
  and LSE_0 = s_00; Sk = 1 gives V_0; ALiBi with Q = 0 gives a truncated
  geometric distribution (tests/golden/hand_alibi_q0.json);
* a library routine: torch's scaled_dot_product_attention in fp64 on the CPU
  (forward, and its autograd backward) for the no-pse mask modes;
* invariants: rows of P sum to 1 (and O = P when V = I), shift invariance in
  K, permutation equivariance of keys, layout equivalence BSH <-> BNSD;
* exact rules for rows with no allowed key (O = 0, LSE = -inf, zero grads).

The formula being pinned is the attention formula of the FlashAttentionScore
guide (sec. 2), in the unfused step order of its sec. 4 step 1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _val(x):
    if isinstance(x, (int, float)):
        return float(x)
    table = {"ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4),
             "-0.75ln3": -0.75 * math.log(3), "0.75ln3": 0.75 * math.log(3)}
    return table[x]


def _arr(nested):
    return np.array([[_val(x) for x in row] if isinstance(row, list) else _val(row)
                     for row in nested], dtype=np.float64)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- worked example

@pytest.mark.parametrize("variant", ["none", "causal"])
def test_hand_two_keys(variant):
    g = json.load(open(os.path.join(GOLD, "hand_two_keys.json")))
    q = _arr(g["q"]).reshape(1, 1, 2, 1)
    k = _arr(g["k"]).reshape(1, 1, 2, 1)
    v = _arr(g["v"]).reshape(1, 1, 2, 1)
    do = _arr(g["dout"]).reshape(1, 1, 2, 1)
    exp = g["expected"][variant]
    causal = variant == "causal"
    out, lse = oracle.fwd(q, k, v, g["scale"], causal=causal)
    np.testing.assert_allclose(out.reshape(-1), _arr(exp["out"]).reshape(-1), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse.reshape(-1), _arr(exp["lse"]).reshape(-1), rtol=0, atol=1e-14)
    dq, dk, dv = oracle.bwd(q, k, v, do, g["scale"], causal=causal)
    np.testing.assert_allclose(dq.reshape(-1), _arr(exp["dq"]).reshape(-1), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk.reshape(-1), _arr(exp["dk"]).reshape(-1), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv.reshape(-1), _arr(exp["dv"]).reshape(-1), rtol=0, atol=1e-14)


def test_alibi_q0_closed_form():
    g = json.load(open(os.path.join(GOLD, "hand_alibi_q0.json")))
    for c in g["cases"]:
        S, slope, causal = c["S"], c["slope"], c["causal"]
        N = 1
        q = np.zeros((1, N, S, 2))
        k = _rand((1, N, S, 2), 3)
        v = np.zeros((1, N, S, 2))
        v[0, 0, :, 0] = np.arange(S)           # v_j = j
        v[0, 0, :, 1] = 1.0
        out, lse = oracle.fwd(q, k, v, 0.7, causal=causal, slopes=np.array([slope]))
        r = math.exp(-slope)
        for i in range(S):
            if causal:
                z = (1 - r ** (i + 1)) / (1 - r)
                # E[j] under weights r^(i-j), j = 0..i: i - E[t] with t = i - j
                # E[t] over t = 0..i of t r^t / z, closed form of the finite sum
                num = r * (1 - (i + 1) * r ** i + i * r ** (i + 1)) / (1 - r) ** 2
                mean_j = i - num / z
            else:
                z = (1 - r ** (i + 1)) / (1 - r) + r * (1 - r ** (S - 1 - i)) / (1 - r)
                mean_j = None
            assert abs(lse[0, 0, i] - math.log(z)) < 1e-13
            assert abs(out[0, 0, i, 1] - 1.0) < 1e-14
            if mean_j is not None:
                assert abs(out[0, 0, i, 0] - mean_j) < 1e-12


def _expr(x):
    """A fixture value written as an exact expression: numbers, fractions,
    natural logs ln(.) and -inf."""
    if x == "-inf":
        return -math.inf
    return float(eval(x, {"__builtins__": {}}, {"ln": math.log}))


@pytest.mark.parametrize("case", ["page_rule", "workload_rule", "image_only_with_diag",
                                  "image_only_no_diag"])
def test_hand_cross_modal_diagonal(case):
    g = json.load(open(os.path.join(GOLD, "hand_cross_modal_diag.json")))
    S = g["shape"]["S"]
    vec = lambda key: np.array([_expr(x) for x in g[key]]).reshape(1, 1, S, 1)
    q, k, v, do = vec("q"), vec("k"), vec("v"), vec("dout")
    ids = np.array([g["ids"]], dtype=np.int32)
    c = g["cases"][case]
    kw = dict(modality_ids=ids, allow=tuple(map(tuple, c["allow"])), allow_diag=c["allow_diag"])
    out, lse = oracle.fwd(q, k, v, g["scale"], **kw)
    np.testing.assert_allclose(out.reshape(-1), [_expr(x) for x in c["out"]], rtol=0, atol=1e-14)
    exp_lse = np.array([_expr(x) for x in c["lse"]])
    assert np.array_equal(np.isneginf(lse.reshape(-1)), np.isneginf(exp_lse))
    fin = np.isfinite(exp_lse)
    np.testing.assert_allclose(lse.reshape(-1)[fin], exp_lse[fin], rtol=0, atol=1e-14)
    if "dq" in c:
        dq, dk, dv = oracle.bwd(q, k, v, do, g["scale"], **kw)
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(got.reshape(-1), [_expr(x) for x in c[name]],
                                       rtol=0, atol=1e-14, err_msg=name)


# ---------------------------------------------------------------- closed forms

MASK_MODES = ["none", "causal", "padding", "bool", "modality", "modality_page",
              "causal+padding"]


def _mask_kwargs(mode, B, N, Sq, Sk, seed=0):
    rng = np.random.default_rng(seed)
    kw = {}
    if "causal" in mode:
        kw["causal"] = True
    if "padding" in mode:
        kw["kv_len"] = rng.integers(1, Sk + 1, size=B).astype(np.int32)
    if mode == "bool":
        kw["mask"] = (rng.random((B, N, Sq, Sk)) < 0.6).astype(np.uint8)
    if mode == "modality":
        assert Sq == Sk
        ids = np.zeros((B, Sk), dtype=np.int32)
        ids[:, Sk // 3:] = 1
        kw["modality_ids"] = ids
        kw["allow"] = ((1, 1), (0, 1))
    if mode == "modality_page":
        # The multimodal page's own cross-modal rule (layer 2,
        # create_cross_modal_mask): a token attends the other modality and
        # itself, never another token of its own modality.
        assert Sq == Sk
        ids = np.zeros((B, Sk), dtype=np.int32)
        ids[:, Sk // 3:] = 1
        kw["modality_ids"] = ids
        kw["allow"] = ((0, 1), (1, 0))
        kw["allow_diag"] = True
    return kw


def _allowed_dense(mode, B, N, Sq, Sk, kw):
    """The allowed(i, j) table built from the mask inputs with torch ops, the
    way the pages build them (tril of ones; doc mask on the key axis; ids
    compared pairwise)."""
    a = torch.ones(B, N, Sq, Sk, dtype=torch.bool)
    if kw.get("causal"):
        a &= torch.ones(Sq, Sk, dtype=torch.bool).tril()
    if "kv_len" in kw:
        kl = torch.as_tensor(kw["kv_len"]).long()
        a &= (torch.arange(Sk)[None, :] < kl[:, None])[:, None, None, :]
    if "mask" in kw:
        a &= torch.as_tensor(kw["mask"]).bool()
    if "modality_ids" in kw:
        ids = torch.as_tensor(kw["modality_ids"]).long()
        allow = torch.as_tensor(kw["allow"]).bool()
        pair = allow[ids[:, :, None], ids[:, None, :]]   # [B, Sq, Sk]
        if kw.get("allow_diag"):
            pair |= torch.eye(Sq, Sk, dtype=torch.bool)[None]
        a &= pair[:, None]
    return a


@pytest.mark.parametrize("mode", MASK_MODES)
def test_q_zero_gives_mean_of_allowed_v(mode):
    B, N, S, D = 2, 3, 9, 5
    q = np.zeros((B, N, S, D))
    k = _rand((B, N, S, D), 1)
    v = _rand((B, N, S, D), 2)
    kw = _mask_kwargs(mode, B, N, S, S, seed=3)
    out, lse = oracle.fwd(q, k, v, 0.3, **kw)
    allowed = _allowed_dense(mode, B, N, S, S, kw).numpy()
    for b in range(B):
        for h in range(N):
            for i in range(S):
                sel = allowed[b, h, i]
                if sel.sum() == 0:
                    assert lse[b, h, i] == -np.inf
                    assert np.all(out[b, h, i] == 0.0)
                    continue
                np.testing.assert_allclose(out[b, h, i], v[b, h][sel].mean(0), atol=1e-13)
                assert abs(lse[b, h, i] - math.log(sel.sum())) < 1e-13


@pytest.mark.parametrize("mode", MASK_MODES)
def test_constant_v_gives_constant(mode):
    B, N, S, D = 2, 2, 11, 4
    q = _rand((B, N, S, D), 4) * 3
    k = _rand((B, N, S, D), 5) * 3
    c = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(c, (B, N, S, D)).copy()
    kw = _mask_kwargs(mode, B, N, S, S, seed=6)
    slopes = np.array([0.5, 0.125])
    out, lse = oracle.fwd(q, k, v, 0.4, slopes=slopes, **kw)
    allowed = _allowed_dense(mode, B, N, S, S, kw).numpy()
    nonempty = allowed.any(-1)
    np.testing.assert_allclose(out[nonempty], np.broadcast_to(c, out[nonempty].shape), atol=1e-13)
    assert np.all(out[~nonempty] == 0.0)


def test_causal_row0_and_sk1():
    B, N, S, D = 2, 3, 6, 4
    q = _rand((B, N, S, D), 7)
    k = _rand((B, N, S, D), 8)
    v = _rand((B, N, S, D), 9)
    slopes = np.array([0.5, 0.25, 0.125])
    out, lse = oracle.fwd(q, k, v, 0.5, causal=True, slopes=slopes)
    np.testing.assert_allclose(out[:, :, 0], v[:, :, 0], atol=1e-15)
    s00 = 0.5 * np.einsum("bnd,bnd->bn", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s00, atol=1e-14)
    # one key: every row returns V_0
    out1, lse1 = oracle.fwd(q, k[:, :, :1], v[:, :, :1], 0.5, slopes=slopes)
    np.testing.assert_allclose(out1, np.broadcast_to(v[:, :, :1], out1.shape), atol=1e-15)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("mode", MASK_MODES)
@pytest.mark.parametrize("sq_sk", [(13, 13), (7, 19)])
def test_matches_torch_sdpa_fwd_bwd(mode, sq_sk):
    Sq, Sk = sq_sk
    if mode.startswith("modality") and Sq != Sk:
        pytest.skip("modality rule is self-attention only")
    B, N, D = 2, 3, 8
    scale = 0.37
    q = torch.randn(B, N, Sq, D, dtype=torch.float64, generator=torch.Generator().manual_seed(10))
    k = torch.randn(B, N, Sk, D, dtype=torch.float64, generator=torch.Generator().manual_seed(11))
    v = torch.randn(B, N, Sk, D, dtype=torch.float64, generator=torch.Generator().manual_seed(12))
    do = torch.randn(B, N, Sq, D, dtype=torch.float64, generator=torch.Generator().manual_seed(13))
    kw = _mask_kwargs(mode, B, N, Sq, Sk, seed=14)
    allowed = _allowed_dense(mode, B, N, Sq, Sk, kw)
    nonempty = allowed.any(-1)
    # torch gives NaN on rows with no allowed key; give those rows a dummy key
    # for the library call and compare only the non-empty rows.
    am = allowed.clone()
    am[~nonempty] = True
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    (ref * do * nonempty[..., None]).sum().backward()
    out, lse = oracle.fwd(q, k, v, scale, **kw)
    ne = nonempty.numpy()
    np.testing.assert_allclose(out[ne], ref.detach().numpy()[ne], atol=1e-12, rtol=0)
    # LSE against torch.logsumexp of the library's masked scores
    s = (q @ k.transpose(-1, -2)) * scale
    s = s.masked_fill(~allowed, float("-inf"))
    ref_lse = torch.logsumexp(s, -1).numpy()
    np.testing.assert_allclose(lse[ne], ref_lse[ne], atol=1e-12, rtol=0)
    dq, dk, dv = oracle.bwd(q, k, v, do * nonempty[..., None], scale, **kw)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12, rtol=0)


# ---------------------------------------------------------------- invariants

def test_rows_of_p_sum_to_one_and_v_identity():
    B, N, S, D = 1, 2, 16, 16
    q = _rand((B, N, S, D), 20)
    k = _rand((B, N, S, D), 21)
    v = np.broadcast_to(np.eye(S), (B, N, S, D)).copy()   # V = I, Sk = D
    kw = dict(causal=True, slopes=np.array([0.3, 0.05]))
    out, lse = oracle.fwd(q, k, v, 0.25, **kw)
    for h in range(N):
        p, lse_p = oracle.probs(q, k, 0.25, 0, h, **kw)
        np.testing.assert_allclose(p.sum(-1), np.ones(S), atol=1e-14)
        np.testing.assert_allclose(out[0, h], p, atol=1e-15)   # O = P V = P
        np.testing.assert_allclose(lse_p, lse[0, h], atol=0)
        assert np.all(np.triu(p, 1) == 0.0)


@pytest.mark.parametrize("mode", ["none", "causal", "padding", "bool"])
def test_shift_invariance_in_k(mode):
    B, N, Sq, Sk, D = 2, 2, 10, 12, 6
    if mode == "causal":
        Sk = Sq
    q = _rand((B, N, Sq, D), 30)
    k = _rand((B, N, Sk, D), 31)
    v = _rand((B, N, Sk, D), 32)
    u = _rand((D,), 33)
    kw = _mask_kwargs(mode, B, N, Sq, Sk, seed=34)
    out, lse = oracle.fwd(q, k, v, 0.6, slopes=np.array([0.2, 0.7]), **kw)
    out2, lse2 = oracle.fwd(q, k + u, v, 0.6, slopes=np.array([0.2, 0.7]), **kw)
    finite = np.isfinite(lse)
    np.testing.assert_allclose(out2, out, atol=1e-12)
    shift = 0.6 * np.einsum("bnid,d->bni", q, u)
    np.testing.assert_allclose(lse2[finite], (lse + shift)[finite], atol=1e-12)


def test_permutation_equivariance_of_keys():
    B, N, Sq, Sk, D = 2, 2, 8, 15, 5
    q = _rand((B, N, Sq, D), 40)
    k = _rand((B, N, Sk, D), 41)
    v = _rand((B, N, Sk, D), 42)
    mask = (np.random.default_rng(43).random((B, N, Sq, Sk)) < 0.7).astype(np.uint8)
    perm = np.random.default_rng(44).permutation(Sk)
    out, lse = oracle.fwd(q, k, v, 0.5, mask=mask)
    out2, lse2 = oracle.fwd(q, k[:, :, perm], v[:, :, perm], 0.5, mask=mask[..., perm])
    np.testing.assert_allclose(out2, out, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)


def test_layout_bsh_equals_bnsd():
    B, N, S, D = 2, 3, 7, 4
    q = _rand((B, S, N * D), 50)
    k = _rand((B, S, N * D), 51)
    v = _rand((B, S, N * D), 52)
    do = _rand((B, S, N * D), 53)
    out, lse = oracle.fwd(q, k, v, 0.5, n_heads=N, layout="BSH", causal=True)
    to4 = lambda x: x.reshape(B, S, N, D).transpose(0, 2, 1, 3)
    out4, lse4 = oracle.fwd(to4(q), to4(k), to4(v), 0.5, causal=True)
    np.testing.assert_allclose(to4(out), out4, atol=0)
    np.testing.assert_allclose(lse, lse4, atol=0)
    g = oracle.bwd(q, k, v, do, 0.5, n_heads=N, layout="BSH", causal=True)
    g4 = oracle.bwd(to4(q), to4(k), to4(v), to4(do), 0.5, causal=True)
    for a, b in zip(g, g4):
        np.testing.assert_allclose(to4(a), b, atol=0)


def test_fully_masked_rows_are_exact():
    B, N, S, D = 1, 2, 6, 4
    q = _rand((B, N, S, D), 60)
    k = _rand((B, N, S, D), 61)
    v = _rand((B, N, S, D), 62)
    do = _rand((B, N, S, D), 63)
    mask = np.ones((B, N, S, S), dtype=np.uint8)
    mask[0, 0, 2, :] = 0          # row 2 of head 0 sees nothing
    mask[0, 1, :, 4] = 0          # key 4 of head 1 is never seen
    out, lse = oracle.fwd(q, k, v, 0.5, mask=mask)
    assert lse[0, 0, 2] == -np.inf and np.all(out[0, 0, 2] == 0.0)
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.5, mask=mask)
    assert np.all(dq[0, 0, 2] == 0.0)
    assert np.all(dk[0, 1, 4] == 0.0) and np.all(dv[0, 1, 4] == 0.0)


# ---------------------------------------------------------------- backward pins

def _loss(q, k, v, do, scale, kw):
    out, _ = oracle.fwd(q, k, v, scale, **kw)
    return float((out * do).sum())


@pytest.mark.parametrize("mode", ["none", "causal", "padding", "bool", "modality",
                                  "modality_page"])
@pytest.mark.parametrize("alibi", [False, True])
def test_bwd_finite_differences(mode, alibi):
    B, N, S, D = 1, 2, 5, 3
    q = _rand((B, N, S, D), 70)
    k = _rand((B, N, S, D), 71)
    v = _rand((B, N, S, D), 72)
    do = _rand((B, N, S, D), 73)
    kw = _mask_kwargs(mode, B, N, S, S, seed=74)
    if alibi:
        kw["slopes"] = np.array([0.6, 0.15])
    scale = 0.8
    dq, dk, dv = oracle.bwd(q, k, v, do, scale, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, scale, kw)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, scale, kw)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("mode", MASK_MODES)
def test_bwd_closed_form_invariants(mode):
    B, N, S, D = 2, 2, 9, 4
    q = _rand((B, N, S, D), 80)
    k = _rand((B, N, S, D), 81)
    v = _rand((B, N, S, D), 82)
    do = _rand((B, N, S, D), 83)
    kw = _mask_kwargs(mode, B, N, S, S, seed=84)
    kw["slopes"] = np.array([0.3, 0.9])
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.7, **kw)
    allowed = _allowed_dense(mode, B, N, S, S, kw).numpy()
    nonempty = allowed.any(-1)
    # sum_j dS_ij = 0 for every row  =>  sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(2), 0.0, atol=1e-12)
    # sum_j p_ij = 1 on non-empty rows  =>  sum_j dV_j = sum_{i non-empty} dO_i
    np.testing.assert_allclose(dv.sum(2), (do * nonempty[..., None]).sum(2), atol=1e-12)
    # Q = 0 and no pse: scores are all 0, so dK = scale * sum_i dS_ij Q_i = 0
    kw.pop("slopes")
    _, dk0, _ = oracle.bwd(np.zeros_like(q), k, v, do, 0.7, **kw)
    assert np.all(dk0 == 0.0)


# ---------------------------------------------------------------- dense additive term
# The general `pse` tensor and the float `atten_mask` of the FlashAttentionScore
# guide (sec. 3.2; sec. 4 step 1 adds the mask to the scaled scores before the
# softmax).  Pinned to the bool-mask path, to a shift invariance, to
# torch's scaled_dot_product_attention with a float attn_mask, to scipy's
# softmax for Q = 0, and to finite differences.

def _bias(shape, seed, scale=2.0):
    return _rand(shape, seed) * scale


@pytest.mark.parametrize("mode", ["none", "causal", "padding", "bool"])
def test_bias_of_zero_and_neginf_equals_the_bool_mask(mode):
    B, N, Sq, Sk, D = 2, 3, 7, 11, 5
    if mode == "causal":
        Sk = Sq
    q, k, v, do = (_rand(s, 90 + n) for n, s in enumerate(
        [(B, N, Sq, D), (B, N, Sk, D), (B, N, Sk, D), (B, N, Sq, D)]))
    kw = _mask_kwargs(mode, B, N, Sq, Sk, seed=95)
    rng = np.random.default_rng(96)
    keep = rng.random((B, N, Sq, Sk)) < 0.55
    keep[0, 1, 2, :] = False            # one row with no key at all
    add = np.where(keep, 0.0, -np.inf)
    base = kw.pop("mask", None)        # "bool": the additive term on top of a bool mask
    both = keep if base is None else (keep & (base != 0))
    kw2 = dict(kw) if base is None else dict(kw, mask=base)
    o1, l1 = oracle.fwd(q, k, v, 0.45, mask=both.astype(np.uint8), **kw)
    o2, l2 = oracle.fwd(q, k, v, 0.45, bias=add, **kw2)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    assert l2[0, 1, 2] == -np.inf and np.all(o2[0, 1, 2] == 0.0)
    g1 = oracle.bwd(q, k, v, do, 0.45, mask=both.astype(np.uint8), **kw)
    g2 = oracle.bwd(q, k, v, do, 0.45, bias=add, **kw2)
    for a, b in zip(g1, g2):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("shape", [(2, 3, 6, 9), (1, 3, 6, 9), (2, 1, 6, 9), (6, 9)])
def test_bias_constant_shift_moves_only_the_lse(shape):
    B, N, Sq, Sk, D = 2, 3, 6, 9, 4
    q, k, v, do = (_rand(s, 100 + n) for n, s in enumerate(
        [(B, N, Sq, D), (B, N, Sk, D), (B, N, Sk, D), (B, N, Sq, D)]))
    add = _bias(shape, 105)
    c = 3.25
    kw = dict(slopes=np.array([0.2, 0.5, 0.05]), kv_len=np.array([9, 4], dtype=np.int32))
    o1, l1 = oracle.fwd(q, k, v, 0.6, bias=add, **kw)
    o2, l2 = oracle.fwd(q, k, v, 0.6, bias=add + c, **kw)
    np.testing.assert_allclose(o2, o1, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l2, l1 + c, atol=1e-12, rtol=0)
    for a, b in zip(oracle.bwd(q, k, v, do, 0.6, bias=add, **kw),
                    oracle.bwd(q, k, v, do, 0.6, bias=add + c, **kw)):
        np.testing.assert_allclose(b, a, atol=1e-12, rtol=0)
    # and a broadcast bias equals its materialised copy
    full = np.broadcast_to(add.reshape((1,) * (4 - add.ndim) + add.shape), (B, N, Sq, Sk))
    o3, l3 = oracle.fwd(q, k, v, 0.6, bias=full.copy(), **kw)
    np.testing.assert_array_equal(o3, o1)
    np.testing.assert_array_equal(l3, l1)


@pytest.mark.parametrize("mode", ["none", "causal", "padding"])
@pytest.mark.parametrize("sq_sk", [(9, 9), (5, 14)])
def test_bias_matches_torch_sdpa_float_mask(mode, sq_sk):
    Sq, Sk = sq_sk
    if mode == "causal" and Sq != Sk:
        pytest.skip("square causal case only")
    B, N, D = 2, 2, 6
    scale = 0.41
    gen = torch.Generator().manual_seed(110)
    q, do = (torch.randn(B, N, Sq, D, dtype=torch.float64, generator=gen) for _ in range(2))
    k, v = (torch.randn(B, N, Sk, D, dtype=torch.float64, generator=gen) for _ in range(2))
    add = torch.randn(1, N, Sq, Sk, dtype=torch.float64, generator=gen) * 1.5
    kw = _mask_kwargs(mode, B, N, Sq, Sk, seed=111)
    allowed = _allowed_dense(mode, B, N, Sq, Sk, kw)
    nonempty = allowed.any(-1)
    am = add.expand(B, N, Sq, Sk).masked_fill(~allowed, float("-inf"))
    am = am.masked_fill(~nonempty[..., None], 0.0)   # torch gives NaN on empty rows
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    (ref * do * nonempty[..., None]).sum().backward()
    out, lse = oracle.fwd(q, k, v, scale, bias=add.numpy(), **kw)
    ne = nonempty.numpy()
    np.testing.assert_allclose(out[ne], ref.detach().numpy()[ne], atol=1e-12, rtol=0)
    s = (q @ k.transpose(-1, -2)) * scale + add
    ref_lse = torch.logsumexp(s.masked_fill(~allowed, float("-inf")), -1).numpy()
    np.testing.assert_allclose(lse[ne], ref_lse[ne], atol=1e-12, rtol=0)
    dq, dk, dv = oracle.bwd(q, k, v, do * nonempty[..., None], scale, bias=add.numpy(), **kw)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12, rtol=0)


def test_bias_q0_closed_form():
    from scipy.special import logsumexp, softmax
    B, N, Sq, Sk, D = 2, 2, 5, 8, 3
    q = np.zeros((B, N, Sq, D))
    k = _rand((B, N, Sk, D), 120)
    v = _rand((B, N, Sk, D), 121)
    add = _bias((B, N, Sq, Sk), 122, scale=3.0)   # not symmetric in (i, j)
    add[1, 0, 3, 5:] = -np.inf
    out, lse = oracle.fwd(q, k, v, 0.9, bias=add)
    np.testing.assert_allclose(lse, logsumexp(add, axis=-1), atol=1e-13, rtol=0)
    want = np.einsum("bnij,bnjd->bnid", softmax(add, axis=-1), v)
    np.testing.assert_allclose(out, want, atol=1e-13, rtol=0)


@pytest.mark.parametrize("mode", ["none", "causal"])
def test_bias_bwd_finite_differences(mode):
    B, N, S, D = 1, 2, 5, 3
    q, k, v, do = (_rand((B, N, S, D), 130 + n) for n in range(4))
    kw = _mask_kwargs(mode, B, N, S, S, seed=134)
    kw["bias"] = _bias((1, N, S, S), 135)
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.8, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q, "k": k, "v": v}
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, 0.8, kw)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, 0.8, kw)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------- dropout (keep_prob < 1)
# The guide's keep_prob (sec. 3.1/3.2).  The generator is Philox-4x32-10
# (Salmon et al., SC'11), pinned to the published known-answer vectors
# (tests/golden/philox4x32_10_kat.json) and to torch's header-only Philox
# engine (ATen/core/PhiloxRNGEngine.h, a library implementation of the same
# algorithm, compiled here with the host C++ compiler); the mask layout and
# the dropout arithmetic are pinned to that engine and to torch autograd.

_ENGINE_SRC = r"""
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
int main() {
  unsigned long long seed, subsequence, offset;
  while (std::scanf("%llu %llu %llu", &seed, &subsequence, &offset) == 3) {
    at::philox_engine e(seed, subsequence, offset);
    unsigned w0 = e(), w1 = e(), w2 = e(), w3 = e();
    std::printf("%u %u %u %u\n", w0, w1, w2, w3);
  }
  return 0;
}
"""
_engine_exe = []


def _torch_philox(triples):
    """First 128-bit block of torch's Philox stream for each (seed,
    subsequence, offset): Philox-4x32-10 at key (seed lo, seed hi) and
    counter (offset lo, offset hi, subsequence lo, subsequence hi)."""
    import subprocess
    import tempfile
    from torch.utils import cpp_extension
    if not _engine_exe:
        inc = cpp_extension.include_paths()[0]
        if not os.path.exists(os.path.join(inc, "ATen", "core", "PhiloxRNGEngine.h")):
            pytest.skip("torch's Philox engine header is not installed")
        d = tempfile.mkdtemp(prefix="philox_engine_")
        src, exe = os.path.join(d, "engine.cpp"), os.path.join(d, "engine")
        with open(src, "w") as f:
            f.write(_ENGINE_SRC)
        subprocess.run(["g++", "-O1", "-std=c++17", "-I", inc, "-o", exe, src], check=True,
                       capture_output=True)
        _engine_exe.append(exe)
    text = "".join(f"{s} {q} {o}\n" for s, q, o in triples)
    out = subprocess.run([_engine_exe[0]], input=text, capture_output=True, text=True,
                         check=True).stdout.split()
    return np.array([int(x) for x in out], dtype=np.uint32).reshape(-1, 4)


def test_philox_known_answer_vectors():
    with open(os.path.join(GOLD, "philox4x32_10_kat.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        words = [int(x, 16) for x in c["counter"]], [int(x, 16) for x in c["key"]]
        want = np.array([int(x, 16) for x in c["out"]], dtype=np.uint32)
        np.testing.assert_array_equal(oracle.philox4x32(*words), want)


def test_philox_matches_torch_engine():
    rng = np.random.default_rng(160)
    triples, words = [], []
    for _ in range(40):
        c = [int(x) for x in rng.integers(0, 2**32, size=4, dtype=np.uint64)]
        k = [int(x) for x in rng.integers(0, 2**32, size=2, dtype=np.uint64)]
        triples.append((k[0] | (k[1] << 32), c[2] | (c[3] << 32), c[0] | (c[1] << 32)))
        words.append((c, k))
    want = _torch_philox(triples)
    for (c, k), w in zip(words, want):
        np.testing.assert_array_equal(oracle.philox4x32(c, k), w)


@pytest.mark.parametrize("offset", [77, 2**64 - 3])
def test_dropout_mask_layout_matches_torch_philox(offset):
    """keep(b, h, i, j): 16-bit field j mod 8 of the block offset + j / 8 of
    torch's Philox stream with that seed and subsequence (b N + h) 2^32 + i;
    the second offset makes the block index wrap past 2^64."""
    B, N, Sq, Sk = 2, 3, 5, 40
    keep_prob, seed = 0.6, 0x1234_5678_9ABC_DEF0
    keep = oracle.dropout_keep_mask(B, N, Sq, Sk, keep_prob, seed, offset)
    t = math.floor(keep_prob * 65536 + 0.5)
    idx = [(b, h, i, jb) for b in range(B) for h in range(N) for i in range(Sq)
           for jb in range((Sk + 7) // 8)]
    blocks = _torch_philox([(seed, ((b * N + h) << 32) | i, (offset + jb) % 2**64)
                            for b, h, i, jb in idx])
    for (b, h, i, jb), words in zip(idx, blocks):
        for j in range(8 * jb, min(8 * jb + 8, Sk)):
            f = j % 8
            u = (int(words[f // 2]) >> (16 * (f % 2))) & 0xFFFF
            assert keep[b, h, i, j] == (u < t), (b, h, i, j)


def test_dropout_keep_rate_and_independence():
    keep = oracle.dropout_keep_mask(2, 4, 128, 256, 0.85, 99, 3).astype(np.float64)
    n = keep.size
    assert abs(keep.mean() - 0.85) < 4 * math.sqrt(0.85 * 0.15 / n)
    # neighbours along keys and along queries are uncorrelated
    for a, b in ((keep[..., 1:], keep[..., :-1]), (keep[:, :, 1:], keep[:, :, :-1])):
        c = np.corrcoef(a.ravel(), b.ravel())[0, 1]
        assert abs(c) < 0.02
    # another offset gives another mask
    other = oracle.dropout_keep_mask(2, 4, 128, 256, 0.85, 99, 4)
    assert np.mean(other != keep) > 0.2


def test_keep_prob_one_reproduces_no_dropout():
    B, N, Sq, Sk, D = 2, 2, 7, 9, 4
    q, k, v, do = (_rand(s, 170 + n) for n, s in enumerate(
        [(B, N, Sq, D), (B, N, Sk, D), (B, N, Sk, D), (B, N, Sq, D)]))
    kw = dict(causal=False, kv_len=np.array([9, 5], dtype=np.int32), slopes=np.array([0.3, 0.1]))
    o1, l1 = oracle.fwd(q, k, v, 0.5, **kw)
    o2, l2 = oracle.fwd(q, k, v, 0.5, dropout=(1.0, 5, 6), **kw)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    for a, b in zip(oracle.bwd(q, k, v, do, 0.5, **kw),
                    oracle.bwd(q, k, v, do, 0.5, dropout=(1.0, 5, 6), **kw)):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("mode", ["none", "causal", "padding"])
def test_dropout_matches_torch_autograd(mode):
    B, N, Sq, Sk, D = 2, 2, 9, 21, 5
    if mode == "causal":
        Sk = Sq
    keep_prob, seed, offset = 0.7, 2024, 11
    gen = torch.Generator().manual_seed(180)
    q, do = (torch.randn(B, N, Sq, D, dtype=torch.float64, generator=gen) for _ in range(2))
    k, v = (torch.randn(B, N, Sk, D, dtype=torch.float64, generator=gen) for _ in range(2))
    kw = _mask_kwargs(mode, B, N, Sq, Sk, seed=181)
    allowed = _allowed_dense(mode, B, N, Sq, Sk, kw)
    keep = torch.as_tensor(oracle.dropout_keep_mask(B, N, Sq, Sk, keep_prob, seed, offset)).bool()
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    s = (qt @ kt.transpose(-1, -2)) * 0.45
    p = torch.softmax(s.masked_fill(~allowed, float("-inf")), -1)
    ref = (p * keep / keep_prob) @ vt
    (ref * do).sum().backward()
    out, lse = oracle.fwd(q, k, v, 0.45, dropout=(keep_prob, seed, offset), **kw)
    np.testing.assert_allclose(out, ref.detach().numpy(), atol=1e-12, rtol=0)
    ref_lse = torch.logsumexp(s.detach().masked_fill(~allowed, float("-inf")), -1).numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.45, dropout=(keep_prob, seed, offset), **kw)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", ["causal", "bool", "modality"])
def test_all_terms_together_match_torch_autograd(mode):
    """A dense additive term, ALiBi, a mask and dropout at once: the scaled
    scores plus ALiBi plus the term are masked, softmaxed, dropped and
    rescaled, then multiply V (guide sec. 2 and sec. 4 step 1, with the
    keep_prob of sec. 3.2); LSE is that of the scores before dropout."""
    B, N, S, D = 2, 3, 11, 4
    keep_prob, seed, offset = 0.6, 77, 5
    gen = torch.Generator().manual_seed(185)
    q, k, v, do = (torch.randn(B, N, S, D, dtype=torch.float64, generator=gen) for _ in range(4))
    bias = torch.randn(B, N, S, S, dtype=torch.float64, generator=gen)
    slopes = np.array([0.5, 0.25, 0.125])
    kw = _mask_kwargs(mode, B, N, S, S, seed=186)
    allowed = _allowed_dense(mode, B, N, S, S, kw)
    keep = torch.as_tensor(oracle.dropout_keep_mask(B, N, S, S, keep_prob, seed, offset)).bool()
    i = torch.arange(S, dtype=torch.float64)
    alibi = -torch.as_tensor(slopes)[:, None, None] * (i[:, None] - i[None, :]).abs()
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    s = (qt @ kt.transpose(-1, -2)) * 0.4 + alibi + bias
    p = torch.softmax(s.masked_fill(~allowed, float("-inf")), -1)
    p = torch.nan_to_num(p, nan=0.0)   # rows with no allowed key give 0
    ref = (p * keep / keep_prob) @ vt
    (ref * do).sum().backward()
    okw = dict(kw, slopes=slopes, bias=bias.numpy(), dropout=(keep_prob, seed, offset))
    out, lse = oracle.fwd(q, k, v, 0.4, **okw)
    np.testing.assert_allclose(out, ref.detach().numpy(), atol=1e-12, rtol=0)
    ref_lse = torch.logsumexp(s.detach().masked_fill(~allowed, float("-inf")), -1).numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.4, **okw)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12, rtol=0)


def test_dropout_bwd_finite_differences():
    B, N, S, D = 1, 2, 5, 3
    q, k, v, do = (_rand((B, N, S, D), 190 + n) for n in range(4))
    kw = dict(causal=True, slopes=np.array([0.4, 0.2]), dropout=(0.6, 7, 1))
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.8, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q, "k": k, "v": v}
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, 0.8, kw)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, 0.8, kw)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-6, (name, err)
