"""Shared helpers of the GPU parity tests: run a Case through the CUDA path
(via the C-ABI binding) and through the fp64 oracle, and compare.

Tolerances (fixed by the problem statement of this operator):
  bf16 or fp16 in/out, fp32 accumulation : max|d| <= 2e-2 and mean|d| <= 2e-3
  fp32 path                      : max|d| <= 1e-4
  rows with no visible key       : out exactly 0, lse exactly -inf
The same bounds are applied to the LSE.  For gradients of large workloads
the bound is also reported relative to the oracle's RMS (see
``grad_report``), but the absolute bound is the pass criterion.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_fwd_bwd_02_b200 import fa

BF16_MAX, BF16_MEAN = 2e-2, 2e-3
F32_MAX = 1e-4


def to_dev(case, device="cuda"):
    d = {}
    for name in ("q", "k", "v", "dout"):
        t = getattr(case, name)
        d[name] = None if t is None else t.to(device)
    d["kv_len"] = None if case.kv_len is None else case.kv_len.to(device)
    d["ids"] = None if case.modality_ids is None else case.modality_ids.to(device)
    d["slopes"] = None if case.slopes is None else case.slopes.to(device)
    return d


def mask_kwargs(case, dev, mask_mode="modality", atten_mask=None, tile_map=None):
    kw = dict(causal=case.causal, padding_kv_len=dev["kv_len"])
    if case.modality_ids is not None:
        if mask_mode == "modality":
            kw.update(modality_ids=dev["ids"], allow=case.allow, allow_diag=case.allow_diag)
        else:  # explicit bool mask built on the GPU from the ids
            m = fa.build_modality_mask(dev["ids"], case.allow, case.allow_diag)
            kw.update(atten_mask=m.unsqueeze(1))
            if mask_mode == "bool+tilemap":
                kw["tile_map"] = fa.build_tile_map(m.unsqueeze(1), dev["q"], dev["k"],
                                                   case.N, case.layout)
    if atten_mask is not None:
        kw["atten_mask"] = atten_mask
        if tile_map is not None:
            kw["tile_map"] = tile_map
    return kw


def gpu_fwd(case, mask_mode="modality", atten_mask=None, tile_map=None):
    dev = to_dev(case)
    kw = mask_kwargs(case, dev, mask_mode, atten_mask, tile_map)
    out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], case.N, case.layout, pse=dev["slopes"],
                      scale=case.scale, **kw)
    fa.sync_status()
    return out, lse


def gpu_bwd(case, out, lse, mask_mode="modality", atten_mask=None, tile_map=None):
    dev = to_dev(case)
    kw = mask_kwargs(case, dev, mask_mode, atten_mask, tile_map)
    dq, dk, dv = fa.bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, case.N,
                        case.layout, pse=dev["slopes"], scale=case.scale, **kw)
    fa.sync_status()
    return dq, dk, dv


def oracle_kwargs(case, atten_mask=None):
    kw = dict(causal=case.causal, kv_len=None if case.kv_len is None else case.kv_len.numpy(),
              slopes=None if case.slopes is None else case.slopes.double().numpy())
    if case.modality_ids is not None:
        kw.update(modality_ids=case.modality_ids.numpy(), allow=case.allow,
                  allow_diag=case.allow_diag)
    if atten_mask is not None:
        kw["mask"] = atten_mask.cpu().numpy()
    return kw


def _bnsd(x, case):
    x = x.detach().to("cpu").double()
    if case.layout == "BSH":
        B, S, H = x.shape
        x = x.reshape(B, S, case.N, H // case.N).permute(0, 2, 1, 3)
    return x.contiguous().numpy()


def oracle_fwd(case, heads=None, atten_mask=None):
    """Oracle (out, lse) in BNSD order, optionally only for (b, h) in heads."""
    q, k, v = (_bnsd(getattr(case, n), case) for n in ("q", "k", "v"))
    kw = oracle_kwargs(case, atten_mask)
    if heads is None:
        return oracle.fwd(q, k, v, case.scale, **kw)
    outs, lses = [], []
    for b, h in heads:
        kwh = _slice_kwargs(kw, case, b, h)
        o, l = oracle.fwd(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                          case.scale, **kwh)
        outs.append(o[0, 0])
        lses.append(l[0, 0])
    return np.stack(outs), np.stack(lses)


def oracle_bwd(case, heads=None, atten_mask=None):
    q, k, v, do = (_bnsd(getattr(case, n), case) for n in ("q", "k", "v", "dout"))
    kw = oracle_kwargs(case, atten_mask)
    if heads is None:
        return oracle.bwd(q, k, v, do, case.scale, **kw)
    res = [[], [], []]
    for b, h in heads:
        kwh = _slice_kwargs(kw, case, b, h)
        g = oracle.bwd(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                       do[b:b + 1, h:h + 1], case.scale, **kwh)
        for r, x in zip(res, g):
            r.append(x[0, 0])
    return tuple(np.stack(r) for r in res)


def _slice_kwargs(kw, case, b, h):
    kwh = dict(kw)
    if kw.get("kv_len") is not None:
        kwh["kv_len"] = kw["kv_len"][b:b + 1]
    if kw.get("slopes") is not None:
        kwh["slopes"] = kw["slopes"][h:h + 1]
    if kw.get("modality_ids") is not None:
        kwh["modality_ids"] = kw["modality_ids"][b:b + 1]
    if kw.get("mask") is not None:
        m = np.asarray(kw["mask"])
        m4 = np.broadcast_to(m.reshape((1,) * (4 - m.ndim) + m.shape),
                             (case.B, case.N, case.Sq, case.Sk))
        kwh["mask"] = np.ascontiguousarray(m4[b:b + 1, h:h + 1])
    return kwh


def gpu_heads(x, case, heads=None, is_lse=False):
    """GPU tensor -> numpy BNSD (optionally the listed (b, h) only); lse is
    already [B, N, Sq]."""
    a = x.detach().cpu().double().numpy() if is_lse else _bnsd(x, case)
    if heads is None:
        return a
    return np.stack([a[b, h] for b, h in heads])


def assert_close(got, ref, dtype, what, max_tol=None, mean_tol=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    ninf = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), ninf), f"{what}: -inf rows differ"
    g, r = got[~ninf], ref[~ninf]
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if g.size == 0:
        return
    d = np.abs(g - r)
    if dtype == torch.float32:
        mx = F32_MAX if max_tol is None else max_tol
        assert d.max() <= mx, f"{what}: max|d| {d.max():.3e} > {mx}"
    else:
        mx = BF16_MAX if max_tol is None else max_tol
        mn = BF16_MEAN if mean_tol is None else mean_tol
        assert d.max() <= mx and d.mean() <= mn, \
            f"{what}: max|d| {d.max():.3e} (<= {mx}), mean|d| {d.mean():.3e} (<= {mn})"


def grad_report(got, ref):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    rms = float(np.sqrt(np.mean(np.square(ref)))) or 1.0
    return dict(max=float(d.max()), mean=float(d.mean()), rel_max=float(d.max()) / rms)
