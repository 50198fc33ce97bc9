"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only draws random tensors and
integer side inputs (padding lengths, modality ids, ALiBi slopes) on the CPU.
Both the CUDA path and the fp64 oracle consume what it returns, so input
rounding (fp32 -> bf16 or fp16, round-to-nearest-even, done once here) is never
counted as kernel error.

Workloads (the shapes and value distributions of the attention call sites on
the source pages; none of the pages' datasets are available, so these
synthetic N(0, 1) tensors stand in for them -- the operator's cost does not
depend on the values):

1. fp32 check: BNSD, B=1, N=2, S=128, D=64, scale 1/8, no mask.
2. causal decoder self-attention: BNSD bf16, B=4, N=32, S=2048, D=128,
   scale 1/sqrt(128), causal (the `tril` mask of the CogVLM page).
3. multimodal joint attention: BSH bf16, B=64, 12 heads, D=64 (H=768),
   8 text + 16 image = 24 tokens (multimodal page, layer 1 example) or
   64 text + 256 image = 320 tokens; modality ids 0 (text) then 1 (image);
   text attends all tokens, image attends image tokens only.
4. retrieval cross-attention: BNSD bf16, query 32 over documents of 256 (or
   512) tokens (retrieval page, layer 1 shapes), B=256, N=12, D=64, valid
   document length uniform in [64, Sk] (the doc padding mask).
5. training fwd+bwd sweep: BNSD bf16, N=16, B*S=16384, S in
   {128,512,1024,2048,4096}, D in {64,128}, causal + ALiBi slopes
   2^(-8(h+1)/N) for 0-based head h.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

ALLOW_TEXT_ALL_IMAGE_IMAGE = ((1, 1), (0, 1))   # allow[id_q][id_k]
ALLOW_CROSS_ONLY = ((0, 1), (1, 0))             # multimodal page default rule


@dataclass
class Case:
    """One synthetic attention problem (CPU tensors)."""
    name: str
    B: int
    N: int
    Sq: int
    Sk: int
    D: int
    dtype: torch.dtype
    layout: str                  # "BNSD" or "BSH"
    scale: float
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: Optional[torch.Tensor] = None
    causal: bool = False
    kv_len: Optional[torch.Tensor] = None         # int32 [B]
    modality_ids: Optional[torch.Tensor] = None   # int32 [B, S]
    allow: tuple = ALLOW_TEXT_ALL_IMAGE_IMAGE
    allow_diag: bool = False
    slopes: Optional[torch.Tensor] = None         # fp32 [N]
    extra: dict = field(default_factory=dict)

    def shape_q(self):
        return _shape(self.layout, self.B, self.N, self.Sq, self.D)

    def shape_kv(self):
        return _shape(self.layout, self.B, self.N, self.Sk, self.D)


def _shape(layout, B, N, S, D):
    if layout == "BNSD":
        return (B, N, S, D)
    if layout == "BSH":
        return (B, S, N * D)
    raise ValueError(layout)


def alibi_slopes(n_heads: int) -> torch.Tensor:
    """ALiBi slopes 2^(-8(h+1)/N), h = 0..N-1 (fp32)."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / n_heads) for h in range(n_heads)],
                        dtype=torch.float32)


def modality_ids_text_image(B: int, n_text: int, n_image: int) -> torch.Tensor:
    """ids = 0 for the n_text text tokens, then 1 for the n_image image tokens."""
    row = torch.cat([torch.zeros(n_text, dtype=torch.int32),
                     torch.ones(n_image, dtype=torch.int32)])
    return row.unsqueeze(0).repeat(B, 1).contiguous()


def make_case(name, B, N, Sq, Sk, D, *, dtype=torch.bfloat16, layout="BNSD",
              seed=0, scale=None, causal=False, kv_len_range=None,
              modality=None, allow=ALLOW_TEXT_ALL_IMAGE_IMAGE, allow_diag=False,
              alibi=False, with_dout=True, value_scale=1.0) -> Case:
    """Draw Q, K, V, dO ~ N(0, 1) fp32 (in that order) then round to ``dtype``.

    ``kv_len_range=(lo, hi)`` draws valid key lengths uniform in [lo, hi]
    after the tensors; ``modality=(n_text, n_image)`` gives text-then-image
    ids; ``alibi`` attaches the standard slope vector."""
    g = torch.Generator().manual_seed(int(seed))
    sq = _shape(layout, B, N, Sq, D)
    sk = _shape(layout, B, N, Sk, D)
    q = torch.randn(sq, generator=g, dtype=torch.float32) * value_scale
    k = torch.randn(sk, generator=g, dtype=torch.float32) * value_scale
    v = torch.randn(sk, generator=g, dtype=torch.float32)
    dout = torch.randn(sq, generator=g, dtype=torch.float32) if with_dout else None
    kv_len = None
    if kv_len_range is not None:
        lo, hi = kv_len_range
        kv_len = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int32)
    ids = None
    if modality is not None:
        n_text, n_image = modality
        assert n_text + n_image == Sq == Sk
        ids = modality_ids_text_image(B, n_text, n_image)
    if dtype not in (torch.float32, torch.bfloat16, torch.float16, torch.float8_e4m3fn):
        raise ValueError(f"unsupported dtype {dtype}")

    def cast(t):
        return t.to(dtype).contiguous()

    q, k, v = cast(q), cast(k), cast(v)
    if dout is not None:  # e4m3 is forward only; its dO (unused) stays bf16
        dout = dout.to(torch.bfloat16 if dtype == torch.float8_e4m3fn else dtype).contiguous()
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return Case(name=name, B=B, N=N, Sq=Sq, Sk=Sk, D=D, dtype=dtype,
                layout=layout, scale=float(scale), q=q, k=k, v=v, dout=dout,
                causal=causal, kv_len=kv_len, modality_ids=ids, allow=allow,
                allow_diag=allow_diag,
                slopes=alibi_slopes(N) if alibi else None)


# ---------------------------------------------------------------------------
# The five workloads at their full sizes.
# ---------------------------------------------------------------------------

def config1():
    return make_case("cfg1_fp32_B1N2S128D64", 1, 2, 128, 128, 64,
                     dtype=torch.float32, seed=1001, scale=1.0 / 8.0,
                     with_dout=True)


def config2(with_dout=True):
    return make_case("cfg2_causal_B4N32S2048D128", 4, 32, 2048, 2048, 128,
                     seed=1002, causal=True, with_dout=with_dout)


def config3(S=24):
    if S == 24:
        n_text, n_image = 8, 16
    elif S == 320:
        n_text, n_image = 64, 256
    else:
        raise ValueError(S)
    return make_case(f"cfg3_multimodal_BSH_B64N12S{S}D64", 64, 12, S, S, 64,
                     layout="BSH", seed=1003, modality=(n_text, n_image))


def config4(Sk=256):
    return make_case(f"cfg4_retrieval_B256N12Sq32Sk{Sk}D64", 256, 12, 32, Sk, 64,
                     seed=1004, kv_len_range=(64, Sk))


def config5(S, D):
    B = 16384 // S
    return make_case(f"cfg5_train_B{B}N16S{S}D{D}", B, 16, S, S, D,
                     seed=1005, causal=True, alibi=True)


CONFIG5_SWEEP = [(s, d) for s in (128, 512, 1024, 2048, 4096) for d in (64, 128)]
