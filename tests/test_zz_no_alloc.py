"""fa_bwd_noalloc: the backward whose scratch lives in a fixed device array
inside the library, for callers that cannot call cudaMalloc (a host
framework whose memory pool already holds the device memory, or a
latency-critical loop that cannot afford cudaMalloc's implicit
synchronisation).  Checked through the C ABI against fa_bwd, which takes a
caller-allocated workspace, on two calls in a row (the second call finds the
first call's data in the shared array and must not depend on it).

This file is collected last on purpose."""
import pytest
import torch

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


@pytest.mark.parametrize("D", [64, 128])
def test_noalloc_matches_workspace_backward(D):
    # Two calls in a row on different inputs and shapes: the second call
    # finds the first call's data in the shared scratch array, and its
    # result must match fa_bwd (caller workspace) on its own inputs.
    cases = [I.make_case(f"noalloc_D{D}_a", 2, 4, 300, 300, D, seed=41, causal=True, alibi=True),
             I.make_case(f"noalloc_D{D}_b", 1, 3, 200, 200, D, seed=42, causal=True)]
    for call, c in enumerate(cases):
        dev = P.to_dev(c)
        kw = dict(pse=dev["slopes"], scale=c.scale, causal=True)
        out, lse = fa.fwd(dev["q"], dev["k"], dev["v"], c.N, "BNSD", **kw)
        ref = fa.bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, c.N, "BNSD", **kw)
        grads = tuple(torch.full_like(t, float("nan")) for t in (dev["q"], dev["k"], dev["v"]))
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        got = fa.bwd_noalloc(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, c.N,
                             "BNSD", dq=grads[0], dk=grads[1], dv=grads[2], **kw)
        fa.sync_status()
        # Nothing was allocated through the caller's allocator, even for a
        # moment (the peak stays at the level before the call).
        assert torch.cuda.max_memory_allocated() <= before, "the call allocated device memory"
        assert all(g is t for g, t in zip(got, grads))
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            P.assert_close(g.double().cpu().numpy(), r.double().cpu().numpy(), c.dtype,
                           f"call {call} {name}")


def test_noalloc_empty_shape_is_a_no_op():
    s = fa.FaShape(0, 4, 128, 128, 64, fa.FA_LAYOUT_BNSD, fa.FA_BF16)
    assert fa.lib().fa_bwd_noalloc(s, None, None, None, None, None, None, None, None,
                                   0.1, 1.0, None, None, None, None, None) == fa.FA_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # fp32 dQ accumulator alone: 1 * 64 * 2048 * 128 * 4 B = 64 MiB > 32 MiB
    s = fa.FaShape(1, 64, 2048, 2048, 128, fa.FA_LAYOUT_BNSD, fa.FA_BF16)
    assert fa.lib().fa_bwd_workspace_size(s) > fa.NOALLOC_SCRATCH_BYTES
    p = torch.empty(16, dtype=torch.uint8, device="cuda")
    ptr = fa._ptr(p)
    rc = fa.lib().fa_bwd_noalloc(s, ptr, ptr, ptr, ptr, ptr, ptr, None, None, 0.1, 1.0,
                                 None, ptr, ptr, ptr, None)
    assert rc == fa.FA_ERR_UNSUPPORTED
