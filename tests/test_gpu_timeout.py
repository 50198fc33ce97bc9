"""Failure handling on the GPU without a fault: every mbarrier wait of the
kernels is bounded (about one second); on expiry the kernel winds down,
releases its tensor memory and sets the library's device status word.

The test-only entry fa_testing_fwd_withhold_q (include/fa_testing.h) runs the
forward with its query tiles never delivered, so the waits on them expire.
The test checks that the status comes back as FA_ERR_TIMEOUT, that reading
it clears it, and that the same context then computes a correct forward."""
import time

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


def test_withheld_query_times_out_and_context_survives():
    # One work item (S = 256 = one CTA): the launch lasts about one second.
    c = I.make_case("timeout", 1, 1, 256, 256, 128, seed=77, causal=True)
    dev = P.to_dev(c)
    fa.sync_status()  # nothing pending before the test
    t0 = time.perf_counter()
    fa.testing_fwd_withhold_q(dev["q"], dev["k"], dev["v"], c.N, "BNSD", scale=c.scale,
                              causal=True)
    with pytest.raises(fa.FaError) as ei:
        fa.sync_status()
    waited = time.perf_counter() - t0
    assert ei.value.status == fa.FA_ERR_TIMEOUT
    assert 0.5 < waited < 30.0, waited
    fa.sync_status()  # the word was cleared by the previous read
    # The context is intact: a normal forward on the same stream is correct.
    out, lse = P.gpu_fwd(c)
    ref_o, ref_l = P.oracle_fwd(c)
    P.assert_close(P.gpu_heads(out, c), ref_o, c.dtype, "out after timeout")
    P.assert_close(P.gpu_heads(lse, c, is_lse=True), ref_l, c.dtype, "lse after timeout")
