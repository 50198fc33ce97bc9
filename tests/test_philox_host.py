"""The kernels' dropout generator (attention_fwd_bwd_02_b200/csrc/philox.cuh),
compiled for the host with the C++ compiler, against the fp64 oracle's keep
mask: the same bits for every (b, h, i, j), so a layout mistake in the
device header shows up without a GPU.  The header is plain integer
arithmetic; the only device intrinsic it uses, __umulhi, gets a host
definition here (the high half of the 64-bit product)."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_fwd_bwd_02_b200", "csrc")

_SRC = r"""
#include <cstdint>
#include <cstdio>
#define __device__
#define __forceinline__ inline
static inline uint32_t __umulhi(uint32_t a, uint32_t b) {
  return uint32_t((uint64_t(a) * b) >> 32);
}
#include "philox.cuh"
int main() {
  unsigned long long seed, offset;
  unsigned keep_t;
  int B, N, Sq, Sk;
  if (std::scanf("%llu %llu %u %d %d %d %d", &seed, &offset, &keep_t, &B, &N, &Sq, &Sk) != 7)
    return 1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < N; ++h)
      for (int i = 0; i < Sq; ++i)
        for (int jb = 0; 8 * jb < Sk; jb += 4)  // 32 keys per call, as the forward
          std::printf("%u\n", fa::dropout_bits32(seed, offset, keep_t, jb, i,
                                                 int64_t(b) * N + h));
  return 0;
}
"""
_exe = []


def _bits(seed, offset, keep_t, B, N, Sq, Sk):
    if not _exe:
        d = tempfile.mkdtemp(prefix="philox_host_")
        src, exe = os.path.join(d, "p.cpp"), os.path.join(d, "p")
        with open(src, "w") as f:
            f.write(_SRC)
        subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-o", exe, src], check=True,
                       capture_output=True)
        _exe.append(exe)
    out = subprocess.run([_exe[0]], input=f"{seed} {offset} {keep_t} {B} {N} {Sq} {Sk}\n",
                         capture_output=True, text=True, check=True).stdout.split()
    words = np.array([int(x) for x in out], dtype=np.uint64).reshape(B, N, Sq, -1)
    j = np.arange(Sk)
    return ((words[..., j // 32] >> (j % 32).astype(np.uint64)) & 1).astype(np.uint8)


@pytest.mark.parametrize("keep_prob,seed,offset", [
    (0.9, 1234, 0),
    (0.5, 0x5EED_0123_4567_89AB, 42),
    (0.125, 2**64 - 1, 2**64 - 5),     # the block index wraps past 2^64
])
def test_device_generator_equals_the_oracle_mask(keep_prob, seed, offset):
    B, N, Sq, Sk = 2, 3, 9, 70          # Sk not a multiple of 8 or 32
    keep_t = int(np.floor(keep_prob * 65536 + 0.5))
    got = _bits(seed, offset, keep_t, B, N, Sq, Sk)
    want = oracle.dropout_keep_mask(B, N, Sq, Sk, keep_prob, seed, offset)
    np.testing.assert_array_equal(got, want)
