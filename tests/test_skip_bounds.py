"""The numerical facts block skipping rests on, checked on the CPU against the constants
the library is built with (read from its source).

Tensor cores: sweep 2 stores r as fp16(r 2^15).  A (tile, block) pair may be left out
only if every one of its r rounds to exactly 0 there, i.e. every log-density is at least
kSkipCut nats below log Z, with room for the two sweeps' rounding differences.
CUDA cores: the statistics keep fp32 r down to expf's underflow.  The cut kSimtSkipCut
must leave out only responsibilities that are negligible even summed over 10^9 points.
"""
import math
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "ivf_quantizer_b200", "csrc", "fgmm_internal.h")


def _const(name):
    text = open(SRC).read()
    m = re.search(r"constexpr float %s = ([0-9.]+)f;" % name, text)
    assert m, name
    return float(m.group(1))


def _fp16_scaled(r):
    """fp16(r 2^15), the value sweep 2 feeds its second GEMM and N_k."""
    return np.float16(np.float32(r) * np.float32(2.0 ** 15))


def test_fp16_zero_threshold():
    # r = 2^-40: r 2^15 = 2^-25, half the smallest fp16 subnormal: rounds (to even) to 0
    assert _fp16_scaled(2.0 ** -40) == 0
    assert _fp16_scaled(2.0 ** -40 * 0.99) == 0
    # just above it the product survives, so the bound is tight
    assert _fp16_scaled(2.0 ** -40 * 1.01) > 0
    assert abs(40 * math.log(2) - 27.7259) < 1e-4


def test_tensor_cut_leaves_out_only_zeros():
    cut = _const("kSkipCut")
    bound = 40 * math.log(2)               # log-density gap at which fp16(r 2^15) is 0
    assert cut > bound + 2.0, (cut, bound)  # > 2 nats of margin for the sweeps' rounding
    assert _fp16_scaled(math.exp(-cut)) == 0
    # the side path's own cut (stiff components) keeps far more than the tensor sweep
    assert _const("kSideCut") >= cut


def test_simt_cut_is_negligible():
    cut = _const("kSimtSkipCut")
    r = math.exp(-cut)
    assert r < 2e-22
    assert 1e9 * r < 1e-12                 # a whole component over 10^9 points
    # and it is not vacuous: expf keeps values well below it (fp32 subnormals)
    assert np.float32(np.exp(np.float32(-cut))) > 0
    assert np.float32(np.exp(np.float64(-104.0))) == 0
