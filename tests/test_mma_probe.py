"""The tensor-core issue-rate diagnostic (tri_attn_probe_mma): it completes
with a clean status, and its rates are physically possible — no instruction
shape may beat the dense bf16 rate of 4096 multiply-adds per cycle per SM
(2.25 PFLOP/s at 148 SMs and 1.965 GHz after rounding), and a wider N may not
take fewer cycles than a narrower one."""

import pytest

import triangle_attention_b200 as ta

pytestmark = pytest.mark.gpu

DENSE_MAC_PER_CYCLE = 4096


def test_rates_are_physical_and_monotone_in_n():
    cyc = {n: ta.probe_mma(n, 0, instructions=8192) for n in (32, 64, 128, 256)}
    for n, c in cyc.items():
        macs = 128 * n * 16
        assert macs / c <= DENSE_MAC_PER_CYCLE * 1.02, (n, c)
    assert cyc[32] <= cyc[64] * 1.02 <= cyc[128] * 1.04 <= cyc[256] * 1.06
    # the MN-major operand form of the gradient products and the tensor-memory
    # operand form of O += P V, at N = 32
    for layout in (1, 2):
        c = ta.probe_mma(32, layout, instructions=8192)
        assert 128 * 32 * 16 / c <= DENSE_MAC_PER_CYCLE * 1.02, (layout, c)
