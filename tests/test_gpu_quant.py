"""The E4M3 quantiser's quotient path on the GPU, checked exhaustively.

The per-token (and requantisation) scale is s = amax / 448 with amax a bf16
value, and every quantised value is a bf16 too, so the pairs (v, amax) with
|v| <= amax are the whole input domain.  The library computes v / s from one
reciprocal per row and a fused-multiply-add correction; the check runs every
pair and compares the E4M3 codes with those of an IEEE fp32 division.
"""
import pytest

import mixture_experts_expert_moe_b200 as m

pytestmark = pytest.mark.gpu


def test_quant_division_exhaustive(cuda_device):
    checked, bad, first = m.run_quant_division_check()
    # sum over amax bits b = 1..0x7F7F of 2 (b + 1) pairs
    n = 0x7F7F
    assert checked == 2 * (n * (n + 1) // 2 + n)
    assert bad == 0, f"{bad} mismatches, e.g. v bits {first >> 16:#06x}, amax bits {first & 0xFFFF:#06x}"
