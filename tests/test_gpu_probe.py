"""The instruction-rate probe behind the secondary bounds: it runs, leaves no
device error, and reports rates in a plausible range for a B200-class SM
(a tcgen05 M128N128K16 MMA cannot beat 8192 FLOP/clk/SM; MUFU ex2 needs at
least one cycle per warp instruction per sub-partition)."""

import pytest

from mixed_precision_attention_tm_b200 import ops

pytestmark = pytest.mark.gpu


def test_probe_rates_plausible():
    r = ops.probe_rates()
    assert ops.get_device_error() == ops.TM_OK
    assert 1.0 <= r["ex2_cycles_per_warp_instr"] <= 64.0
    assert 0.5 <= r["cvt_s32_f32_cycles_per_warp_instr"] <= 64.0
    assert 0.5 <= r["magic_conversion_cycles_per_warp_value"] <= 64.0
    # 2*128*128*16 FLOP per MMA at no more than 8192 FLOP/clk/SM -> >= 64 cycles
    assert 63.0 <= r["mma_f16_m128n128k16_cycles"] <= 1000.0
    assert 63.0 <= r["mma_i8_m128n128k32_cycles"] <= 1000.0
