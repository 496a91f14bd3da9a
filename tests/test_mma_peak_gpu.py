"""The tensor-core throughput loop (mxattn_mxf4_mma_loop): the block-scaled
FP4 MMA shape of the attention kernel, issued back to back on shared-memory
operands, finishes without a timeout, its time grows with the work, and its
rate per SM clock (from the cycles each CTA records) lies just under the
tensor core's 32,768 dense FP4 flop per clock per SM."""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_quantization_b200 import mxattn as mx

pytestmark = pytest.mark.gpu


def _time(ctas, iters, cycles=None):
    mx.mxattn_mxf4_mma_loop(ctas, iters, cycles=cycles)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    st = mx.mxattn_mxf4_mma_loop(ctas, iters, cycles=cycles)
    e1.record()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return e0.elapsed_time(e1)


def test_mma_loop_completes_scales_and_rate_per_clock():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    t1 = _time(sms, 2000)
    t2 = _time(sms, 8000, cycles)
    assert 2.5 < t2 / t1 < 5.0, (t1, t2)
    c = cycles.cpu().numpy().astype(np.float64)
    assert np.all(c > 0)
    per_clk = 8000 * mx.MXF4_LOOP_FLOP_PER_ITER / c
    tflops = sms * 8000 * mx.MXF4_LOOP_FLOP_PER_ITER / (t2 / 1e3) / 1e12
    print(f"[mxf4 loop] {sms} CTAs x 8000 iterations: {t2:.3f} ms, {tflops:.0f} TFLOP/s wall; "
          f"{np.median(per_clk):.0f} flop per clock per SM (min {per_clk.min():.0f}, max {per_clk.max():.0f})")
    assert 0.8 * 32768 < np.median(per_clk) < 1.02 * 32768, np.median(per_clk)


@pytest.mark.parametrize("ctas", [1, 7, 296])
def test_mma_loop_other_grids(ctas):
    assert _time(ctas, 500) > 0
