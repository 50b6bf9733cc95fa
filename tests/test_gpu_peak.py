"""The dense-FP4 calibration kernel (nvfp4_fp4_peak_probe) runs in both forms,
covers the GPU with one CTA per SM, and reports a rate in the range the
hardware can have (above a quarter and below twice the vendor's nominal
dense FP4 figure of about 9 PFLOP/s)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_gemm_b200 as nv
    nv.lib()
    return nv


@pytest.mark.parametrize("pair", [False, True])
def test_fp4_peak_probe_runs_and_is_plausible(nv, pair):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    steps = 20000
    nv.fp4_peak_probe(pair, 1000)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ctas = nv.fp4_peak_probe(pair, steps)
    e1.record()
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    assert (ctas == sms) if not pair else (ctas % 2 == 0 and sms - 8 <= ctas <= sms)
    tflops = steps * ctas * nv.FP4_PEAK_FLOPS_PER_STEP / (e0.elapsed_time(e1) / 1e3) / 1e12
    assert 2250 < tflops < 18000, tflops


def test_fp4_peak_probe_rejects_bad_arguments(nv):
    with pytest.raises(nv.Nvfp4Error):
        nv.fp4_peak_probe(False, 0)
