"""The tensor-pipe rate probe (nvfp4_selftest_mma_rate): the GEMM's own
block-scaled MMA stage on resident operands, the measured FP4 peak that the
benchmark reports beside the derived one.  NVFP4 on Blackwell's tensor cores:
nerdman.de, section "Was konkret passiert ist"; the two scale formats:
aisight.pl, section "Architektura NVFP4 kontra ograniczenia mikroskalowania"."""
import pytest
import torch

pytestmark = pytest.mark.gpu

FLOP_PER_ROUND = 4 * 2 * 256 * 256 * 64  # four M256 N256 K64 MMAs of a CTA pair


@pytest.mark.parametrize("mx", [False, True], ids=["nvfp4", "mxfp4"])
def test_mma_rate_probe(mx, cuda_lib):
    B = cuda_lib
    dev = torch.device("cuda", 0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ws = B.workspace(256, dev)
    cycles = torch.zeros(sms // 2, dtype=torch.int64, device=dev)
    iters = 4000
    B.nvfp4_selftest_mma_rate(cycles, ws, 100, mx=mx)  # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    pairs = B.nvfp4_selftest_mma_rate(cycles, ws, iters, mx=mx)
    e1.record()
    B.nvfp4_check(ws)  # no timeout recorded
    assert 1 <= pairs <= sms // 2
    c = cycles[:pairs].cpu()
    assert bool((c > 0).all()) and bool((cycles[pairs:].cpu() == 0).all())
    per_round = float(c.double().median()) / iters
    tflops = pairs * iters * FLOP_PER_ROUND / (e0.elapsed_time(e1) * 1e-3) / 1e12
    # a round cannot beat the tensor pipe's documented order of magnitude (9 PFLOP/s dense FP4 per GPU)
    assert 200.0 < per_round < 20000.0, per_round
    assert 500.0 < tflops < 20000.0, tflops
    print("mma rate probe (%s): %d pairs, %.1f cycles per round, %.0f TFLOP/s" % (
        "mxfp4" if mx else "nvfp4", pairs, per_round, tflops))
