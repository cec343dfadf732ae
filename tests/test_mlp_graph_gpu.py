"""The MLP block step captured in a CUDA graph (mlp.MlpStep.capture) replays the
same kernels: bit-identical outputs to the eager step on the same inputs, and a
replay after new inputs are copied into the step's buffers matches an eager
step on those inputs (the MLP block: hyper.ai, "NVIDIA revolutioniert
KI-Praetrainingsgeschwindigkeit mit 4-Bit-Genauigkeit")."""
import pytest
import torch

from nvfp4_bit_precision_quantize_b200 import workloads as W
from nvfp4_bit_precision_quantize_b200.mlp import MlpStep

pytestmark = pytest.mark.gpu

OUT = ("Y1", "h", "Y2", "dY1", "dX", "dW1", "dW2")


def _inputs(dev, data_seed):
    w = W.mlp(seed=5, M=512, H=256, F=768, data_seed=data_seed)
    return {k: W.bits_to_torch_bf16(v).to(dev) for k, v in w.items()}


def test_graph_replay_matches_eager(cuda_lib):
    dev = torch.device("cuda", 0)
    a, b = _inputs(dev, 1), _inputs(dev, 2)
    st = MlpStep({k: v.clone() for k, v in a.items()})
    g = st.capture()
    g.replay()
    torch.cuda.synchronize()
    got_a = {k: getattr(st, k).clone() for k in OUT}
    st.d["X"].copy_(b["X"])
    st.d["dY2"].copy_(b["dY2"])
    g.replay()
    torch.cuda.synchronize()
    got_b = {k: getattr(st, k).clone() for k in OUT}
    for inputs, got in ((a, got_a), (b, got_b)):
        ref = MlpStep(inputs)
        ref.step()
        torch.cuda.synchronize()
        for k in OUT:
            assert torch.equal(getattr(ref, k), got[k]), k
    assert not torch.equal(got_a["Y2"], got_b["Y2"])
