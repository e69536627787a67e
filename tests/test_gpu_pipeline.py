"""HostPipeline: steps fed from pinned host memory with the copies on their
own streams give, batch by batch, exactly the outputs of the same steps run
one at a time (same kernels, same inputs: bit-identical)."""
import pytest
import torch

from fp8_fine_grained_x1_b200 import linear, synth
from fp8_fine_grained_x1_b200.pipeline import HostPipeline

from gpu_util import dev


def test_pipeline_needs_two_step_copies():
    with pytest.raises(ValueError):
        HostPipeline([object()])


@pytest.mark.gpu
@pytest.mark.parametrize("depth", [2, 3])
def test_pipeline_matches_serial_steps(depth):
    d = dev()
    M, N, K = 256, 384, 512
    w = synth.normal((N, K), 0.02, 7).to(torch.bfloat16)
    xs = [synth.activations(M, K, seed=10 + i, outlier_seed=20 + i).to(torch.bfloat16)
          for i in range(7)]
    steps = [linear.FpropStep(torch.empty_like(xs[0], device=d), torch.empty_like(w, device=d))
             for _ in range(depth)]
    pipe = HostPipeline(steps, d)
    w_pin = w.pin_memory()
    outs = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in xs]
    torch.cuda.synchronize()
    pipe.run([([x.pin_memory(), w_pin], o) for x, o in zip(xs, outs)])
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        ref = linear.FpropStep(x.to(d), w.to(d))().cpu()
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
