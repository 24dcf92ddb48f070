"""bq.StepGraph: a sequence of C-ABI calls captured once and replayed gives the eager calls'
results bit for bit, on fresh inputs copied into the captured buffers (needs a B200)."""
import numpy as np
import pytest

import bq_inputs as I
from tests.parity_util import to_dev_bf16, to_dev_f32, torch_mods

pytestmark = pytest.mark.gpu


def test_step_graph_replays_the_eager_calls():
    torch, bq = torch_mods()
    la = bq.QuantLinear("bitnet", to_dev_f32(I.weights(300, 1280, seed=1)))
    lb = bq.QuantLinear("abq", to_dev_f32(I.weights(200, 1280, seed=2)), w_bits=4, a_bits=8)
    lc = bq.QuantLinear("abq", to_dev_f32(I.weights(150, 1280, seed=3)), w_bits=8, a_bits=8)
    x1 = torch.empty((1, 1280), dtype=torch.bfloat16, device="cuda")
    x40 = torch.empty((40, 1280), dtype=torch.bfloat16, device="cuda")
    ya, yb, yc = (torch.empty((m, n), device="cuda") for m, n in ((1, 300), (1, 200), (40, 150)))

    def issue():
        la.linear(x1, ya)
        lb.linear(x1, yb)
        lc.linear(x40, yc)   # 40 tokens: the act kernel, then the tensor-core GEMM

    g = bq.StepGraph(issue)
    for step in range(3):
        x1.copy_(to_dev_bf16(I.activations(1, 1280, seed=10 + step)))
        x40.copy_(to_dev_bf16(I.activations(40, 1280, seed=20 + step)))
        g.replay()
        torch.cuda.synchronize()
        got = [y.cpu().numpy().copy() for y in (ya, yb, yc)]
        issue()
        torch.cuda.synchronize()
        bq.bq_device_check()
        for a, b in zip(got, (ya, yb, yc)):
            assert np.array_equal(a, b.cpu().numpy())
