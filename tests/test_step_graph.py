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


def test_step_graph_with_readbacks_forked_onto_a_copy_stream():
    """The pattern of the bench's end-to-end step: each call's output is read back to pinned
    host memory on a copy stream as soon as the call is done, inside the captured step, and
    the copy stream joins before the step ends. Every replay's host copies equal the eager
    results of the same inputs."""
    torch, bq = torch_mods()
    layers = [bq.QuantLinear("bitnet", to_dev_f32(I.weights(n, 1280, seed=5 + i))) for i, n in enumerate((300, 200, 150))]
    x = torch.empty((1, 1280), dtype=torch.bfloat16, device="cuda")
    ys = [torch.empty((1, L.N), device="cuda") for L in layers]
    hs = [torch.empty((1, L.N)).pin_memory() for L in layers]
    copy_stream = torch.cuda.Stream()

    def issue():
        for L, y, h in zip(layers, ys, hs):
            L.linear(x, y)
            done = torch.cuda.Event()
            done.record()
            copy_stream.wait_event(done)
            with torch.cuda.stream(copy_stream):
                h.copy_(y, non_blocking=True)
        torch.cuda.current_stream().wait_stream(copy_stream)

    g = bq.StepGraph(issue)
    for step in range(3):
        x.copy_(to_dev_bf16(I.activations(1, 1280, seed=30 + step)))
        g.replay()
        torch.cuda.synchronize()
        got = [h.numpy().copy() for h in hs]
        for L, y in zip(layers, ys):
            L.linear(x, y)
        torch.cuda.synchronize()
        bq.bq_device_check()
        for a, y in zip(got, ys):
            assert np.array_equal(a, y.cpu().numpy())
