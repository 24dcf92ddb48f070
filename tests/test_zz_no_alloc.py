"""bq_linear_static_scratch (fixed library scratch instead of a caller workspace) against
bq_linear, through the C ABI, on two calls in a row (needs a B200). Collected last."""
import numpy as np
import pytest

import bq_inputs as I
from tests.parity_util import RTOL, assert_y_close, to_dev_bf16, to_dev_f32, torch_mods

pytestmark = pytest.mark.gpu


def _layer(fmt, N, K, rank=32, seed=0):
    torch, bq = torch_mods()
    inp = I.layer_inputs(fmt, N, K, 1, seed, rank)
    kw = {}
    if fmt == "ternary":
        kw.update(lora_rank=rank, lora_alpha=0.1, lora_A=to_dev_f32(inp["lora_A"]), lora_B=to_dev_f32(inp["lora_B"]))
    if fmt == "abq":  # W8A8; the scratch holds the act buffer (with its tensor-core section at 16..64 tokens)
        kw.update(w_bits=8, a_bits=8)
    return bq.QuantLinear(fmt, to_dev_f32(inp["W"]), **kw)


@pytest.mark.parametrize("fmt,N,K,M,rank", [("ternary", 2048, 2048, 4, 32), ("ternary", 300, 1280, 16, 64),
                                            ("bitnet", 4096, 4096, 1, 0), ("abq", 300, 4096, 8, 0),
                                            ("abq", 4096, 4096, 64, 0), ("abq", 200, 1280, 17, 0),
                                            ("bvsr", 512, 1280, 16, 0), ("bvsr", 300, 5120, 64, 0)])
def test_static_scratch_matches_workspace_call(fmt, N, K, M, rank):
    torch, bq = torch_mods()
    ql = _layer(fmt, N, K, rank)
    for call in range(2):  # the same scratch array serves consecutive calls
        x = to_dev_bf16(I.activations(M, K, seed=100 + call))
        y_ref = torch.full((M, N), float("nan"), device="cuda")
        acc_ref = torch.zeros((M, N), dtype=torch.int64, device="cuda")
        ql.linear(x, y_ref, acc_ref)
        y = torch.full((M, N), float("nan"), device="cuda")
        acc = torch.zeros((M, N), dtype=torch.int64, device="cuda")
        bq.bq_linear_static_scratch(ql.layer, x, M, y, acc)
        torch.cuda.synchronize()
        bq.bq_device_check()
        y_h, y_ref_h = y.cpu().numpy(), y_ref.cpu().numpy()
        assert np.array_equal(acc.cpu().numpy(), acc_ref.cpu().numpy())
        assert_y_close(y_h, y_ref_h, f"{fmt} call {call}")
        assert RTOL == 1e-3


def test_static_scratch_rejects_oversize():
    torch, bq = torch_mods()
    K = 16512                      # K_pad / 256 = 65 tiles: 65 * 64 * 64 * 4 > 1 MiB
    ql = _layer("ternary", 16, K, rank=64)
    assert bq.bq_linear_workspace_bytes(ql.layer, 64) > bq.BQ_STATIC_SCRATCH_BYTES
    x = torch.zeros((64, K), dtype=torch.bfloat16, device="cuda")
    y = torch.full((64, 16), 7.0, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_linear_static_scratch(ql.layer, x, 64, y)
    assert e.value.status == bq.BQ_ERR_SIZE
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    # at the limit it runs
    assert bq.bq_linear_workspace_bytes(ql.layer, 63) <= bq.BQ_STATIC_SCRATCH_BYTES
    bq.bq_linear_static_scratch(ql.layer, x[:63], 63, y[:63])
    torch.cuda.synchronize()
    bq.bq_device_check()
