"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up, reports through the workspace status word, and leaves the
CUDA context usable for the next call of the layer."""
import pytest

import seeded_inputs
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_stays_usable():
    import torch
    import lora_linear_fine_b200 as L
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert L.lora_linear_workspace_init(ws.data_ptr(), ws.numel(), stream) == 0
    assert L.lora_linear_device_status(ws.data_ptr(), stream) == (0, 0)
    # 2^16 cycles: well under a millisecond at any SM clock
    assert L.lora_linear_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 16, stream) == 0
    st, word = L.lora_linear_device_status(ws.data_ptr(), stream)
    assert st == 7 and word == 0x1, (st, word)     # LORA_ERR_DEVICE_STATUS, wait-timeout bit
    assert L.lora_linear_workspace_init(ws.data_ptr(), ws.numel(), stream) == 0
    assert L.lora_linear_device_status(ws.data_ptr(), stream) == (0, 0)
    # the same context still runs the layer correctly
    M, d_in, d_out, r = 200, 320, 264, 8
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=11)
    out = G.run_library(inp, M, d_in, d_out, r, 2.0, "identity")
    ref = G.run_oracle(inp, 2.0, "identity")
    G.assert_all_ok(G.compare_all(out, ref, "identity", r))
