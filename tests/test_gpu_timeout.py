"""Failure detection without a GPU fault: a bounded device wait that nothing
completes (a producer that issues nothing) gives up after a short limit and
comes back as MOE_Q4_ETIMEOUT in the status word; the context stays usable
and the next layer forward succeeds."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import bit_codebook_quantized_router_b200 as q4
from bit_codebook_quantized_router_b200 import _lib, inputs
from tests import gpu_support
from tests.test_gpu_forward import _small_device_layer

pytestmark = pytest.mark.gpu


def test_wait_that_nobody_completes_reports_timeout_and_the_next_call_works():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    rc = q4.lib().moe_q4_selftest_wait(_lib._ptr(status), 2000, ctypes.c_void_p(stream.cuda_stream))  # 2 ms
    assert rc == _lib.OK
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.ETIMEOUT
    # the context is intact: a layer forward right after runs and matches the oracle
    w = inputs.WORKLOADS["tiny"]
    L, dev = _small_device_layer(w)
    x, lg = inputs.activations(w), inputs.router_logits(w)
    out32 = torch.empty((w.T, w.shape.H), dtype=torch.float32, device="cuda")
    ws = q4.alloc_workspace(q4.forward_workspace(dev, w.T, w.shape.k))
    q4.forward(dev, x.cuda(), lg.cuda(), w.shape.k, ws=ws, out_f32=out32)
    assert q4.forward_status(ws) == _lib.OK
    ref = oracle.moe_tokens(L, inputs.bf16_bits(x), lg.numpy(), w.shape.k)
    gpu_support.check_out(out32, ref, "forward after a timed-out wait")


def test_selftest_rejects_bad_limits():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = q4.lib()
    assert L.moe_q4_selftest_wait(_lib._ptr(status), 0, None) == _lib.EINVAL
    assert L.moe_q4_selftest_wait(_lib._ptr(status), 3000000, None) == _lib.EINVAL
    assert L.moe_q4_selftest_wait(None, 10, None) == _lib.EINVAL
