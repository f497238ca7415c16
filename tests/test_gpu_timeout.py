"""The bounded in-kernel wait on the GPU: a wait on a barrier that nothing
completes runs out after its limit, records WAN_ETIMEOUT in the device
status word, returns, and leaves the context usable for the next call."""

import math
import time

import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, cuda, f64
from oracle import attention as oattn
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def test_completed_wait_leaves_status_clear():
    wan.device_status(clear=True)
    wan.wait_selftest(1)
    torch.cuda.synchronize()
    assert wan.device_status() == 0


def test_wait_runs_out_and_context_survives():
    wan.device_status(clear=True)
    t0 = time.monotonic()
    wan.wait_selftest(0)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert 1.5 <= elapsed <= 20.0, elapsed
    assert wan.device_status(clear=True) == wan.WAN_ETIMEOUT
    assert wan.device_status() == 0
    # the context still runs the attention kernel correctly
    g = wan.grid(2, 4, 4)
    q, k, v = (inputs.randn_bf16((1, 32, 2, 128), inputs.seed_for(0, r))
               for r in ("q", "k", "v"))
    o = torch.empty((1, 32, 2, 128), dtype=torch.bfloat16, device="cuda")
    wan.self_attn(cuda(q), cuda(k), cuda(v), o, g)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    want = oattn.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128))
    assert_attn_close(f64(o), want, "after timeout")


def test_rejects_bad_argument():
    with pytest.raises(wan.WanError):
        wan.wait_selftest(2)
