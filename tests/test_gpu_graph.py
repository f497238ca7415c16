"""The library's calls inside a CUDA graph: one hot-path step (RoPE pass,
self-attention, cross-attention, CFG + Euler step, and a UniPC stop) is
captured once, replayed on refilled inputs, and must reproduce the eager
results bit for bit (the calls take only pointers, sizes and a stream, and
their host-side set-up is cached after a first eager call)."""

import numpy as np
import pytest
import torch

from gpu_common import cuda
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def test_step_graph_replay_matches_eager():
    g = wan.grid(5, 30, 52)            # 480p 17 frames: 7,800 tokens
    B, H, L, Lk = 1, 12, 7800, 512
    lens = [333]
    q0 = inputs.randn_bf16((B, L, H, 128), 71)
    k0 = inputs.randn_bf16((B, L, H, 128), 72)
    v = cuda(inputs.randn_bf16((B, L, H, 128), 73))
    kc = cuda(inputs.randn_bf16((B, Lk, H, 128), 74))
    vc = cuda(inputs.randn_bf16((B, Lk, H, 128), 75))
    n = 499200
    x0 = inputs.randn_f32((n,), 76)
    c = cuda(inputs.randn_f32((n,), 77))
    u = cuda(inputs.randn_f32((n,), 78))
    xc0, m10, m20 = (inputs.randn_f32((n,), s) for s in (79, 80, 81))
    table = wan.rope3d_table(g)
    sig = wan.fm_sigmas(40, 5.0)

    def make():
        return {"q": cuda(q0.clone()), "k": cuda(k0.clone()),
                "o": torch.empty((B, L, H, 128), dtype=torch.bfloat16,
                                 device="cuda"),
                "oc": torch.empty((B, L, H, 128), dtype=torch.bfloat16,
                                  device="cuda"),
                "x": cuda(x0.clone()), "ux": cuda(x0.clone()),
                "xc": cuda(xc0.clone()), "m1": cuda(m10.clone()),
                "m2": cuda(m20.clone())}

    def step(d):
        wan.rope3d_qk(d["q"], d["k"], g, table)
        wan.self_attn(d["q"], d["k"], v, d["o"], g)
        wan.cross_attn(d["o"], kc, vc, d["oc"], lens)
        wan.fm_step(d["x"], c, u, 4.0, sig[3], sig[4])
        wan.unipc_step(d["ux"], d["xc"], d["m1"], d["m2"], d["m2"], c, u,
                       4.0, sig, 3)

    eager = make()
    step(eager)                       # also warms every call's host set-up
    torch.cuda.synchronize()

    d = make()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step(d)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    # capture does not run the work: refill the in-place inputs and replay
    for key, src in (("q", q0), ("k", k0), ("x", x0), ("ux", x0),
                     ("xc", xc0), ("m1", m10), ("m2", m20)):
        d[key].copy_(cuda(src))
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        assert wan.device_status() == 0
        for key in ("q", "k", "o", "oc", "x", "ux", "xc", "m2"):
            assert torch.equal(d[key], eager[key]), key
        for key, src in (("q", q0), ("k", k0), ("x", x0), ("ux", x0),
                         ("xc", xc0), ("m1", m10), ("m2", m20)):
            d[key].copy_(cuda(src))
    del graph
