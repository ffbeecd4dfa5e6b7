"""deco_moe_forward_static: the forward pass for callers that cannot allocate.

Some hosts cannot hand the library a device workspace while they run layers:
their memory budget is fixed and handed out before they start, or they call
the layer from inside another runtime that owns every allocation, where a
cudaMalloc would fail or stall the device.  For them the library offers an
entry point that uses a scratch array compiled into the library instead of a
workspace.  These tests call it through the C ABI and check that it gives the
same output as the workspace entry point, on two calls in a row (the second
call reuses the scratch the first one left behind), and that shapes needing
more scratch than it has are refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_util import case, to_gpu


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["edge_decode_t16", "large_t16", "tiny_f32"])
def test_static_scratch_forward_matches_workspace_forward(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    xs = [G["x"], torch.flip(G["x"], dims=[0]).contiguous()]      # two different batches
    for x in xs:                                                  # two calls in a row
        ref = lib.forward(x, G, eps=shape.eps)
        sh = lib.layer_shape(x, G, shape.eps)
        w = lib._weights(G)
        out = torch.empty_like(x)
        rc = lib._lib.deco_moe_forward_static(ctypes.byref(sh), x.data_ptr(), ctypes.byref(w),
                                              out.data_ptr(), lib._stream(None))
        assert rc == 0, lib._lib.deco_status_string(rc)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the same bits
        assert torch.equal(out, ref), name
        assert lib.static_device_error() == 0


def test_static_scratch_rejects_shapes_that_do_not_fit(lib):
    # rejected on the host, before any device call
    sh = lib.make_shape(4096, 2048, 64, 256, 1024, lib.DECO_BF16)
    need = lib.workspace_size(sh)
    assert need > lib.STATIC_SCRATCH_BYTES
    w = lib.Weights(*[0x10000 + 0x1000 * i for i in range(8)])
    rc = lib._lib.deco_moe_forward_static(ctypes.byref(sh), 0x100000, ctypes.byref(w), 0x200000,
                                          None)
    assert rc == 3
    small = lib.make_shape(16, 2048, 64, 256, 1024, lib.DECO_BF16)
    assert lib.workspace_size(small) <= lib.STATIC_SCRATCH_BYTES


@pytest.mark.gpu
def test_static_scratch_reports_device_errors(lib):
    # a NaN router input sets bit 1 of the error word kept in the built-in
    # scratch; the accessor reads it, clears it, and a clean call leaves 0
    shape, L = case("edge_decode_t4")
    G = to_gpu(L, lib)
    x = G["x"].clone()
    x[1, 5] = float("nan")
    lib.forward_static(x, G, eps=shape.eps)
    assert lib.static_device_error() == 1
    assert lib.static_device_error() == 0
    lib.forward_static(G["x"], G, eps=shape.eps)
    assert lib.static_device_error() == 0
