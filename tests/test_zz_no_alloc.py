"""The allocation-free weight quantiser (bitlinear_quantize_weights_static).

It exists for callers that may not allocate device memory (a plugin inside a
host application that owns the device-memory budget, or a loop in which
cudaMalloc/cudaFree and their synchronisation are not allowed); its scratch is
a fixed array inside the library.  Called through the C ABI, two calls in a
row must give exactly the packed weights and α of the workspace-taking entry
point.  This file is collected last so that a failure here comes after every
other test has run."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
from bitlinear_w1_a8_03_b200 import synth

pytestmark = pytest.mark.gpu


def _static_call(W):
    L = bl.lib()
    N, K = W.shape
    packed = torch.empty((N, bl.packed_row_bytes(K)), dtype=torch.uint8, device="cuda")
    alpha = torch.empty(1, dtype=torch.float32, device="cuda")
    dt = bl.BL_F32 if W.dtype == torch.float32 else bl.BL_BF16
    st = L.bitlinear_quantize_weights_static(W.data_ptr(), dt, N, K, packed.data_ptr(), alpha.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    bl.check(st, "bitlinear_quantize_weights_static")
    return packed, alpha


def test_static_scratch_matches_workspace_entry_point_twice():
    shapes = [(2048, 4096, torch.float32, 11), (333, 1000, torch.bfloat16, 12)]
    for N, K, dt, seed in shapes:  # two calls in a row, different sizes
        W = torch.from_numpy(synth.weights(seed, N, K, 0.02)).cuda().to(dt)
        p_static, a_static = _static_call(W)
        p_ref, a_ref = bl.bitlinear_quantize_weights(W)
        torch.cuda.synchronize()
        assert a_static.cpu().numpy()[0] == a_ref.cpu().numpy()[0]
        assert np.array_equal(p_static.cpu().numpy(), p_ref.cpu().numpy())


def test_static_rejects_shapes_beyond_the_shared_limit():
    """N·K above 2^40 is refused before anything is launched.  The static
    entry point shares this limit with the workspace one; its own scratch-size
    check cannot fire for accepted shapes (the partial-sum grid is capped at
    the scratch size, pinned by a static_assert in the library)."""
    L = bl.lib()
    P = 0x7F0000000000
    assert L.bitlinear_quantize_weights_static(P, 0, 1 << 30, 1 << 20, P, P, None) == 2  # BL_ERR_SHAPE
