"""mxq_act_sqmean_noalloc: the h pass for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: their device memory belongs to another
allocator or a fixed arena, or they must not allocate after start-up because an allocation
can synchronise the device. For them the library offers an h pass that takes no workspace
and uses a 1 MiB static device array inside the library instead. This test calls it through
the C-ABI, twice in a row (the second call reuses the array the first one wrote), and
checks each result against the workspace version, mxq_act_sqmean. Both run the same two
kernels with the same row chunks in the same fixed order, so the results must be equal bit
for bit (a wrong offset or leading dimension in the scratch path would show up even where
it moves h only slightly); the shapes include the widest scratch use (a one-wave grid of
256-column strips) and the widest accepted input. It also checks that a width beyond the
array's limit is rejected before any launch. It must pass alone in a fresh process and after the rest of
the suite, so it lives in a file that is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mxq():
    from block_scaled_weight_b200.build import build
    build()
    from block_scaled_weight_b200 import mxq as m
    return m


def call_noalloc(mxq, X, h):
    """The entry point, called through the C-ABI with plain pointers."""
    R, K = X.shape
    st = torch.cuda.current_stream(X.device).cuda_stream
    return mxq._lib.mxq_act_sqmean_noalloc(ctypes.c_void_p(X.data_ptr()), 1 if X.dtype == torch.bfloat16 else 0,
                                           R, K, X.stride(0), ctypes.c_void_p(h.data_ptr()),
                                           ctypes.c_void_p(st))


@pytest.mark.parametrize("rows,cols,dtype", [(244449 // 8, 9728, torch.bfloat16),
                                             (1000, 264, torch.bfloat16),
                                             (512, 256, torch.float32),
                                             # 4 strips x 111 chunks: ~0.9 MB of scratch
                                             (65536, 1024, torch.bfloat16),
                                             # the widest accepted input, many rows
                                             (2048, 131072, torch.bfloat16)])
def test_noalloc_matches_workspace_version_twice(mxq, rows, cols, dtype):
    from block_scaled_weight_b200 import synth
    for call in range(2):
        X = synth.activations(rows, cols, 100 + call, dtype=dtype, device=DEV)
        ref = mxq.mxq_act_sqmean(X)
        h = torch.full((cols,), float("nan"), dtype=torch.float32, device=DEV)
        assert call_noalloc(mxq, X, h) == 0, mxq._lib.mxq_last_error()
        torch.cuda.synchronize()
        assert np.array_equal(h.cpu().numpy(), ref.cpu().numpy())
        del X


def test_noalloc_rejects_widths_beyond_the_static_scratch(mxq):
    X = torch.empty(16, 131072 + 256, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(X.shape[1], dtype=torch.float32, device=DEV)
    assert call_noalloc(mxq, X, h) == 2                    # MXQ_ERR_SHAPE, nothing launched
    assert b"scratch" in mxq._lib.mxq_last_error()
    X = torch.zeros(16, 131072, dtype=torch.bfloat16, device=DEV)
    h = torch.empty(X.shape[1], dtype=torch.float32, device=DEV)
    assert call_noalloc(mxq, X, h) == 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(h).item() == 0
