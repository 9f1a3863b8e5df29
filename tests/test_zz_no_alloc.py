"""fp4_preshift_calibrate_noalloc: calibration for callers that cannot
obtain device memory when they calibrate (a runtime whose device-memory plan
is fixed at start-up, a plug-in handed tensors but no allocator).  It keeps
its scratch in a 256 KB buffer inside the library instead of a workspace, so
its results must equal those of fp4_preshift_calibrate bit for bit, call
after call, whatever an earlier call left in that buffer.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

from w4a16_gemm_fp4_b200 import synth


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _calibrate_ws(L, X, stream):
    M, K = X.shape
    shift = torch.empty(K, dtype=torch.int8, device=X.device)
    rho = torch.empty(1, dtype=torch.float32, device=X.device)
    nb = L.fp4_preshift_workspace_size(M, K)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=X.device)
    rc = L.fp4_preshift_calibrate(_ptr(X), M, K, _ptr(shift), _ptr(rho), _ptr(ws), nb, stream)
    assert rc == 0
    return shift, rho


def _calibrate_noalloc(L, X, stream):
    M, K = X.shape
    shift = torch.full((K,), 77, dtype=torch.int8, device=X.device)
    rho = torch.full((1,), -1.0, dtype=torch.float32, device=X.device)
    rc = L.fp4_preshift_calibrate_noalloc(_ptr(X), M, K, _ptr(shift), _ptr(rho), stream)
    assert rc == 0
    return shift, rho


@pytest.mark.gpu
def test_noalloc_calibrate_matches_workspace_entry():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from w4a16_gemm_fp4_b200 import api, build
    build.build()
    L = api.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rng = np.random.default_rng(99)
    cases = []
    # a large calibration set first (many row slabs), then a smaller one, so
    # the second call runs over what the first left in the shared buffer
    for (M, K) in ((2048, 4096), (300, 11008)):
        Xb, _ = synth.outlier_activations(rng, M, K)
        Xb[:, 5] = 0  # an all-zero channel
        X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.int16)
        cases.append(X)
    for X in cases:
        ref_shift, ref_rho = _calibrate_ws(L, X, stream)
        for _ in range(2):
            shift, rho = _calibrate_noalloc(L, X, stream)
            torch.cuda.synchronize()
            assert torch.equal(shift, ref_shift)
            assert rho.item() == ref_rho.item()
    st = api.device_status(clear=True)
    assert st == 0


def test_noalloc_rejects_k_beyond_its_buffer():
    """K above the buffer's 65536 columns is refused before anything runs."""
    from w4a16_gemm_fp4_b200 import api, build
    build.build()
    L = api.lib()
    fake = ctypes.c_void_p(1 << 20)
    assert L.fp4_preshift_calibrate_noalloc(fake, 4, 65536 + 8, fake, fake, None) == 4   # FP4_ERR_WORKSPACE
    assert L.fp4_preshift_calibrate_noalloc(fake, 4, 12, fake, fake, None) == 2          # K % 8
