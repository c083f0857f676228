"""The allocation-free W2A8 GEMM entry point (bitnet_w2a8_gemm_noalloc).

It serves callers that cannot allocate device memory and therefore cannot pass
the workspace bitnet_w2a8_gemm may need; it uses the library's one built-in
scratch array instead.  These tests call it through the C ABI and check it
against the oracle and against the workspace entry point on the same inputs,
two calls in a row with different data (the shared scratch keeps the previous call's contents, so a
stale read would show), including a shape whose plan does use scratch.  This
file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import oracle
import ternary_weight_bit_w2a8_b200 as bn
from ternary_weight_bit_w2a8_b200 import synth


def test_noalloc_rejects_problems_beyond_its_scratch():
    # checked on the host before any device work; the fake pointers are never
    # used, and the test is skipped where a GPU is present so a wrong
    # expectation cannot become a launch on them.  K not a multiple of 16 with
    # M >= 2: the activations are repacked into M * K_pad bytes of scratch
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake-pointer host check runs only where no GPU is present")
    lib = bn.lib()
    A = ctypes.c_void_p(0x10000)
    M, N, K = 4, 64, (1 << 21) - 1
    assert lib.bitnet_workspace_bytes(M, N, K) > 1048576
    assert lib.bitnet_w2a8_gemm_noalloc(A, A, A, M, N, K, None) == bn.BITNET_ERR_WORKSPACE
    assert lib.bitnet_w2a8_gemm_noalloc(A, A, A, 0, N, K, None) == bn.BITNET_OK


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = bn.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # these use the scratch array: (1, 640, 131072) splits K (its activations do
    # not fit one CTA's shared memory) and keeps int32 partials there; (3, 129,
    # 1000) and (2, 64, 999) have K not a multiple of 16, so their activations
    # are repacked there for the tensor-core path; the others need none
    cases = [(1, 640, 131072), (3, 129, 1000), (2, 64, 999), (1, 300, 2560), (5, 96, 2560), (1, 7, 100)]
    for (M, N, K) in cases:
        for call in range(2):
            q, w = synth.uniform_int8_ternary(N, K, seed=1000 * call + M + N, M=M)
            qd = torch.from_numpy(q).cuda()
            packed = bn.bitnet_pack_weights(torch.from_numpy(w).cuda())
            y_ref = bn.bitnet_w2a8_gemm(qd, packed, N)
            y = torch.full((M, N), -7, dtype=torch.int32, device="cuda")
            rc = lib.bitnet_w2a8_gemm_noalloc(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(packed.data_ptr()),
                                              ctypes.c_void_p(y.data_ptr()), M, N, K, stream)
            assert rc == bn.BITNET_OK, bn.status_string(rc)
            torch.cuda.synchronize()
            assert np.array_equal(y.cpu().numpy(), oracle.gemm_i32(q, w)), (M, N, K, call)
            assert torch.equal(y, y_ref), (M, N, K, call)
    assert bn.bitnet_get_device_error() == 0
