"""The entry point that allocates nothing: bitnet_quantize_pack_weights_noalloc.

Some callers cannot allocate device memory (a runtime that only lends the library the tensors
it owns, code running where cudaMalloc is not allowed), so they cannot provide the workspace of
bitnet_quantize_pack_weights.  The _noalloc variant keeps its partial sums in a fixed scratch
array inside the library.  This test calls it straight through the C ABI (ctypes, raw device
pointers) twice in a row and checks each result against the workspace entry point, bit for bit
(the tolerance of every packed-weight test): the second call also shows that the scratch left
by the first call does not leak into the next result.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_activation_linear_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from bit_activation_linear_b200 import binding, build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return binding.load_library()


def reference(lib, W, N, K):
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    need = lib.bitnet_weight_workspace_bytes(N, K)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    rc = lib.bitnet_quantize_pack_weights(W.data_ptr(), N, K, Wp.data_ptr(), g.data_ptr(),
                                          ws.data_ptr(), ws.numel(),
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.bitnet_last_error().decode()
    return Wp, g


def no_alloc(lib, W, N, K):
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    rc = lib.bitnet_quantize_pack_weights_noalloc(W.data_ptr(), N, K, Wp.data_ptr(), g.data_ptr(),
                                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.bitnet_last_error().decode()
    return Wp, g


def test_no_alloc_matches_workspace_entry_twice(lib):
    # weight matrices back to back, largest first: 4096 x 4096 (16.8 M weights) takes the
    # full 1184 partial sums the fixed array holds; the smaller ones after it use fewer, so a
    # stale partial from the first call would show in their gamma
    for (N, K, seed) in ((4096, 4096, 13), (2048, 2048, 11), (264, 384, 12)):
        W = synth.to_torch_bf16(synth.latent_weights(N, K, seed=seed)).cuda()
        Wp_ref, g_ref = reference(lib, W, N, K)
        Wp, g = no_alloc(lib, W, N, K)
        assert lib.bitnet_sync_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        assert g.item() == g_ref.item()
        assert torch.equal(Wp, Wp_ref)


def test_no_alloc_rejects_bad_arguments(lib):
    W = torch.zeros((8, 100), dtype=torch.bfloat16, device="cuda")
    Wp = torch.empty((8, 25), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    rc = lib.bitnet_quantize_pack_weights_noalloc(W.data_ptr(), 8, 100, Wp.data_ptr(),
                                                  g.data_ptr(), None)
    assert rc == -1 and "multiple of 128" in lib.bitnet_last_error().decode()
