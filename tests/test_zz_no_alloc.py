"""svsa_build_perm_noalloc: the permutation build for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Called through the C ABI and compared with svsa_build_perm, which takes a
caller-allocated workspace: the permutations are integers, so they must match
bit for bit.  Two calls in a row share the library's scratch, so the second
call also checks that nothing left over from the first one leaks into it.
This file runs last in a full collection and also passes alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_hilbert_b200 as svsa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    svsa.lib()


def _with_workspace(s, order, N, Npad):
    perm = torch.full((Npad,), -7, dtype=torch.int32, device="cuda")
    iperm = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(svsa.svsa_perm_workspace_bytes(s, order), 16), dtype=torch.uint8, device="cuda")
    svsa.svsa_build_perm(s, order, perm, iperm, ws, ws.numel())
    return perm, iperm


def _without_allocation(s, order, N, Npad):
    perm = torch.full((Npad,), -7, dtype=torch.int32, device="cuda")
    iperm = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = svsa.lib().svsa_build_perm_noalloc(s, order, perm.data_ptr(), iperm.data_ptr(), stream)
    assert status == 0, svsa.lib().svsa_last_error().decode()
    return perm, iperm


@pytest.mark.parametrize("order", [svsa.ORDER_HILBERT, svsa.ORDER_RASTER])
def test_matches_workspace_variant_on_two_calls(order):
    # a large grid first, then a small one: the second call reuses the scratch
    for T, H, W in [(126, 30, 52), (4, 8, 8)]:
        s = svsa.shape(1, 1, T, H, W, 128)
        N = T * H * W
        Npad = -(-N // 64) * 64
        ref = _with_workspace(s, order, N, Npad)
        got = _without_allocation(s, order, N, Npad)
        svsa.svsa_sync_status()
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
        assert np.array_equal(np.sort(got[0].cpu().numpy()[:N]), np.arange(N))


def test_rejects_grids_beyond_the_fixed_scratch():
    s = svsa.shape(1, 1, 2, 129, 3, 64)                    # longest side 129 > 128
    perm = torch.empty(2 * 129 * 3 + 64, dtype=torch.int32, device="cuda")
    iperm = torch.empty(2 * 129 * 3, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = svsa.lib().svsa_build_perm_noalloc(s, svsa.ORDER_HILBERT, perm.data_ptr(), iperm.data_ptr(), stream)
    assert status == 2
    assert "128" in svsa.lib().svsa_last_error().decode()


def test_two_streams_ordered_by_an_event():
    # The calls share one scratch array: on two streams they are correct only
    # when ordered.  Both calls are queued back to back with no host
    # synchronisation between them; stream b waits for an event recorded
    # after the call on stream a, so both results must equal the workspace
    # variant's.
    T, H, W = 21, 30, 52
    s = svsa.shape(1, 1, T, H, W, 128)
    N = T * H * W
    Npad = -(-N // 64) * 64
    ref = _with_workspace(s, svsa.ORDER_HILBERT, N, Npad)
    outs = [(torch.full((Npad,), -7, dtype=torch.int32, device="cuda"),
             torch.full((N,), -7, dtype=torch.int32, device="cuda")) for _ in range(2)]
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    done = torch.cuda.Event()
    for n, ((perm, iperm), stream) in enumerate(zip(outs, (sa, sb))):
        if n == 1:
            stream.wait_event(done)
        status = svsa.lib().svsa_build_perm_noalloc(s, svsa.ORDER_HILBERT, perm.data_ptr(), iperm.data_ptr(),
                                                    ctypes.c_void_p(stream.cuda_stream))
        assert status == 0, svsa.lib().svsa_last_error().decode()
        if n == 0:
            done.record(stream)
    torch.cuda.synchronize()
    svsa.svsa_sync_status()
    for perm, iperm in outs:
        assert torch.equal(perm, ref[0]) and torch.equal(iperm, ref[1])
