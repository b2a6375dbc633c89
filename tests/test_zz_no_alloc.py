"""The allocation-free projection (llama_op_linear_noalloc) against the
projection that takes a caller workspace (llama_op_linear).

llama_op_linear_noalloc serves callers that cannot allocate device memory:
its split-tile scratch is a fixed array inside the library instead of a
caller buffer.  Both entry points run the same kernel with the same split of
the work over the SMs, and split partials are added in a fixed order, so the
outputs must be bit-identical to the workspace entry point's and from call to
call (the shared array keeps the previous call's contents, which must not
leak into the next result), and match fp64 like the workspace entry point
does.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


def _inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
    return A, W


def _close_to_workspace_result(got, ref):
    # same kernel, same work split, partials added in the same order
    assert np.array_equal(got, ref)


def _rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("M,N,K", [(4, 4096, 4096), (16, 12288, 4096), (1, 1000, 4160), (7, 4096, 11008)])
def test_noalloc_matches_workspace_projection_twice(llb, M, N, K):
    A, W = _inputs(M, N, K, 100 * M + K)
    ref = torch.empty(M, N, device="cuda")
    llb.op_linear(A, W, ref)
    torch.cuda.synchronize()
    want = A.double().cpu().numpy() @ W.double().cpu().numpy().T
    first = None
    for call in range(2):
        out = torch.full((M, N), float("nan"), device="cuda")
        rc = llb.lib().llama_op_linear_noalloc(A.data_ptr(), W.data_ptr(), M, N, K, out.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)
        assert rc == llb.LLAMA_OK, llb.last_error()
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all(), call
        _close_to_workspace_result(got, ref.cpu().numpy())
        assert _rel_l2(got, want) < 2e-5
        if first is None:
            first = got
        else:
            assert np.array_equal(got, first), "second call differs from the first"


def test_noalloc_second_shape_after_first(llb):
    """A call with other shapes right after a larger one: leftovers in the shared
    array must not show up in the result."""
    for (M, N, K) in [(16, 22016, 4096), (3, 4096, 4096)]:
        A, W = _inputs(M, N, K, 7 + M)
        ref = torch.empty(M, N, device="cuda")
        llb.op_linear(A, W, ref)
        out = torch.empty(M, N, device="cuda")
        llb.op_linear_noalloc(A, W, out)
        torch.cuda.synchronize()
        _close_to_workspace_result(out.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_array(llb):
    A, W = _inputs(17, 256, 256, 3)
    out = torch.empty(17, 256, device="cuda")
    rc = llb.lib().llama_op_linear_noalloc(A.data_ptr(), W.data_ptr(), 17, 256, 256, out.data_ptr(), None)
    assert rc == llb.LLAMA_ERR_CAPACITY
    assert "16" in llb.last_error()
