"""tp_csr_transpose_noalloc: the transpose for callers that cannot allocate device memory.

Some hosts cannot give the library a workspace (device memory owned by a pool they do not
control, a framework that reserved nearly all of the GPU, or a loop that must avoid the
device synchronisation of cudaMalloc/cudaFree).  This entry point keeps its scratch in a
fixed array inside the library; these checks compare it, through the C ABI, with the
workspace-taking tp_csr_transpose on two calls in a row (the second call must not see
anything the first left in the shared array).  Integer results, so the tolerance is zero.
This file is named to be collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    from equivariant_tensor_product_b200 import _lib
    lib = _lib.load()
    f = lib.tp_csr_transpose_noalloc
    f.restype = C.c_int
    f.argtypes = [C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    return lib


def _graph(seed, n, deg_hi, n_senders):
    rng = np.random.default_rng(seed)
    deg = rng.integers(0, deg_hi + 1, n)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    src = rng.integers(0, n_senders, int(rowptr[-1])).astype(np.int32)
    return rowptr, src


def _noalloc(lib, rowptr, src, n):
    dev = lambda a: torch.as_tensor(a).cuda()
    r, s = dev(rowptr), dev(src)
    colptr = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((len(src),), -7, dtype=torch.int32, device="cuda")
    st = lib.tp_csr_transpose_noalloc(n, len(src), r.data_ptr(), s.data_ptr() if len(src) else None,
                                      colptr.data_ptr(), perm.data_ptr() if len(src) else None,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return colptr.cpu().numpy(), perm.cpu().numpy()


def _existing(rowptr, src, n):
    import equivariant_tensor_product_b200 as tp
    colptr, perm = tp.tp_csr_transpose(torch.as_tensor(rowptr).cuda(), torch.as_tensor(src).cuda(), n)
    return colptr.cpu().numpy(), perm.cpu().numpy()


def test_noalloc_matches_workspace_transpose_twice_in_a_row(lib):
    # a large graph (many senders) then a small one (few senders, many repeats)
    cases = [_graph(1, 20000, 60, 20000) + (20000,), _graph(2, 3000, 9, 37) + (3000,)]
    for rowptr, src, n in cases:
        got = _noalloc(lib, rowptr, src, n)
        want = _existing(rowptr, src, n)
        np.testing.assert_array_equal(got[0], want[0])
        np.testing.assert_array_equal(got[1], want[1])
        np.testing.assert_array_equal(got[1], np.argsort(src, kind="stable"))
    torch.cuda.synchronize()


def test_noalloc_at_its_limits_and_when_empty(lib):
    """The largest accepted graph (N = 131,072, E = 1,048,576: the last sender's counter and
    the last slot of every scratch region in use), then graphs without edges or nodes, then a
    small graph again, each against tp_csr_transpose and a stable numpy argsort."""
    rng = np.random.default_rng(9)
    N, E = 1 << 17, 1 << 20
    src = rng.integers(0, N, E).astype(np.int32)
    src[-4096:] = N - 1
    rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
    cases = [(rowptr, src, N),
             (np.zeros(11, np.int32), np.zeros(0, np.int32), 10),
             (np.zeros(1, np.int32), np.zeros(0, np.int32), 0),
             _graph(4, 500, 12, 499) + (500,)]
    for rowptr, src, n in cases:
        got = _noalloc(lib, rowptr, src, n)
        want = _existing(rowptr, src, n)
        np.testing.assert_array_equal(got[0], want[0])
        np.testing.assert_array_equal(got[1], want[1])
        np.testing.assert_array_equal(got[1], np.argsort(src, kind="stable"))
        np.testing.assert_array_equal(got[0], np.concatenate([[0], np.cumsum(np.bincount(src, minlength=n))]))
    torch.cuda.synchronize()


def test_noalloc_rejects_graphs_beyond_its_array(lib):
    fake = C.c_void_p(0x10000)   # never touched: the size check comes first
    assert lib.tp_csr_transpose_noalloc(1 << 17 | 1, 10, fake, fake, fake, fake, None) == 2
    assert lib.tp_csr_transpose_noalloc(10, (1 << 20) + 1, fake, fake, fake, fake, None) == 2
    assert lib.tp_csr_transpose_noalloc(-1, 10, fake, fake, fake, fake, None) == 1
