"""The no-allocation Hessian entry point, through the C ABI.

qat4_hessian_noalloc exists for callers that must not allocate device memory
themselves (an engine that owns all device memory, a loop where cudaMalloc is
not acceptable); its scratch is a static array inside the library.  This file
runs last so that a failure here does not hide any other test's result, and it
passes both alone in a fresh process and after the rest of the suite."""
import ctypes as ct

import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs
from hessian_check import check_hessian

pytestmark = pytest.mark.gpu


def _call(fn_name, X, H, *extra):
    L = q4.lib()
    st = ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    n, C = X.shape
    return getattr(L, fn_name)(ct.c_void_p(X.data_ptr()), n, C, ct.c_void_p(H.data_ptr()), *extra, st)


def _frob(a, b):
    return float(torch.linalg.norm((a - b).double()) / torch.linalg.norm(b.double()))


def test_noalloc_matches_workspace_entry_point_twice_in_a_row(oracle_mod):
    # a shape whose n is split, so the scratch is really used (18 MiB at 65536 x 2048 would also do)
    n, C = 8192, 1024
    assert q4.hessian_workspace_bytes(n, C) > 0
    results = []
    for seed in (1, 2):     # two calls in a row with different data: no stale scratch leaks
        Xb = inputs.activations(n, C, seed=seed, cfg=70, name="X", outliers=10)
        X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
        H_noalloc = torch.empty((C, C), dtype=torch.float32, device="cuda")
        assert _call("qat4_hessian_noalloc", X, H_noalloc) == 0
        H_ref = torch.empty((C, C), dtype=torch.float32, device="cuda")
        ws = torch.empty(q4.hessian_workspace_bytes(n, C), dtype=torch.uint8, device="cuda")
        assert _call("qat4_hessian", X, H_ref, ct.c_void_p(ws.data_ptr()), ws.numel()) == 0
        q4.sync_check()
        assert _frob(H_noalloc, H_ref) <= 1e-3
        assert torch.equal(H_noalloc, H_ref)      # same kernels, same order: identical bits
        # and against the float64 oracle, block by block over every upper tile
        check_hessian(H_noalloc.cpu().numpy(), Xb, oracle_mod, np.random.default_rng(seed), n_random=4)
        results.append(H_noalloc)
    assert not torch.equal(results[0], results[1])


def test_noalloc_argument_errors():
    X = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    H = torch.empty((64, 64), dtype=torch.float32, device="cuda")
    L = q4.lib()
    st = ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.qat4_hessian_noalloc(None, 64, 64, ct.c_void_p(H.data_ptr()), st) == 1
    assert L.qat4_hessian_noalloc(ct.c_void_p(X.data_ptr()), 64, 48, ct.c_void_p(H.data_ptr()), st) == 2
