"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before anything is launched."""
import ctypes as ct
import os
import re

import numpy as np
import pytest

import int4_group_wise_b200 as q4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qat4.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qat4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound():
    L = q4.lib()
    names = _declared()
    assert "qat4_hessian" in names and "qat4_scale_search" in names and len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert sorted(q4.EXPORTS) == names
    assert L.qat4_abi_version() == 1


def test_status_strings():
    for code, name in q4.STATUS.items():
        assert q4.status_string(code).startswith(name)
    assert "UNKNOWN" in q4.status_string(99)


def test_grad_scale_constant():
    assert q4.GRAD_SCALE == float(np.float32(1.0 / np.sqrt(224.0)))


# Fake, 16-byte aligned non-null "device" addresses: validation rejects the
# call before any pointer is dereferenced or any CUDA call is made.
A = ct.c_void_p(0x10000)
B = ct.c_void_p(0x20000)
MIS = ct.c_void_p(0x20004)


@pytest.mark.parametrize("args,code", [
    ((None, 8, 64, A, A), 1),
    ((A, 8, 64, None, A), 1),
    ((A, 0, 64, A, A), 2),
    ((A, 8, 48, A, A), 2),
    ((A, 8, 0, A, A), 2),
    ((MIS, 8, 64, A, A), 3),
    ((A, 8, 64, A, MIS), 3),
])
def test_lsq_fwd_validation(args, code):
    W, R, C, d, Q = args
    assert q4.lib().qat4_lsq_fwd(W, d, R, C, Q, None) == code


def test_lsq_bwd_and_fused_validation():
    L = q4.lib()
    assert L.qat4_lsq_bwd(A, A, None, 0, 4, 64, ct.c_float(1.0), A, A, None) == 1
    assert L.qat4_lsq_bwd(A, A, A, 7, 4, 64, ct.c_float(1.0), A, A, None) == 4
    assert L.qat4_lsq_bwd(A, A, MIS, 1, 4, 64, ct.c_float(1.0), A, A, None) == 3
    assert L.qat4_lsq_fwd_bwd(A, A, A, 1, 4, 64, ct.c_float(1.0), None, A, A, None) == 1
    assert L.qat4_lsq_fwd_bwd(A, A, A, 1, 4, 33, ct.c_float(1.0), A, A, A, None) == 2


def test_pack_search_hessian_validation():
    L = q4.lib()
    assert L.qat4_pack_w4a16(A, A, 4, 64, None, A, None) == 1
    assert L.qat4_pack_w4a16(A, A, -1, 64, A, A, None) == 2
    assert L.qat4_pack_w4a16(A, A, 4, 64, A, MIS, None) == 3
    assert L.qat4_scale_search(A, 4, 64, A, 64, A, 0, A, A, None, None) == 2      # K = 0
    assert L.qat4_scale_search(A, 4, 64, A, 32, A, 5, A, A, None, None) == 2      # ldh < C
    assert L.qat4_scale_search(A, 4, 64, A, 66, A, 5, A, A, None, None) == 3      # ldh not 16-B multiple
    assert L.qat4_scale_search(A, 4, 64, A, 64, None, 5, A, A, None, None) == 1
    assert L.qat4_hessian(None, 64, 64, A, None, 0, None) == 1
    assert L.qat4_hessian(A, 0, 64, A, None, 0, None) == 2
    assert L.qat4_hessian(A, 64, 40, A, None, 0, None) == 2
    assert L.qat4_hessian(MIS, 64, 64, A, None, 0, None) == 3
    assert L.qat4_selftest_bounded_wait(0, None) == 2


@pytest.mark.parametrize("args,code", [
    ((None, 1, A, A, 8, 64, 32, A), 1),
    ((A, 1, A, None, 8, 64, 32, A), 1),
    ((A, 0, A, A, 8, 64, 32, A), 2),          # no token
    ((A, 1, A, A, 8, 48, 32, A), 2),          # C not a multiple of 32
    ((A, 1, A, A, 8, 64, 16, A), 2),          # group below 32
    ((A, 1, A, A, 8, 96, 64, A), 2),          # group does not divide C
    ((A, 1, A, A, 0, 64, 32, A), 2),
    ((MIS, 1, A, A, 8, 64, 32, A), 3),
    ((A, 1, A, MIS, 8, 64, 32, A), 3),
])
def test_w4a16_gemv_validation(args, code):
    x, M, packed, scales, R, C, group, y = args
    assert q4.lib().qat4_w4a16_gemv(x, M, packed, scales, R, C, group, y, None) == code


def test_fq_gemm_validation():
    L = q4.lib()
    assert L.qat4_fq_gemm(None, 8, A, A, 8, 64, A, None) == 1
    assert L.qat4_fq_gemm(A, 0, A, A, 8, 64, A, None) == 2
    assert L.qat4_fq_gemm(A, 8, A, A, 8, 48, A, None) == 2
    assert L.qat4_fq_gemm(A, 8, A, A, 0, 64, A, None) == 2
    assert L.qat4_fq_gemm(A, 8, MIS, A, 8, 64, A, None) == 3
    assert L.qat4_fq_gemm(A, 8, A, A, 8, 64, MIS, None) == 3
    need = L.qat4_fq_gemm_staged_workspace_bytes(8, 64)
    assert need == 1024
    assert L.qat4_fq_gemm_staged(A, 8, A, A, 8, 64, A, None, need, None) == 1
    assert L.qat4_fq_gemm_staged(A, 8, A, A, 8, 48, A, A, need, None) == 2
    assert L.qat4_fq_gemm_staged(A, 8, A, A, 8, 64, A, MIS, need, None) == 3
    assert L.qat4_fq_gemm_staged(A, 8, A, A, 8, 64, A, A, need - 256, None) == 5


def test_hessian_partial_validation():
    L = q4.lib()
    assert L.qat4_hessian_partial(None, 64, 64, 64, A, None, 0, None) == 1
    assert L.qat4_hessian_partial(A, 64, 64, 63, A, None, 0, None) == 2      # n_total < n
    assert L.qat4_hessian_partial(A, 64, 40, 64, A, None, 0, None) == 2
    assert L.qat4_hessian_partial(MIS, 64, 64, 128, A, None, 0, None) == 3


def test_refine_validation():
    L = q4.lib()
    assert L.qat4_refine(None, 4, 64, A, 64, A, 5, 1, A, A, None, A, 1 << 20, None) == 1
    assert L.qat4_refine(A, 4, 64, A, 64, A, 0, 1, A, A, None, A, 1 << 20, None) == 2      # K = 0
    assert L.qat4_refine(A, 4, 64, A, 64, A, 5, -1, A, A, None, A, 1 << 20, None) == 2     # sweeps < 0
    assert L.qat4_refine(A, 4, 64, A, 32, A, 5, 1, A, A, None, A, 1 << 20, None) == 2      # ldh < C
    assert L.qat4_refine(A, 4, 64, A, 66, A, 5, 1, A, A, None, A, 1 << 20, None) == 3      # ldh % 4
    assert L.qat4_refine(A, 4, 64, A, 64, A, 5, 1, A, A, None, A, 16, None) == 5           # workspace
    assert L.qat4_refine_workspace_bytes(4, 64) == 2 * 4 * 64 * 8


def test_lsq_host_validation():
    L = q4.lib()
    ws = q4.lsq_fwd_bwd_host_workspace_bytes(3000, 1024, q4.QAT4_BF16)
    assert ws > 0 and q4.lsq_fwd_bwd_host_workspace_bytes(3000, 48, q4.QAT4_BF16) == 0
    assert q4.lsq_fwd_bwd_host_workspace_bytes(3000, 1024, 7) == 0
    f = L.qat4_lsq_fwd_bwd_host
    s = ct.c_float(q4.GRAD_SCALE)
    assert f(None, A, A, 1, 3000, 1024, s, A, A, A, B, ws, None, None) == 1          # null W
    assert f(A, A, A, 1, 3000, 1024, s, A, A, A, None, ws, None, None) == 1          # null workspace
    assert f(A, A, A, 1, 3000, 40, s, A, A, A, B, ws, None, None) == 2               # C % 32
    assert f(A, A, A, 5, 3000, 1024, s, A, A, A, B, ws, None, None) == 4             # dtype
    assert f(A, A, A, 1, 3000, 1024, s, A, A, A, B, ws - 1, None, None) == 5         # small workspace
    assert f(A, A, A, 1, 3000, 1024, s, A, A, A, ct.c_void_p(0x20010), ws, None, None) == 3  # alignment


def _plan_workspace(n, C):
    """The split of the calibration rows as the Hessian's planner states it: T upper 256x256 tiles
    on 74 SM pairs; the tiles of the last (or only) wave are cut into min(74 // r, ceil(n/128) // 16)
    parts when that is at least 2, and each cut tile keeps one 256x256 float32 partial per part."""
    nb = -(-C // 256)
    T = nb * (nb + 1) // 2
    r = T if T <= 74 else T % 74
    s = min(74 // r if r else 1, -(-n // 128) // 16)
    return 0 if (s < 2 or r == 0) else r * s * 256 * 256 * 4


@pytest.mark.parametrize("n,C", [(262144, 2048), (40000, 3072), (262144, 8192), (131072, 14336),
                                 (131072, 4096), (1000, 2048), (4096, 512), (16, 32), (262144, 65536)])
def test_hessian_workspace_follows_the_split_plan(n, C):
    """Host-side plan, no GPU: the workspace the library asks for is the plan's partial tiles."""
    import int4_group_wise_b200 as q4
    assert q4.hessian_workspace_bytes(n, C) == _plan_workspace(n, C)


def test_hessian_workspace_examples():
    """The 1B-class up-projection splits all 36 tiles in two (18.9 MB of partials); 78 tiles put the
    4 of the second wave in 18 parts; 528 tiles leave 10 for the last wave, cut in 7."""
    import int4_group_wise_b200 as q4
    assert q4.hessian_workspace_bytes(262144, 2048) == 36 * 2 * 262144
    assert q4.hessian_workspace_bytes(40000, 3072) == 4 * 18 * 262144
    assert q4.hessian_workspace_bytes(262144, 8192) == 10 * 7 * 262144
    assert q4.hessian_workspace_bytes(0, 2048) == 0 and q4.hessian_workspace_bytes(100, 48) == 0
