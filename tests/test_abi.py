"""Host-only checks of the C ABI: the library loads, exports every declared entry
point, and rejects bad arguments before touching the GPU."""

import os
import re

import pytest

from exact_io_aware_91_b200 import api
from exact_io_aware_91_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return api.library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    assert sorted(declared_functions()) == sorted(api.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARG"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_MISALIGNED"), (4, "FA_ERR_CUDA"), (5, "FA_ERR_TIMEOUT"), (6, "FA_ERR_RANGE")]:
        assert api.status_str(code) == name
    assert api.status_str(99) == "FA_ERR_UNKNOWN"


# blocks of the streaming passes that leave per-block maxima in the workspaces
PRE_BLOCKS = 148 * 8     # backward preprocess: 4 tensors x 4 bytes per block
VPASS_BLOCKS = 148 * 16  # forward V pass: 4 bytes per block


def _ws_expected(B, H, N, d):
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    Np = (N + 127) // 128 * 128
    # fp16 Q, dO, K, V; D and LSE*log2(e); control block (counters, exponents); maxima
    return 4 * a(B * H * N * d * 2) + 2 * a(B * H * Np * 4) + 256 + a(16 * PRE_BLOCKS)


@pytest.mark.parametrize("shape", [(1, 1, 1, 64), (4, 16, 2048, 128), (2, 32, 8192, 128), (1, 8, 131072, 128),
                                   (3, 5, 1000, 64)])
def test_workspace_size_is_linear_in_n(lib, shape):
    assert api.fa_bwd_workspace_size(*shape) == _ws_expected(*shape)


def _ws_expected_gqa(B, H, Hkv, N, d):
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    Np = (N + 127) // 128 * 128
    # few key/value tiles: the group's query heads are split over CTAs with fp32 partial dK, dV
    # (one unit per key tile; at d = 256 the dV and dK kernels each have that many)
    group, units = H // Hkv, B * Hkv * ((N + 127) // 128)
    split = next((s for s in range(1, group) if group % s == 0 and units * s >= 4 * 148), group)
    part = 2 * a(split * B * Hkv * N * d * 4) if split > 1 else 0
    return (2 * a(B * H * N * d * 2) + 2 * a(B * Hkv * N * d * 2) + 2 * a(B * H * Np * 4) + part + 256 +
            a(16 * PRE_BLOCKS))


@pytest.mark.parametrize("shape", [(1, 4, 1, 1, 64), (2, 32, 8, 8192, 128), (1, 8, 1, 131072, 128),
                                   (3, 6, 3, 1000, 64), (2, 16, 16, 2048, 128), (1, 8, 2, 9472, 256)])
def test_gqa_workspace_size(lib, shape):
    B, H, Hkv, N, d = shape
    assert api.fa_bwd_gqa_workspace_size(*shape) == _ws_expected_gqa(*shape)
    if H == Hkv:
        assert api.fa_bwd_gqa_workspace_size(*shape) == api.fa_bwd_workspace_size(B, H, N, d)


def test_gqa_head_counts_are_checked(lib):
    assert api.fa_bwd_gqa_workspace_size(1, 6, 4, 64, 64) == 0  # 6 is not a multiple of 4
    assert api.fa_bwd_gqa_workspace_size(1, 6, 0, 64, 64) == 0
    fwd_gqa = lambda H, Hkv: lib.fa_fwd_gqa(A, A, A, A, A, None, 1, H, Hkv, 16, 64, 0.125, 0, None)  # noqa: E731
    assert fwd_gqa(6, 4) == api.FA_ERR_INVALID_ARG
    assert fwd_gqa(6, 0) == api.FA_ERR_INVALID_ARG
    assert fwd_gqa(6, -3) == api.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_gqa(None, None, None, None, None, None, 1, 0, 0, 16, 64, 0.125, 0, None) == api.FA_OK
    bwd_gqa = lambda H, Hkv: lib.fa_bwd_gqa(A, A, A, A, A, A, A, A, A, A, 1, H, Hkv, 16, 64, 0.125, 0, A,  # noqa: E731
                                             1 << 40, None)
    assert bwd_gqa(8, 3) == api.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_gqa(A, A, A, A, A, A, A, A, A, A, 1, 8, 2, 16, 64, 0.125, 0, A,
                          _ws_expected_gqa(1, 8, 2, 16, 64) - 1, None) == api.FA_ERR_INVALID_ARG


def test_forward_workspace(lib):
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # fp16 V, control block (work counter, the copy's exponent), the V pass's maxima
    assert api.fa_fwd_workspace_size(2, 8, 8192, 128) == a(2 * 8 * 8192 * 128 * 2) + 256 + a(4 * VPASS_BLOCKS)
    assert api.fa_fwd_workspace_size(1, 1, 300, 64) == a(300 * 64 * 2) + 256 + a(4 * VPASS_BLOCKS)
    assert api.fa_fwd_workspace_size(0, 8, 100, 64) == 0
    assert api.fa_fwd_workspace_size(1, 1, 100, 96) == 0
    ws = lambda ptr=A, n=1 << 40, H=4, Hkv=2: lib.fa_fwd_ws(A, A, A, A, A, None, 1, H, Hkv, 16, 64, 0.125, 0,  # noqa: E731
                                                            ptr, n, None)
    assert ws(ptr=None) == api.FA_ERR_INVALID_ARG
    assert ws(n=api.fa_fwd_workspace_size(1, 2, 16, 64) - 1) == api.FA_ERR_INVALID_ARG
    assert ws(ptr=A + 16) == api.FA_ERR_MISALIGNED
    assert ws(H=6, Hkv=4) == api.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_ws(None, None, None, None, None, None, 1, 4, 2, 0, 64, 0.125, 0, None, 0, None) == api.FA_OK


def test_descriptor_entry_points_check_their_arguments(lib):
    import ctypes

    pr = api.FaAttnProblem(1, 4, 2, 300, 64, 0.125, 1, 16, -1)
    assert api.fa_attn_fwd_workspace_size(pr) == api.fa_fwd_workspace_size(1, 2, 300, 64)
    assert api.fa_attn_bwd_workspace_size(pr) == api.fa_bwd_gqa_workspace_size(1, 4, 2, 300, 64)
    assert lib.fa_attn_fwd_workspace_size(None) == 0 and lib.fa_attn_bwd_workspace_size(None) == 0
    bad = api.FaAttnProblem(1, 4, 2, 300, 64, 0.125, 1, -2, -1)
    assert api.fa_attn_fwd_workspace_size(bad) == 0
    fwd = lambda p, ws=A: lib.fa_attn_fwd(ctypes.byref(p), A, A, A, A, A, None, ws, 1 << 40, None)  # noqa: E731
    bwd = lambda p: lib.fa_attn_bwd(ctypes.byref(p), A, A, A, A, A, A, A, A, A, A, A, 1 << 40, None)  # noqa: E731
    assert fwd(bad) == api.FA_ERR_INVALID_ARG
    assert bwd(bad) == api.FA_ERR_INVALID_ARG
    assert fwd(pr, ws=None) == api.FA_ERR_INVALID_ARG  # the forward needs its workspace
    assert lib.fa_attn_fwd(None, A, A, A, A, A, None, A, 1 << 40, None) == api.FA_ERR_INVALID_ARG
    assert fwd(api.FaAttnProblem(1, 6, 4, 300, 64, 0.125, 1, -1, -1)) == api.FA_ERR_INVALID_ARG


def test_workspace_size_of_empty_or_bad_problem_is_zero(lib):
    assert api.fa_bwd_workspace_size(0, 1, 10, 64) == 0
    assert api.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    assert api.fa_bwd_workspace_size(1, 1, 10, 96) == 0
    assert api.fa_bwd_workspace_size(-1, 1, 10, 64) == 0


# Fake device addresses: never dereferenced, because every call below is rejected
# (or is empty) before anything is launched.
A = 0x10000  # 16-byte (and 256-byte) aligned
MIS = 0x10008


# fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream) and
# fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, stream):
# the boundary's plain signatures
def fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=16, d=64, scale=0.125, causal=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, None)


def bwd(lib, ptr=A, ws=A, B=1, H=1, N=16, d=64, scale=0.125, causal=0, dq=A):
    return lib.fa_bwd(ptr, ptr, ptr, ptr, ptr, ptr, dq, ptr, ptr, B, H, N, d, scale, causal, ws, None)


# the grouped entry points carry the residual and the workspace size
def fwd_gqa(lib, resid=None, B=1, H=1, N=16, d=64):
    return lib.fa_fwd_gqa(A, A, A, A, A, resid, B, H, H, N, d, 0.125, 0, None)


def bwd_gqa(lib, ws_bytes=1 << 40, resid=A, B=1, H=1, N=16, d=64):
    return lib.fa_bwd_gqa(A, A, A, A, resid, A, A, A, A, A, B, H, H, N, d, 0.125, 0, A, ws_bytes, None)


def test_forward_argument_errors(lib):
    assert fwd(lib, q=None) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, o=None) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, N=-1) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=0.0) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=float("nan")) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=float("inf")) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, causal=2) == api.FA_ERR_INVALID_ARG
    assert fwd(lib, d=96) == api.FA_ERR_UNSUPPORTED
    assert fwd(lib, d=256) == api.FA_ERR_UNSUPPORTED
    assert fwd(lib, q=MIS) == api.FA_ERR_MISALIGNED
    assert fwd(lib, o=MIS) == api.FA_ERR_MISALIGNED
    assert fwd(lib, lse=A + 2) == api.FA_ERR_MISALIGNED
    assert fwd_gqa(lib, resid=A + 8) == api.FA_ERR_MISALIGNED
    assert fwd(lib, B=1 << 25) == api.FA_ERR_UNSUPPORTED


def test_empty_problems_are_no_ops(lib):
    # nothing to compute: FA_OK even with null pointers, nothing launched
    assert fwd(lib, q=None, k=None, v=None, o=None, lse=None, N=0) == api.FA_OK
    assert fwd(lib, q=None, k=None, v=None, o=None, lse=None, B=0) == api.FA_OK
    assert bwd(lib, ptr=None, ws=None, dq=None, H=0) == api.FA_OK
    assert lib.fa_fwd_f32(None, None, None, None, None, 1, 1, 0, 64, 0.125, 0, None) == api.FA_OK


def test_backward_argument_errors(lib):
    assert bwd(lib, ptr=None) == api.FA_ERR_INVALID_ARG
    assert bwd(lib, ws=None) == api.FA_ERR_INVALID_ARG
    assert bwd_gqa(lib, ws_bytes=_ws_expected(1, 1, 16, 64) - 1) == api.FA_ERR_INVALID_ARG
    assert bwd(lib, d=32) == api.FA_ERR_UNSUPPORTED
    assert bwd(lib, causal=-1) == api.FA_ERR_INVALID_ARG
    assert bwd(lib, dq=MIS) == api.FA_ERR_MISALIGNED
    assert bwd_gqa(lib, resid=MIS) == api.FA_ERR_MISALIGNED
    assert bwd(lib, ws=A + 16) == api.FA_ERR_MISALIGNED  # workspace needs 256-byte alignment


def bwd_ws(lib, fws=A, fws_bytes=1 << 40, ws_bytes=1 << 40, B=1, H=1, N=16, d=64):
    return lib.fa_bwd_ws(A, A, A, A, A, A, A, A, A, A, B, H, H, N, d, 0.125, 0, fws, fws_bytes, A, ws_bytes, None)


@pytest.mark.parametrize("shape", [(1, 4, 1, 1, 64), (2, 32, 8, 8192, 128), (2, 16, 16, 2048, 128),
                                   (1, 2, 2, 300, 256), (3, 6, 3, 1000, 64)])
def test_backward_with_forward_workspace_sizes(lib, shape):
    # fa_bwd_gqa's workspace without its fp16 copy of V (B * H_kv * N * d halves)
    B, H, Hkv, N, d = shape
    assert api.fa_bwd_ws_workspace_size(*shape) == api.fa_bwd_gqa_workspace_size(*shape) - _align256(B * Hkv * N * d * 2)


def test_backward_with_forward_workspace_checks_its_arguments(lib):
    # every call here is rejected on the host (or is empty): nothing reaches a GPU
    fneed = api.fa_fwd_workspace_size(1, 1, 16, 64)
    assert bwd_ws(lib, fws=None) == api.FA_ERR_INVALID_ARG
    assert bwd_ws(lib, fws_bytes=fneed - 1) == api.FA_ERR_INVALID_ARG
    assert bwd_ws(lib, fws=A + 16) == api.FA_ERR_MISALIGNED
    assert bwd_ws(lib, ws_bytes=api.fa_bwd_ws_workspace_size(1, 1, 1, 16, 64) - 1) == api.FA_ERR_INVALID_ARG
    assert bwd_ws(lib, d=512) == api.FA_ERR_UNSUPPORTED
    assert bwd_ws(lib, d=96) == api.FA_ERR_UNSUPPORTED
    assert bwd_ws(lib, fws=None, N=0) == api.FA_OK  # empty problem: nothing to do


def test_f32_forward_argument_errors(lib):
    assert lib.fa_fwd_f32(None, A, A, A, A, 1, 1, 8, 64, 0.125, 0, None) == api.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_f32(A + 2, A, A, A, A, 1, 1, 8, 64, 0.125, 0, None) == api.FA_ERR_MISALIGNED
    assert lib.fa_fwd_f32(A, A, A, A, A, 1, 1, 8, 48, 0.125, 0, None) == api.FA_ERR_UNSUPPORTED


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_a_gpu_fails_loudly(lib):
    # all arguments valid: the call reaches the CUDA runtime, which has no device here
    assert fwd(lib) == api.FA_ERR_CUDA


def test_fp8_forward_checks_its_arguments(lib):
    import ctypes

    pr = api.FaAttnProblem(1, 4, 2, 300, 128, 0.125, 1, -1, -1)
    assert api.fa_attn_fwd_fp8_workspace_size(pr) == 256
    assert lib.fa_attn_fwd_fp8_workspace_size(None) == 0
    assert api.fa_attn_fwd_fp8_workspace_size(api.FaAttnProblem(1, 4, 2, 300, 128, 0.125, 1, -3, -1)) == 0

    def call(p=pr, q=A, o=A, lse=A, ws=A, ws_bytes=256, ds=(1.0, 1.0, 1.0)):
        return lib.fa_attn_fwd_fp8(None if p is None else ctypes.byref(p), q, A, A, *ds, o, lse, ws, ws_bytes, None)

    assert call(p=None) == api.FA_ERR_INVALID_ARG
    assert call(ds=(0.0, 1.0, 1.0)) == api.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, -1.0, 1.0)) == api.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, 1.0, float("inf"))) == api.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, float("nan"), 1.0)) == api.FA_ERR_INVALID_ARG
    assert call(p=api.FaAttnProblem(1, 4, 2, 300, 256, 0.0625, 1, -1, -1)) == api.FA_ERR_UNSUPPORTED  # d = 128, 64
    assert call(p=api.FaAttnProblem(1, 4, 2, 300, 96, 0.1, 1, -1, -1)) == api.FA_ERR_UNSUPPORTED
    assert call(p=api.FaAttnProblem(1, 6, 4, 300, 128, 0.125, 1, -1, -1)) == api.FA_ERR_INVALID_ARG
    assert call(q=None) == api.FA_ERR_INVALID_ARG
    assert call(ws=None) == api.FA_ERR_INVALID_ARG
    assert call(ws_bytes=255) == api.FA_ERR_INVALID_ARG
    assert call(q=MIS) == api.FA_ERR_MISALIGNED
    assert call(lse=A + 2) == api.FA_ERR_MISALIGNED
    assert call(ws=A + 16) == api.FA_ERR_MISALIGNED
    empty = api.FaAttnProblem(1, 4, 2, 0, 128, 0.125, 1, -1, -1)
    assert lib.fa_attn_fwd_fp8(ctypes.byref(empty), None, None, None, 1.0, 1.0, 1.0, None, None, None, 0,
                               None) == api.FA_OK


def test_head_dim_256_is_a_forward_with_workspace(lib):
    assert api.fa_fwd_workspace_size(1, 2, 300, 256) == _align256(1 * 2 * 300 * 256 * 2) + 256 + \
        _align256(4 * VPASS_BLOCKS)
    pr = api.FaAttnProblem(1, 4, 2, 300, 256, 0.0625, 1, -1, -1)
    assert api.fa_attn_fwd_workspace_size(pr) == api.fa_fwd_workspace_size(1, 2, 300, 256)
    # the backward takes d = 256 (one kernel per gradient, each with one unit per key tile)
    assert api.fa_bwd_workspace_size(1, 2, 300, 256) == _ws_expected(1, 2, 300, 256)
    assert api.fa_bwd_gqa_workspace_size(1, 4, 2, 300, 256) == _ws_expected_gqa(1, 4, 2, 300, 256)
    assert fwd(lib, d=256) == api.FA_ERR_UNSUPPORTED  # fa_fwd: no workspace, no d = 256 kernel
    # fa_fwd_ws without its workspace: the problem is valid, the missing workspace is the error
    assert lib.fa_fwd_ws(A, A, A, A, A, None, 1, 4, 2, 300, 256, 0.0625, 1, None, 0, None) == api.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_ws(A, A, A, A, A, None, 1, 4, 2, 300, 512, 0.0625, 1, A, 1 << 40, None) == \
        api.FA_ERR_UNSUPPORTED
    # rejected on the host before any launch: a missing workspace, an unsupported head dimension
    assert bwd(lib, d=256, ws=None) == api.FA_ERR_INVALID_ARG
    assert bwd(lib, d=512) == api.FA_ERR_UNSUPPORTED


def _align256(x):
    return (x + 255) // 256 * 256
