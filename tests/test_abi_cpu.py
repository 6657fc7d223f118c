"""The C-ABI library without a GPU: it builds, loads, exports every symbol
include/mmf.h declares, and its host-side logic (sizes, status strings,
argument checks that return before any CUDA call) behaves as documented."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mmf.h")


@pytest.fixture(scope="module")
def L():
    from bitlinear_rmsnorm_quant_b200 import build, mmf
    build.build()
    return mmf.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mmf_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("mmf_pack_ternary", "mmf_bitlinear_fwd", "mmf_quantize_act", "mmf_ternary_acc",
                 "mmf_check_async", "mmf_workspace_bytes", "mmf_packed_bytes"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    from bitlinear_rmsnorm_quant_b200 import mmf
    for name in declared_functions():
        assert hasattr(L, name), f"{name} not exported"
        assert name in mmf.SIGNATURES, f"{name} not bound"


def test_library_is_sm100a_only():
    from bitlinear_rmsnorm_quant_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)


def test_sizes(L):
    assert L.mmf_packed_bytes(2560, 6912) == 2560 * 6912 // 4
    assert L.mmf_packed_bytes(-1, 128) == 0
    # up to 3 tokens take the fused CUDA-core decode kernel: no workspace
    assert L.mmf_workspace_bytes(1, 2560, 2560) == 0
    assert L.mmf_workspace_bytes(3, 6912, 2560) == 0
    # 4 .. 32 tokens: the codes in the decode tensor-core kernel's operand layout
    # (16 or 32 token rows per 128-wide K chunk) + absmax + qsum, 256-byte aligned
    assert L.mmf_workspace_bytes(4, 6912, 2560) == 16 * 6912 + 2 * 256
    assert L.mmf_workspace_bytes(9, 6912, 2560) == 16 * 6912 + 2 * 256
    # large M: int8 codes + absmax + qsum, each 256-byte aligned
    M, K = 8192, 2048
    assert L.mmf_workspace_bytes(M, K, 5632) == M * K + 2 * ((4 * M + 255) // 256 * 256)
    assert L.mmf_workspace_bytes(9, 256, 100) >= 9 * 256
    # unsupported K
    assert L.mmf_workspace_bytes(100, 100, 100) == 0


def test_status_strings(L):
    from bitlinear_rmsnorm_quant_b200 import mmf
    for code, name in mmf.STATUS.items():
        assert L.mmf_status_string(code).decode() == name
    assert L.mmf_status_string(99).decode() == "MMF_ERR_UNKNOWN"
    assert L.mmf_version().decode().startswith("mmf ")


# Fake, never-dereferenced device addresses: the checks below return before
# the library touches CUDA.
A = 0x10000
MIS = 0x10008


def test_argument_errors_need_no_device(L):
    # null pointers
    assert L.mmf_pack_ternary(None, 16, 128, 1e-5, A, A, None) == 1
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, None, A, 1, 128, 16, A, None, 0, None) == 1
    assert L.mmf_quantize_act(A, None, 1e-6, 1, 128, A, A, None) == 1
    assert L.mmf_ternary_acc(A, A, 1, 128, 16, None, None, 0, None) == 1
    # bad eps
    assert L.mmf_pack_ternary(A, 16, 128, -1.0, A, A, None) == 1
    assert L.mmf_quantize_act(A, A, float("nan"), 1, 128, A, A, None) == 1
    # K not a positive multiple of 128, or above the limit
    for K in (0, 64, 100, 130, 65536 + 128):
        assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 1, K, 16, A, None, 0, None) == 2
    # negative sizes
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, -1, 128, 16, A, None, 0, None) == 1
    # misaligned pointers
    assert L.mmf_bitlinear_fwd(MIS, A, 1e-6, A, A, 1, 128, 16, A, None, 0, None) == 3
    assert L.mmf_pack_ternary(A, 16, 128, 1e-5, MIS, A, None) == 3
    assert L.mmf_hbm_copy(A, MIS, 64, None) == 3
    assert L.mmf_hbm_copy(A, A, 15, None) == 1
    # missing or short workspace on the large-M path
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 4096, 2048, 2048, A, None, 0, None) == 4
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 4096, 2048, 2048, A, A, 1024, None) == 4
    assert L.mmf_ternary_acc(A, A, 4096, 2048, 2048, A, None, 0, None) == 4
    # empty problems are no-ops that launch nothing
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 0, 128, 16, A, None, 0, None) == 0
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 3, 128, 0, A, None, 0, None) == 0
    assert L.mmf_pack_ternary(A, 0, 128, 1e-5, A, A, None) == 0
    assert L.mmf_hbm_copy(A, A, 0, None) == 0


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_no_device_is_reported(L):
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 1, 128, 16, A, None, 0, None) == 7
    assert L.mmf_check_async(None) == 7


def test_binding_fails_loudly_without_library(monkeypatch):
    from bitlinear_rmsnorm_quant_b200 import mmf
    monkeypatch.setattr(mmf, "_lib", None)
    monkeypatch.setattr(mmf, "LIB_PATH", "/nonexistent/libmmf.so")
    with pytest.raises(RuntimeError, match="missing"):
        mmf.lib()


def test_group_argument_errors(L):
    from bitlinear_rmsnorm_quant_b200 import mmf
    arr = (mmf.Projection * 1)()
    arr[0] = mmf.Projection(A, A, A, 16)
    f = L.mmf_bitlinear_fwd_group
    assert f(A, A, 1e-6, 1, 128, None, 1, None, 0, 0, None) == 1          # no descriptors
    assert f(A, A, 1e-6, 1, 128, arr, 0, None, 0, 0, None) == 1           # count 0
    assert f(A, A, 1e-6, 1, 128, arr, 9, None, 0, 0, None) == 1           # count above the limit
    assert f(A, A, 1e-6, 1, 128, arr, 1, None, 0, 4, None) == 1           # unknown flag
    assert f(A, A, 1e-6, 1, 100, arr, 1, None, 0, 0, None) == 2           # bad K
    arr[0] = mmf.Projection(A, A, None, 16)
    assert f(A, A, 1e-6, 1, 128, arr, 1, None, 0, 0, None) == 1           # null y
    arr[0] = mmf.Projection(A, MIS, A, 16)
    assert f(A, A, 1e-6, 1, 128, arr, 1, None, 0, 1, None) == 3           # misaligned scale
    arr[0] = mmf.Projection(None, None, None, 0)
    assert f(None, None, 1e-6, 1, 128, arr, 1, None, 0, 0, None) == 0     # empty group
    arr[0] = mmf.Projection(A, A, A, 16)
    assert f(A, A, 1e-6, 4096, 2048, arr, 1, None, 0, 0, None) == 4       # large M needs workspace


def test_glu_argument_errors(L):
    f = L.mmf_bitlinear_fwd_glu
    assert f(A, None, A, 1e-6, A, A, 1, 128, 16, A, None, 0, 0, None) == 1      # no u
    assert f(A, A, A, 1e-6, A, A, 1, 128, 16, A, None, 0, 2, None) == 1        # unknown flag
    assert f(A, A, A, -1.0, A, A, 1, 128, 16, A, None, 0, 0, None) == 1        # bad eps
    assert f(A, A, A, 1e-6, A, A, 1, 100, 16, A, None, 0, 0, None) == 2        # bad K
    assert f(A, MIS, A, 1e-6, A, A, 1, 128, 16, A, None, 0, 0, None) == 3      # misaligned u
    assert f(A, A, A, 1e-6, A, A, 4096, 2048, 2048, A, None, 0, 0, None) == 4  # missing workspace
    assert f(None, None, None, 1e-6, None, None, 0, 128, 16, None, None, 0, 0, None) == 0  # empty


def test_mlgru_scan_argument_errors(L):
    f = L.mmf_mlgru_scan
    assert f(A, A, A, None, 1, 4, 65, A, A, None) == 2      # odd D
    assert f(A, A, A, None, -1, 4, 64, A, A, None) == 1     # negative size
    assert f(A, None, A, None, 1, 4, 64, A, A, None) == 1   # missing input
    assert f(A, A, A, MIS, 1, 4, 64, A, A, None) == 3       # misaligned h0
    assert f(None, None, None, None, 0, 4, 64, None, None, None) == 0  # empty


def test_bwd_argument_errors(L):
    f = L.mmf_bitlinear_bwd
    need = L.mmf_bwd_workspace_bytes(64, 256, 128)
    assert need >= 64 * 256 * 4
    assert f(A, A, A, 1e-6, A, A, 64, 256, 128, A, A, A, None, 0, None) == 1       # no workspace
    assert f(A, A, A, 1e-6, A, A, 64, 100, 128, A, A, A, A, need, None) == 2       # bad K
    assert f(A, A, A, 1e-6, A, A, 64, 256, 128, A, A, MIS, A, need, None) == 3     # misaligned dW
    assert f(A, A, A, 1e-6, A, A, 64, 256, 128, A, A, A, A, need - 1, None) == 4   # short workspace


def test_shape_limits(L):
    f = L.mmf_bitlinear_fwd
    big_ws = 1 << 62  # claimed workspace size: the shape checks come first
    # tokens beyond the forward's stated limit (65535 * 256); a weight matrix beyond 2^40 elements
    assert f(A, A, 1e-6, A, A, 65535 * 256 + 1, 128, 16, A, A, big_ws, None) == 2
    assert f(A, A, 1e-6, A, A, 16, 65536, (1 << 24) + 16, A, A, big_ws, None) == 2
    # the allocation-free call refuses shapes whose workspace exceeds its static scratch
    assert L.mmf_bitlinear_fwd_noalloc(A, A, 1e-6, A, A, 65536, 2048, 2048, A, None) == 4
    # the backward's dgamma grid limit (K beyond the fused RMSNorm backward's)
    need = L.mmf_bwd_workspace_bytes(65535 * 64 + 1, 8320, 16)
    assert L.mmf_bitlinear_bwd(A, A, A, 1e-6, A, A, 65535 * 64 + 1, 8320, 16, A, A, A, A, need, None) == 2
    # the timeout self-test needs a limit within the library's own
    assert L.mmf_selftest_timeout(0, None, None) == 1


def test_launch_counts_follow_the_path(L):
    # up to 3 tokens: one launch; 4 .. 32 tokens: quantiser + contraction; more: quantiser + one per projection
    assert L.mmf_fwd_launches(1, 2560, 7680, 3) == 1
    assert L.mmf_fwd_launches(3, 2560, 7680, 3) == 1
    assert L.mmf_fwd_launches(4, 2560, 7680, 3) == 2
    assert L.mmf_fwd_launches(9, 2560, 7680, 3) == 2
    assert L.mmf_fwd_launches(32, 6912, 2560, 1) == 2
    assert L.mmf_fwd_launches(33, 2560, 7680, 3) == 4
    assert L.mmf_fwd_launches(8192, 2048, 2048, 1) == 2
    assert L.mmf_fwd_launches(0, 2560, 2560, 1) == 0 and L.mmf_fwd_launches(4, 100, 2560, 1) == 0


def test_workspace_sizes_follow_the_path(L):
    # up to 3 tokens (the CUDA-core decode kernel) need none; 4 .. 32 tokens (the
    # decode tensor-core kernel) need the codes as 16 or 32 operand rows per K
    # chunk and the per-token absmax and code sums; the large-M path the codes,
    # absmax and sums of every token
    a256 = lambda v: (v + 255) // 256 * 256
    for K in (128, 2560, 6912):
        assert L.mmf_workspace_bytes(1, K, 256) == 0
        assert L.mmf_workspace_bytes(3, K, 256) == 0
        for M in (4, 8, 9, 16):
            assert L.mmf_workspace_bytes(M, K, 256) == a256(16 * K) + 2 * a256(4 * M)
        for M in (17, 32):
            assert L.mmf_workspace_bytes(M, K, 256) == a256(32 * K) + 2 * a256(4 * M)
        assert L.mmf_workspace_bytes(33, K, 256) == a256(33 * K) + 2 * a256(4 * 33)
        assert L.mmf_workspace_bytes(8192, K, 256) >= 8192 * K + 8 * 8192
    # a single token too wide for the decode kernel's shared memory takes the large-M path
    assert L.mmf_workspace_bytes(1, 65536, 256) >= 65536


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_largest_k_passes_the_shape_checks(L):
    # K = 65536 is inside the limit: the call gets as far as looking for a device
    assert L.mmf_bitlinear_fwd(A, A, 1e-6, A, A, 1, 65536, 16, A, A, 1 << 30, None) == 7
    assert L.mmf_quantize_act(A, A, 1e-6, 4096, 65536, A, A, None) == 7
