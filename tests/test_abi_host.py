"""Host-side checks of the C ABI: no GPU needed, no kernel launched."""
import ctypes
import math
import os
import re
from fractions import Fraction

import pytest

from moe_layer_gemm_b200 import abi, build
from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def _header_functions():
    src = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_every_header_function_is_exported(lib):
    names = _header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(abi.EXPORTED) == names


def test_status_strings_and_version(lib):
    assert abi.moe_version() >= 100
    for s in (0, -1, -2, -3, -4, -5):
        assert abi.moe_status_str(s).startswith("MOE_")
    assert abi.moe_status_str(-99) == "unknown status"


@pytest.mark.parametrize("T,K,E,cf", [
    (8192, 4, 60, 1.0), (64, 2, 8, 1.25), (30, 2, 3, 0.8), (30, 2, 3, 0.75), (1, 1, 1, 1e-30),
    (16384, 2, 8, 1.1), (4096, 8, 256, 0.3), (777, 3, 7, 2.0 / 3.0), (100, 2, 8, 0.0), (100, 2, 8, -1.0),
    (5, 1, 2, 1e6)])
def test_capacity_matches_oracle(lib, T, K, E, cf):
    d = abi.Dims(T, 128, 256, E, K, cf)
    want = O.capacity(T, K, E, cf)
    assert abi.moe_capacity(d) == (-1 if want is None else want)


def test_dims_validation(lib):
    good = abi.Dims(64, 128, 256, 8, 2)
    assert abi.moe_workspace_size(good) > 0
    bad = [abi.Dims(0, 128, 256, 8, 2), abi.Dims(64, 128, 256, 8, 9), abi.Dims(64, 128, 256, 0, 1),
           abi.Dims(64, 128, 256, 300, 2), abi.Dims(64, 8, 256, 8, 2), abi.Dims(1 << 25, 128, 256, 8, 2)]
    for d in bad:
        with pytest.raises(abi.MoEError) as e:
            abi.moe_workspace_size(d)
        assert e.value.status == abi.MOE_EINVAL
    with pytest.raises(abi.MoEError) as e:
        abi.moe_workspace_size(abi.Dims(64, 136, 256, 8, 2))  # d_model not a multiple of 16
    assert e.value.status == abi.MOE_EUNSUPPORTED
    assert abi.moe_capacity(abi.Dims(0, 128, 256, 8, 2)) < -1


def test_null_arguments_are_rejected_before_any_launch(lib):
    d = abi.Dims(64, 128, 256, 8, 2).c()
    ws_bytes = abi.moe_workspace_size(d)
    nul = None
    assert lib.moe_route(ctypes.byref(d), nul, nul, nul, nul, nul, nul, nul, nul, ws_bytes, nul) == abi.MOE_EINVAL
    assert lib.moe_permute(ctypes.byref(d), nul, nul, nul, nul, nul, nul, nul, nul, nul, nul, 0, nul) == abi.MOE_EINVAL
    assert lib.moe_combine(ctypes.byref(d), nul, nul, nul, nul, 0, nul) == abi.MOE_EINVAL
    assert lib.moe_layer_forward(ctypes.byref(d), nul, nul, nul, 0.0, nul, nul, nul, 0, nul, nul, 0, nul) == abi.MOE_EINVAL
    assert lib.moe_bias_update(ctypes.byref(d), nul, 0.001, nul, nul) == abi.MOE_EINVAL
    assert lib.moe_pack_weights(None, nul, nul, nul, nul, nul, nul) == abi.MOE_EINVAL


def test_workspace_too_small_and_misaligned(lib):
    d = abi.Dims(64, 128, 256, 8, 2).c()
    n = abi.moe_workspace_size(d)
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the size check fails first
    st = lib.moe_route_from_logits(ctypes.byref(d), fake, None, fake, fake, None, fake, n - 1, None)
    assert st == abi.MOE_EWORKSPACE
    st = lib.moe_route_from_logits(ctypes.byref(d), fake, None, fake, fake, None, ctypes.c_void_p(0x10008), n, None)
    assert st == abi.MOE_EINVAL


def test_workspace_grows_with_problem(lib):
    small = abi.moe_workspace_size(abi.Dims(64, 128, 256, 8, 2))
    big = abi.moe_workspace_size(abi.Dims(16384, 4096, 14336, 8, 2))
    assert big > small
    # at least x_perm + h + y_perm for the big case
    A = 16384 * 2
    assert big >= A * 4096 * 2 + A * 14336 * 2 + A * 4096 * 4


def test_noalloc_dispatch_rejects_oversize_on_the_host(lib):
    d = abi.Dims(70000, 64, 64, 256, 8).c()   # ceil(T/256) * E = 70144 > 65536 scratch entries
    fake = ctypes.c_void_p(0x10000)            # never dereferenced: the size check fails first
    st = lib.moe_permute_noalloc(ctypes.byref(d), fake, None, fake, fake, fake, fake, fake, None, None, None)
    assert st == abi.MOE_ESCRATCH
    assert abi.moe_status_str(abi.MOE_ESCRATCH).startswith("MOE_ESCRATCH")


def test_ffn_kernel_choice_by_shape(lib):
    # decode-sized groups with 256-multiple widths: weight-major CTA pairs
    assert abi.moe_ffn_kernel(abi.Dims(256, 4096, 14336, 8, 2)) == "grouped_gemm_2sm_kernel"
    # prefill-sized groups: token-major CTA pairs
    assert abi.moe_ffn_kernel(abi.Dims(16384, 4096, 14336, 8, 2)) == "grouped_gemm_2sm_kernel"
    # mid-sized groups (mean 546 rows) keep single-CTA tiles
    assert abi.moe_ffn_kernel(abi.Dims(8192, 2048, 1408, 60, 4, 1.0)) == "grouped_gemm_kernel"
    # widths that are not multiples of 256 cannot take 256-wide pair tiles
    assert abi.moe_ffn_kernel(abi.Dims(64, 128, 256, 8, 2)) == "grouped_gemm_kernel"
    bad = abi.Dims(0, 4096, 14336, 8, 2)
    with pytest.raises(abi.MoEError):
        abi.moe_ffn_kernel(bad)


def test_layer_launch_counts(lib):
    # decode: fused router, one-launch dispatch + gather, both GEMMs, combine (+ statistics tail)
    assert abi.moe_layer_launch_count(abi.Dims(256, 4096, 14336, 8, 2), True, False) == 4
    # statistics and the bias update add no launch
    assert abi.moe_layer_launch_count(abi.Dims(256, 4096, 14336, 8, 2), True, True) == 4
    # prefill (T > 4096): transpose + logits GEMM + top-K router, hist / scan / rank + gather, GEMMs, combine
    assert abi.moe_layer_launch_count(abi.Dims(16384, 4096, 14336, 8, 2), True, False) == 9
    # up to 4096 tokens the fused router: one launch
    assert abi.moe_layer_launch_count(abi.Dims(4096, 4096, 14336, 8, 2), True, False) == 7
    # E > 32: transpose + logits GEMM + top-K router; DeepSeek-like T = 4096 > 1024
    assert abi.moe_layer_launch_count(abi.Dims(4096, 7168, 2048, 256, 8), True, True) == 9


def test_layer_outputs_struct_matches_header():
    src = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    body = src[src.index("typedef struct moe_layer_outputs {"):src.index("} moe_layer_outputs;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\*\s*(\w+)\s*;", body)
    assert names == [n for n, _ in abi.moe_layer_outputs._fields_]


def test_chunked_workspace_and_host_checks(lib):
    big = abi.Dims(16384, 4096, 14336, 8, 2)
    full = abi.moe_workspace_size(big)
    chunked = abi.moe_chunked_workspace_size(big, 2048)
    # the expert stage buffers (x_perm, H, Y_perm) shrink with the chunk
    A_c = 2048 * 2
    assert chunked < full / 4
    assert chunked >= A_c * 4096 * 2 + A_c * 14336 * 2 + A_c * 4096 * 4
    # one chunk covering the batch needs about the unchunked workspace
    assert abi.moe_chunked_workspace_size(big, 16384) >= full
    # the last, shorter chunk may need more per-token room (a reduction split): it is covered
    odd = abi.Dims(4096 + 100, 1024, 2048, 8, 2)
    assert abi.moe_chunked_workspace_size(odd, 4096) >= abi.moe_workspace_size(abi.Dims(100, 1024, 2048, 8, 2))
    with pytest.raises(abi.MoEError):
        abi.moe_chunked_workspace_size(big, 0)
    # a capacity is defined over the whole batch: rejected before any launch
    d = abi.Dims(1000, 128, 256, 8, 2, 1.0).c()
    fake = ctypes.c_void_p(0x10000)   # never dereferenced
    st = lib.moe_layer_forward_chunked(ctypes.byref(d), 256, fake, fake, None, 0.0, fake, fake, fake, 0, None,
                                       fake, 1 << 30, None)
    assert st == abi.MOE_EUNSUPPORTED
    d = abi.Dims(1000, 128, 256, 8, 2).c()
    st = lib.moe_layer_forward_chunked(ctypes.byref(d), 0, fake, fake, None, 0.0, fake, fake, fake, 0, None,
                                       fake, 1 << 30, None)
    assert st == abi.MOE_EINVAL
    n = abi.moe_chunked_workspace_size(abi.Dims(1000, 128, 256, 8, 2), 256)
    st = lib.moe_layer_forward_chunked(ctypes.byref(d), 256, fake, fake, None, 0.0, fake, fake, fake, 0, None,
                                       fake, n - 1, None)
    assert st == abi.MOE_EWORKSPACE


def test_chunked_launch_counts(lib):
    # Mixtral prefill in 4 chunks of 4096: the router of the whole batch (16384 tokens: transpose + logits
    # GEMM + top-K) + 4 x (hist/scan/rank + gather, GEMMs, combine, counts) + the statistics CTA
    d = abi.Dims(16384, 4096, 14336, 8, 2)
    assert abi.moe_layer_chunked_launch_count(d, 4096, True, False) == 3 + 4 * (4 + 3) + 1
    # chunks of 1024 take the one-launch dispatch
    assert abi.moe_layer_chunked_launch_count(d, 1024, True, False) == 3 + 16 * (1 + 3) + 1
    # no statistics, no bias: no statistics CTA
    assert abi.moe_layer_chunked_launch_count(d, 16384, False, False) == 3 + (4 + 3)
    # a batch of 4096 tokens is routed by the fused router
    assert abi.moe_layer_chunked_launch_count(abi.Dims(4096, 4096, 14336, 8, 2), 1024, True, False) == 1 + 4 * (1 + 3) + 1
