"""The expert GEMMs' device-side timeout paths, run on purpose without a fault.

moe_test_set_wait_limits shortens the kernels' bounded waits and makes the
down projection's readiness target unreachable.  Every CTA (or CTA pair)
then gives up on its first down-projection tile: the wait records
MOE_ETIMEOUT with detail 6 (the readiness wait) in the workspace status
flag, raises the abort flag so every other role stops, the producer drains
the copies in flight (the pair leader after reconciling with its peer), the
MMA issuer waits for its last MMAs, and TMEM is freed before the kernel
returns.  The tests check that status, that the call ends quickly, that the
GPU still answers, and that a normal call in the same process afterwards
matches the oracle.  Nothing here can fault: no access changes, only the
value a wait compares with.
"""
import time

import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from tests.gpu_util import LayerInputs, oracle_layer
from tests.test_gpu_layer import _check, _forward

pytestmark = pytest.mark.gpu

DEP_TIMEOUT = 6


def _aborted_then_normal(name, T, kernel):
    inp = LayerInputs(synth.get_workload(name), T=T)
    assert abi.moe_ffn_kernel(inp.dims) == kernel
    y = torch.empty(inp.T, inp.wl.d_model, dtype=torch.float32, device=inp.x.device)
    abi.moe_reset_device_status(inp.ws)
    torch.cuda.synchronize()
    try:
        abi.moe_test_set_wait_limits(1 << 20, 1 << 14, True)
        t0 = time.perf_counter()
        abi.moe_layer_forward(inp.dims, inp.x, inp.Wr, None, 0.0, inp.W13p, inp.W2p, y, inp.ws)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        abi.moe_test_set_wait_limits(0, 0, False)
    st, detail = abi.moe_get_device_status(inp.ws)
    assert st == abi.MOE_ETIMEOUT and detail == DEP_TIMEOUT, (st, detail)
    assert elapsed < 10.0, elapsed
    # the context is intact: plain work runs, then the layer itself
    z = torch.arange(1 << 20, device=inp.x.device, dtype=torch.float32)
    assert float(z.sum().item()) == float((1 << 20) * ((1 << 20) - 1) / 2)
    yn, outs = _forward(inp)   # resets the status and asserts it stays clear
    tokens = sorted(set(np.linspace(0, T - 1, min(T, 24)).astype(int).tolist()))
    ref = oracle_layer(inp, tokens=tokens)
    _check(inp, yn, outs, ref, tokens=tokens)


def test_timeout_single_cta_kernel():
    _aborted_then_normal("tiny", 64, "grouped_gemm_kernel")


def test_timeout_cta_pair_kernel():
    _aborted_then_normal("mixtral_decode", 64, "grouped_gemm_2sm_kernel")


def test_timeout_cta_pair_token_major_tiles():
    # groups of ~1024 rows: token-major 256 x 256 pair tiles
    _aborted_then_normal("mixtral_prefill", 4096, "grouped_gemm_2sm_kernel")


def test_timeout_cta_pair_both_queues():
    # skewed groups above and below 128 rows: token-major pairs (two k-blocks
    # per stage) and weight-major pairs (one) abort and drain in one launch
    _aborted_then_normal("deepseek_bias", 1024, "grouped_gemm_2sm_kernel")
