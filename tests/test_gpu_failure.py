"""Failure detection on the GPU without a fault: the GEMM kernel's bounded
mbarrier waits are made to run out (its first X tile is never loaded, a flag
nothing sets), the kernel sets the library's device error word and exits,
bnb4_device_status reports the timeout, and the context stays usable for a
correct GEMM afterwards.  Nothing traps or hangs."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_nf4_b200 as bnb4
import oracle
import synth
from parity import check_linear, cpu_bits

pytestmark = pytest.mark.gpu


def _problem(M=256, N=256, K=512):
    W = synth.weight_bf16(N, K, seed=99)
    X = synth.activations_bf16(M, K, seed=98)
    st = oracle.quantize(synth.bf16_bits(W.view(-1)), 64, oracle.NF4, True)
    return X, st, N


def test_withheld_stage_times_out_and_context_survives():
    X, st, N = _problem()
    M, K = X.shape
    g = bnb4.state_from_arrays(st)
    Xd = X.cuda()
    stream = torch.cuda.current_stream().cuda_stream
    assert bnb4.bnb4_device_status(stream, True) == bnb4.OK
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    rc = bnb4.bnb4_debug_gemm_withhold(Xd.data_ptr(), M, K, g.cstruct(), N,
                                       Y.data_ptr(), 20000, stream)
    assert rc == bnb4.OK
    assert bnb4.bnb4_device_status(stream, True) == bnb4.ERR_DEVICE_TIMEOUT
    assert bnb4.bnb4_device_status(stream, True) == bnb4.OK   # cleared
    # the context is still usable: a normal GEMM is correct
    Y2 = bnb4.gemm_4bit(Xd, g, N)
    torch.cuda.synchronize()
    assert bnb4.bnb4_device_status(stream, True) == bnb4.OK
    What = oracle.dequantize(st, oracle.BF16).reshape(N, K)
    Xb = synth.bf16_bits(X)
    check_linear(cpu_bits(Y2), oracle.linear_ref(Xb, What), Xb, What)


def test_debug_entry_checks_its_limit():
    X, st, N = _problem(M=128, N=64, K=128)
    g = bnb4.state_from_arrays(st)
    Y = torch.empty(128, N, dtype=torch.bfloat16, device="cuda")
    Xd = X.cuda()
    for bad in (0, 1000001):
        assert bnb4.bnb4_debug_gemm_withhold(Xd.data_ptr(), 128, 128, g.cstruct(), N,
                                             Y.data_ptr(), bad, None) == bnb4.ERR_INVALID_ARG
