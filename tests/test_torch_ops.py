"""The bnb4:: torch operators and the Linear4bit module, without a GPU: the
operators are registered, their fake (shape-only) implementations give the
shapes, dtypes and devices the real ones return (so a graph calling them can
be traced), and the module holds its full-precision weight until it is moved
to a CUDA device."""
import pytest
import torch
from torch._subclasses.fake_tensor import FakeTensorMode

import bit_blockwise_weight_nf4_b200 as bnb4
from bit_blockwise_weight_nf4_b200 import torch_ops


def test_operators_registered():
    for name in ("quantize_4bit", "dequantize_4bit", "gemv_4bit", "gemm_4bit", "linear_4bit"):
        assert hasattr(torch.ops.bnb4, name), name


@pytest.mark.parametrize("n,bs,dq", [(1000, 64, True), (4096 * 3 + 7, 32, True),
                                     (129, 256, False)])
def test_quantize_fake_shapes(n, bs, dq):
    nb = -(-n // bs)
    with FakeTensorMode():
        x = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        codes, absmax, absmax_q, scale2, offset = torch.ops.bnb4.quantize_4bit(x, bs, bnb4.NF4, dq)
    assert codes.shape == ((n + 1) // 2,) and codes.dtype == torch.uint8
    assert absmax.shape == (nb,) and absmax.dtype == torch.float32
    if dq:
        assert absmax_q.shape == (nb,) and scale2.shape == (-(-nb // 256),)
        assert offset.shape == (1,)
    else:
        assert absmax_q.numel() == 0 and scale2.numel() == 0 and offset.numel() == 0
    assert codes.device.type == "cuda"


def test_linear_and_dequant_fake_shapes():
    with FakeTensorMode():
        W = torch.empty(384, 1024, dtype=torch.float16, device="cuda")
        st = torch.ops.bnb4.quantize_4bit(W, 64, bnb4.FP4, True)
        x = torch.empty(17, 1024, dtype=torch.float16, device="cuda")
        b = torch.empty(384, dtype=torch.float16, device="cuda")
        y = torch.ops.bnb4.linear_4bit(x, *st, 384, 64, bnb4.FP4, True, b)
        w = torch.ops.bnb4.dequantize_4bit(*st, 384 * 1024, 64, bnb4.FP4, True, torch.float16)
        g = torch.ops.bnb4.gemm_4bit(x.bfloat16(), *st, 384, 64, bnb4.FP4, True)
        v = torch.ops.bnb4.gemv_4bit(x[:2].bfloat16(), *st, 384, 64, bnb4.FP4, True)
    assert y.shape == (17, 384) and y.dtype == torch.float16
    assert w.shape == (384 * 1024,) and w.dtype == torch.float16
    assert g.shape == (17, 384) and g.dtype == torch.bfloat16
    assert v.shape == (2, 384)


def test_linear4bit_module_before_quantization():
    m = torch_ops.Linear4bit(64, 32, bias=True, compute_dtype=torch.float16)
    assert not m.quantized
    assert set(m.state_dict()) == {"weight", "bias"}
    assert m.weight.dtype == torch.float16
    ref = torch.nn.Linear(64, 32).half()
    m.load_state_dict(ref.state_dict())
    assert torch.equal(m.weight, ref.weight)
    with pytest.raises(RuntimeError, match="CUDA"):
        m(torch.zeros(2, 64, dtype=torch.float16))
    with pytest.raises(TypeError):
        torch_ops.Linear4bit(64, 32, compute_dtype=torch.float32)
