"""Seeded synthetic inputs for the 4-bit quantization path.

This module is shared by the tests (oracle side and GPU side alike), the
smoke check and the benchmark.  It only draws random numbers and names the
workload shapes; none of the quantization arithmetic lives here.

Recipe (every draw uses torch's own generator, seeded per tensor):
  * weights ~ N(0, 0.02^2): ``torch.randn`` in fp32 times 0.02;
  * outliers: ``torch.randperm`` picks ``round(frac * numel)`` positions whose
    fp32 values are multiplied by the outlier factor before any bf16 cast;
  * activations ~ N(0, 1): ``torch.randn`` in fp32;
  * bf16 tensors are the fp32 draw cast with ``.to(torch.bfloat16)``
    (round to nearest even).
The Llama-7B shapes follow the torch Linear convention W[out, in].
"""
from dataclasses import dataclass

import torch

WEIGHT_STD = 0.02
OUTLIER_FRAC = 0.001
OUTLIER_SCALE = 20.0


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_f32(shape, seed, std=1.0, device="cpu"):
    """fp32 N(0, std^2) tensor."""
    x = torch.randn(shape, generator=_gen(seed, device), dtype=torch.float32,
                    device=device)
    if std != 1.0:
        x.mul_(std)
    return x


def weight_bf16(rows, cols, seed, std=WEIGHT_STD, outlier_frac=0.0,
                outlier_scale=OUTLIER_SCALE, device="cpu"):
    """bf16 [rows, cols] weight ~ N(0, std^2) with an optional fraction of
    uniformly placed positions scaled by ``outlier_scale`` before the cast."""
    w = normal_f32((rows, cols), seed, std, device)
    if outlier_frac > 0.0:
        n = rows * cols
        k = int(round(outlier_frac * n))
        pos = torch.randperm(n, generator=_gen(seed + 7919, device),
                             device=device)[:k]
        w.view(-1)[pos] *= outlier_scale
    return w.to(torch.bfloat16)


def activations_bf16(B, K, seed, device="cpu"):
    """bf16 [B, K] activations ~ N(0, 1)."""
    return normal_f32((B, K), seed, 1.0, device).to(torch.bfloat16)


def bf16_bits(t):
    """numpy uint16 bit patterns of a CPU bf16 tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


# ---------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Linear:
    name: str
    N: int  # out features (W rows)
    K: int  # in features (W cols)


HIDDEN = 4096
FFN = 11008
N_LAYERS = 32


def llama7b_layer():
    """The seven linears of one Llama-7B decoder layer, W[out, in]."""
    return [Linear("q", HIDDEN, HIDDEN), Linear("k", HIDDEN, HIDDEN),
            Linear("v", HIDDEN, HIDDEN), Linear("o", HIDDEN, HIDDEN),
            Linear("gate", FFN, HIDDEN), Linear("up", FFN, HIDDEN),
            Linear("down", HIDDEN, FFN)]


def llama7b_stack(n_layers=N_LAYERS):
    """(layer, Linear) for every linear of the 32-layer stack, in order."""
    return [(l, lin) for l in range(n_layers) for lin in llama7b_layer()]


def stack_weight_seed(layer, idx):
    """Seed of weight ``idx`` (0..6) of decoder layer ``layer``."""
    return 1000 + 7 * layer + idx


# Named workloads (sizes of the five configurations of the method's brief).
ROUNDTRIP_N = 1 << 20              # fp32 vector, seed 0, blocksize 64, dq
MATRIX_4096 = (4096, 4096)         # bf16, 0.1% outliers x20, NF4 and FP4
GEMV_SHAPES = [(FFN, HIDDEN), (HIDDEN, FFN)]           # (N, K)
GEMV_BATCHES = [1, 8]
GEMM_M = 2048
GEMM_SHAPES = [(HIDDEN, HIDDEN), (FFN, HIDDEN), (HIDDEN, FFN)]  # (N, K)
