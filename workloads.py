"""Seeded synthetic inputs for the W4A4 linear layer.

This module is shared by the tests, the benchmark and the oracle checks.  It
draws random numbers and nothing else: no rotation, quantisation or GEMM
arithmetic lives here.  Every tensor is made on the CPU from a seeded
``torch.Generator`` so that the CUDA path and the oracle see identical bits.

Distributions (stand-ins for the diffusion-transformer activations and
weights the pages measure on, which are not available):
  * activations x: bf16, i.i.d. N(0, 1), with a fraction p of the K input
    channels (round(p*K) distinct columns, chosen by a seeded permutation)
    multiplied by an outlier factor f in fp32 before the bf16 cast;
  * weights W: fp32, i.i.d. N(0, 0.02);
  * bias: bf16, i.i.d. N(0, 0.01).
"""

from dataclasses import dataclass, field

import torch


def make_activation(M, K, seed, outlier_frac=0.0, outlier_scale=1.0):
    """bf16 [M, K] activations with outlier channels (CPU tensor)."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn(M, K, generator=gen, dtype=torch.float32)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        cols = torch.randperm(K, generator=gen)[:n_out]
        x[:, cols] *= float(outlier_scale)
    return x.to(torch.bfloat16)


def make_weight(N, K, seed, std=0.02):
    """fp32 [N, K] weights (CPU tensor)."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed) + 1_000_003)
    return torch.randn(N, K, generator=gen, dtype=torch.float32) * std


def make_bias(N, seed, std=0.01):
    """bf16 [N] bias (CPU tensor)."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed) + 2_000_003)
    return (torch.randn(N, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)


def bf16_bits(t):
    """Raw uint16 bit patterns of a bf16 CPU tensor, as a numpy array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


@dataclass
class Linear:
    """One W4A4 linear workload: y[M, N] = x[M, K] W[N, K]^T (+ bias)."""
    name: str
    M: int
    K: int
    N: int
    g: int = 128
    seed: int = 0
    outlier_frac: float = 0.005
    outlier_scale: float = 30.0
    bias: bool = True
    act: int = 0                      # 0: none, 1: exact GELU before rotation
    notes: dict = field(default_factory=dict)

    def ops(self):
        return 2 * self.M * self.N * self.K

    def bytes(self):
        """Algorithmic HBM bytes of the fused layer: read x (bf16), the packed
        weight and its scales (and bias), write y (bf16)."""
        b = 2 * self.M * self.K + self.N * self.K // 2 + 4 * self.N + 2 * self.M * self.N
        if self.bias:
            b += 2 * self.N
        return b

    def make(self):
        x = make_activation(self.M, self.K, self.seed, self.outlier_frac, self.outlier_scale)
        w = make_weight(self.N, self.K, self.seed)
        b = make_bias(self.N, self.seed) if self.bias else None
        return x, w, b


# The workloads, named by what they are.
TINY = Linear("tiny 16x256->128 g128", M=16, K=256, N=128, g=128, seed=0,
              outlier_frac=0.01, outlier_scale=20.0, bias=False)
SQUARE = Linear("square 4608x3072->3072 g128", M=4608, K=3072, N=3072, g=128, seed=1)
MLP_UP = Linear("mlp up 4608x3072->12288 g128", M=4608, K=3072, N=12288, g=128, seed=2)
MLP_DOWN = Linear("mlp down 4608x12288->3072 g128 (gelu input)", M=4608, K=12288, N=3072,
                  g=128, seed=2, act=1)


def small_m_sweep():
    """Decode-like sweep: M in {1, 8, 16, 64} over four weight shapes."""
    out = []
    for (N, K) in [(12288, 3072), (3072, 12288), (5120, 5120), (3072, 3072)]:
        for M in (1, 8, 16, 64):
            out.append(Linear(f"small-m {M}x{K}->{N} g128", M=M, K=K, N=N, g=128,
                              seed=3, bias=False))
    return out


def block_stack(g=128, M=32760, blocks=10):
    """Transformer-block linear stack: per block q, k, v, out (5120x5120) and
    an MLP 5120->13824->5120; q/k/v read one shared quantised activation."""
    layers = []
    for b in range(blocks):
        for nm, K, N in (("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120),
                         ("out", 5120, 5120), ("up", 5120, 13824), ("down", 13824, 5120)):
            layers.append(Linear(f"block{b}.{nm} {M}x{K}->{N} g{g}", M=M, K=K, N=N, g=g,
                                 seed=4 + b, act=1 if nm == "down" else 0))
    return layers
