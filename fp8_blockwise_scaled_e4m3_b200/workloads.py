"""Seeded synthetic inputs for the blockwise-FP8 linear path.

This module only draws random tensors of the right shapes and distributions; it holds
none of the quantisation or GEMM arithmetic, so both the CUDA path and the CPU oracle
can take their inputs from it.

Shapes are those of a Qwen3-1.7B-shaped transformer block with an untied LM head
(jj-blog "PuRo-2B: ... RTX 5090 ...", the paragraph on the training recipe: Qwen3-1.7B
configuration, untied embedding and LM head, sequence length 4096): hidden 2048,
QKV 2048->4096, O 2048->2048, fused gate/up 2048->12288, down 6144->2048, vocabulary
151936, 28 blocks.

Distributions (drawn in FP32 with a seeded torch.Generator, then rounded to BF16):
  activations   N(0, 1); 1% of entries (Bernoulli) replaced by Student-t(3) draws
  weights       N(0, 0.02^2)
  output grads  1e-3 x (the activation recipe)
  dlogits       softmax(z) - onehot(target), z iid N(0, 2048 * 0.02^2) (the logit
                distribution a unit-variance hidden state meets at initialisation),
                targets uniform over the vocabulary
  small GEMM    A ~ N(0, 1) with columns {17, 130, 131, 400} multiplied by 50,
                W ~ N(0, 0.02^2)
Every tensor has its own generator, seeded from (workload seed, tensor index).
"""

import math

import torch

HIDDEN = 2048
FFN = 6144
QKV_OUT = 4096
VOCAB = 151936
LAYERS = 28
WEIGHT_STD = 0.02
GRAD_STD = 1e-3
HEAVY_FRAC = 0.01
HEAVY_NU = 3

# (name, N_out, K_in) of the four linears of one block, in forward order.
LINEARS = (
    ("qkv", QKV_OUT, HIDDEN),
    ("o", HIDDEN, HIDDEN),
    ("gate_up", 2 * FFN, HIDDEN),
    ("down", HIDDEN, FFN),
)
LM_HEAD = ("lm_head", VOCAB, HIDDEN)

SMALL_GEMM = dict(M=256, K=512, N=384, outlier_cols=(17, 130, 131, 400), outlier_scale=50.0)


def generator(seed: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 24) + int(index))
    return g


def normal(shape, std, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def heavy_tailed(shape, std, g, device) -> torch.Tensor:
    """N(0,1) with a Bernoulli(1%) mask of entries replaced by Student-t(3), times std."""
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(HEAVY_NU):
        chi2 += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
    t = z / torch.sqrt(chi2 / HEAVY_NU)
    mask = torch.rand(shape, generator=g, device=device) < HEAVY_FRAC
    x = torch.where(mask, t, x)
    return x * std


def bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def dlogits(tokens, vocab, g, device, hidden=HIDDEN, weight_std=WEIGHT_STD) -> torch.Tensor:
    """softmax(z) - onehot(target) per row, BF16 [tokens, vocab] (no 1/T loss scale)."""
    z = torch.randn((tokens, vocab), generator=g, device=device, dtype=torch.float32)
    z *= math.sqrt(hidden) * weight_std
    p = torch.softmax(z, dim=1)
    del z
    target = torch.randint(0, vocab, (tokens,), generator=g, device=device)
    p[torch.arange(tokens, device=device), target] -= 1.0
    return bf16(p)


def small_gemm(seed=0, device="cpu"):
    """A [256, 512] with outlier channels and W [384, 512], BF16."""
    c = SMALL_GEMM
    a = normal((c["M"], c["K"]), 1.0, generator(seed, 0, device), device)
    cols = torch.tensor(c["outlier_cols"], device=device)
    a[:, cols] *= c["outlier_scale"]
    w = normal((c["N"], c["K"]), WEIGHT_STD, generator(seed, 1, device), device)
    return bf16(a), bf16(w)


def layer_forward(seed, tokens, device, layer=0):
    """Inputs and weights of one block's four linears: [(name, X, W)], BF16."""
    out = []
    for i, (name, n_out, k_in) in enumerate(LINEARS):
        base = 64 * layer + 2 * i
        x = heavy_tailed((tokens, k_in), 1.0, generator(seed, base, device), device)
        w = normal((n_out, k_in), WEIGHT_STD, generator(seed, base + 1, device), device)
        out.append((name, bf16(x), bf16(w)))
    return out


def layer_grads(seed, tokens, device, layer=0):
    """Output gradients dY [tokens, N_out] of one block's four linears: [(name, dY)]."""
    out = []
    for i, (name, n_out, _) in enumerate(LINEARS):
        g = generator(seed, 64 * layer + 32 + i, device)
        out.append((name, bf16(heavy_tailed((tokens, n_out), GRAD_STD, g, device))))
    return out


def lm_head(seed, tokens, device, vocab=VOCAB):
    """Hidden states H [tokens, 2048], W_head [vocab, 2048], dlogits [tokens, vocab]."""
    h = normal((tokens, HIDDEN), 1.0, generator(seed, 10_000, device), device)
    w = normal((vocab, HIDDEN), WEIGHT_STD, generator(seed, 10_001, device), device)
    dl = dlogits(tokens, vocab, generator(seed, 10_002, device), device)
    return bf16(h), bf16(w), dl


def bf16_bits(t: torch.Tensor):
    """BF16 tensor -> NumPy uint16 array of its bit patterns (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
