"""Parameter and FLOP accounting of the oracle (test infrastructure only).

The model is the Qwen3-1.7B architecture with an untied embedding and LM head, about
2B parameters (jj-blog "PuRo-2B: ... RTX 5090 ...", the paragraph on the training
recipe). Its linear layers, per transformer block, are
  QKV  2048 -> 4096   (16 query + 8 key + 8 value heads of 128)
  O    2048 -> 2048
  gate/up 2048 -> 12288 (fused, 2 x 6144)
  down 6144 -> 2048
with 28 blocks, hidden size 2048 and a vocabulary of 151936.

Training compute uses the convention C = 6 N D, N the parameter count and D the tokens
(jj-blog page, the paragraph after Table 1, which names the formula; the walkthrough's
section "Cost decomposes into price times time" uses the same convention, its formula
lost in the page's text). For one linear layer with weight
[N_out, K_in] over T tokens, forward, dgrad and wgrad are three GEMMs of 2*T*N_out*K_in
FLOPs each, i.e. 6 * (N_out*K_in) * T: the linear part of 6ND.
"""

HIDDEN = 2048
LAYERS = 28
HEAD_DIM = 128
Q_HEADS = 16
KV_HEADS = 8
FFN = 6144
VOCAB = 151936


def layer_linears():
    """(name, N_out, K_in) of the four linear layers of one transformer block."""
    qkv_out = (Q_HEADS + 2 * KV_HEADS) * HEAD_DIM
    return [
        ("qkv", qkv_out, HIDDEN),
        ("o", HIDDEN, Q_HEADS * HEAD_DIM),
        ("gate_up", 2 * FFN, HIDDEN),
        ("down", HIDDEN, FFN),
    ]


def lm_head():
    return ("lm_head", VOCAB, HIDDEN)


def linear_params() -> int:
    """Weights that run through the blockwise-FP8 GEMMs: 28 blocks plus the LM head."""
    per_layer = sum(n * k for _, n, k in layer_linears())
    _, vn, vk = lm_head()
    return LAYERS * per_layer + vn * vk


def total_params() -> int:
    """All parameters: linears, the untied input embedding and the RMSNorm weights.

    Norms per block: two hidden-size norms plus the per-head query and key norms of
    the Qwen3 architecture; one final norm.
    """
    norms = LAYERS * (2 * HIDDEN + 2 * HEAD_DIM) + HIDDEN
    embedding = VOCAB * HIDDEN
    return linear_params() + embedding + norms


def flops_6nd(n_params: float, tokens: float) -> float:
    return 6.0 * n_params * tokens


def gemm_flops(m: int, n: int, k: int) -> int:
    """FLOPs of one GEMM C[m, n] = A[m, k] B[n, k]^T (one multiply + one add per MAC)."""
    return 2 * m * n * k


def microstep_gemms(tokens: int, layers: int = LAYERS, with_head: bool = True):
    """(op, name, M, N, K) of every blockwise GEMM of one micro-step over ``tokens``.

    fprop  Y  = X  W^T : M = T,     N = N_out, K = K_in
    dgrad  dX = dY W   : M = T,     N = K_in,  K = N_out
    wgrad  dW = dY^T X : M = N_out, N = K_in,  K = T
    """
    lins = [lin for _ in range(layers) for lin in layer_linears()]
    if with_head:
        lins.append(lm_head())
    out = []
    for name, n_out, k_in in lins:
        out.append(("fprop", name, tokens, n_out, k_in))
        out.append(("dgrad", name, tokens, k_in, n_out))
        out.append(("wgrad", name, n_out, k_in, tokens))
    return out


def microstep_flops(tokens: int, layers: int = LAYERS, with_head: bool = True) -> int:
    return sum(gemm_flops(m, n, k) for _, _, m, n, k in microstep_gemms(tokens, layers, with_head))
