"""Seeded synthetic workloads for the 2:4 activation-sparse linear layer.

This module only draws random inputs; it holds none of the layer's arithmetic
(no selection, compensation or matrix products), so both the CUDA path and the
CPU oracle can be fed from it without sharing any of the method.

Every tensor is returned as a numpy ``uint16`` array of bf16 bit patterns.
Values are drawn in float32 with ``numpy.random.default_rng`` and rounded to
bf16 by torch's float32 -> bfloat16 conversion (round to nearest even).

Shapes and distributions are those of the DiT linear layers the RT-Lynx pages
measure (qingkeai.online article section 05; neuraltrendhub summary: only
about 5-10% of neurons are active per token):

* activation mixture -- each element independently is "large" with
  probability 0.08 and then N(0, 1), else N(0, 0.05) (sigma = std-dev);
* GELU inputs (MLP down-projection) -- GELU (tanh form) of N(-0.5, 1), computed
  in float32 and then rounded;
* W ~ N(0, 1/sqrt(K)), bias ~ N(0, 0.02), LoRA A [r,K] and B [N,r] ~ N(0, 0.01),
  r = 64.
"""
from dataclasses import dataclass

import numpy as np

LORA_RANK = 64


@dataclass(frozen=True)
class LinearShape:
    name: str
    M: int
    K: int
    N: int
    r: int = LORA_RANK
    seed: int = 0
    x_kind: str = "mixture"  # "mixture" or "gelu"

    @property
    def dense_flops(self) -> int:
        """Dense-equivalent work 2*M*N*K of the main product."""
        return 2 * self.M * self.N * self.K


CONFIGS = {
    "tiny": LinearShape("tiny", M=256, K=512, N=512, seed=0),
    "attn_out": LinearShape("attn_out", M=4096, K=3072, N=3072, seed=2),
    "mlp_up": LinearShape("mlp_up", M=4608, K=3072, N=12288, seed=3),
    "mlp_down": LinearShape("mlp_down", M=4608, K=12288, N=3072, seed=4, x_kind="gelu"),
}

# Full DiT block sweep: M = 8192 tokens (two 1024^2 latents), hidden 3072.
SWEEP_M = 8192
SWEEP_LAYERS = (
    ("qkv", 3072, 9216, "mixture"),
    ("out", 3072, 3072, "mixture"),
    ("up", 3072, 12288, "mixture"),
    ("down", 12288, 3072, "gelu"),
)
SWEEP_BLOCKS = 8
SWEEP_SEED = 5


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) with torch; return uint16 bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _gelu_tanh_f32(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float32)
    c = np.float32(np.sqrt(2.0 / np.pi))
    return (np.float32(0.5) * z *
            (np.float32(1.0) + np.tanh(c * (z + np.float32(0.044715) * z * z * z)))).astype(np.float32)


def draw_activations(rng: np.random.Generator, M: int, K: int, kind: str) -> np.ndarray:
    """Activation X [M,K] as float32 (before rounding)."""
    if kind == "mixture":
        large = rng.random((M, K), dtype=np.float32) < np.float32(0.08)
        x = rng.standard_normal((M, K), dtype=np.float32)
        return np.where(large, x, x * np.float32(0.05)).astype(np.float32)
    if kind == "gelu":
        z = rng.standard_normal((M, K), dtype=np.float32) + np.float32(-0.5)
        return _gelu_tanh_f32(z)
    raise ValueError(f"unknown activation kind {kind!r}")


def make_linear_inputs(M: int, K: int, N: int, r: int = LORA_RANK, seed=0,
                       x_kind: str = "mixture", bias: bool = True, lora: bool = True) -> dict:
    """Inputs of one linear layer, in a fixed drawing order: X, W, bias, A, B.

    ``seed`` is anything ``numpy.random.default_rng`` accepts (an int or a
    sequence of ints).  Returns bf16 bit arrays ``X`` [M,K], ``W`` [N,K],
    ``bias`` [N] or None, ``A`` [r,K] / ``B`` [N,r] or None.
    """
    rng = np.random.default_rng(seed)
    X = f32_to_bf16_bits(draw_activations(rng, M, K, x_kind))
    W = f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / np.sqrt(K)))
    b = f32_to_bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(0.02))
    A = f32_to_bf16_bits(rng.standard_normal((r, K), dtype=np.float32) * np.float32(0.01))
    B = f32_to_bf16_bits(rng.standard_normal((N, r), dtype=np.float32) * np.float32(0.01))
    return {"X": X, "W": W, "bias": b if bias else None,
            "A": A if lora else None, "B": B if lora else None}


def make_config_inputs(name: str, **kw) -> dict:
    c = CONFIGS[name]
    return make_linear_inputs(c.M, c.K, c.N, c.r, seed=c.seed, x_kind=c.x_kind, **kw)


def make_rank_inputs(name: str, rank: int, **kw) -> dict:
    """One data-parallel rank's inputs of a named workload.

    Token rows are independent, so the layer shards by rows: every rank holds
    the same W, bias, A and B (the config's own draws) and its own batch of
    activations.  Rank 0's batch is the config's X; rank q > 0 draws a fresh X
    of the same shape and kind from the seed ``[config seed, q]``.
    """
    c = CONFIGS[name]
    inp = make_config_inputs(name, **kw)
    if rank > 0:
        rng = np.random.default_rng([c.seed, rank])
        inp["X"] = f32_to_bf16_bits(draw_activations(rng, c.M, c.K, c.x_kind))
    return inp


def sweep_skip_blocks() -> list:
    """The 2 of 8 blocks whose linears are left dense (selective layer skipping)."""
    rng = np.random.default_rng(SWEEP_SEED)
    return sorted(int(b) for b in rng.choice(SWEEP_BLOCKS, 2, replace=False))


def sweep_layer_seed(block: int, layer: int):
    """Independent seed of one linear of the block sweep."""
    return [SWEEP_SEED, block, layer]


def sweep_plan(M: int = SWEEP_M):
    """List of (block, layer_name, M, K, N, x_kind, skip, seed) for the block sweep."""
    skip = set(sweep_skip_blocks())
    plan = []
    for b in range(SWEEP_BLOCKS):
        for li, (lname, K, N, kind) in enumerate(SWEEP_LAYERS):
            plan.append((b, lname, M, K, N, kind, b in skip, sweep_layer_seed(b, li)))
    return plan
