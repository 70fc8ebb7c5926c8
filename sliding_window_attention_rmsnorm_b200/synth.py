"""Seeded synthetic inputs for the attention core.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests; it holds no attention or normalisation arithmetic, only random draws.

Inputs are i.i.d. N(0, 1) drawn in fp32 on the CPU with a torch.Generator and
rounded to bf16, so every consumer sees the same bits.  The pages train on
tokenised web text; the core itself only ever sees q, k, v and dO, whose
statistics after the QK norm are what matters, hence Gaussian stand-ins.

Seed of one tensor: 1000 * config + 10 * layer + {q: 0, k: 1, v: 2, dO: 3, ve: 4,
g: 5}; ve is a value embedding [B, T, Hkv, D] and g the gate logits [B, T, Hkv]
of the layers that mix one in (N(0,1) like the rest).
"""
import torch

_ROLE = {"q": 0, "k": 1, "v": 2, "dO": 3, "ve": 4, "g": 5}


def seed_of(config: int, layer: int, role: str) -> int:
    return 1000 * int(config) + 10 * int(layer) + _ROLE[role]


def normal_bf16(shape, seed: int) -> torch.Tensor:
    """N(0,1) drawn in fp32 from a seeded CPU generator, rounded to bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def layer_inputs(config: int, layer: int, B: int, T: int, H: int, D: int,
                 roles=("q", "k", "v", "dO")):
    """Dict role -> bf16 CPU tensor [B, T, H, D] for one layer of one workload."""
    return {r: normal_bf16((B, T, H, D), seed_of(config, layer, r)) for r in roles}


def peaked_keys(q: torch.Tensor, seed: int, noise: float = 0.1) -> torch.Tensor:
    """Keys close to the queries (k = q + noise * N(0,1)), to drive logits
    towards their bound; a stress input, bf16."""
    n = normal_bf16(tuple(q.shape), seed).float()
    return (q.float() + noise * n).to(torch.bfloat16)


def value_embedding(config: int, layer: int, B: int, T: int, Hkv: int, D: int):
    """(ve [B, T, Hkv, D], g [B, T, Hkv]) bf16 CPU tensors, seeded like the rest."""
    return (normal_bf16((B, T, Hkv, D), seed_of(config, layer, "ve")),
            normal_bf16((B, T, Hkv), seed_of(config, layer, "g")))
