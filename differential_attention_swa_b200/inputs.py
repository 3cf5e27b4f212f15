"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it draws N(0, 1) values from a
seeded CPU generator, rounds them to bf16, and lists the workload shapes.
Both the CUDA path and the CPU oracle consume what it produces.

Recipe: generator ``torch.Generator('cpu').manual_seed(seed + k)`` with
k = 0, 1, 2, ... for the tensors in the order listed (Q, K, V; or Q1, K1, Q2,
K2, V), fp32 ``randn``, then round-to-nearest-even to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


def randn_bf16(shape, seed: int) -> torch.Tensor:
    g = torch.Generator("cpu").manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def attn_inputs(B, Hq, Hkv, N, dqk, dv=None, seed: int = 0):
    dv = dqk if dv is None else dv
    q = randn_bf16((B, Hq, N, dqk), seed + 0)
    k = randn_bf16((B, Hkv, N, dqk), seed + 1)
    v = randn_bf16((B, Hkv, N, dv), seed + 2)
    return q, k, v


def diff_inputs(B, Hq, Hkv, N, dqk, dv, seed: int = 0):
    q1 = randn_bf16((B, Hq, N, dqk), seed + 0)
    k1 = randn_bf16((B, Hkv, N, dqk), seed + 1)
    q2 = randn_bf16((B, Hq, N, dqk), seed + 2)
    k2 = randn_bf16((B, Hkv, N, dqk), seed + 3)
    v = randn_bf16((B, Hkv, N, dv), seed + 4)
    return q1, k1, q2, k2, v


def decode_inputs(T, B, Hq, Hkv, d, W, seed: int = 0):
    """Cache pre-filled with W tokens, then T steps of new tokens."""
    k_cache = randn_bf16((B, Hkv, W, d), seed + 0)
    v_cache = randn_bf16((B, Hkv, W, d), seed + 1)
    q = randn_bf16((T, B, Hq, d), seed + 2)
    k_new = randn_bf16((T, B, Hkv, d), seed + 3)
    v_new = randn_bf16((T, B, Hkv, d), seed + 4)
    return q, k_new, v_new, k_cache, v_cache


def diff_decode_inputs(T, B, Hq, Hkv, dk, dv, W, seed: int = 0):
    """Caches pre-filled with W tokens (K1, K2, V), then T steps of new
    tokens and both maps' queries."""
    k1_cache = randn_bf16((B, Hkv, W, dk), seed + 0)
    k2_cache = randn_bf16((B, Hkv, W, dk), seed + 1)
    v_cache = randn_bf16((B, Hkv, W, dv), seed + 2)
    q1 = randn_bf16((T, B, Hq, dk), seed + 3)
    q2 = randn_bf16((T, B, Hq, dk), seed + 4)
    k1_new = randn_bf16((T, B, Hkv, dk), seed + 5)
    k2_new = randn_bf16((T, B, Hkv, dk), seed + 6)
    v_new = randn_bf16((T, B, Hkv, dv), seed + 7)
    return q1, q2, k1_new, k2_new, v_new, k1_cache, k2_cache, v_cache


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "swa", "strided", "global", "dilated", "swa_bwd", "diff", "decode", "diff_decode"
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    W: int
    S: int = 0
    dv: int | None = None
    lam: float = 0.0
    steps: int = 0  # decode steps
    pos0: int = 0  # decode: absolute position of the first step
    extra: dict = field(default_factory=dict)

    @property
    def dv_(self) -> int:
        return self.d if self.dv is None else self.dv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The workloads, by what they are. The decode cache holds the W tokens at
# positions pos0 - W .. pos0 - 1; step t adds position pos0 + t.
WORKLOADS = {
    "tiny_swa": Workload("tiny_swa", "swa", 1, 2, 2, 256, 64, 64),
    "tiny_strided": Workload("tiny_strided", "strided", 1, 2, 2, 256, 64, 16, S=8),
    "mistral_swa_prefill": Workload("mistral_swa_prefill", "swa", 2, 32, 8, 8192, 128, 4096),
    "local_strided_prefill": Workload("local_strided_prefill", "strided", 1, 16, 16, 16384, 64, 128, S=128),
    "diff_causal": Workload("diff_causal", "diff", 1, 16, 16, 4096, 64, 4096, dv=128, lam=0.8),
    "gemma_swa_prefill": Workload("gemma_swa_prefill", "swa", 1, 16, 8, 131072, 128, 1024),
    # the backward of the Mistral-style window attention (gradients of Q, K, V)
    "mistral_swa_backward": Workload("mistral_swa_backward", "swa_bwd", 2, 32, 8, 8192, 128, 4096),
    # the backward of the local + strided mask
    "local_strided_backward": Workload("local_strided_backward", "swa_bwd", 1, 16, 16, 16384, 64, 128, S=128),
    # window + global tokens with a Longformer-like shape (16 heads of 64,
    # a 512-token window, 64 global tokens at the start); S carries g
    "longformer_global_prefill": Workload("longformer_global_prefill", "global", 1, 16, 16, 16384, 64, 512, S=64),
    # the same shape with a dilated window (dilation 2, S carries it)
    "longformer_dilated_prefill": Workload("longformer_dilated_prefill", "dilated", 1, 16, 16, 16384, 64, 512, S=2),
    "gemma_swa_decode": Workload("gemma_swa_decode", "decode", 64, 16, 8, 0, 128, 1024, steps=256,
                                 pos0=131072),
    # the same decode with 4 attention-sink slots ahead of the window
    "gemma_sink_decode": Workload("gemma_sink_decode", "decode", 64, 16, 8, 0, 128, 1024, steps=256,
                                  pos0=131072, extra={"n_sink": 4}),
    # differential decode with the differential prefill's head dims and
    # context (4096-token window), GQA groups of 2: both maps share V
    "diff_gqa_decode": Workload("diff_gqa_decode", "diff_decode", 64, 16, 8, 0, 64, 4096, dv=128, lam=0.8,
                                steps=256, pos0=4096),
}
