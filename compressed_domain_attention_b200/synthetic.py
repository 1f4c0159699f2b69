"""Seeded synthetic K/V/q generators shared by the tests, the smoke check and the bench.

This module draws random numbers only; it holds none of the method's arithmetic
(no rotation, no quantisation, no attention). Both the CUDA path and the CPU
oracle consume exactly the tensors it returns.

Recipe (stands in for the pages' real-model workloads: Llama-3.1-70B,
Llama-3-8B, Gemma-3-1B shaped heads; no weights or datasets are used). One
``torch.Generator`` seeded with the workload's seed is drawn in this order:

1. K base ~ N(0, 1), shape [B][T][Hkv][D] (ragged workloads: one [len_b][Hkv][D]
   block per sequence, in sequence order);
2. per (kv-head, channel) log-scales z ~ N(0, 1); K is multiplied by e^z
   (log-normal channel scales, sigma = 1);
3. per kv-head outlier channels ``randperm(D)[:D // 32]`` (4 at D = 128, 8 at
   D = 256), multiplied by a further 10;
4. V ~ N(0, 1), same shape as K;
5. q ~ N(0, 1), shape [B][Hq][D];
6. the appended-token K (times the same channel multipliers) and V, shape
   [B][n_append][Hkv][D].

The tensors are then cast to the workload dtype (bf16 by round-to-nearest-even,
or kept fp32). Ragged lengths are drawn first, from their own generator with the
same seed, as ``randint(lo, hi + 1, (B,))``.

Step 2 draws z before step 1's K is scaled, so the draw order above is the
order in which the generator is consumed: K base, z, outlier permutations, V, q,
appended K, appended V.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_lens: List[int]          # prefix length per sequence already in the cache
    dtype: torch.dtype           # dtype of k, v, q as handed to the library
    seed: int
    n_append: int = 0            # tokens appended per sequence after the prefix
    max_seq: Optional[int] = None
    sm_scale: Optional[float] = None
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def capacity(self) -> int:
        if self.max_seq is not None:
            return self.max_seq
        return max(self.seq_lens) + self.n_append

    @property
    def scale(self) -> float:
        return self.sm_scale if self.sm_scale is not None else self.head_dim ** -0.5


def tiny_single_head() -> Workload:
    """B1, 1 q-head / 1 kv-head, D128, 256-token context, fp32, seed 0, one decode query."""
    return Workload("tiny_single_head_d128_t256_fp32", 1, 1, 1, 128, [256], torch.float32, 0)


def llama3_8b_layer() -> Workload:
    """B1, 32/8 heads (GQA 4), D128, 4096-token prefix, bf16, seed 1; plus a 1-token append."""
    return Workload("llama3_8b_gqa4_d128_t4096_bf16", 1, 32, 8, 128, [4096], torch.bfloat16, 1, n_append=1)


def gemma3_1b_sweep(T: int) -> Workload:
    """B1, 4/1 heads, D256, context T in {256 .. 4096}, bf16, seed 2."""
    return Workload(f"gemma3_1b_mqa4_d256_t{T}_bf16", 1, 4, 1, 256, [T], torch.bfloat16, 2)


def llama31_70b_long() -> Workload:
    """B1, 64/8 heads (GQA 8), D128, 131072-token context, bf16, seed 3."""
    return Workload("llama31_70b_gqa8_d128_t131072_bf16", 1, 64, 8, 128, [131072], torch.bfloat16, 3)


def ragged_lengths(seed: int, batch: int, lo: int, hi: int) -> List[int]:
    g = torch.Generator("cpu").manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g)]


def ragged_serving() -> Workload:
    """32 sequences, lengths U{1024..32768} (seed 4), 32/8 heads, D128, bf16; per step 1 appended token each."""
    lens = ragged_lengths(4, 32, 1024, 32768)
    return Workload("ragged_serving_b32_gqa4_d128_bf16", 32, 32, 8, 128, lens, torch.bfloat16, 4,
                    n_append=1, notes="prefill of one 4096-token sequence is timed separately")


GEMMA_SWEEP = (256, 512, 1024, 2048, 4096)

# Hot-tail sizes for the delegated cache (the pages name the mode but give no
# window): the most recent 256 V tokens stay binary16, folded 64 at a time.
DELEGATED_WINDOW = 256
DELEGATED_FOLD = 64


def all_workloads() -> List[Workload]:
    return [tiny_single_head(), llama3_8b_layer(), *[gemma3_1b_sweep(t) for t in GEMMA_SWEEP],
            llama31_70b_long(), ragged_serving()]


@dataclass
class Tensors:
    k: List[torch.Tensor]        # per sequence [len_b][Hkv][D] (workload dtype)
    v: List[torch.Tensor]
    q: torch.Tensor              # [B][Hq][D]
    k_new: torch.Tensor          # [B][n_append][Hkv][D]
    v_new: torch.Tensor
    channel_mult: torch.Tensor   # [Hkv][D] fp32


def generate(w: Workload, device: str = "cpu", seq_subset: Optional[List[int]] = None) -> Tensors:
    """Draw the workload's tensors in the documented order.

    ``device="cuda"`` draws from a CUDA generator (a different stream than the
    CPU one; the bench uses it to avoid host-side generation of gigabytes).
    ``seq_subset`` keeps only those sequences' prefix blocks (the draws for the
    others still happen, so the kept values are identical to a full draw).
    """
    g = torch.Generator(device).manual_seed(w.seed)
    Hkv, D = w.n_kv_heads, w.head_dim
    keep = set(range(w.batch)) if seq_subset is None else set(seq_subset)
    base = []
    for b, L in enumerate(w.seq_lens):
        x = torch.randn((L, Hkv, D), generator=g, device=device)
        base.append(x if b in keep else None)  # the draw happens either way
    z = torch.randn((Hkv, D), generator=g, device=device)
    mult = torch.exp(z)
    n_out = D // 32
    for h in range(Hkv):
        idx = torch.randperm(D, generator=g, device=device)[:n_out]
        mult[h, idx] *= 10.0
    k = [(base[b] * mult).to(w.dtype) if b in keep else None for b in range(w.batch)]
    del base
    v = []
    for b, L in enumerate(w.seq_lens):
        x = torch.randn((L, Hkv, D), generator=g, device=device)
        v.append(x.to(w.dtype) if b in keep else None)
    q = torch.randn((w.batch, w.n_q_heads, D), generator=g, device=device).to(w.dtype)
    kn = (torch.randn((w.batch, w.n_append, Hkv, D), generator=g, device=device) * mult).to(w.dtype)
    vn = torch.randn((w.batch, w.n_append, Hkv, D), generator=g, device=device).to(w.dtype)
    return Tensors(k, v, q, kn, vn, mult)
