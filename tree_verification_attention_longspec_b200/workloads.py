"""The synthetic verification workloads, named by what they are.

The LongSpec pages run their verification on long-context models (Vicuna, LongChat,
LLaMA-3.1, QwQ) over long documents (gist.science summary, section 3). No dataset is
shipped here; these shapes stand in for one attention layer of such a model during
one tree-verification step.
"""
from __future__ import annotations

from .inputs import Workload

TINY = Workload("tiny_L1k_T16_h4x1_d64", batch=1, num_q_heads=4, num_kv_heads=1,
                head_dim=64, tree_size=16, prefix=1024, tree="uniform",
                input_scale=0.125)  # N(0,1)/sqrt(64)
LLAMA8B = Workload("llama8b_L16k_T64_h32x8_d128", batch=1, num_q_heads=32, num_kv_heads=8,
                   head_dim=128, tree_size=64, prefix=16384, tree="window8")
QWEN7B = Workload("qwen7b_L64k_T64_h28x4_d128", batch=1, num_q_heads=28, num_kv_heads=4,
                  head_dim=128, tree_size=64, prefix=65536, tree="window8")
DEEP70B = Workload("70b_L128k_T128_h64x8_d128_bfs", batch=1, num_q_heads=64, num_kv_heads=8,
                   head_dim=128, tree_size=128, prefix=131072, tree="bfs")
RAGGED = Workload("ragged_b8_L4k-32k_T64_h32x8_d128", batch=8, num_q_heads=32, num_kv_heads=8,
                  head_dim=128, tree_size=64, prefix=(4096, 32768), tree="window8")

# Per-sequence trees: the ragged batch with T_b ~ U{16..128} nodes per sequence.
RAGGED_TREES = Workload("ragged_trees_b8_L4k-32k_T16-128_h32x8_d128", batch=8, num_q_heads=32, num_kv_heads=8,
                        head_dim=128, tree_size=128, prefix=(4096, 32768), tree="window8",
                        tree_size_range=(16, 128))

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B, QWEN7B, DEEP70B, RAGGED, RAGGED_TREES)}
# The headline workload: a Qwen2.5-7B-shaped layer at L = 64k, T = 64.
HEADLINE = QWEN7B


def algorithmic_bytes(B, Hq, Hkv, d, T, total_L) -> int:
    """Bytes a perfect implementation must move: K/V prefix + K/V tree + q in, out + lse."""
    return (4 * total_L * Hkv * d + 4 * B * T * Hkv * d + 2 * B * T * Hq * d
            + 2 * B * T * Hq * d + 4 * B * T * Hq)


def algorithmic_flops(Hq, d, T, lengths) -> int:
    """QK^T and PV over every (query, visible-or-not tree key) pair: 4*T*H_q*d*(L_b+T) per sequence."""
    return int(sum(4 * T * Hq * d * (int(L) + T) for L in lengths))
