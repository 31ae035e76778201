"""The attention workloads the library is measured and checked on, and their work counts.

Shapes follow the pages' own examples: B=2, H=8, N=1024, d=64 (page "Flash Attention 3.7
核心原理与实战" §3.2); B=2, N=4096, model dim 512 in 8 heads (page "显存神技：必学FlashAttention！");
B=32, H=16, N=2048, d=64 (page "告别OOM和训练慢…(含A100环境配置)" §1); 8192 tokens with
head_dim 128 and a sliding window (page "PyTorch-CUDA-v2.9镜像…" on 8k sequences, page
"Flash Attention 3.7 …" §5, page "告别OOM和训练慢…" §4.2 `window_size`).

Work convention for throughput: forward 4*B*H*N^2*d flops, backward 2.5x the forward
(fwd+bwd = 3.5x), halved for causal; a sliding window counts its visible (query, key)
pairs, 4*B*H*d*pairs for the forward.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    window: tuple  # (left, right), -1 = unbounded
    backward: bool
    seed_index: int
    scale: float | None = None  # None: 1/sqrt(d)
    alibi: bool = False         # linear bias -m_h |i - j| with the slopes of alibi_slopes()
    varlen: bool = False        # variable-length batch with the lengths of seq_lengths()
    fp8: bool = False           # e4m3 Q, K, V (forward only)
    packed: bool = False        # with varlen: the sequences back to back, (total, H, d)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    def seq_lengths(self) -> list:
        """The real lengths of a variable-length batch: seeded, uniform in [N/4, N]."""
        if not self.varlen:
            return [self.N] * self.B
        import numpy as np
        rng = np.random.default_rng(0x5EED0000 + 16 * self.seed_index + 7)
        return [int(x) for x in rng.integers(self.N // 4, self.N + 1, size=self.B)]

    def visible_pairs(self, N: int | None = None) -> int:
        """Exact number of visible (query, key) pairs of one (batch, head) of length N."""
        N = self.N if N is None else N
        left, right = self.window
        if self.causal:
            right = 0
        total = 0
        # rows are grouped by which clip is active; closed form per row is
        # hi - lo + 1 with lo = max(0, i-left) and hi = min(N-1, i+right)
        for i in range(N):
            lo = 0 if left < 0 else max(0, i - left)
            hi = N - 1 if right < 0 else min(N - 1, i + right)
            total += hi - lo + 1
        return total

    def fwd_flops(self) -> float:
        """Forward flops by the metric's convention (a variable-length batch counts the
        pairs of its real lengths)."""
        if self.varlen:
            return 4.0 * self.H * self.d * sum(self.visible_pairs(L) for L in self.seq_lengths())
        base = 4.0 * self.B * self.H * self.N * self.N * self.d
        if self.window != (-1, -1) and self.window[0] >= 0:
            return 4.0 * self.B * self.H * self.d * self.visible_pairs()
        return base / 2 if self.causal else base

    def step_flops(self) -> float:
        """Flops of one step: forward, plus backward (2.5x) when the workload has one."""
        return self.fwd_flops() * (3.5 if self.backward else 1.0)

    def tensor_bytes(self) -> int:
        return self.B * self.H * self.N * self.d * 2

    def fwd_bytes(self) -> int:
        """Compulsory device-memory traffic of the forward: read Q, K, V; write O, LSE."""
        return 4 * self.tensor_bytes() + 4 * self.B * self.H * self.N

    def bwd_bytes(self) -> int:
        """Compulsory traffic of the backward: read Q, K, V, O, dO, LSE; write dQ, dK, dV."""
        return 8 * self.tensor_bytes() + 4 * self.B * self.H * self.N


WORKLOADS = {
    "c1": Workload("c1_tiny_b1h2n128d64", 1, 2, 128, 64, False, (-1, -1), True, 0, scale=0.125),
    "c2": Workload("c2_fwd_b2h8n1024d64", 2, 8, 1024, 64, False, (-1, -1), False, 1),
    "c3": Workload("c3_b2h8n4096d64", 2, 8, 4096, 64, False, (-1, -1), True, 2),
    "c4": Workload("c4_causal_b32h16n2048d64", 32, 16, 2048, 64, True, (-1, -1), True, 3),
    "c5c": Workload("c5_causal_b2h32n8192d128", 2, 32, 8192, 128, True, (-1, -1), True, 4),
    "c5w": Workload("c5_window1024_b2h32n8192d128", 2, 32, 8192, 128, True, (1024, 0), True, 4),
    # C4 with the ALiBi bias of the `alibi_slopes` parameter (page "告别OOM和训练慢…" §4.2)
    "c4a": Workload("c4_causal_alibi_b32h16n2048d64", 32, 16, 2048, 64, True, (-1, -1), True, 3,
                    alibi=True),
    # C4 as a variable-length batch: real lengths uniform in [512, 2048] (the `lengths` of
    # the dynamic batching of page "告别OOM和训练慢…" §6); work counted on the real pairs
    "c4v": Workload("c4_causal_varlen_b32h16n2048d64", 32, 16, 2048, 64, True, (-1, -1), True,
                    3, varlen=True),
    # the same batch packed back to back with no padding (cumulative lengths): the page's
    # dynamic batching groups sequences to avoid padding waste
    "c4p": Workload("c4_causal_packed_b32h16n2048d64", 32, 16, 2048, 64, True, (-1, -1), True,
                    3, varlen=True, packed=True),
    # the long-sequence causal forward on e4m3 inputs (FP8 support, page "告别OOM和训练慢…" §6)
    "c5f8": Workload("c5_causal_fp8_fwd_b2h32n8192d128", 2, 32, 8192, 128, True, (-1, -1), False,
                     4, fp8=True),
}


def alibi_slopes(H: int) -> list:
    """The geometric ALiBi slopes 2^(-8 h / H), h = 1..H (one per head)."""
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
