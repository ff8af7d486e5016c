"""The five attention workloads: shapes, mask modes, passes and seeds.

Each workload draws Q, K, V and dO i.i.d. N(0,1) (rounded to bf16) with base
seed 42 + its index in ``WORKLOADS``. The softmax scale is 1/sqrt(d).
"""

from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: tuple
    passes: tuple = ("fwd", "bwd")
    fp8: bool = False
    outlier_rate: float = 0.0
    seed: int = 42
    nq: int = 0  # query rows when fewer than N (decoding against a cache); 0 = N
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return self.d ** -0.5

    def fwd_flops(self, causal: bool) -> float:
        """4*B*Hq*N^2*d, halved for a causal mask."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if causal else f

    def bwd_flops(self, causal: bool) -> float:
        """2.5x the forward count."""
        return 2.5 * self.fwd_flops(causal)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 128, 64, (False, True), seed=42,
                     notes="tiny oracle check"),
    "gpt2": Workload("gpt2", 8, 16, 16, 2048, 64, (False, True), seed=43,
                     notes="GPT-2-style training shape"),
    "long128": Workload("long128", 2, 16, 16, 8192, 128, (True,), seed=44,
                        notes="long sequence, head dim 128"),
    "gqa": Workload("gqa", 2, 32, 8, 8192, 128, (True,), seed=45,
                    notes="grouped-query attention, 4 query heads per KV head"),
    "fp8": Workload("fp8", 1, 16, 16, 16384, 128, (False,), passes=("fwd",), fp8=True,
                    outlier_rate=0.001, seed=46,
                    notes="FP8 e4m3 forward with outliers, 64xd block scales, Hadamard rotation"),
    # not one of the five: one decode step (a query row per head) against a
    # 16K-token cache, GQA 32/8
    "decode": Workload("decode", 16, 32, 8, 16384, 128, (True,), passes=("fwd",), seed=47, nq=1,
                       notes="decode step: 1 query row per head, 16384-key cache, GQA 4:1"),
}
