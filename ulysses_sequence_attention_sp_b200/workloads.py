"""The synthetic workloads the tests and the benchmark run (shapes only, no arithmetic).

Each is named for what it is. Token and head splits follow the balanced rule
(earlier ranks take the remainder); ``prefix`` rows are a replicated cls token.
"""

from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq_len: int          # tokens that are split across ranks (cls excluded)
    prefix: int           # replicated leading tokens (cls), 0 or 1
    heads: int
    head_dim: int
    world: int            # virtual sequence-parallel ranks
    dtype: str            # "bf16" or "fp32"
    std: float
    seed: int
    num_chunks: tuple     # head-chunk counts the workload is run with
    kv_heads: int = 0     # k/v heads (grouped-query attention); 0 means `heads`
    ring: int = 1         # Ulysses + Ring hybrid: ring size (world // ring ranks per Ulysses group)

    @property
    def heads_kv(self) -> int:
        return self.kv_heads or self.heads

    @property
    def tokens(self) -> int:
        return self.prefix + self.seq_len

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def tensor_bytes(self) -> int:
        return self.batch * self.tokens * self.heads * self.head_dim * self.elem_bytes

    @property
    def attention_flop(self) -> int:
        t = self.tokens
        return 4 * self.batch * self.heads * t * t * self.head_dim


TINY = Workload("tiny-ragged-T37-H6-D16-P4-fp32", 1, 37, 0, 6, 16, 4, "fp32", 1.0, 1001, (1, 2))
RESHARD = Workload("reshard-T32768-H32-D128-P8-bf16", 1, 32768, 0, 32, 128, 8, "bf16", 1.0, 1002, (1,))
VIDEO = Workload("video-T75600-H24-D128-P7-bf16", 1, 75600, 0, 24, 128, 7, "bf16", 1.0, 1003, (1,))
VIT = Workload("vit-B16-cls1+576-H16-D80-P4-bf16", 16, 576, 1, 16, 80, 4, "bf16", 0.5, 1004, (1,))
CHUNKED = Workload("chunked-T16384-H40-D128-P8-bf16", 1, 16384, 0, 40, 128, 8, "bf16", 1.0, 1005, (3, 1))

# The video latent on 8 ranks as a Ulysses + Ring hybrid: 2 groups of 4 (6 heads per rank), 2-step ring.
HYBRID = Workload("hybrid-video-T75600-H24-D128-U4xR2-bf16", 1, 75600, 0, 24, 128, 8, "bf16", 1.0, 1006, (1,),
                  ring=2)

ALL = (TINY, RESHARD, VIDEO, VIT, CHUNKED, HYBRID)
BY_NAME = {w.name: w for w in ALL}
