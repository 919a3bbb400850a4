"""Workload shapes for the IA layer hot path (synthetic inputs only).

Each workload names the layer shape it stands for.  The pages measure
language models of 125M-1.3B parameters trained on a web-text corpus; no
dataset is needed here because the layer's cost does not depend on the input
values, so seeded Gaussian inputs of those layers' q/k/v shapes stand in.
``M`` is the number of complex S4D modes, ``d_xi`` the feature width of q and
k (R = d_h in the paper), ``d_v`` the value width.
"""
from dataclasses import dataclass, field
from typing import Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d_xi: int
    d_v: int
    M: int
    dtype: str          # "f32" or "bf16" input dtype; states and outputs are fp32
    seed: int           # torch CPU generator seed for this workload's inputs
    kind: str = "fwd"   # "fwd", "fwd_bwd" or "decode"
    decode_batches: Tuple[int, ...] = field(default_factory=tuple)

    @property
    def tokens(self) -> int:
        return self.B * self.N


WORKLOADS = {
    # tiny fp32 layer: parity at 1e-4 against the fp64 oracle
    "tiny_f32": Workload("tiny_f32", 1, 2, 256, 16, 16, 16, "f32", 1000),
    # 125M-layer-shaped prefill forward
    "prefill_125m": Workload("prefill_125m", 8, 12, 2048, 64, 64, 64, "bf16", 1001),
    # 1.3B-layer-shaped prefill forward
    "prefill_1p3b": Workload("prefill_1p3b", 4, 16, 2048, 128, 128, 64, "bf16", 1002),
    # training step (forward + backward) at 350M-layer shape
    "train_350m": Workload("train_350m", 8, 16, 2048, 64, 64, 64, "bf16", 1003, kind="fwd_bwd"),
    # length extrapolation: prefill of 3.5 x 2048 at the 1.3B shape
    "prefill_1p3b_7168": Workload("prefill_1p3b_7168", 1, 16, 7168, 128, 128, 64, "bf16", 1004),
    # single-token decode after a 7168-token prefix at the 1.3B shape
    "decode_1p3b": Workload("decode_1p3b", 64, 16, 1, 128, 128, 64, "bf16", 1004, kind="decode",
                            decode_batches=(1, 16, 64)),
}
