"""The synthetic workloads the tests and the benchmark run.

Each workload is a MoE layer (or the dense E=1 MLP) of the Jamba family with
seeded random tensors drawn by :mod:`synth`:

* activations ``x`` ~ N(0, 1) rounded to bf16,
* router ``W_r`` ~ N(0, 0.02) in fp32,
* expert weights ~ N(0, 0.02) rounded to bf16 (then quantised to INT8 by the
  library under test),
* seed = 20240822 + workload index.

The shapes are the Jamba-1.5-Mini (d_model 4096, d_ff 14336) and
Jamba-1.5-Large (d_model 8192, d_ff 24576) expert shapes with 16 experts and
top-2 routing (Jamba-1.5 summary, "The Jamba Hybrid Block Structure": n = 16,
K = 2, d_model = 8192 for Large).  The skewed workload adds +2.0 to the router
logits of experts 0 and 1, so that about 40 % of the assignments land on them.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

SEED0 = 20240822
SIGMA_X = 1.0
SIGMA_W = 0.02
SIGMA_R = 0.02


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    d_model: int
    d_ff: int
    E: int = 16
    top_k: int = 2
    bias: Optional[Tuple[float, ...]] = None  # per-expert router logit bias
    dense: bool = False  # the E=1 dense MLP entry (no router)
    regime: str = "decode"  # "decode" (HBM bound) or "prefill" (tensor-core bound)

    @property
    def seed(self) -> int:
        return SEED0 + self.index

    @property
    def A(self) -> int:
        return self.T * self.top_k

    def describe(self) -> dict:
        d = {"workload": self.name, "T": self.T, "d_model": self.d_model, "d_ff": self.d_ff,
             "experts": self.E, "top_k": self.top_k, "seed": self.seed}
        if self.bias is not None:
            d["router_bias"] = "+2.0 on experts 0,1"
        return d


def _skew(E: int) -> Tuple[float, ...]:
    return tuple(2.0 if e < 2 else 0.0 for e in range(E))


TINY = Workload("tiny_T64_d256_f512_E16_top2", 0, 64, 256, 512, regime="launch")
MINI_DECODE = Workload("mini_decode_T8_d4096_f14336_E16_top2", 1, 8, 4096, 14336)
MINI_PREFILL = Workload("mini_prefill_T16384_d4096_f14336_E16_top2", 2, 16384, 4096, 14336,
                        regime="prefill")
MINI_DENSE = Workload("mini_dense_mlp_T16384_d4096_f14336_E1", 2, 16384, 4096, 14336,
                      E=1, top_k=1, dense=True, regime="prefill")
LARGE_DECODE = Workload("large_decode_T32_d8192_f24576_E16_top2", 3, 32, 8192, 24576)
LARGE_PREFILL_SKEW = Workload("large_prefill_skewed_T8192_d8192_f24576_E16_top2", 4, 8192, 8192,
                              24576, bias=_skew(16), regime="prefill")

# generalised routing at Mini size: 64 experts, top-4 (a wider MoE, as in the
# routing settings the layer also supports)
MINI_DECODE_E64 = Workload("mini_decode_T8_d4096_f14336_E64_top4", 5, 8, 4096, 14336, E=64,
                           top_k=4)

ALL = [TINY, MINI_DECODE, MINI_PREFILL, MINI_DENSE, LARGE_DECODE, LARGE_PREFILL_SKEW,
       MINI_DECODE_E64]
BY_NAME = {w.name: w for w in ALL}
