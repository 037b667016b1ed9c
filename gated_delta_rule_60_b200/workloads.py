"""The five KDA workloads, by name and size.

  tiny_fp32     B=1, H=2,  T=64,        d=16,  fp32, S0=0
  k3_prefill    B=1, H=96, T=8192,      d=128, bf16, S0=0
  varlen_h0     24 sequences, lengths uniform on [256, 8192], H=96, d=128,
                bf16, h0 ~ N(0, 0.02^2) fp32
  long_1m       B=1, H=16, T=1,048,576, d=128, bf16, S0=0
  decode_256    256 sequences x 96 heads, d=128, fp32 state built by a
                512-token prefill, then 128 single-token decode steps

Seeds: 1000 + index for the prefill inputs; decode step s draws with seed
5000 + s.  Chunk length is 16 throughout (the 16-token tile of the pages).
"""
from dataclasses import dataclass
from typing import List, Optional

import torch

from . import inputs


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    lengths: tuple
    h0_std: Optional[float] = None

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def T_tot(self) -> int:
        return int(sum(self.lengths))

    def make(self) -> inputs.PrefillInputs:
        return inputs.make_prefill(list(self.lengths), self.H, self.dk,
                                   self.dv, self.dtype, self.seed,
                                   self.h0_std)


def _varlen_lengths() -> List[int]:
    return inputs.draw_lengths(24, 256, 8192, seed=1002)


TINY = Workload("tiny_fp32", 0, 2, 16, 16, torch.float32, (64,))
K3_PREFILL = Workload("k3_prefill", 1, 96, 128, 128, torch.bfloat16, (8192,))
VARLEN = Workload("varlen_h0", 2, 96, 128, 128, torch.bfloat16,
                  tuple(_varlen_lengths()), h0_std=0.02)
LONG = Workload("long_1m", 3, 16, 128, 128, torch.bfloat16, (1 << 20,))

DECODE_B = 256
DECODE_H = 96
DECODE_D = 128
DECODE_PREFILL = 512
DECODE_STEPS = 128
DECODE_SEED = 1004
DECODE_STEP_SEED0 = 5000

ALL_PREFILL = (TINY, K3_PREFILL, VARLEN, LONG)


def by_name(name: str) -> Workload:
    for w in ALL_PREFILL:
        if w.name == name:
            return w
    raise KeyError(name)
