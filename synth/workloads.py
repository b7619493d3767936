"""The five synthetic workloads (shapes, distributions, seeds) of the
BitLinear forward, as lazily generated cases.

Each case names one BitLinear call: activations x (bf16 [M, K]), a weight
W (fp32 [N, K], nn.Linear's [out, in]) and an optional bf16 bias [N].  The
seed of workload c is 0xB1700 + c; each tensor has its own stream id, so any
tensor can be regenerated alone.  Nothing here computes any part of the
method: the recipes only fix shapes and value distributions.

1. single small layer: x N(0,1) [8,256]; W N(0,0.02) [512,256]; no bias.
2. decode sweep: M in {1,4,16}; (K,N) = (4096,4096) and (4096,11008);
   x N(0,1) with 1% of the channels scaled x20; W N(0,0.02); bias N(0,0.01).
3. prefill: M in {512,2048,8192}; (K,N) = (3200,8640) and (8640,3200);
   x Student-t(4); W N(0,0.02); no bias.
4. 3B-class projection stack: 26 layers x (q,k,v,o 3200x3200; gate,up
   3200->8640; down 8640->3200) of independent W N(0,0.02); x N(0,1), one
   input shared by q/k/v, one for o, one shared by gate/up, one [M,8640] for
   down; M in {1, 2048}; no bias.
5. 100B-class FFN: hidden 8192, FFN 28672 (gate/up 8192->28672, down
   28672->8192); 13 independent layers; x N(0,1); W N(0,0.01); M in
   {1,8,64,512}; no bias.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Optional

import torch

from . import normal_bf16, normal_f32, normal_with_outliers_bf16, student_t4_bf16

SEED0 = 0xB1700


def seed_of(workload: int) -> int:
    return SEED0 + workload


@dataclass
class Case:
    """One BitLinear call of a workload; tensors are generated on demand."""
    name: str
    M: int
    N: int
    K: int
    make_x: Callable[[], torch.Tensor]
    make_w: Callable[[], torch.Tensor]
    make_bias: Optional[Callable[[], torch.Tensor]] = None
    tags: dict = field(default_factory=dict)

    def x(self) -> torch.Tensor:
        return self.make_x()

    def w(self) -> torch.Tensor:
        return self.make_w()

    def bias(self) -> Optional[torch.Tensor]:
        return None if self.make_bias is None else self.make_bias()


def workload1() -> list[Case]:
    s = seed_of(1)
    return [Case("w1_single_8x256x512", 8, 512, 256,
                 lambda: normal_bf16(s, 1, (8, 256)),
                 lambda: normal_f32(s, 2, (512, 256), 0.02))]


DECODE_SHAPES = ((4096, 4096), (4096, 11008))   # (K, N)
DECODE_MS = (1, 4, 16)


def workload2() -> list[Case]:
    s = seed_of(2)
    cases = []
    for si, (K, N) in enumerate(DECODE_SHAPES):
        for M in DECODE_MS:
            cases.append(Case(
                f"w2_decode_M{M}_K{K}_N{N}", M, N, K,
                (lambda M=M, K=K: normal_with_outliers_bf16(s, 100 + M, (M, K))),
                (lambda N=N, K=K, si=si: normal_f32(s, 200 + si, (N, K), 0.02)),
                (lambda N=N, si=si: normal_bf16(s, 300 + si, (N,), 0.01)),
                tags={"shape": si}))
    return cases


PREFILL_SHAPES = ((3200, 8640), (8640, 3200))   # (K, N)
PREFILL_MS = (512, 2048, 8192)


def workload3() -> list[Case]:
    s = seed_of(3)
    cases = []
    for si, (K, N) in enumerate(PREFILL_SHAPES):
        for M in PREFILL_MS:
            cases.append(Case(
                f"w3_prefill_M{M}_K{K}_N{N}", M, N, K,
                (lambda M=M, K=K, si=si: student_t4_bf16(s, 100 + 10 * si + M % 7, (M, K))),
                (lambda N=N, K=K, si=si: normal_f32(s, 200 + si, (N, K), 0.02))))
    return cases


STACK3B_LAYERS = 26
HID3B, FFN3B = 3200, 8640
# projection id -> (name, K, N, input id)
PROJ3B = ((0, "q", HID3B, HID3B, 0), (1, "k", HID3B, HID3B, 0), (2, "v", HID3B, HID3B, 0),
          (3, "o", HID3B, HID3B, 1), (4, "gate", HID3B, FFN3B, 2), (5, "up", HID3B, FFN3B, 2),
          (6, "down", FFN3B, HID3B, 3))


def workload4(M: int, layers=None) -> list[Case]:
    s = seed_of(4)
    layers = range(STACK3B_LAYERS) if layers is None else layers
    cases = []
    for L in layers:
        for pid, pname, K, N, xin in PROJ3B:
            cases.append(Case(
                f"w4_stack3b_M{M}_L{L}_{pname}", M, N, K,
                (lambda L=L, K=K, xin=xin: normal_bf16(s, 10_000 + 100 * L + 10 * xin + (M % 5), (M, K))),
                (lambda L=L, pid=pid, N=N, K=K: normal_f32(s, 16 * L + pid, (N, K), 0.02)),
                tags={"layer": L, "proj": pname}))
    return cases


STACK100B_LAYERS = 13
HID100B, FFN100B = 8192, 28672
PROJ100B = ((0, "gate", HID100B, FFN100B, 0), (1, "up", HID100B, FFN100B, 0),
            (2, "down", FFN100B, HID100B, 1))
MS100B = (1, 8, 64, 512)


def workload5(M: int, layers=None) -> list[Case]:
    s = seed_of(5)
    layers = range(STACK100B_LAYERS) if layers is None else layers
    cases = []
    for L in layers:
        for pid, pname, K, N, xin in PROJ100B:
            cases.append(Case(
                f"w5_ffn100b_M{M}_L{L}_{pname}", M, N, K,
                (lambda L=L, K=K, xin=xin: normal_bf16(s, 10_000 + 100 * L + 10 * xin + (M % 5), (M, K))),
                (lambda L=L, pid=pid, N=N, K=K: normal_f32(s, 16 * L + pid, (N, K), 0.01)),
                tags={"layer": L, "proj": pname}))
    return cases
