"""The synthetic workloads: shapes, seeds and value distributions.

Model widths follow the pages' three model sizes (370M, 1.3B and 2.7B
parameters; jiqizhixin.com, section "实验") and their channel mixer, a
MatMul-free GLU built from BitLinear layers (datacamp.com, section "Các thành
phần lõi: MLGRU và GLU").  Every input is drawn by ``inputs`` from a seed; no
dataset is read.

A ``Projection`` is one BitLinear d_in -> d_out.  ``input_index`` names which
activation tensor feeds it: projections with the same index share one x.  In
the token mixer (MLGRU) the f, c and g projections read the mixer's input and
o reads the gated hidden state g*h, its own input; in the channel mixer (GLU)
gate and up share the mixer's input and down reads their product.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Projection:
    name: str
    K: int            # d_in
    N: int            # d_out
    input_index: int  # which activation tensor feeds it


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    seed: int
    M: int
    projections: tuple
    outlier_frac: float = 0.0
    eps: float = 1e-6
    eps_w: float = 1e-5
    extra: dict = field(default_factory=dict)

    @property
    def weights(self) -> int:
        return sum(p.N * p.K for p in self.projections)

    def inputs(self):
        """(input_index, K) of every distinct activation tensor."""
        seen = {}
        for p in self.projections:
            seen.setdefault(p.input_index, p.K)
        return sorted(seen.items())


def _set_1p3b():
    d, f = 2048, 5632
    return (
        Projection("f", d, d, 0), Projection("c", d, d, 0),
        Projection("g", d, d, 0), Projection("o", d, d, 1),
        Projection("gate", d, f, 2), Projection("up", d, f, 2),
        Projection("down", f, d, 3),
    )


def _set_2p7b():
    d, f = 2560, 6912
    return (
        Projection("f", d, d, 0), Projection("c", d, d, 0),
        Projection("g", d, d, 0), Projection("o", d, d, 1),
        Projection("gate", d, f, 2), Projection("up", d, f, 2),
        Projection("down", f, d, 3),
    )


SMOKE = Workload(
    "smoke-256", "single fused BitLinear, M=16, 256->256", seed=0, M=16,
    projections=(Projection("w", 256, 256, 0),))

DECODE_370M = Workload(
    "decode-370m", "decode GEMV at 370M width, M=1: 1024->1024, 1024->2816, 2816->1024",
    seed=1, M=1,
    projections=(Projection("proj", 1024, 1024, 0), Projection("gate", 1024, 2816, 1),
                 Projection("down", 2816, 1024, 2)))


def decode_2p7b(M: int = 1) -> Workload:
    assert M in (1, 8, 32)
    return Workload(
        f"decode-2.7b-m{M}",
        f"decode at 2.7B width, M={M}: 4x 2560->2560, 2x 2560->6912, 6912->2560; "
        "1% outlier channels x20",
        seed=2, M=M, projections=_set_2p7b(), outlier_frac=0.01)


PREFILL_1P3B = Workload(
    "prefill-1.3b", "prefill at 1.3B width, M=8192: 2048->2048, 2048->5632, 5632->2048",
    seed=3, M=8192,
    projections=(Projection("proj", 2048, 2048, 0), Projection("up", 2048, 5632, 1),
                 Projection("down", 5632, 2048, 2)))

PREFILL_2P7B = Workload(
    "prefill-2.7b", "prefill at 2.7B width, M=8192: 2560->2560, 2560->6912, 6912->2560; 1% outlier channels x20",
    seed=6, M=8192,
    projections=(Projection("proj", 2560, 2560, 0), Projection("up", 2560, 6912, 1),
                 Projection("down", 6912, 2560, 2)),
    outlier_frac=0.01)

TRAIN_FWD_1P3B = Workload(
    "train-fwd-1.3b",
    "training-batch forward at 1.3B width, M=2^8*2048=524288, full BitLinear set "
    "(4x 2048->2048, 2x 2048->5632, 5632->2048)",
    seed=4, M=524288, projections=_set_1p3b())


ALL = {w.name: w for w in (SMOKE, DECODE_370M, decode_2p7b(1), decode_2p7b(8),
                           decode_2p7b(32), PREFILL_1P3B, PREFILL_2P7B, TRAIN_FWD_1P3B)}
