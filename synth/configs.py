"""The five synthetic workloads (seed 0 throughout).

cfg1  256x512 layer, 1 base, fp32 row/col scales, fp32 x, rank-8 binary correction, M=1
cfg2  Llama-7B attention projection 4096x4096, 2 bases, bf16 scales, no correction, M=1
cfg3  Llama-7B MLP: gate/up 4096->11008 (out=11008, in=4096) and down 11008->4096
      (out=4096, in=11008), 2 bases, 1% salient input columns in int8, M in {1, 4, 16}
cfg4  5120x5120, 2 bases, rank-512 binary correction, x with 0.1% outlier channels x20,
      M in {1, 2, 4, 8}
cfg5  32-layer Llama-7B decoder weight stream (q/k/v/o 4096^2, gate/up 4096->11008,
      down 11008->4096), 2 bases, rank-256 correction, M in {1..128}

Shapes follow the (out, in) convention: Y[M, out] = X[M, in] @ W[out, in]^T.
"""

from dataclasses import dataclass
from typing import Iterator, List, Tuple

from .gen import Layer, make_activations, make_layer

SEED = 0

LLAMA7B_MATRICES = [  # (name, out, in)
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
]


@dataclass(frozen=True)
class Spec:
    name: str
    out: int
    in_: int
    K: int
    scale_dtype: str
    x_dtype: str
    rank: int = 0
    sal_frac: float = 0.0
    outlier_frac: float = 0.0
    outlier_factor: float = 1.0


CONFIGS = {
    1: dict(Ms=[1], specs=[Spec("cfg1", 256, 512, 1, "f32", "f32", rank=8)]),
    2: dict(Ms=[1], specs=[Spec("cfg2_attn", 4096, 4096, 2, "bf16", "bf16")]),
    3: dict(Ms=[1, 4, 16], specs=[Spec("cfg3_gate_up", 11008, 4096, 2, "bf16", "bf16", sal_frac=0.01),
                                  Spec("cfg3_down", 4096, 11008, 2, "bf16", "bf16", sal_frac=0.01)]),
    4: dict(Ms=[1, 2, 4, 8], specs=[Spec("cfg4", 5120, 5120, 2, "bf16", "bf16", rank=512,
                                         outlier_frac=0.001, outlier_factor=20.0)]),
    5: dict(Ms=[1, 2, 4, 8, 16, 32, 64, 128],
            specs=[Spec(f"cfg5_l{l}_{n}", o, i, 2, "bf16", "bf16", rank=256)
                   for l in range(32) for (n, o, i) in LLAMA7B_MATRICES]),
}


def spec_key(cfg: int, spec_index: int, M: int) -> Tuple[int, int, int]:
    return (cfg, spec_index, M)


def build(cfg: int, spec_index: int, M: int, seed: int = SEED) -> Tuple[Layer, "object"]:
    """(layer, X) for one spec of a config at batch M.

    The weights do not depend on M except through salient selection (which uses X);
    X depends on M. Salient layers are keyed by M so each batch has its own selection.
    """
    s = CONFIGS[cfg]["specs"][spec_index]
    wkey = (cfg, spec_index, M if s.sal_frac > 0 else 0)
    xkey = (cfg, spec_index, 1000 + M)
    X = make_activations(seed, xkey, M, s.in_, s.x_dtype, s.outlier_frac, s.outlier_factor)
    L = make_layer(seed, wkey, s.out, s.in_, s.K, s.scale_dtype, rank=s.rank, sal_frac=s.sal_frac,
                   x_for_salience=X if s.sal_frac > 0 else None, x_dtype=s.x_dtype, name=s.name)
    return L, X


def config_layers(cfg: int, M: int, seed: int = SEED) -> Iterator[Tuple[Layer, "object"]]:
    for i in range(len(CONFIGS[cfg]["specs"])):
        yield build(cfg, i, M, seed)


def spec(cfg: int, spec_index: int = 0) -> Spec:
    return CONFIGS[cfg]["specs"][spec_index]


def all_specs(cfg: int) -> List[Spec]:
    return list(CONFIGS[cfg]["specs"])
