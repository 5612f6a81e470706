"""The five decode-attention workloads: shapes, value distributions, scale.

Plain data, no arithmetic of the method. Each entry is one synthetic
workload; the inputs module draws its tensors from a seed.

Context lengths follow "Flash-Decoding for long-context inference" (section
"Motivation"): contexts grew from 2k to 32k and 100k tokens, and decoding at
batch size 1 over such contexts is where splitting the keys/values pays.
"""
from dataclasses import dataclass
import math


@dataclass(frozen=True)
class Workload:
    name: str
    B: int            # sequences in the batch
    Hq: int           # query heads
    Hkv: int          # key/value heads (Hq % Hkv == 0; query head i reads kv head i // (Hq/Hkv))
    D: int            # head dimension
    Lmax: int         # allocated cache length per sequence
    ragged: bool      # seqlens drawn uniform in [1, Lmax] instead of all = Lmax
    sigma_q: float = 1.0
    sigma_k: float = 1.0
    sigma_v: float = 1.0
    nan_pad: bool = False   # fill positions >= seqlen with NaN in K and V
    description: str = ""

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "Workload":
        d = self.__dict__.copy()
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny_mha": Workload(
        "tiny_mha", B=1, Hq=4, Hkv=4, D=64, Lmax=1024, ragged=False,
        description="tiny MHA decode, B=1 Hq=Hkv=4 D=64 L=1024, N(0,1); run with 1 and with 4 splits"),
    "mha_16k": Workload(
        "mha_16k", B=1, Hq=32, Hkv=32, D=128, Lmax=16384, ragged=False,
        description="7B-style MHA long context, B=1 Hq=Hkv=32 D=128 L=16384, N(0,1)"),
    "gqa_128k": Workload(
        "gqa_128k", B=1, Hq=64, Hkv=8, D=128, Lmax=131072, ragged=False,
        description="GQA very long context, B=1 Hq=64 Hkv=8 (group 8) D=128 L=131072, N(0,1)"),
    "batch_4k": Workload(
        "batch_4k", B=64, Hq=32, Hkv=8, D=128, Lmax=4096, ragged=False,
        description="batch-bound decode, B=64 Hq=32 Hkv=8 D=128 L=4096 for every sequence, N(0,1)"),
    "ragged_64k": Workload(
        "ragged_64k", B=32, Hq=32, Hkv=8, D=128, Lmax=65536, ragged=True,
        sigma_k=4.0, nan_pad=True,
        description="ragged batch with peaked softmax, B=32 Hq=32 Hkv=8 D=128 Lmax=65536, "
                    "seqlens ~ U[1,65536], q,V ~ N(0,1), K ~ N(0,4^2), NaN beyond seqlen"),
}

# Order in which the workloads are listed everywhere (tiny case first).
ORDER = ["tiny_mha", "mha_16k", "gqa_128k", "batch_4k", "ragged_64k"]

# The workload the benchmark reports by default: batch-1 MHA over a 16k context.
HEADLINE = "mha_16k"
