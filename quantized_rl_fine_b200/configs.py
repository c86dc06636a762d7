"""The five synthetic workloads of the low-bit MoE layer, named by what they are.

Shapes follow the layers the Orbit article trains in one 8xB200 node
(trillion-parameter INT4 MoE, FP4 MoE); the distributions are the ones the
workload list fixes (BF16 N(0,1) activations, N(0,0.02) weights quantized to
the 4-bit base, router logits N(0,1), U[0,1) or N(0,1) + Zipf bias, adapter
I + N(0, 1e-3), upstream gradient N(0,1)).
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    E: int            # experts
    k: int            # experts per token
    d: int            # hidden size
    f: int            # expert FFN width
    T: int            # tokens
    fmt: str          # "int4" (BF16 group scales) or "mxfp4" (E8M0 group scales)
    swiglu: bool      # gate/up + down with SwiGLU; False = single up-projection
    logits: str       # "normal", "uniform" or "zipf"
    adapter: bool     # BF16 block-diagonal adapter on the gate/up input
    train: bool       # also run the backward to activations and adapter
    seed: int
    chunk_size: int = 8

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    @property
    def M(self) -> int:
        return self.T * self.k


TINY_INT4 = MoEConfig("tiny_int4_E8_k2_d256_f512_T64", E=8, k=2, d=256, f=512, T=64,
                      fmt="int4", swiglu=True, logits="normal", adapter=False, train=False,
                      seed=1001)

MXFP4_UP = MoEConfig("mxfp4_up_E64_k4_d2048_f1024_T1024", E=64, k=4, d=2048, f=1024, T=1024,
                     fmt="mxfp4", swiglu=False, logits="uniform", adapter=False, train=False,
                     seed=1002)

TRILLION_INT4 = MoEConfig("trillion_int4_E384_k8_d7168_f2048", E=384, k=8, d=7168, f=2048,
                          T=2048, fmt="int4", swiglu=True, logits="normal", adapter=False,
                          train=False, seed=1003)
TRILLION_T_SWEEP = (128, 2048, 16384)
CHUNK_SWEEP = (8, 16, 32)

ZIPF_MXFP4 = MoEConfig("zipf_mxfp4_E256_k8_d4096_f1536_T8192", E=256, k=8, d=4096, f=1536,
                       T=8192, fmt="mxfp4", swiglu=True, logits="zipf", adapter=False,
                       train=False, seed=1004)

TRAIN_INT4 = MoEConfig("train_int4_adapter_E384_k8_d7168_f2048_T4096", E=384, k=8, d=7168,
                       f=2048, T=4096, fmt="int4", swiglu=True, logits="normal", adapter=True,
                       train=True, seed=1005)

ALL = {c.name: c for c in (TINY_INT4, MXFP4_UP, TRILLION_INT4, ZIPF_MXFP4, TRAIN_INT4)}
