"""The five HiLS forward workloads (shapes and synthetic-input recipes).

Shapes stand in for the pages' 7B OLMo3-style model at 128K / 512K context
(32 query heads, 8 KV heads, head_dim 128) and for a small model; the chunk
size is 64 throughout.  The input recipe of each workload is applied by
``synth.py``; nothing here computes any part of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int            # prefill length, or KV-cache length N for decode
    d: int
    C: int
    topk: int
    M: int            # query-group size for the chunk union (prefill only)
    dtype: str        # "f32" or "bf16"
    decode: bool = False
    q_kind: str = "iid"      # "iid" N(0,1) or "ar1" (stationary AR(1) walk)
    q_sigma: float = 0.0     # AR(1) innovation std
    needles: int = 0         # planted needle chunks per KV head
    needle_amp: float = 2.0  # needle key shift = amp * sqrt(d) * u_h
    lmk_noise: float = 0.0   # landmark = chunk-mean(keys) + N(0, lmk_noise^2); 0 -> iid N(0,1)
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5

    @property
    def n_lmk(self) -> int:
        """Landmark keys per KV head: one per complete chunk."""
        return self.L // self.C

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny_prefill_f32_L4096", B=1, Hq=1, Hkv=1, L=4096, d=64, C=64, topk=8,
                    M=16, dtype="f32", seed=1000)
SMALL_32K = Workload("small_prefill_bf16_L32768", B=2, Hq=16, Hkv=16, L=32768, d=64, C=64,
                     topk=16, M=64, dtype="bf16", needles=4, lmk_noise=0.5, seed=1001)
PREFILL_128K = Workload("prefill_7b_gqa_bf16_L131072", B=1, Hq=32, Hkv=8, L=131072, d=128,
                        C=64, topk=32, M=64, dtype="bf16", q_kind="ar1", q_sigma=0.05,
                        lmk_noise=0.5, seed=1002)
DECODE_512K = Workload("decode_gqa_bf16_B16_N524288", B=16, Hq=32, Hkv=8, L=524288, d=128,
                       C=64, topk=64, M=64, dtype="bf16", decode=True, lmk_noise=0.5, seed=1003)
PREFILL_512K = Workload("prefill_7b_gqa_bf16_L524288", B=1, Hq=32, Hkv=8, L=524288, d=128,
                        C=64, topk=64, M=128, dtype="bf16", q_kind="ar1", q_sigma=0.02,
                        needles=64, lmk_noise=0.5, seed=1004)

WORKLOADS = [TINY_F32, SMALL_32K, PREFILL_128K, DECODE_512K, PREFILL_512K]
BY_NAME = {w.name: w for w in WORKLOADS}
