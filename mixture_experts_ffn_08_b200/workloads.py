"""The five MoE-layer workloads this library is measured and tested on.

Shapes follow the configuration table of the "MoE" chapter index (llm-infra-atlas,
§3 "一组贯穿全文的数字": Mixtral 8x7B H=4096 I=14336 E=8 top-2; DeepSeek-V3
H=7168, 256 routed experts, top-8, 1 shared expert) and the GroupedTopK setup of
"MoE 路由入门：从 Dense FFN 到 GroupedTopK" (§十: 8 groups of 32 experts, keep 4).

A workload is plain data: sizes and routing options. No arithmetic lives here.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1

DTYPE_BF16 = 0
DTYPE_FP8 = 1
DTYPE_FP8_FP4 = 2      # e4m3 activations, e2m1 weights with UE8M0 scales per 32 K elements


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    I: int                 # intermediate size of one routed expert
    E: int                 # routed experts
    K: int                 # experts chosen per token
    score_fn: int = SCORE_SOFTMAX
    n_group: int = 1       # expert groups (1 = plain top-k)
    topk_group: int = 1    # groups kept
    group_topn: int = 1    # group score = sum of the top-n selection scores in the group
    renormalize: bool = True
    routed_scale: float = 1.0
    has_bias: bool = False  # selection-only bias, fp32 [E]
    I_shared: int = 0       # intermediate size of the always-active shared expert (0 = none)
    dtype: int = DTYPE_BF16
    skewed: bool = False    # Zipf-shaped router for the skew stress case
    block_m: int = 0        # bucket row alignment: 128, 256 (two-SM GEMM tiles), 0 = library choice
    fused_combine: bool = False  # down projection adds into the output (atomic, non-deterministic)
    masked_cap: int = 0     # 0 = contiguous buckets; > 0 = masked layout, expert e owns rows [e*cap, (e+1)*cap)

    @property
    def P(self) -> int:
        return self.T * self.K

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny", T=64, H=256, I=128, E=8, K=2)

MIXTRAL_PREFILL = Workload("mixtral_prefill", T=4096, H=4096, I=14336, E=8, K=2)

DSV3_PREFILL = Workload(
    "dsv3_prefill", T=8192, H=7168, I=2048, E=256, K=8,
    score_fn=SCORE_SIGMOID, n_group=8, topk_group=4, group_topn=2,
    renormalize=True, routed_scale=2.5, has_bias=True, I_shared=2048)

DSV3_DECODE = DSV3_PREFILL.with_(name="dsv3_decode", T=128)

SKEWED_FP8 = Workload("skewed_fp8", T=16384, H=4096, I=1536, E=128, K=8,
                      dtype=DTYPE_FP8, skewed=True)

# FP8 x FP4 expert GEMMs ("DeepGEMM质变" §5.3, the Mega MoE compute unit) on the
# DeepSeek-V3 routed experts: decode (expert weights streamed from HBM at half the FP8
# bytes) and prefill.  Routed experts only: the shared expert stays a bf16-only feature.
DSV3_DECODE_FP4 = DSV3_DECODE.with_(name="dsv3_decode_fp4", dtype=DTYPE_FP8_FP4, I_shared=0)
DSV3_PREFILL_FP4 = DSV3_PREFILL.with_(name="dsv3_prefill_fp4", dtype=DTYPE_FP8_FP4, I_shared=0)

ALL = {w.name: w for w in (TINY, MIXTRAL_PREFILL, DSV3_PREFILL, DSV3_DECODE, SKEWED_FP8)}
FP4 = {w.name: w for w in (DSV3_DECODE_FP4, DSV3_PREFILL_FP4)}

# Stand-ins small enough for a full profiler capture (a few GB on the device) that keep
# the tile structure of a full workload: DeepSeek-V3 expert shapes with 32 experts and
# the same ~256 rows per expert as the 256-expert prefill.
PROFILE = {w.name: w for w in (
    DSV3_PREFILL.with_(name="dsv3_prefill_e32", T=1024, E=32),
    SKEWED_FP8.with_(name="skewed_fp8_e32", T=4096, E=32),
    DSV3_DECODE.with_(name="dsv3_decode_fp4_e64", T=32, E=64, dtype=DTYPE_FP8_FP4, I_shared=0),
    DSV3_DECODE.with_(name="dsv3_decode_e32", T=16, E=32),
)}
