"""Workloads of the fused decode FFN half-layer: shapes, number formats, rows,
seeds and layer counts, plus the input recipe the generator follows.

Input recipe (every tensor seeded, synthetic; std is the standard deviation):
  hc_in       [R][S][H]   N(0, 1)                       -> hc element type
  mix_w       [S*H][24]   N(0, 1/sqrt(S*H))             -> fp32
  norm_w      [H]         1 + N(0, 0.1)                 -> norm element type
  router_w    [H][E]      N(0, 1/sqrt(H))               -> fp32
  router_bias [E]         U(-0.1, 0.1)                  -> fp32 (selection only)
  gate, up    [E+1][I][H] N(0, 1/sqrt(H))               -> expert format
  down        [E+1][H][I] N(0, 1/sqrt(I))               -> expert format
Slot E is the shared expert.  Quantised formats are encoded per output row:
FP8 e4m3 with an fp32 scale per 128 inputs, MXFP4 e2m1 with an e8m0 scale per
32 inputs.  Independent rows select mostly disjoint experts (about 57 unique
of 256 at 8 rows, top-8).
"""

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    n_routed: int
    top_k: int
    inter: int
    rows: int
    seed: int
    hc_dtype: str  # "f32" | "bf16"
    norm_dtype: str  # "f32" | "bf16"
    w_dtype: str  # "f32" | "bf16" | "fp8" | "mxfp4"
    round_bf16: bool
    n_layers: int = 1
    hc: int = 4
    rms_eps: float = 1e-6
    pre_eps: float = 1e-6
    post_mult: float = 2.0
    route_scale: float = 2.5
    denom_clamp: float = 1e-20
    sinkhorn_iters: int = 20
    mx_spread: int = 0   # MXFP4: block magnitudes within a row span up to 2^mx_spread
    dense: bool = False  # a dense MLP of width (n_routed + 1) * inter over every slot, no router
    act_mx8: bool = False  # MXFP4 experts: activations quantised to MXFP8 before each expert matvec

    def with_(self, **kw):
        return replace(self, **kw)

    @property
    def mix_cols(self):
        return 2 * self.hc + self.hc * self.hc


def _flash(name, rows, seed, w_dtype, n_layers=1):
    return Workload(name, hidden=5120, n_routed=256, top_k=8, inter=2048, rows=rows, seed=seed,
                    hc_dtype="bf16", norm_dtype="bf16", w_dtype=w_dtype, round_bf16=True,
                    n_layers=n_layers)


# the five configurations of the target layer
TINY_FP32 = Workload("tiny-fp32-r1", hidden=256, n_routed=16, top_k=2, inter=128, rows=1, seed=0,
                     hc_dtype="f32", norm_dtype="f32", w_dtype="f32", round_bf16=False)
FLASH_BF16_R1 = _flash("v41flash-bf16-r1", 1, 1, "bf16")
FLASH_BF16_R6 = _flash("v41flash-bf16-r6", 6, 2, "bf16")
FLASH_BF16_R8 = _flash("v41flash-bf16-r8", 8, 2, "bf16")
FLASH_FP8_R4 = _flash("v41flash-fp8b128-r4", 4, 3, "fp8")
FLASH_MXFP4_CHAIN4_R8 = _flash("v41flash-mxfp4-chain4-r8", 8, 4, "mxfp4", n_layers=4)

FULL = [TINY_FP32, FLASH_BF16_R1, FLASH_BF16_R6, FLASH_BF16_R8, FLASH_FP8_R4, FLASH_MXFP4_CHAIN4_R8]

# a dense layer of the same model family: SwiGLU width 6 x 2048 = 12288 run as
# six expert-shaped slices (five routed slots and the shared slot), weight 1
DENSE6_BF16_R1 = Workload("v41flash-dense6-bf16-r1", hidden=5120, n_routed=5, top_k=5, inter=2048, rows=1, seed=7,
                          hc_dtype="bf16", norm_dtype="bf16", w_dtype="bf16", round_bf16=True, dense=True)


def scaled(w: Workload, hidden=1024, n_routed=32, top_k=4, inter=512, **kw) -> Workload:
    """A smaller copy of a workload that the oracle finishes in seconds while
    still spanning several tiles per CTA and a ragged tail."""
    return w.with_(name=w.name + f"-h{hidden}", hidden=hidden, n_routed=n_routed, top_k=top_k,
                   inter=inter, **kw)


# the MXFP4 chain with the MXFP8-activation numerics (vLLM MonoKernel page,
# Numerics): not one of the five configurations; a parity and bench case
FLASH_MXFP4_MX8_CHAIN4_R8 = FLASH_MXFP4_CHAIN4_R8.with_(name="v41flash-mxfp4-mx8act-chain4-r8", act_mx8=True)

BY_NAME = {w.name: w for w in FULL + [DENSE6_BF16_R1, FLASH_MXFP4_MX8_CHAIN4_R8]}
