"""Workload table for the MoE layer with zero-computation experts.

Shapes follow the LongCat-Flash Technical Report, §2.1 (zero-computation
experts) and §2.4 (model information: hidden 6144, expert intermediate 2048,
512 FFN experts + 256 zero experts, 12 experts per token).  The smaller
shapes are synthetic stand-ins at the same structure.

Notation (as in §2.1, Eq. (1) and Eq. (2)):
    T tokens, d hidden size, N FFN experts, Z zero-computation experts,
    E = N + Z, K experts per token, I expert intermediate size,
    K_e target number of FFN experts per token.
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    N: int
    Z: int
    K: int
    I: int
    dtype: str          # "f32" or "bf16": the storage type of x and of every weight
    w_std: float        # std of the N(0, w_std) weight draws
    bias_kind: str      # "zero" or "uniform" (U(-bias_amp, bias_amp))
    bias_amp: float = 0.0
    gamma: float = 1.0  # §2.3.2, Eq. (8) scale; 1 unless stated
    mu: float = 0.1     # bias adaptation rate of Eq. (2)
    steps: int = 1      # bias-control steps (skewed-routing workload only)
    skewed: bool = False

    @property
    def E(self) -> int:
        return self.N + self.Z

    @property
    def K_e(self) -> float:
        # Target FFN experts per token.  §2.4 gives K_e = 8 for N=512, Z=256,
        # K=12; that equals K*N/E, which is the reading used for every shape.
        return self.K * self.N / self.E

    def with_T(self, T: int, name: str) -> "MoEConfig":
        return replace(self, T=T, name=name)


TINY_F32 = MoEConfig("tiny_f32_T256_d256_N16_Z8_K4_I128", T=256, d=256, N=16, Z=8, K=4,
                     I=128, dtype="f32", w_std=0.02, bias_kind="zero")
MID_BF16 = MoEConfig("mid_bf16_T4096_d2048_N64_Z32_K6_I1024", T=4096, d=2048, N=64, Z=32,
                     K=6, I=1024, dtype="bf16", w_std=0.02, bias_kind="uniform",
                     bias_amp=0.05)
LONGCAT_PREFILL = MoEConfig("longcat_prefill_bf16_T8192_d6144_N512_Z256_K12_I2048", T=8192,
                            d=6144, N=512, Z=256, K=12, I=2048, dtype="bf16",
                            w_std=0.006, bias_kind="zero")
# The LongCat expert geometry (d=6144, I=2048, K=12, ~128 rows per expert) on
# 32 FFN experts: a few GB, for profiling captures and quick parity runs.
LONGCAT_SLICE = MoEConfig("longcat_slice_bf16_T512_d6144_N32_Z16_K12_I2048", T=512, d=6144,
                          N=32, Z=16, K=12, I=2048, dtype="bf16", w_std=0.006, bias_kind="zero")
DECODE_T16 = MID_BF16.with_T(16, "decode_bf16_T16_d2048_N64_Z32_K6_I1024")
DECODE_T64 = MID_BF16.with_T(64, "decode_bf16_T64_d2048_N64_Z32_K6_I1024")
DECODE_T256 = MID_BF16.with_T(256, "decode_bf16_T256_d2048_N64_Z32_K6_I1024")
SKEWED_BIAS_CONTROL = replace(TINY_F32, name="skewed_f32_T16384_d256_N16_Z8_K4_steps200",
                              T=16384, steps=200, skewed=True)

CONFIGS = {c.name: c for c in (TINY_F32, MID_BF16, LONGCAT_PREFILL, DECODE_T16, DECODE_T64,
                               DECODE_T256, SKEWED_BIAS_CONTROL, LONGCAT_SLICE)}
