"""The five synthetic workloads of the SSD layer scan, by name and size.

Each workload fixes the tensor shapes of the Mamba-2 SSD sequence mixer
(batch b, sequence length L, heads H, head dimension P, state dimension N,
B/C groups G, chunk length Q), the element type of x/B/C/y, and whether a
nonzero initial state is passed.  The value distributions are drawn by
``inputs.make_inputs``; this module holds sizes only.

Sizes follow the layer shapes the pages discuss: state dimension 64-256 and
multi-head SSMs (crackai.dev "Transformers are SSMs", How It Works), chunk
lengths 64-256 (mohakchugh.is-a.dev "Mamba-2", Block Decomposition).
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str            # "f32" or "bf16": element type of x, B, C and y
    init_state: bool      # nonzero fp32 initial state ~ N(0, 0.1^2)
    seed: int
    decode: bool = False  # consumed one token per call by the decode update
    nseq: int = 0         # > 0: batch 1 holds nseq packed sequences of uneven length

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Parity-sized fp32 case the oracle finishes in well under a second.
SSD_F32_SMALL = Workload("ssd_fwd_f32_b1_L256_H2_P64_N64_Q64", 1, 256, 2, 64, 64, 1, 64,
                         "f32", False, 1000)
# ~370M-parameter Mamba-2 layer (d_inner = 1536).
SSD_370M = Workload("ssd_fwd_bf16_b2_L2048_H24_P64_N128_Q256", 2, 2048, 24, 64, 128, 1, 256,
                    "bf16", False, 1001)
# 2.7B-parameter Mamba-2 layer (d_model 2560, expand 2 -> 80 heads of 64), final states returned.
SSD_2P7B = Workload("ssd_fwd_bf16_b4_L4096_H80_P64_N128_Q256", 4, 4096, 80, 64, 128, 1, 256,
                    "bf16", False, 1002)
# Long context: 256 chunks of state passing, 8 groups, nonzero initial state.
SSD_LONG = Workload("ssd_fwd_bf16_b1_L65536_H32_P64_N128_G8_Q256_init", 1, 65536, 32, 64, 128, 8,
                    256, "bf16", True, 1003)
# Recurrent decode: 1000 consecutive single-token updates of a (128, 80, 64, 128) fp32 state.
SSD_DECODE = Workload("ssd_decode_bf16_b128_H80_P64_N128_1000steps", 128, 1000, 80, 64, 128, 1,
                      256, "bf16", True, 1004, decode=True)

# Packed variable-length sequences: the 2.7B layer's 16384 tokens as 12 sequences of uneven
# length in one row, each with its own nonzero initial state and final state.
SSD_VARLEN = Workload("ssd_varlen_bf16_T16384_seq12_H80_P64_N128_Q256_init", 1, 16384, 80, 64,
                      128, 1, 256, "bf16", True, 1005, nseq=12)

ALL = (SSD_F32_SMALL, SSD_370M, SSD_2P7B, SSD_LONG, SSD_DECODE, SSD_VARLEN)
BY_NAME = {w.name: w for w in ALL}
