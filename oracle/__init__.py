"""CPU oracle (test infrastructure only; see ``w4a16_oracle``)."""
from .w4a16_oracle import (  # noqa: F401
    GROUP,
    QuantRangeError,
    awq_alpha_grid,
    awq_clip_search,
    awq_scale_search,
    awq_scales,
    channel_mean_abs,
    clip_ratio_grid,
    dequantize,
    fp16_round_up,
    gemm,
    gemm_entries,
    pack_nibbles,
    quantize_pack,
    quantize_rtn,
    unpack_nibbles,
)
