"""Uno draft-and-verify hot path on NVIDIA B200 (sm_100a).

The computation lives in libuno.so (CUDA kernels behind the C ABI of include/uno.h):
the row-gated LoRA linear, the lossless block verify and the TV self-distillation loss.
This package is its thin Python binding (plus `driver`, the decode step chained on one
stream); `workloads` holds the seeded synthetic inputs.
"""
from ._lib import (  # noqa: F401
    UNO_BF16, UNO_F32, UNO_OK, UnoError, load, uno_block_noise, uno_block_verify, uno_block_verify_workspace_size,
    uno_block_verify_min_workspace_size,
    uno_gated_lora_linear, uno_gated_lora_linear_workspace_size, uno_read_device_status, uno_tv_loss,
    uno_tv_loss_workspace_size, uno_version,
)
