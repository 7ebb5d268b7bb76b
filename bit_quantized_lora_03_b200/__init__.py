"""QLoRA NF4 frozen-base linear layer for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library libqlora_nf4.so (hand-written CUDA kernels);
`binding` marshals torch tensors into it. `inputs` draws the seeded synthetic workloads.
"""

from .binding import (PackedNF4, codebook, last_status, nf4_dequantize, nf4_quantize,  # noqa: F401
                      qlora_linear_bwd, qlora_linear_fwd)
