"""B200 (sm_100a) heterogeneous multi-adapter LoRA linear layer.

The compute lives in the in-tree CUDA library ``liblora_b200.so`` behind the C
ABI declared in ``include/lora.h``; ``lora_adapter_execution_b200.abi`` is a
thin ctypes binding with the same names (argument marshalling only). There is
no CPU fallback: if the library is missing, every call raises.
"""

from . import abi  # noqa: F401
from .abi import (LoraError, Plan, base_gemm, bwd_workspace_size, device_status, dropout_keep_bits, dropout_mask,  # noqa: F401
                  dropout_seed_for_rows, Switch, bwd_multi_workspace_size, linear_bwd_multi, linear_fwd_fused,
                  fused_gemm, linear_bwd, linear_bwd_static, linear_fwd, linear_fwd_host, linear_shrink, load_library,
                  selftest_bounded_wait, tsqr, tsqr_workspace_size, Compressor,
                  compress_allocate)
