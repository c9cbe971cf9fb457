"""CSA2 sparse attention over a shared FP4 global KV cache, for NVIDIA B200 (sm_100a).

The computation lives in libcsa2.so (hand-written CUDA, C ABI in include/csa2.h);
this package only marshals PyTorch tensors into that ABI.
"""
from . import capi  # noqa: F401
from .capi import (CSA2_FULL, CSA2_REINDEX, CSA2_REUSE, Csa2Error, csa2_fp4_quantize,  # noqa: F401
                   csa2_index_topk, csa2_layer_stack, csa2_sparse_attn, csa2_status_string,
                   csa2_workspace_bytes)
from .ops import (LayerStack, Status, Workspace, cache_append, fp4_compress, fp4_quantize,  # noqa: F401
                  index_topk,
                  sparse_attn)
