"""B200-native looped Recurrent Block of the OpenMythos Recurrent-Depth Transformer.

The compute path is librdt.so (hand-written sm_100a CUDA kernels behind the C ABI in
include/rdt.h); this package is its Python binding.  Build the library with
``python -m recurrent_depth_moe_b200.build``.
"""
from ._native import RdtError, RDT_FLAG_TRANSFORMER_OFF, load as load_library  # noqa: F401
from .api import (RecurrentBlock, KVCache, Trace, Block, Generator, DecodeGraph, DepthBatch, block_forward,  # noqa: F401
                  embed, head,
                  model_forward, generate, greedy_tokens, to_model_dtype, config_struct, dense_config_struct,
                  workspace_size, alloc_workspace)
