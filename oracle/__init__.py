"""CPU fp64 oracle of MILO's compressed-KV decode path.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
restatement of the method that the CUDA path is checked against.  Only the
tests, the smoke check and the benchmark's CPU-baseline leg may import it;
the library itself never does, and it shares no code with the library.

Sources (page "MILO: Efficient Many-shot In-Context Learning with Block-wise
Low-rank Compression", a section summary of the paper):
  §4.2  block-wise low-rank compression of keys and values, block by block;
  §4.3  entropy-driven rank allocation under a fixed total budget;
  §4.4  workflow: encode (partition, entropy, low-rank store), then decode;
  §5.3  composition with asymmetric INT8 quantisation (oracle/quant.py);
  §3, §4.5  pre-RoPE key factors, reconstructed and rotated at decode (oracle/rope.py).

Every function states the passage it follows and the reading taken where the
page is silent.
"""
from .milo import (  # noqa: F401
    ALLOC_RULES,
    POOL_SCOPES,
    BudgetError,
    allocate_blocks,
    allocate_ranks,
    allocate_ranks_greedy,
    allocate_ranks_random,
    allocate_ranks_uniform,
    block_svd,
    compress_layer,
    compress_layer_rule,
    compress_pool,
    decode_attention,
    decode_attention_dense,
    rank_total,
    reconstruct_pool,
    spectral_entropy,
    stored_factors,
)
from .hestenes import hestenes_svd  # noqa: F401
from .quant import (dequantize_channel, quantize_block, quantize_channel, quantize_channel_symmetric,  # noqa: F401
                    quantize_layer, quantize_pool)
from .rope import apply_rope, decode_attention_rope, inv_freq, rotated_prefix_keys  # noqa: F401
from .tiefree import cut_gap, greedy_cut_gap, tiefree_taus  # noqa: F401
