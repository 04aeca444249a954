"""fp64 CPU oracle of one MiniMax-H3 transformer block (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA library never does.
"""
from .h3_block import (  # noqa: F401
    BlockOracle, adaln, apply_rope, attention, documents, int8_matmul_exact,
    modulation, prepare_int8_weight, qk_rmsnorm, quantize_rows, rmsnorm,
    rope_angles, rope_frequencies, rotate_blocks, silu, softmax, swiglu,
    sylvester_hadamard, w8a8_linear,
)
from .h3_modulation import (  # noqa: F401
    modulation_table, produce, sinusoidal_embedding, time_mlp, timestep_frequencies, two_time_embedding,
)
from .h3_model import ModelOracle, affine, norm_out, refine_text, scatter_rows  # noqa: F401
from .h3_sparse import block_scores, select, sparse_attention, sparse_block_attention  # noqa: F401
