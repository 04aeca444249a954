"""B200-native forward of one MiniMax-H3 transformer block, and of the model
shell (input projections, token refiner, block stack, heads) around it.

The compute lives in libh3blk.so (hand-written sm_100a CUDA kernels behind the
C-ABI declared in include/h3blk.h). This package is its ctypes binding and a
thin torch-tensor wrapper; importing it fails if the library is not built.
"""
from ._binding import (  # noqa: F401
    EXPORTS, H3BLK_OK, H3BlkError, LIB_PATH, STAGE, STAGES, h3blk_config, h3blk_weights,
)
from . import _binding as capi  # noqa: F401
from .block import (  # noqa: F401
    DeviceWeights, H3Block, ModulationWeights, gemm_bf16, gemm_s8_s32, make_config, modulation_table, rotate_quantize,
)
from .model import DeviceInputs, DeviceModel, Model, ModelGraph  # noqa: F401
