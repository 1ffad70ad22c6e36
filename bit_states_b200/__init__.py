"""bit_states_b200 - FlashOptim-style fused compressed-state optimizer step for
NVIDIA B200 (sm_100a).

The product is ``libfo.so`` (C ABI in ``include/fo.h``); ``fo`` is its ctypes
binding and ``state`` allocates the compressed buffers with torch.
"""
from . import fo  # noqa: F401
from .fo import (FoError, TensorState, descriptors, fo_adamw_hparams, fo_adamw_step,  # noqa: F401
                 fo_decode_master, fo_encode_master, fo_format, fo_sgdm_hparams, fo_sgdm_step,
                 fo_stream_copy, fo_tensor, make_format)
