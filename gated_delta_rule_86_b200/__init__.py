"""B200-native (sm_100a) KDA operator: chunkwise prefill and recurrent decode.

The computation lives in ``libkda_b200.so`` (C ABI in ``include/kda.h``);
``ops`` is its thin Python binding.  Importing the package does not load the
library; the first call does, and fails loudly if it has not been built.
"""
from ._lib import EXPORTED, KdaError, load  # noqa: F401
from .ops import (device_error, gdn_chunk_fwd, gdn_decode_step, gdn_recurrent_fwd, kda_chunk,  # noqa: F401
                  kda_chunk_bwd, kda_chunk_fwd, kda_chunk_fwd_fused, kda_decode_step, kda_decode_step_fused,
                  kda_recurrent_fwd)

__all__ = ["kda_chunk_fwd", "kda_recurrent_fwd", "kda_decode_step", "kda_chunk_fwd_fused", "kda_decode_step_fused",
           "gdn_chunk_fwd", "gdn_recurrent_fwd", "gdn_decode_step", "kda_chunk", "kda_chunk_bwd", "device_error",
           "KdaError", "load"]
