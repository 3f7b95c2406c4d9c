"""B200-native gated local/full decode attention (On-Demand Attention's hot path).

The compute lives in liboda.so (CUDA for sm_100a, C ABI in include/oda.h);
``gated_local_full_b200.oda`` is its thin Python binding.
"""

from .oda import (  # noqa: F401
    BF16, F32, EXPORTS, LIB_PATH, MAX_BATCH, OdaConfig, OdaContext, OdaError, OdaGraph,
    OdaStepDesc, layout, lib, make_config, ptr, version,
)
