"""B200-native hybrid compressed attention (CSA / HCA) for sm_100a.

The work is done by libhcsa.so (hand-written CUDA behind the C ABI declared in
include/hca_csa.h); this package is its ctypes binding plus layer helpers that
allocate device buffers with torch and issue the calls in order.
"""
from ._lib import *  # noqa: F401,F403
from ._lib import EXPORTS, HcsaError, load, make_cache, make_params  # noqa: F401
from .layer import DecodeLayer, PrefillLayer, params_for, torch_dtype  # noqa: F401
from .sharded import ShardedDecodeLayer, ShardedPrefillLayer, entry_range, shard_cache, zigzag_chunks  # noqa: F401
