"""B200-native paged-KV hot path: store_kvcache, paged decode, varlen prefill.

The CUDA library is loaded on first use; see ``_binding``.
"""
from ._binding import *  # noqa: F401,F403
from ._binding import load_library  # noqa: F401
