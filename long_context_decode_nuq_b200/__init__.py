"""KVQuant quantized-KV decode path for NVIDIA B200: Python binding of libkvq.so."""
from .kvq import *  # noqa: F401,F403
from .kvq import (  # noqa: F401
    Cache, Cfg, Codebook, KvqError, load, make_cfg, EXPORTS, LIB_PATH,
)
