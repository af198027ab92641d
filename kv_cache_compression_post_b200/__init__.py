"""kvb: historical KV-bank management (DensityKV, Forcing-KV) on sm_100a.

The binding lives in ``kv_cache_compression_post_b200.kvb`` (loaded on first
use: importing it fails loudly if ``libkvb.so`` has not been built with
``python -m kv_cache_compression_post_b200.build``).  Names such as
``kv_cache_compression_post_b200.kvb_admit`` are forwarded to it.
"""


def __getattr__(name):
    if name.startswith("kvb_") or name in ("KvbError", "make_config", "lib", "LIB_PATH", "Bank", "PAGES_PRESET") \
            or name.startswith("KVB_"):
        from . import kvb as _kvb
        return getattr(_kvb, name)
    raise AttributeError(name)
