"""ssa: structured sparse attention (DAM diagonal + vertical patterns) for B200.

The compute lives in ``libssa.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/ssa.h``); ``binding`` is the thin ctypes layer over it.
The binding is imported lazily so that the seeded input generator (``inputs``)
can be used without loading the CUDA library.
"""

_BINDING_NAMES = ("attn_maps", "capture", "extend", "refill", "attn_fwd", "attn_ws_bytes", "attn_decode", "set_wait_limit_ns",
                  "SSAError", "Plan", "load")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
