"""B200 (sm_100a) FlashAttention forward/backward with the Generalized Sliding
Window mask, behind the C ABI of include/attn.h (libattn.so).

The binding loads the library on first use and raises if it is missing.
"""

from . import synth  # noqa: F401  (seeded inputs; no attention arithmetic)

_BINDING_NAMES = {
    "forward", "backward", "allowed_pairs", "tile_plan", "tile_plan_bwd", "device_status",
    "lib", "AttnError", "FwdParams", "BwdParams", "WINDOW_INF", "CAUSAL_TOP_LEFT",
    "CAUSAL_BOTTOM_RIGHT",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
