"""B200-native Mixture-of-Lookup-Experts (MoLE) lookup path.

The compute lives in ``libmole.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in ``include/mole.h``).  ``mixture_lookup_experts_b200.mole`` is
the thin ctypes binding with the same entry-point names; importing it loads the
library and raises if it is missing -- there is no CPU fallback.
``mixture_lookup_experts_b200.inputs`` draws the seeded synthetic inputs.
"""
__version__ = "0.1.0"


def __getattr__(name):
    # Load the CUDA binding lazily so that ``inputs`` can be used without it.
    if name.startswith("mole_") or name in ("MoleError", "lib"):
        from . import mole
        return getattr(mole, name)
    raise AttributeError(name)
