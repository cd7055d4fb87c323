"""B200-native 32-bit two-state optimizer step (Adam/AdamW, AdEMAMix).

The work happens in libopt2s.so (hand-written CUDA for sm_100a behind the C
ABI of include/opt2s.h); ``binding`` is its thin ctypes front end, ``synth``
makes seeded synthetic inputs, ``shard`` splits a collection across ranks.
"""
from .binding import (ALGOS, DTYPES, Hyper, Opt2sError, Plan, TensorList,  # noqa: F401
                      TensorList8, lib, make_hyper, opt2s_release_cache, opt2s_step,
                      opt2s_step_8bit, opt2s_step_lamb, opt2s_step_max_unorm)

__all__ = ["ALGOS", "DTYPES", "Hyper", "Opt2sError", "Plan", "TensorList", "TensorList8", "lib",
           "make_hyper", "opt2s_release_cache", "opt2s_step", "opt2s_step_8bit", "opt2s_step_lamb",
           "opt2s_step_max_unorm"]
