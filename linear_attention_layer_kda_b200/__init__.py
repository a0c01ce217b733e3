"""B200 (sm_100a) KDA layer-half decode step.

The compute path is the CUDA library ``libkda_decode.so`` (C ABI in
include/kda_decode.h), reached through ``binding`` (ctypes, argument
marshalling only).  ``inputs`` makes seeded synthetic workloads; ``tensors``
moves them into torch CUDA tensors; ``tp`` splits a layer half by heads over
ranks.  There is no CPU implementation of the decode step in this package.
"""
from .binding import (KdaDecoder, KdaError, kda_config, kda_weights, load, make_config,  # noqa: F401
                      weights_from_tensors)

__all__ = ["KdaDecoder", "KdaError", "kda_config", "kda_weights", "load", "make_config", "weights_from_tensors"]
