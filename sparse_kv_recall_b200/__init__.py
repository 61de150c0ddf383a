"""B200 (sm_100a) decode hot path of On-Demand Attention and Declarative Attention block
masks: liboda.so (CUDA kernels behind a C ABI, include/oda.h) and its ctypes binding."""
from . import da, oda  # noqa: F401
from .oda import OdaError, StepGraph, load  # noqa: F401

__version__ = "0.1.0"
