"""B200-native batch-1 q4_0 decode step: libq4g (CUDA, sm_100a) and its Python binding."""
from . import q4g  # noqa: F401
