"""B200-native PowerSGD compression step: a C-ABI CUDA library (libpsgd.so,
include/psgd.h) and its thin ctypes binding."""
from ._lib import PowerSGD, PsgdError, load, LIB_PATH  # noqa: F401
