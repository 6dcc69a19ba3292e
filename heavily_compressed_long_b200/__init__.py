"""B200-native CSA / HCA hybrid-attention hot path (libhcl: CUDA kernels for sm_100a behind a
C ABI, include/hcl.h).  `api` is the Python binding with the C ABI's names."""
from . import api  # noqa: F401
from ._lib import lib  # noqa: F401
