"""B200-native scaled quantize / dequantize.

`_bq` is the ctypes binding of libbq.so (one function per C entry point,
same names); `api` adds helpers that allocate outputs with torch. Importing
this package loads libbq.so and fails if it has not been built.
"""

from . import _bq  # noqa: F401  (loads libbq.so or raises ImportError)
from ._bq import *  # noqa: F401,F403
from . import api  # noqa: F401
