"""B200-native Reduced Matrix Multiplication (RMM).

`rmm` is the ctypes binding over librmm.so (the C ABI in include/rmm.h);
`inputs` draws the seeded synthetic workloads; `build` compiles the library.
Importing the package does not load the shared library; the first call does.
"""
from . import inputs  # noqa: F401
