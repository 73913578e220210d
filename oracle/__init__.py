"""The oracle: a plain, slow CPU restatement of the binary convolution (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``bconv_oracle.c`` (plain C, double accumulation, one multiply per
bit).  This module compiles it with gcc on first use and marshals numpy arrays through
ctypes; it holds none of the method's arithmetic itself.
"""
from .oracle import (  # noqa: F401
    ORACLE_AND,
    ORACLE_BINARY_WEIGHTS,
    ORACLE_XNOR,
    SOURCE_PATH,
    Variant,
    compile_source,
    binarize,
    build,
    conv,
    conv_out_dims,
    fc,
    num_threads,
)
