"""B200-native (sm_100a) CODA GEMM-epilogue kernels for the
GEMM-Residual-RMSNorm-GEMM(+SwiGLU) block and the SwiGLU MLP.

The compute path is ``lib/libcoda.so`` (C ABI in ``include/coda.h``); the
``binding`` module marshals torch tensors into it.  ``synth`` draws the seeded
synthetic inputs.  Import is cheap: the library loads on first use.
"""

__version__ = "0.1.0"
