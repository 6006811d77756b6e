"""B200 (sm_100a) fused quantized linear layer of ZeroQuant (arXiv 2206.01861).

The compute lives in ``libzq.so`` (CUDA kernels behind the C ABI of
``include/zq.h``); ``zq`` is its Python binding.  Import ``zq`` explicitly:
it fails loudly when the library has not been built.
"""
