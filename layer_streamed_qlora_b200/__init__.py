"""B200 (sm_100a) layer-streamed LoRA training over a frozen NF4/bf16 base.

The compute path is the CUDA library ``libsoup.so`` (C ABI in
``include/soup.h``); ``_lib`` binds it with ctypes.  Importing this package does
not load the library; the first call into ``_lib`` does, and fails loudly if the
library has not been built.
"""
