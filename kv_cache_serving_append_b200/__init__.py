"""B200-native KV-cache upkeep and FP8 attention for batch-size-one
autoregressive video diffusion serving.

``kv_cache_serving_append_b200.rtv`` is the Python binding of the C-ABI
library ``librtv.so`` (argument marshalling only; every step runs in the
library's CUDA kernels).  ``configs`` and ``synth`` hold workload shapes and
seeded synthetic inputs.  Importing this package does not load the library;
importing ``.rtv`` does, and fails loudly if it is missing.
"""
