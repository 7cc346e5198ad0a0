"""B200-native hybrid prefill + decode attention (POD-Attention's hot path).

The product is ``libpod_attn.so`` (CUDA for sm_100a behind a C ABI declared in
``include/pod_attn.h``). :mod:`.pod_attn` is the thin ctypes binding over it;
:mod:`.workloads` draws the seeded synthetic batches the tests and the
benchmark use.
"""
