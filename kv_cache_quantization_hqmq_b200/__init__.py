"""HQMQ (Hurwitz Quaternion Multiplicative Quantization) KV-cache codec for
NVIDIA B200 (sm_100a).

* ``csrc/``      CUDA kernels and the C ABI of include/hqmq.h (libhqmq.so)
* ``hqmq``       thin ctypes binding of that ABI (raises if the library is missing)
* ``workloads``  seeded synthetic KV-cache inputs shaped like the pages' models
* ``build``      in-tree nvcc build of libhqmq.so
"""
__version__ = "1.0"
