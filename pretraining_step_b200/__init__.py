"""B200 (sm_100a) base-pretraining step of the depth-parametrised nanochat GPT.

The computation lives in libnc_b200.so (C ABI: include/nc.h), built by
pretraining_step_b200/build.py; `binding` is its ctypes binding and
`inputs` the seeded synthetic-input generators.
"""
__all__ = ["inputs", "binding", "build"]
