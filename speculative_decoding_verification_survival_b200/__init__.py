"""B200-native (sm_100a) hot path of DSpark confidence-scheduled speculative-decoding verification.

The compute lives in libdspark.so (CUDA kernels behind the C ABI declared in include/dspark.h);
`dspark` is its thin ctypes binding (importing it fails loudly when the library is missing) and
`step.VerifyStep` issues one whole verify step.  `build` compiles the library in-tree.
"""
import importlib


def __getattr__(name):
    if name == "dspark":
        return importlib.import_module(".dspark", __name__)
    if name == "VerifyStep":
        return importlib.import_module(".step", __name__).VerifyStep
    raise AttributeError(name)
