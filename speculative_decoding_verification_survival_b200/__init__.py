"""B200-native (sm_100a) hot path of DSpark confidence-scheduled speculative-decoding verification.

The compute lives in libdspark.so (CUDA kernels behind the C ABI declared in include/dspark.h);
`dspark` is its thin ctypes binding (importing it fails loudly when the library is missing) and
`step.VerifyStep` issues one whole verify step and `pipeline.RoundPipeline` replays verify rounds
as CUDA graphs chained on the device.  `build` compiles the library in-tree.
"""
import importlib


def __getattr__(name):
    if name == "dspark":
        return importlib.import_module(".dspark", __name__)
    if name == "VerifyStep":
        return importlib.import_module(".step", __name__).VerifyStep
    if name == "RoundPipeline":
        return importlib.import_module(".pipeline", __name__).RoundPipeline
    raise AttributeError(name)
