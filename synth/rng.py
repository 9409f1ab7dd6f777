"""ctypes front end of ``gen.c`` (counter-based SplitMix64 + Box-Muller)."""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

# Named streams: every array of a workload draws from its own stream.
STREAM_PARAM = 1
STREAM_GRAD = 2
STREAM_SHAPES = 3
STREAM_SAMPLE = 4


def build(force=False):
    """Compile gen.c into libsynth.so beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
             "-o", _LIB, _SRC, "-lm"])
    return _LIB


def load_lib():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        lib.synth_key.restype = u64
        lib.synth_key.argtypes = [u64, u64]
        lib.synth_u64.restype = u64
        lib.synth_u64.argtypes = [u64, u64]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, ctypes.c_void_p]
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, dbl, ctypes.c_void_p]
        lib.synth_uniform_f64.argtypes = [u64, u64, i64, ctypes.c_void_p]
        _lib = lib
    return _lib


def stream_key(seed, stream):
    return int(load_lib().synth_key(int(seed) & (2**64 - 1), int(stream)))


def normal_f32(key, first, count, sigma, out=None):
    """float32 array of sigma*N(0,1) for element indices [first, first+count)."""
    if out is None:
        out = np.empty(count, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size >= count
    load_lib().synth_normal_f32(key, int(first), int(count), float(sigma), out.ctypes.data)
    return out


def normal_bf16(key, first, count, sigma, out=None):
    """uint16 array of bf16 bit patterns of sigma*N(0,1), same indexing."""
    if out is None:
        out = np.empty(count, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size >= count
    load_lib().synth_normal_bf16(key, int(first), int(count), float(sigma), out.ctypes.data)
    return out


def uniform_f64(key, first, count):
    out = np.empty(count, dtype=np.float64)
    load_lib().synth_uniform_f64(key, int(first), int(count), out.ctypes.data)
    return out
