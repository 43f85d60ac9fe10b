"""External pin of the oracle's Philox4x32-10 (the SR random stream): cuRAND's
Philox4_32_10 device generator, an independent implementation of the same
published algorithm (Salmon et al., SC'11), evaluated at the counters the
stochastic-rounding mapping uses, must give the same 128-bit blocks."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests.gpu_util import needs_gpu

pytestmark = needs_gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def curand_lib(tmp_path_factory):
    out = tmp_path_factory.mktemp("curand") / "libcurand_philox.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", "-o", str(out),
                    os.path.join(HERE, "support", "curand_philox.cu")], check=True)
    L = ctypes.CDLL(str(out))
    L.curand_philox_blocks.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                       ctypes.c_int, ctypes.c_void_p]
    L.curand_philox_blocks.restype = ctypes.c_int
    return L


@pytest.mark.parametrize("seed,stream", [(1234, 0), (1234, 1), (0, 0), (0xFFFFFFFFFFFFFFFF, 7),
                                         (0x0123456789ABCDEF, 3)])
def test_oracle_philox_matches_curand(curand_lib, seed, stream):
    rng = np.random.default_rng(seed & 0xFFFF)
    g = np.concatenate([np.arange(64, dtype=np.uint64),
                        rng.integers(0, 2**61, 192, dtype=np.uint64),
                        np.array([2**32 - 1, 2**32, 2**61 - 1], dtype=np.uint64)])
    got = np.zeros((g.size, 4), dtype=np.uint32)
    rc = curand_lib.curand_philox_blocks(seed, stream, g.ctypes.data, g.size, got.ctypes.data)
    assert rc == 0
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for i, gi in enumerate(g):
        ctr = [int(gi) & 0xFFFFFFFF, int(gi) >> 32, stream, 0]
        assert np.array_equal(oracle.philox4x32_10(ctr, key), got[i]), (seed, stream, int(gi))
    # the SR uniforms are the halves of these words
    L = np.array([8 * int(g[5]) + j for j in range(8)], dtype=np.uint64)
    r = oracle.sr_u16(seed, stream, L)
    words = got[5]
    want = [(words[j >> 1] >> (16 * (j & 1))) & 0xFFFF for j in range(8)]
    assert list(r) == want
