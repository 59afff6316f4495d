"""The oracle's Philox4x32-10 against cuRAND's device-side Philox (curand_kernel.h, compiled here
into a small test library), on counters whose high words are nonzero.

curand_init(seed, subsequence, offset) keys the generator with the 64-bit seed and starts it at
counter (offset / 4 as a 64-bit value over words 0-1, subsequence over words 2-3); curand4 then
returns the four words of that counter.  Subsequences of 2^32 and above set counter word 3,
which the host-generator pin of the CPU suite never reaches.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

_SRC = r"""
#include <cstdint>
#include <curand_kernel.h>

__global__ void philox_first_block(unsigned long long seed, const unsigned long long* subseq,
                                   const unsigned long long* offset, uint4* out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    curandStatePhilox4_32_10_t st;
    curand_init(seed, subseq[i], offset[i], &st);
    out[i] = curand4(&st);
}

extern "C" int philox_first_blocks(unsigned long long seed, const unsigned long long* subseq,
                                   const unsigned long long* offset, unsigned int* out, int n) {
    philox_first_block<<<(n + 63) / 64, 64>>>(seed, subseq, offset, reinterpret_cast<uint4*>(out), n);
    return static_cast<int>(cudaDeviceSynchronize());
}
"""


@pytest.fixture(scope="module")
def curand_lib(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    d = tmp_path_factory.mktemp("curand_philox")
    src, lib = d / "probe.cu", d / "libprobe.so"
    src.write_text(_SRC)
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", str(src), "-o", str(lib)], check=True)
    L = ctypes.CDLL(str(lib))
    L.philox_first_blocks.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_int]
    L.philox_first_blocks.restype = ctypes.c_int
    oracle.build()
    return L


def test_philox_matches_curand_device_api(curand_lib):
    rng = np.random.default_rng(17)
    n = 256
    sub = rng.integers(0, 2 ** 63, n, dtype=np.uint64)
    sub[:4] = [1 << 32, (1 << 32) + 5, 2 ** 63 - 1, 7]          # word 3 set, and one small case
    blocks = rng.integers(0, 2 ** 40, n, dtype=np.uint64)
    blocks[:4] = [0, 3, 1 << 33, 0]
    for seed in (0x0123456789ABCDEF, 2 ** 64 - 1, 42):
        s_d = torch.from_numpy(sub.view(np.int64)).cuda()
        o_d = torch.from_numpy((blocks * np.uint64(4)).view(np.int64)).cuda()
        out = torch.zeros(4 * n, dtype=torch.int32, device="cuda")
        assert curand_lib.philox_first_blocks(seed, s_d.data_ptr(), o_d.data_ptr(), out.data_ptr(), n) == 0
        got = out.cpu().numpy().view(np.uint32).reshape(n, 4)
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for i in range(n):
            c, s = int(blocks[i]), int(sub[i])
            ref = oracle.philox4x32_10([c & 0xFFFFFFFF, c >> 32, s & 0xFFFFFFFF, s >> 32], key)
            assert np.array_equal(got[i], ref), (hex(seed), hex(s), hex(c))
