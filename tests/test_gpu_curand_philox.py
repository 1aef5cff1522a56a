"""The oracle's Philox4x32-10 against calls to cuRAND's Philox4_32_10
generator (B200; compiles a small CUDA program with nvcc at test time).

cuRAND's generator, initialised with curand_init(seed, subsequence, 0),
returns from its n-th curand4() call the Philox block of counter
(n, 0, lo32(subsequence), hi32(subsequence)) under key (lo32(seed),
hi32(seed)) -- the same generator the oracle restates from Salmon et al.
(SC'11).  With subsequence = (tag << 24 | k << 12 | pos) << 32 | step the
counter is exactly the oracle's keyed counter (c0 = n, b = 0, step,
tag << 24 | k << 12 | pos), so every word must agree.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

SOURCE = r"""
#include <cstdio>
#include <curand_kernel.h>

__global__ void draw(unsigned long long seed, unsigned long long sub, int n, uint4* out) {
  curandStatePhilox4_32_10_t s;
  curand_init(seed, sub, 0ull, &s);
  for (int i = 0; i < n; ++i) out[i] = curand4(&s);
}

int main(int argc, char** argv) {
  const int n = 8;
  uint4* d = nullptr;
  cudaMalloc(&d, n * sizeof(uint4));
  unsigned long long seed, sub;
  while (std::scanf("%llu %llu", &seed, &sub) == 2) {
    draw<<<1, 1>>>(seed, sub, n, d);
    uint4 h[n];
    if (cudaMemcpy(h, d, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
    for (int i = 0; i < n; ++i) std::printf("%u %u %u %u\n", h[i].x, h[i].y, h[i].z, h[i].w);
  }
  cudaFree(d);
  return 0;
}
"""


def test_oracle_philox_matches_curand(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.fail("nvcc not found")
    src = tmp_path / "curand_philox.cu"
    exe = tmp_path / "curand_philox"
    src.write_text(SOURCE)
    subprocess.check_call([nvcc, "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-o",
                           str(exe), str(src)])
    cases = [(0, 0, 1, 0, 0), (1, 7, 2, 0, 3), (2**63 + 11, 99, 3, 5, 4),
             (0xDEADBEEFCAFEF00D, 2**32 - 1, 4, 31, 63), (12345, 123456, 2, 0, 17)]
    lines = []
    for seed, step, tag, k, pos in cases:
        hi = (tag << 24) | (k << 12) | pos
        lines.append(f"{seed} {(hi << 32) | step}")
    r = subprocess.run([str(exe)], input="\n".join(lines) + "\n", capture_output=True,
                       text=True, timeout=120, check=True)
    got = np.array([[int(x) for x in ln.split()] for ln in r.stdout.splitlines()],
                   dtype=np.uint64).reshape(len(cases), 8, 4)
    for c, (seed, step, tag, k, pos) in enumerate(cases):
        for n in range(8):
            want = [oracle.stream_word(seed, step, tag, 0, k, pos, n, w) for w in range(4)]
            assert got[c, n].tolist() == want, (seed, step, tag, k, pos, n)
