"""The CUDA path's dropout generator (csrc/philox.cuh) on the host: its
Philox4x32-10 and the dropout counter layout, compiled with g++ from the
same header the kernels include, equal the oracle's independent generator
and keep mask bit for bit; the device path compiles for sm_100a."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "io_aware_exact_33_b200", "csrc")

HARNESS = r"""
#include <stdio.h>
#include <stdlib.h>
#include "philox.cuh"
// mode 0: stdin lines "c0 c1 c2 c3 k0 k1" -> four output words
// mode 1: argv B H Nq Nk t seed offset -> keep mask, one 0/1 per element
int main(int argc, char** argv) {
  if (atoi(argv[1]) == 0) {
    unsigned c0, c1, c2, c3, k0, k1;
    while (scanf("%u %u %u %u %u %u", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
      attn::Philox4 r = attn::philox4x32_10(c0, c1, c2, c3, k0, k1);
      printf("%u %u %u %u\n", r.w[0], r.w[1], r.w[2], r.w[3]);
    }
    return 0;
  }
  const int B = atoi(argv[2]), H = atoi(argv[3]), Nq = atoi(argv[4]), Nk = atoi(argv[5]);
  const unsigned t = (unsigned)atoi(argv[6]);
  const unsigned long long seed = strtoull(argv[7], 0, 10);
  const unsigned offset = (unsigned)strtoul(argv[8], 0, 10);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < Nq; ++i)
        for (int j = 0; j < Nk; ++j) {
          attn::Philox4 r = attn::dropout_block(seed, offset, b * H + h, i / 4, j / 4);
          unsigned u = (r.w[i % 4] >> (8 * (j % 4))) & 0xFFu;
          putchar(attn::dropout_factor(u, t) != 0.f ? '1' : '0');
        }
  return 0;
}
"""

DEVICE_USE = r"""
#include "philox.cuh"
__global__ void use(unsigned* out, unsigned long long seed) {
  attn::Philox4 r = attn::dropout_block(seed, 1u, blockIdx.x, threadIdx.x, 3u);
  out[blockIdx.x * blockDim.x + threadIdx.x] = r.w[0] ^ r.w[3];
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("philox")
    src = d / "h.cpp"
    src.write_text(HARNESS)
    exe = d / "h"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)], check=True)
    return str(exe)


def test_generator_matches_oracle(harness):
    rng = np.random.default_rng(5)
    rows = rng.integers(0, 2 ** 32, size=(400, 6), dtype=np.uint64).tolist()
    rows += [[0, 0, g, 0, 0xDEADBEEF, 0x12345] for g in range(8)]
    rows += [[2 ** 32 - 1] * 6, [0] * 6]
    inp = "\n".join(" ".join(str(x) for x in r) for r in rows) + "\n"
    out = subprocess.run([harness, "0"], input=inp, capture_output=True, text=True, check=True)
    got = [list(map(int, line.split())) for line in out.stdout.strip().splitlines()]
    assert len(got) == len(rows)
    for r, g in zip(rows, got):
        assert g == oracle.philox4x32_10(r[:4], r[4:]), f"counter {r}"


@pytest.mark.parametrize("p,seed,offset", [(0.1, 0x0123456789ABCDEF, 0), (0.5, 7, 12345),
                                           (0.9, 2 ** 64 - 1, 2 ** 32 - 1)])
def test_keep_mask_matches_oracle(harness, p, seed, offset):
    B, H, Nq, Nk = 2, 3, 13, 10  # ragged in both block directions
    t = oracle.dropout_threshold(p)
    out = subprocess.run([harness, "1", str(B), str(H), str(Nq), str(Nk), str(t), str(seed),
                          str(offset)], capture_output=True, text=True, check=True).stdout
    got = np.frombuffer(out.encode(), dtype=np.uint8).reshape(B, H, Nq, Nk) - ord("0")
    want = oracle.dropout_keep(B, H, Nq, Nk, p, seed, offset)
    assert np.array_equal(got, want)


def test_device_path_compiles(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "d.cu"
    src.write_text(DEVICE_USE)
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-c",
                    "-o", str(tmp_path / "d.o"), str(src)], check=True)
