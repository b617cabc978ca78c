"""The FP4 quantiser of the cache-append kernel, run on the host.

`csrc/append_quant.cuh` holds the kernel's per-group quantiser as a
__host__ __device__ function built on CUDA's float -> FP8 / FP4 conversions.
This test compiles a small host program around it with nvcc (no GPU needed)
and checks its scale and code bytes against the oracle's quantiser taking its
decisions in float32 (fp4_quantize(..., decide_in_f32=True)): bit for bit, on
N(0,1) latents at three magnitudes, nearest-even ties of both formats,
saturation, tiny and zero groups.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import v41

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "latent_kv_decode_b200", "csrc")

DRIVER = r'''
#include <cstdio>
#include "append_quant.cuh"
int main() {
  float x[16];
  while (fread(x, sizeof(float), 16, stdin) == 16) {
    uint8_t c[8];
    const uint8_t s = mla::fp4_quantize_group16(x, c);
    fwrite(c, 1, 8, stdout);
    fwrite(&s, 1, 1, stdout);
  }
  return 0;
}
'''


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    nv = _nvcc()
    if nv is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("aq")
    src, exe = d / "drv.cu", d / "drv"
    src.write_text(DRIVER)
    r = subprocess.run([nv, "-O2", "-std=c++17", "-Wno-deprecated-gpu-targets", "-I", CSRC, str(src),
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return str(exe)


def _run(exe, x):
    x = np.ascontiguousarray(x, np.float32)
    out = subprocess.run([exe], input=x.tobytes(), capture_output=True, check=True).stdout
    r = np.frombuffer(out, np.uint8).reshape(x.shape[0], 32, 9)
    return np.concatenate([r[:, :, :8].reshape(x.shape[0], 256), r[:, :, 8]], axis=1)


def test_matches_oracle_f32_decisions(driver):
    rng = np.random.Generator(np.random.PCG64(47))
    x = rng.standard_normal((1500, 512)).astype(np.float32)
    x[500:1000] *= np.float32(1e-3)
    x[1000:] *= np.float32(300.0)
    x[0] = 0.0
    x[1, :16] = 1e-9
    x[2, :16] = 5000.0          # amax / 6 above 448: the scale saturates
    x[3, :16] = -1e-30
    np.testing.assert_array_equal(_run(driver, x), v41.fp4_quantize(x.astype(np.float64), decide_in_f32=True))


def test_ties_and_saturation(driver):
    x = np.zeros((2, 512), np.float32)
    # scale 1 (amax 6); the other 15 sit on E2M1 midpoints, both signs, and one
    # small negative that rounds to -0
    x[0, :16] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.1]
    # amax / 6 exactly between two E4M3 values (0.125 and 0.140625)
    x[1, :16] = 6 * 0.125 * (1 + 1 / 16)
    got = _run(driver, x)
    want = v41.fp4_quantize(x.astype(np.float64), decide_in_f32=True)
    np.testing.assert_array_equal(got, want)
    codes = np.stack([got[0, :8] & 0xF, got[0, :8] >> 4], axis=1).reshape(-1)
    # by hand: ties go to the even code (0/0.5 -> 0, 0.5/1 -> 1 (2), 1/1.5 -> 1 (2), 1.5/2 -> 2 (4),
    # 2/3 -> 2 (4), 3/4 -> 4 (6), 4/6 -> 4 (6)); negatives add the sign bit 8
    assert list(codes) == [7, 0, 2, 2, 4, 4, 6, 6, 8, 10, 10, 12, 12, 14, 14, 8]
