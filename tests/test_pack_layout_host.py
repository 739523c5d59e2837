"""The packed weight layout's index maps (csrc/svdq_quant.cuh: gemm_row_of / orig_row_of,
tile_col_of_packed / packed_of_tile_col, wgt_sf_offset), compiled by nvcc into a host program and
checked on the CPU for every tile width the packs use, with and without the SwiGLU interleave:
- the packed-row map is a permutation of the weight rows, and orig_row_of inverts it;
- within a tile, the first half of the tile columns are gate rows and the second half the matching
  up rows (SwiGLU);
- at the 384-wide tile, CTA c of the pair stages exactly tile columns [128c, 128c + 128) and
  [256 + 64c, 256 + 64c + 64), each in one contiguous box of 192 packed rows;
- the scale offsets of all rows and K blocks are distinct, inside the scale region, and put a tile
  column into atom column / 128 of its (tile, K atom).
These are the layouts the GEMM kernel's TMA boxes and MMA scale reads assume; the GPU parity tests
check the same through the kernels' outputs."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_diffusion_transformer_svdquant_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "svdq_quant.cuh"
using namespace svdq;

static int fail(const char* what, int a, int b, int c) {
  std::printf("FAIL %s %d %d %d\n", what, a, b, c);
  return 1;
}

static int check(int N, int K, int n_tile, int swiglu) {
  std::vector<int> seen(N, 0);
  for (int n = 0; n < N; ++n) {
    const int p = gemm_row_of(n, N, n_tile, swiglu);
    if (p < 0 || p >= N) return fail("row out of range", N, n_tile, n);
    if (seen[p]++) return fail("row collision", N, n_tile, n);
    if (orig_row_of(p, N, n_tile, swiglu) != n) return fail("orig_row_of", N, n_tile, n);
  }
  for (int nb = 0; nb < N / n_tile; ++nb)
    for (int t = 0; t < n_tile; ++t) {
      const int p = nb * n_tile + packed_of_tile_col(t, n_tile);
      if (tile_col_of_packed(p - nb * n_tile, n_tile) != t) return fail("tile column round trip", N, n_tile, t);
      if (swiglu) {
        const int half = n_tile / 2, o = orig_row_of(p, N, n_tile, 1);
        const int want = t < half ? nb * half + t : N / 2 + nb * half + (t - half);
        if (o != want) return fail("gate/up interleave", N, n_tile, t);
      }
    }
  if (n_tile == 384)
    for (int c = 0; c < 2; ++c) {
      std::vector<int> cols(384, 0);
      for (int q = 192 * c; q < 192 * c + 192; ++q) cols[tile_col_of_packed(q, 384)] = 1;
      for (int t = 0; t < 384; ++t) {
        const bool mine = (t >= 128 * c && t < 128 * c + 128) || (t >= 256 + 64 * c && t < 256 + 64 * c + 64);
        if (cols[t] != (mine ? 1 : 0)) return fail("CTA box columns", c, t, cols[t]);
      }
    }
  const int atoms = (n_tile + 127) / 128;
  const size_t sf_bytes = static_cast<size_t>(N / n_tile) * (K / 64) * atoms * 512;
  std::vector<unsigned char> hit(sf_bytes, 0);
  for (int p = 0; p < N; ++p)
    for (int kb = 0; kb < K / 16; ++kb) {
      const size_t off = wgt_sf_offset(p, kb, K, n_tile);
      if (off >= sf_bytes) return fail("scale offset out of range", N, n_tile, p);
      if (hit[off]++) return fail("scale offset collision", N, n_tile, p);
      const int nb = p / n_tile, t = tile_col_of_packed(p - nb * n_tile, n_tile);
      const size_t atom = off >> 9;
      const size_t want = (static_cast<size_t>(nb) * (K / 64) + kb / 4) * atoms + t / 128;
      if (atom != want) return fail("scale atom", N, n_tile, p);
    }
  return 0;
}

int main() {
  int bad = 0;
  bad |= check(1536, 512, 384, 0);
  bad |= check(768, 256, 384, 0);
  bad |= check(1536, 512, 384, 1);   // the maps themselves; the packs use 384 only without SwiGLU
  bad |= check(1024, 256, 256, 0);
  bad |= check(1024, 256, 256, 1);
  bad |= check(768, 256, 192, 0);
  bad |= check(384, 512, 192, 1);
  bad |= check(640, 256, 128, 0);
  bad |= check(640, 256, 128, 1);
  if (!bad) std::printf("ok\n");
  return bad;
}
"""


def test_pack_layout_maps(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    src = tmp_path / "layout.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "layout"
    r = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                        str(src), "-o", str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout[-2000:] + out.stderr[-2000:]
