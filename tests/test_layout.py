"""Host-side check of the shared-memory image layouts (csrc/layout.cuh):
sl_index is a bijection on [0, D*D'), sl_coords inverts it, the split form
(feature base + column offset) agrees with it, and the weight image index is
a bijection too, for every supported (D, D'); so is the K-pieced image of the
general feature map's weights."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_attention_video_chunked_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "layout.cuh"
using namespace rehyat;
int main() {
  int bad = 0;
  const int Ds[] = {32, 64, 128}, Dps[] = {32, 64, 128, 256};
  for (int D : Ds) for (int Dp : Dps) {
    std::vector<int> seen(D * Dp, 0), seen_w(D * Dp, 0);
    for (int f = 0; f < Dp; ++f) for (int d = 0; d < D; ++d) {
      const long long o = sl_index(f, d, D, Dp);
      if (o < 0 || o >= (long long)D * Dp) { ++bad; continue; }
      seen[o]++;
      int f2, d2;
      sl_coords(o, D, Dp, &f2, &d2);
      if (f2 != f || d2 != d) ++bad;
      if (sl_feature_base(f, D, Dp) + sl_column_offset(f, d) != o) ++bad;
      if (D >= 64) {
        const long long w = wimg_index(f, d, D, Dp);
        if (w < 0 || w >= (long long)D * Dp) ++bad; else seen_w[w]++;
      }
    }
    for (int i = 0; i < D * Dp; ++i) {
      if (seen[i] != 1) ++bad;
      if (D >= 64 && seen_w[i] != 1) ++bad;
    }
  }
  // K-pieced weight images of the general feature map: W_a^T [Dh][128] and
  // W_b^T [Dp][Dh] are bijections onto [0, N*K).
  const int Ns[] = {64, 128, 256, 384, 512}, Ks[] = {128, 256, 384, 512};
  for (int N : Ns) for (int K : Ks) {
    std::vector<int> seen_k((size_t)N * K, 0);
    for (int n = 0; n < N; ++n) for (int k = 0; k < K; ++k) {
      const long long o = kpiece_img_index(n, k, N);
      if (o < 0 || o >= (long long)N * K) { ++bad; continue; }
      seen_k[o]++;
      // 16-byte chunks stay within their 128-byte row; row r of a box at r * 64.
      const int rp = N < 128 ? N : 128;
      if ((o % 64) / 8 != (((k & 127) >> 3) & 7 ^ ((n % rp) & 7))) ++bad;
    }
    for (long long i = 0; i < (long long)N * K; ++i) if (seen_k[i] != 1) ++bad;
  }
  std::printf("%d\n", bad);
  return bad != 0;
}
"""


def test_image_layouts_are_bijections(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "t.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "t"
    subprocess.run([nvcc, "-std=c++17", "-I" + CSRC, str(src), "-o", str(exe)], check=True,
                   capture_output=True, timeout=300)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "0", res.stdout
