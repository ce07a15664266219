"""CPU checks of the C ABI: the library builds, loads without a GPU, exports
every entry point that include/lemo.h declares, and rejects bad arguments
on the host before touching CUDA.  Also checks the tile enumeration of the
scoring kernel (compiled with g++ from the same header the kernel uses)."""

import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

from contextual_token_sparsity_b200 import build as lemo_build
from contextual_token_sparsity_b200 import lemo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lemo.h")


@pytest.fixture(scope="module")
def lib():
    if shutil.which("nvcc") or os.path.exists("/usr/local/cuda/bin/nvcc"):
        lemo_build.build()
    if not os.path.exists(lemo.LIB_PATH):
        pytest.skip("liblemo.so not built and nvcc unavailable")
    return lemo.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LEMO_API\s+[\w\s\*]+?\b(lemo_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ["lemo_score_blocks", "lemo_select", "lemo_gather_pad", "lemo_scatter_residual",
              "lemo_workspace_size", "lemo_get_error"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    nm = shutil.which("nm")
    if nm:
        out = subprocess.run([nm, "-D", "--defined-only", lemo.LIB_PATH], capture_output=True,
                             text=True).stdout
        exported = set(re.findall(r"\bT\s+(lemo_\w+)", out))
        assert set(names) <= exported
        # nothing else of ours leaks out of the library
        assert exported == set(names)


def test_binding_covers_header(lib):
    assert set(declared_functions()) == set(lemo._SIGS)


def test_status_strings(lib):
    for code, name in lemo.STATUS.items():
        assert lib.lemo_status_string(code).decode() == name


def _shape(batch=1, total_L=1024, max_seqlen=1024, H=8, dh=64, block=64, cu=0x1000):
    return lemo.lemo_shape(batch, cu, total_L, max_seqlen, H, dh, block)


def test_workspace_size_matches_layout(lib):
    def align(v):
        return (v + 255) // 256 * 256
    for batch, total_L, maxL, b in [(1, 1024, 1024, 64), (4, 10240, 4096, 64),
                                    (1, 32768, 32768, 128), (3, 0, 0, 64)]:
        s = _shape(batch, total_L, maxL, block=b)
        got = lib.lemo_workspace_size(ctypes.byref(s))
        off = align(32)                      # header
        off = align(off + 8 * (batch + 1))   # tile prefix
        off = align(off + 4 * (batch + 1))   # block prefix
        off = align(off + 8 * (batch + 1))   # block-max prefix
        nlb = -(-total_L // 2048) if total_L else 1
        off = align(off + 8 * nlb)           # look-back descriptors
        m_cap = (-(-maxL // b)) * ((total_L + batch * (b - 1)) // b)
        off = align(off + 4 * m_cap)
        assert got == off, (batch, total_L, got, off)


def test_workspace_size_rejects_bad_shapes(lib):
    for kw in [dict(batch=0), dict(total_L=-1), dict(block=32), dict(block=0),
               dict(max_seqlen=(1 << 22) + 1), dict(max_seqlen=0)]:
        s = _shape(**kw)
        assert lib.lemo_workspace_size(ctypes.byref(s)) == 0, kw
    s = _shape()
    s.cu_seqlens = None
    assert lib.lemo_workspace_size(ctypes.byref(s)) == 0


def test_block_max_elems(lib):
    assert lemo.lemo_block_max_elems([4096, 3072, 2048, 1024], 64) == 64**2 + 48**2 + 32**2 + 16**2
    assert lemo.lemo_block_max_elems([65, 0, 1], 64) == 4 + 0 + 1
    assert lemo.lemo_block_max_elems([32768], 128) == 256**2


def test_host_validation_returns_before_cuda(lib):
    """Argument errors come back from the host checks (no CUDA call needed)."""
    s = _shape(H=8, dh=96)
    buf = 0x10000  # never dereferenced: the checks fail first
    assert lib.lemo_score_blocks(ctypes.byref(s), buf, buf, 1.0, None, buf, buf, 1 << 20,
                                 None) == lemo.LEMO_ERR_UNSUPPORTED
    s = _shape()
    assert lib.lemo_score_blocks(ctypes.byref(s), buf + 8, buf, 1.0, None, buf, buf, 1 << 20,
                                 None) == lemo.LEMO_ERR_INVALID_ARG       # misaligned q
    assert lib.lemo_score_blocks(ctypes.byref(s), buf, buf, -1.0, None, buf, buf, 1 << 20,
                                 None) == lemo.LEMO_ERR_INVALID_ARG       # scale <= 0
    assert lib.lemo_score_blocks(ctypes.byref(s), buf, buf, 1.0, None, buf, buf, 16,
                                 None) == lemo.LEMO_ERR_INVALID_ARG       # workspace too small
    assert lib.lemo_select(ctypes.byref(s), buf, 0.0, buf, buf, buf, None, buf, 1 << 20,
                           None) == lemo.LEMO_ERR_INVALID_ARG             # no kept_total
    # gather / scatter: d % 8, strides, alignment, null pointers
    assert lib.lemo_gather_pad(buf, 12, 10, 12, buf, buf, 128, buf, 12, 128,
                               None) == lemo.LEMO_ERR_UNSUPPORTED
    assert lib.lemo_gather_pad(buf, 8, 10, 16, buf, buf, 128, buf, 16, 128,
                               None) == lemo.LEMO_ERR_INVALID_ARG         # ld_x < d
    assert lib.lemo_gather_pad(buf + 2, 16, 10, 16, buf, buf, 128, buf, 16, 128,
                               None) == lemo.LEMO_ERR_INVALID_ARG         # misaligned x
    assert lib.lemo_gather_pad(buf, 16, 10, 16, buf, buf, 0, buf, 16, 128,
                               None) == lemo.LEMO_ERR_INVALID_ARG         # pad_to < 1
    assert lib.lemo_scatter_residual(None, 16, 10, 16, buf, 16, buf, buf,
                                     None) == lemo.LEMO_ERR_INVALID_ARG


def test_segment_loss_workspace_and_validation(lib):
    def align(v):
        return (v + 255) // 256 * 256
    for T, V, S in [(16384, 32000, 1024), (300, 1000, 64), (5, 13, 64), (0, 7, 3)]:
        ld = -(-V // 8) * 8
        rows = min(S, max(T, 1)) if T < S else S
        want = align(4)
        want = align(want + 4 * max(T, 1))
        want = align(want + 4 * rows * ld)
        nseg = -(-T // S) if T > 0 else 1
        want = align(want + 2 * min(nseg, 4) * rows * ld)          # up to four dz segments
        want = align(want + 8 * rows * 2 * (-(-V // 256)))          # per-row softmax partials
        assert lemo.lemo_segment_loss_workspace_size(T, V, S) == want, (T, V, S)
    # the peak part scales with the segment rows, not with T
    a = lemo.lemo_segment_loss_workspace_size(16384, 32000, 1024)
    b = lemo.lemo_segment_loss_workspace_size(16384, 32000, 16384)
    assert (b - a) == align(4 * 16384 * 32000) + align(2 * 16384 * 32000) - \
        align(4 * 1024 * 32000) - align(2 * 4 * 1024 * 32000) + \
        align(8 * 16384 * 250) - align(8 * 1024 * 250)
    assert lemo.lemo_segment_loss_workspace_size(-1, 10, 4) == 0
    assert lemo.lemo_segment_loss_workspace_size(10, 0, 4) == 0
    assert lemo.lemo_segment_loss_workspace_size(10, 10, 0) == 0
    buf, big = 0x10000, 1 << 40
    f = lib.lemo_segment_loss
    ok = [buf, 64, 10, 64, buf, 64, 100, buf, -100, 4, buf, None, buf, 64, buf, 64, buf, big, None]
    def call(**kw):
        args = list(ok)
        names = ["h", "ld_h", "T", "d", "w", "ld_w", "V", "y", "ign", "seg", "loss", "tl", "dh",
                 "ld_dh", "dw", "ld_dw", "ws", "ws_bytes", "st"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)
    assert call(d=12, ld_h=16, ld_w=16, ld_dh=16, ld_dw=16) == lemo.LEMO_ERR_UNSUPPORTED
    assert call(ld_h=60) == lemo.LEMO_ERR_INVALID_ARG        # stride < d
    assert call(ld_w=68) == lemo.LEMO_ERR_INVALID_ARG        # stride not a multiple of 8
    assert call(h=buf + 8) == lemo.LEMO_ERR_INVALID_ARG      # misaligned h
    assert call(seg=0) == lemo.LEMO_ERR_INVALID_ARG
    assert call(loss=None) == lemo.LEMO_ERR_INVALID_ARG
    assert call(ws_bytes=1024) == lemo.LEMO_ERR_INVALID_ARG  # workspace too small
    assert call(ws=buf + 16) == lemo.LEMO_ERR_INVALID_ARG    # workspace not 256-aligned
    assert call(dw=buf, ld_dw=32) == lemo.LEMO_ERR_INVALID_ARG


TILE_CHECK = r"""
#include <cstdio>
#include <vector>
#include "tile_plan.h"
using namespace lemo_plan;
int main() {
  const int Ls[] = {1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 300, 511, 512, 513, 1000,
                    1024, 2047, 2049, 3072, 4096, 8192, 16384, 32768};
  for (int L : Ls) {
    const int nq = (int)query_tiles(L);
    const long long T = seq_tiles(L);
    long long brute = 0;
    for (int q = 0; q < nq; ++q)
      for (int k = 0; k * TN <= q * TM + TM - 1; ++k) ++brute;
    if (brute != T) { printf("count L=%d %lld %lld\n", L, T, brute); return 1; }
    std::vector<int> seen((size_t)nq * nq, 0);
    int prev_group = -1;
    for (long long t = 0; t < T; ++t) {
      int qi, kj; decode_tile(L, t, &qi, &kj);
      if (qi < 0 || qi >= nq || kj < 0 || kj > qi) { printf("range L=%d t=%lld\n", L, t); return 1; }
      int g = qi / GROUP;
      if (g < prev_group) { printf("group order L=%d\n", L); return 1; }
      prev_group = g;
      if (seen[(size_t)qi * nq + kj]++) { printf("dup L=%d\n", L); return 1; }
    }
    for (int b : {64, 128}) {             // every score block n >= m in exactly one tile
      const int nb = (L + b - 1) / b;
      std::vector<int> cov((size_t)nb * nb, 0);
      for (long long t = 0; t < T; ++t) {
        int qi, kj; decode_tile(L, t, &qi, &kj);
        for (int n = qi * TM / b; n < (qi + 1) * TM / b; ++n)
          for (int m = kj * TN / b; m < (kj + 1) * TN / b; ++m)
            if (n < nb && m <= n) cov[(size_t)n * nb + m]++;
      }
      for (int n = 0; n < nb; ++n)
        for (int m = 0; m <= n; ++m)
          if (cov[(size_t)n * nb + m] != 1) { printf("cover L=%d b=%d n=%d m=%d c=%d\n", L, b, n, m, cov[(size_t)n*nb+m]); return 1; }
    }
  }
  printf("ok\n");
  return 0;
}
"""


def test_tile_enumeration_covers_every_block(tmp_path):
    gxx = shutil.which("g++")
    if not gxx:
        pytest.skip("g++ unavailable")
    src = tmp_path / "tile_check.cc"
    src.write_text(TILE_CHECK)
    exe = tmp_path / "tile_check"
    inc = os.path.join(ROOT, "contextual_token_sparsity_b200", "csrc")
    subprocess.run([gxx, "-O2", "-std=c++17", "-I" + inc, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout


SHARD_CHECK = r"""
#include <cstdio>
#include <vector>
#include "tile_plan.h"
using namespace lemo_plan;
int main() {
  const int Ls[] = {1, 200, 256, 257, 1000, 4096, 5000, 8192, 16384, 32768};
  const int Gs[] = {1, 2, 3, 4, 5, 8};
  for (int L : Ls) {
    const int nq = (int)query_tiles(L);
    for (int G : Gs) {
      std::vector<int> seen((size_t)nq * nq, 0);
      long long total = 0, most = 0;
      for (int r = 0; r < G; ++r) {
        const long long T = shard_seq_tiles(L, r, G);
        total += T;
        if (T > most) most = T;
        int prev_group = -1;
        for (long long t = 0; t < T; ++t) {
          int qi, kj; decode_tile_shard(L, t, r, G, &qi, &kj);
          if (qi < 0 || qi >= nq || kj < 0 || kj > qi) { printf("range L=%d G=%d\n", L, G); return 1; }
          if (!owns_key_tile(kj, r, G)) { printf("owner L=%d G=%d\n", L, G); return 1; }
          if (qi / GROUP < prev_group) { printf("group order L=%d G=%d\n", L, G); return 1; }
          prev_group = qi / GROUP;
          if (seen[(size_t)qi * nq + kj]++) { printf("dup L=%d G=%d\n", L, G); return 1; }
          if (G == 1) {
            int q1, k1; decode_tile(L, t, &q1, &k1);
            if (q1 != qi || k1 != kj) { printf("order L=%d\n", L); return 1; }
          }
        }
      }
      if (total != seq_tiles(L)) { printf("total L=%d G=%d\n", L, G); return 1; }
      // snake order keeps the shards within one column of each other
      if (G > 1 && most * G > total + (long long)G * nq) { printf("balance L=%d G=%d\n", L, G); return 1; }
    }
  }
  // ownership table for the Python mirror: G = 1..5, kj = 0..39
  for (int G = 1; G <= 5; ++G)
    for (int kj = 0; kj < 40; ++kj)
      for (int r = 0; r < G; ++r)
        if (owns_key_tile(kj, r, G)) printf("%d ", r);
  printf("\nok\n");
  return 0;
}
"""


def test_shard_enumeration_partitions_the_tiles(tmp_path):
    """Key-tile shards: every tile of the unsharded enumeration is computed by
    exactly one shard, only on key tiles the shard owns, in group order; one
    shard reproduces the unsharded order; and the Python mirror of the
    ownership rule (used by the host logic of the split) agrees."""
    from contextual_token_sparsity_b200 import split
    gxx = shutil.which("g++")
    if not gxx:
        pytest.skip("g++ unavailable")
    src = tmp_path / "shard_check.cc"
    src.write_text(SHARD_CHECK)
    exe = tmp_path / "shard_check"
    inc = os.path.join(ROOT, "contextual_token_sparsity_b200", "csrc")
    subprocess.run([gxx, "-O2", "-std=c++17", "-I" + inc, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    lines = r.stdout.strip().split("\n")
    assert r.returncode == 0 and lines[-1] == "ok", r.stdout
    owners = [int(v) for v in lines[0].split()]
    want = [split.key_tile_owner(kj, G) for G in range(1, 6) for kj in range(40)]
    assert owners == want
