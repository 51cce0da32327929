"""The decode's launch-shape rule (table layout and CTA width), checked on the host.

The rule lives in csrc/decode_launch.h as host code; a small probe compiled with the host compiler
evaluates it for given (frequency-total bits, largest tile, tile count, CTA count, wide_ok) and
prints the per-warp tile buffer of every (layout, width) pair. Checked here:
  * the buffer sizes equal the shared-memory budget arithmetic (227 KB per CTA, 4 KB alignment
    slack, the table block, 64 B of barriers, 80 + 8 B per warp, 16 B), rounded down to 16 B;
  * the shapes the design lists for the measured workloads (148 SMs);
  * every choice's buffers hold the largest tile, and its cost is the least among usable shapes
    under the documented model: ceil(n / (warps * ctas)) rounds x chain weight x (48 + warps);
  * 16-warp-only launches (the allocation-free entry point) and tiles no buffer holds.
"""
import itertools
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dit_weight_compression_b200", "csrc")

PROBE = r"""
#include "decode_launch.h"
#include <cstdio>
#include <cstdlib>
int main(int argc, char** argv) {
    using namespace ep::dec;
    for (int i = 1; i + 4 < argc; i += 5) {
        const LaunchShape s = launch_shape(atoi(argv[i]), strtoull(argv[i + 1], 0, 10), strtoull(argv[i + 2], 0, 10),
                                           strtoull(argv[i + 3], 0, 10), atoi(argv[i + 4]) != 0);
        printf("shape %d %d\n", s.lay, s.warps);
    }
    for (int lay : {10, 11, 12, 13, 14, 15})
        for (int w : {16, 20, 24, 32}) printf("buf %d %d %u %d\n", lay, w, tile_buffer_bytes(w, lay), int(width_ok(w, lay)));
    return 0;
}
"""

# Table block per layout: 15 tables of 4 KB (10-bit packed words, or 12-bit symbol bytes); 12-bit
# per-symbol entries 16 x 256 x 4 B + 64 B skew; hybrids: (1 + 2D) direct tables of 16 KB,
# 2(7 - D) symbol-byte tables of 4 KB and 2(7 - D) entry rows of 1 KB, + 64 B skew.
TABLE_BYTES = {
    10: 15 * 4096,
    11: 1 * 16384 + 14 * 4096 + 14 * 1024 + 64,
    12: 15 * 4096 + 16 * 256 * 4 + 64,
    15: 3 * 16384 + 12 * 4096 + 12 * 1024 + 64,
    13: 5 * 16384 + 10 * 4096 + 10 * 1024 + 64,
    14: 7 * 16384 + 8 * 4096 + 8 * 1024 + 64,
}
WIDTHS = {10: (16, 20, 24, 32), 11: (16, 20, 24, 32), 12: (16, 20, 24, 32), 13: (16, 20), 14: (16,),
          15: (16, 20, 24, 32)}
WEIGHT = {10: 8, 14: 12, 13: 13, 15: 14, 11: 15, 12: 16}


def expected_buffer(lay, w):
    return ((232448 - 4096 - TABLE_BYTES[lay] - 64 - w * 88 - 16) // w) & ~15


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("shape")
    src, exe = d / "probe.cpp", d / "probe"
    src.write_text(PROBE)
    cuda_inc = "/usr/local/cuda/include"
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-I", cuda_inc,
                    str(src), "-o", str(exe)], check=True)

    def run(cases):
        args = [str(v) for c in cases for v in (c[0], c[1], c[2], c[3], int(c[4]))]
        out = subprocess.run([str(exe), *args], check=True, capture_output=True, text=True).stdout.split("\n")
        shapes = [tuple(map(int, l.split()[1:])) for l in out if l.startswith("shape")]
        bufs = {(int(p[1]), int(p[2])): (int(p[3]), bool(int(p[4]))) for p in (l.split() for l in out) if p and p[0] == "buf"}
        return shapes, bufs
    return run


def test_buffer_sizes_follow_the_shared_memory_budget(probe):
    _, bufs = probe([])
    for lay in (10, 11, 12, 13, 14, 15):
        for w in (16, 20, 24, 32):
            size, ok = bufs[(lay, w)]
            assert ok == (w in WIDTHS[lay]), (lay, w)
            if ok:
                assert size == expected_buffer(lay, w), (lay, w)


# (name, bits, largest tile, tiles) with 148 CTAs -> the shape the design lists and the GPU runs
DOCUMENTED = [
    ("4096x4096 @4", 12, 4064, 2048, (14, 16)),
    ("4096x4096 @4, 10-bit", 10, 4064, 2048, (10, 16)),
    ("4096x11008 @0.5", 12, 4128, 688, (14, 16)),
    ("4096x11008 @2", 12, 4096, 2752, (13, 20)),
    ("4096x11008 @3.5", 12, 7152, 2752, (12, 20)),
    ("4096x11008 @6", 12, 6144, 5504, (11, 20)),
    ("4096x11008 @11", 12, 5696, 11008, (15, 20)),
    ("DiT set, grouped", 12, 5136, 5376, (15, 20)),
    ("DiT 3072x3072 alone", 12, 5136, 576, (13, 16)),
    ("large-layer stream, grouped", 12, 4080, 4 * 28672, (11, 32)),
    ("large-layer stream, 10-bit", 10, 4080, 4 * 28672, (10, 32)),
]


@pytest.mark.parametrize("name,pb,tile,n,shape", DOCUMENTED, ids=[d[0] for d in DOCUMENTED])
def test_documented_workload_shapes(probe, name, pb, tile, n, shape):
    (got,), _ = probe([(pb, tile, n, 148, True)])
    assert got == shape


def _cost(lay, w, n, ctas):
    slots = w * max(ctas, 1)
    return -(-n // slots) * WEIGHT[lay] * (48 + w)


def test_choice_is_usable_and_cheapest(probe):
    cases = [(pb, tile, n, ctas, True)
             for pb in (10, 12)
             for tile in (160, 2000, 3584, 4064, 4288, 4432, 4433, 4656, 4700, 4800, 5120, 5744, 5792, 5840, 6176, 6848,
                          6912, 7248, 7424, 8240, 8656, 9296)
             for n in (1, 4, 148, 2368, 2369, 2960, 3552, 4144, 4736, 10000, 114688)
             for ctas in (148, 132)]
    shapes, bufs = probe(cases)
    for (pb, tile, n, ctas, _), (lay, w) in zip(cases, shapes):
        lays = (10,) if pb == 10 else (14, 13, 15, 11, 12)
        usable = [(l, x) for l in lays for x in WIDTHS[l] if bufs[(l, x)][0] >= tile]
        assert (lay == 10) == (pb == 10)
        if not usable:
            continue
        assert (lay, w) in usable, (pb, tile, n, ctas, lay, w)
        assert _cost(lay, w, n, ctas) == min(_cost(l, x, n, ctas) for l, x in usable), (pb, tile, n, ctas, lay, w)


def test_sixteen_warp_launches_and_oversized_tiles(probe):
    cases = list(itertools.product((10, 12), (4064, 5000, 6000, 7000, 8000, 9000, 12000), (100, 100000), (148,), (False,)))
    cases += [(12, 12000, 100000, 148, True), (10, 12000, 100000, 148, True), (12, 9296, 100000, 148, True)]
    shapes, bufs = probe(cases)
    for (pb, tile, n, ctas, wide), (lay, w) in zip(cases, shapes):
        if not wide:
            assert w == 16 and lay != 14
            if pb == 12 and tile <= bufs[(12, 16)][0]:
                assert lay == (13 if tile <= bufs[(13, 16)][0] else 15 if tile <= bufs[(15, 16)][0]
                               else 11 if tile <= bufs[(11, 16)][0] else 12)
        if tile > 10336:  # no buffer holds it: 16 warps, tiles read from global memory
            assert w == 16 and lay == (10 if pb == 10 else 12)
    assert shapes[-1] == (12, 16)   # fits 16-warp layout-12 buffers only
