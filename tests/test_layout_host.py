"""The device layouts' index maps, compiled for the host from csrc/layout.h
(CPU only): the Q2_K quant lane order is a bijection onto the 64 bytes of a
super-block, and lane q of an MMA quad finds, in its own four words, the four
quants of every sub-block at the bytes the integer MMA's A fragment wants; the
MXFP4 scale-atom index is a bijection onto each 512-byte atom."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "routed_expert_ffn_05_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")

PROG = r"""
#include <cstdio>
#include "layout.h"
int main() {
    for (int e = 0; e < 256; ++e) std::printf("%d %d\n", moe::q2k_word(e), moe::q2k_bit(e));
    // one 128-row x 256-K tile of an expert with N = 256, K = 512: atom index of (n, kb)
    for (int n = 0; n < 256; ++n)
        for (int kb = 0; kb < 16; ++kb)
            std::printf("%lld\n", (long long)moe::mxfp4_tile_index(1, n, kb, 256, 512));
    return 0;
}
"""


@pytest.fixture(scope="module")
def maps():
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "m.cpp"), os.path.join(d, "m")
        with open(src, "w") as f:
            f.write(PROG)
        r = subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, "-I", INCLUDE, src, "-o", exe],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    q2 = np.array([[int(v) for v in l.split()] for l in out[:256]])
    mx = np.array([int(l) for l in out[256:256 + 256 * 16]]).reshape(256, 16)
    return q2, mx


def test_q2k_lane_order_is_a_bijection(maps):
    q2, _ = maps
    word, bit = q2[:, 0], q2[:, 1]
    assert word.min() == 0 and word.max() == 15 and bit.min() == 0 and bit.max() == 30
    assert np.all(bit % 2 == 0)
    assert len({(w, b) for w, b in zip(word, bit)}) == 256   # every 2-bit slot used once


def test_q2k_lane_reads_its_a_fragment(maps):
    """Quant e = 16 c + 4 q + i (sub-block c, quad lane q, byte i) is in word
    4 q + c / 4, and (word >> 2 (c % 4)) & 0x03030303 puts it in byte i."""
    q2, _ = maps
    rng = np.random.default_rng(5)
    quants = rng.integers(0, 4, 256)
    words = np.zeros(16, dtype=np.uint64)
    for e in range(256):
        words[q2[e, 0]] |= np.uint64(int(quants[e]) << int(q2[e, 1]))
    for c in range(16):
        for q in range(4):
            w = int(words[4 * q + c // 4])
            reg = (w >> (2 * (c % 4))) & 0x03030303
            got = [(reg >> (8 * i)) & 3 for i in range(4)]
            assert got == [int(quants[16 * c + 4 * q + i]) for i in range(4)], (c, q)


def test_mxfp4_scale_atoms_are_bijective(maps):
    """Expert 1 of a 256 x 512 matrix: its 2 x 4 atoms of 512 bytes are filled
    exactly once each, atom (n / 128, kb / 4), byte (n % 32) 16 + (n % 128) / 32 4 + kb % 4."""
    _, mx = maps
    base = (1 * 2 * 4) * 512
    off = mx - base
    assert off.min() == 0 and off.max() == 2 * 4 * 512 - 1
    assert len(np.unique(off)) == off.size
    n, kb = np.meshgrid(np.arange(256), np.arange(16), indexing="ij")
    atom = (n // 128) * 4 + kb // 4
    assert np.array_equal(off // 512, atom)
    assert np.array_equal(off % 512, (n % 32) * 16 + ((n % 128) // 32) * 4 + kb % 4)
