"""Host checks of the packed chunk layout of the derivative-saving epilogues
(SP24_EPI_GELU_DERIV_PACKED / SP24_EPI_MUL_AUX_PACKED), no device needed.

The layout is the epilogue's register fragment: for each block of 16 tokens x 32
features, half h and lane l hold four 32-bit registers i, register i packing
tokens 8(i/2) + 2(l%4) + {0, 1} of feature 16h + 8(i%2) + l/4.  The library's
host map goes the other way, from (token, feature) to the offset; the tests
build the packed buffer by walking lanes and registers as the kernel does and
compare."""
import numpy as np
import pytest

import structured_sparse_transformer_b200 as sp


def _pack_by_fragment(a):
    """Packed buffer of row-major uint16 a [T, M] by enumerating blocks, halves,
    lanes, registers and the two 16-bit halves of each register."""
    T, M = a.shape
    nbt, nbf = -(-T // 16), -(-M // 32)
    out = np.zeros(nbt * nbf * 512, dtype=np.uint16)
    for bt in range(nbt):
        for bf in range(nbf):
            base = (bt * nbf + bf) * 512
            for h in range(2):
                for lane in range(32):
                    for i in range(4):
                        for e in range(2):
                            t = 16 * bt + 8 * (i // 2) + 2 * (lane % 4) + e
                            m = 32 * bf + 16 * h + 8 * (i % 2) + lane // 4
                            if t < T and m < M:
                                out[base + 256 * h + 8 * lane + 2 * i + e] = a[t, m]
    return out


@pytest.mark.parametrize("T,M", [(16, 32), (37, 48), (1, 16), (64, 208), (100, 96)])
def test_pack_matches_the_fragment_walk_and_round_trips(T, M):
    rng = np.random.default_rng(T * 1000 + M)
    a = rng.integers(1, 65535, size=(T, M), dtype=np.uint16)
    packed = sp.sp24_aux_pack(a, T, M)
    assert packed.size * 2 == sp.sp24_aux_packed_size(T, M) == -(-T // 16) * -(-M // 32) * 1024
    assert np.array_equal(packed, _pack_by_fragment(a))
    assert np.array_equal(sp.sp24_aux_unpack(packed, T, M), a)


def test_every_entry_lands_once():
    T, M = 48, 96
    a = np.arange(T * M, dtype=np.uint16).reshape(T, M) + 1
    packed = sp.sp24_aux_pack(a, T, M)
    vals = packed[packed != 0]
    assert vals.size == T * M and np.array_equal(np.sort(vals), np.sort(a.reshape(-1)))


def test_packed_size_and_bad_arguments():
    assert sp.sp24_aux_packed_size(0, 0) == 0
    assert sp.sp24_aux_packed_size(17, 33) == 2 * 2 * 1024
    assert sp.aux_elements(17, 33, "mul_aux_packed") == 2048
    assert sp.aux_elements(17, 33, "mul_aux") == 17 * 33
    with pytest.raises(ValueError, match="packed aux has"):
        sp.sp24_aux_unpack(np.zeros(10, dtype=np.uint16), 16, 32)
