"""Host-side check of the arithmetic the GA kernels use to stage rows whose byte length is not a
multiple of 16 (gather_copy / gather_align in scan_fwd_seq.cuh), restated here from that
description and compared with plain byte slicing:

  * a row's window for stage k is the 144 bytes from the 16-byte-aligned address below its step
    0, plus 128 k; chunk c (16 bytes) of it is copied only if it holds a byte of steps 0 .. L-1
    (start of chunk, from step 0: 128 k - sh + 16 c < L * size), else zero-filled, so no read
    leaves the tensor (rounded out to 16 bytes);
  * chunk 8 of stage k's window is chunk 0 of stage k + 1's window (copied as part of stage k + 1,
    or of one extra stage past the last);
  * lane c rebuilds output chunk c from three 8-byte words read at window byte 16 c + (sh & 8),
    keeping the words from (sh & 4) on and funnel-shifting right by 8 (sh & 3) bits;
  * output bytes past the row's steps are zeroed on the row's last window.
"""
import numpy as np
import pytest


def funnel_r(lo, hi, s):
    return ((hi << 32 | lo) >> s) & 0xFFFFFFFF


def shifted_chunk(window, sh, c):
    """Output chunk c of a stage from its 144-byte window, as the kernel forms it."""
    words = []
    for i in range(3):
        b = 16 * c + (sh & 8) + 8 * i
        assert b % 8 == 0 and (b + 8 <= 128 or b >= 128)  # an 8-byte read never straddles windows
        words += [int.from_bytes(bytes(window[b + 4 * j:b + 4 * j + 4]), "little") for j in range(2)]
    u5 = [words[i + 1] if sh & 4 else words[i] for i in range(5)]
    return b"".join(funnel_r(u5[m], u5[m + 1], (sh & 3) * 8).to_bytes(4, "little") for m in range(4))


@pytest.mark.parametrize("es", [2, 4])
def test_shift_matches_byte_slice(es):
    rng = np.random.default_rng(es)
    for _ in range(200):
        window = rng.integers(0, 256, 144, dtype=np.uint8)
        for sh in range(0, 16, es):
            for c in range(8):
                assert shifted_chunk(window, sh, c) == bytes(window[sh + 16 * c:sh + 16 * c + 16])


@pytest.mark.parametrize("es", [2, 4])
@pytest.mark.parametrize("L", [1, 7, 63, 64, 65, 127, 129, 1001, 2047])
def test_staged_rows_equal_the_tensor(es, L):
    # A tensor of rows of L elements at a 16-byte-aligned base; every row staged stage by stage
    # through the copy rule, the next-window chunk and the shift must equal its steps, zero
    # past L, and every copied chunk must overlap the row's own bytes.
    rows = 11
    tc = 128 // es
    row_bytes = L * es
    total = rows * row_bytes
    rng = np.random.default_rng(L * es)
    mem = rng.integers(1, 256, total, dtype=np.uint8)
    nst = (L + tc - 1) // tc

    def window(r, k):
        at = r * row_bytes
        sh = at & 15
        out = np.zeros(144, np.uint8)
        for kk, base in ((k, 0), (k + 1, 128)):
            for c in range(8 if base == 0 else 1):
                off = kk * 128 - sh + 16 * c  # chunk start, from step 0 of the row
                if off < row_bytes:  # the chunk holds a byte of the row's steps
                    start = at + off
                    assert start + 16 > at and start < at + row_bytes
                    assert start % 16 == 0
                    lo, hi = max(start, 0), min(start + 16, total)
                    chunk = np.zeros(16, np.uint8)
                    chunk[lo - start:hi - start] = mem[lo:hi]
                    out[base + 16 * c:base + 16 * c + 16] = chunk
        return out, sh

    for r in range(rows):
        for k in range(nst):
            win, sh = window(r, k)
            nbytes = min(tc, L - k * tc) * es
            got = bytearray()
            for c in range(8):
                ch = bytearray(shifted_chunk(win, sh, c))
                keep = nbytes - 16 * c
                for i in range(max(keep, 0), 16):
                    ch[i] = 0
                got += ch
            exp = np.zeros(128, np.uint8)
            s0 = r * row_bytes + k * 128
            exp[:nbytes] = mem[s0:s0 + nbytes]
            assert bytes(got) == exp.tobytes(), (r, k)
