"""The seeded generator (synth/): Philox4x32-10 against the published known-answer vectors
of its authors' Random123 library, and the C host fill against the numpy implementation."""
import numpy as np
import pytest

import synth

# (counter, key) -> output, the known-answer vectors published with Philox4x32-10
KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF), (0xFFFFFFFF, 0xFFFFFFFF),
     (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,want", KAT)
def test_philox_known_answers(ctr, key, want):
    out = synth.philox4x32_10(np.array([ctr], np.uint32), key)
    assert tuple(int(v) for v in out[0]) == want


@pytest.mark.parametrize("kind,count,start,layer,token,attempt", [
    (synth.W_GU, 1_000_003, 12_345, 2, 0, 0),   # unaligned start, odd count
    (synth.ATTN, 8192, 0, 0, 5, 3),
    (synth.W_O, 77, 3, 7, 0, 0),
    (synth.GAMMA, 7168, 0, 0, 0, 0),
    (synth.W_DOWN, 9, 2**33 + 5, 1, 0, 0),        # counter above 32 bits
])
def test_host_fill_matches_numpy(kind, count, start, layer, token, attempt):
    synth.build_host_fill()
    seed = 0x123456789 + kind
    a = synth.gen_bf16(seed, kind, count, layer=layer, token=token, attempt=attempt, start=start)
    b = synth.gen_bf16_numpy(seed, kind, count, layer=layer, token=token, attempt=attempt, start=start)
    assert a.dtype == np.uint16 and np.array_equal(a, b)
