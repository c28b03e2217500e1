"""Host checks of the documented byte layouts (no GPU): every formula in the
public header that places an element must be a bijection onto its buffer."""
import numpy as np


def sx_nvfp4_offsets(rows128, K_pad):
    """Byte offset of (row r, 16-group g, replica q) in the NVFP4 activation
    scale layout, as the header states it."""
    r = np.arange(rows128)[:, None, None]
    g = np.arange(K_pad // 16)[None, :, None]
    q = np.arange(4)[None, None, :]
    kb = g // 4
    L = r % 32 + 32 * q
    return ((((r // 128) * (K_pad // 256) + kb // 4) * 2 + (kb % 4) // 2) * 4096 + (L // 8) * 256
            + (kb % 2) * 128 + (L % 8) * 16 + ((r % 128) // 32) * 4 + g % 4)


def test_replicated_activation_scales_fill_their_buffer_once():
    for rows128, K_pad in ((128, 256), (256, 768), (384, 3072)):
        off = sx_nvfp4_offsets(rows128, K_pad).ravel()
        assert off.size == 4 * rows128 * K_pad // 16
        assert np.array_equal(np.sort(off), np.arange(off.size))


def test_replicas_of_one_word_are_its_four_lane_copies():
    # the four bytes of (row, 64-block) are adjacent; the replicas of a byte
    # differ only in the lane: 32 lanes apart = 4 lane groups of 256 bytes
    off = sx_nvfp4_offsets(128, 256)
    assert np.all(np.diff(off[:, :, 0].reshape(128, -1, 4), axis=2) == 1)
    assert np.all(np.diff(off, axis=2) == 4 * 256)


def test_atom_layout_of_weight_scales_fills_its_buffer_once():
    N_pad, K_pad = 512, 768
    n = np.arange(N_pad)[:, None]
    k16 = np.arange(K_pad // 16)[None, :]
    off = ((n // 128) * (K_pad // 64) + k16 // 4) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + k16 % 4
    assert np.array_equal(np.sort(off.ravel()), np.arange(N_pad * K_pad // 16))
