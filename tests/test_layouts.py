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


# ---------------------------------------------------------------- emit mode's L1 fragments
def l1frag_offset(k, r):
    """bf16 offset of L1 element (k, r) in emit mode's fragment-ordered copy,
    as kernels.h states it."""
    G, kk = k >> 4, k & 15
    t = 4 * (r & 7) + (kk >> 2)
    return ((G * 32 + t) * 8 + 2 * (r >> 3)) * 2 + (kk & 3)


def test_l1frag_formula_is_the_one_in_the_kernel_header():
    import os
    src = open(os.path.join(os.path.dirname(__file__), "..", "rank_gemm_b200", "csrc", "kernels.h")).read()
    assert "const int G = k >> 4, kk = k & 15, t = 4 * (r & 7) + (kk >> 2);" in src
    assert "return (((size_t)G * 32 + t) * 8 + 2 * (r >> 3)) * 2 + (kk & 3);" in src


def test_l1frag_fills_its_buffer_once():
    K_pad = 512
    k = np.arange(K_pad)[:, None]
    r = np.arange(32)[None, :]
    off = l1frag_offset(k, r).ravel()
    assert np.array_equal(np.sort(off), np.arange(32 * K_pad))


def test_emit_lr_partial_fragments_multiply_to_the_product():
    """One warp's LR partial over one 16-column group, simulated lane by lane:
    A fragments as tcgen05.ld.16x256b returns them from the bf16-pair stash
    (lane t: rows t/4 and t/4 + 8 of its 16-row half, TMEM columns 2(t%4) and
    2(t%4)+1, each column one pair of adjacent k), assigned to the mma slots
    as the kernel does (a0 = r0, a1 = r2, a2 = r1, a3 = r3); B fragments read
    from the l1frag buffer (words 2 nt, 2 nt + 1 of the lane); the product
    formed with mma.m16n8k16's fragment semantics (PTX ISA: A a0 (row g,
    k 2q, 2q+1), a1 (row g+8), a2/a3 the same at k + 8; B b0 (k 2q, 2q+1,
    col g), b1 at k + 8; D d0 d1 (row g, cols 2q, 2q+1), d2 d3 at row g+8;
    g = lane / 4, q = lane % 4).  Integer data, so equality is exact."""
    rng = np.random.default_rng(5)
    G = 3                                              # the group's index along K
    A = rng.integers(-8, 9, size=(32, 16))             # this warp's 32 rows x the group's 16 k
    L1 = rng.integers(-8, 9, size=(16 * (G + 1), 32))  # L1 rows for groups 0..G, 32 ranks
    buf = np.zeros(32 * 16 * (G + 1), dtype=np.int64)
    for kk in range(16 * (G + 1)):
        for rr in range(32):
            buf[l1frag_offset(kk, rr)] = L1[kk, rr]

    def pair(row, col):                                # TMEM column col of a row: k = 2 col, 2 col + 1
        return (A[row, 2 * col], A[row, 2 * col + 1])

    D = np.zeros((32, 32), dtype=np.int64)
    for h in range(2):                                 # the two 16-row halves
        Aslot = np.zeros((16, 16), dtype=np.int64)     # the A the mma sees (slot k order)
        for t in range(32):
            g, q = t >> 2, t & 3
            r0 = pair(16 * h + g, 2 * q)
            r1 = pair(16 * h + g, 2 * q + 1)
            r2 = pair(16 * h + g + 8, 2 * q)
            r3 = pair(16 * h + g + 8, 2 * q + 1)
            a = (r0, r2, r1, r3)                       # the kernel's slot assignment
            Aslot[g, 2 * q: 2 * q + 2] = a[0]
            Aslot[g + 8, 2 * q: 2 * q + 2] = a[1]
            Aslot[g, 2 * q + 8: 2 * q + 10] = a[2]
            Aslot[g + 8, 2 * q + 8: 2 * q + 10] = a[3]
        for nt in range(4):
            Bslot = np.zeros((16, 8), dtype=np.int64)
            for t in range(32):
                g, q = t >> 2, t & 3
                w = (G * 32 + t) * 8 + 2 * nt          # the lane's word 2 nt (b0), 2 nt + 1 (b1)
                Bslot[2 * q: 2 * q + 2, g] = buf[2 * w: 2 * w + 2]
                Bslot[2 * q + 8: 2 * q + 10, g] = buf[2 * w + 2: 2 * w + 4]
            Dt = Aslot @ Bslot
            D[16 * h: 16 * h + 16, 8 * nt: 8 * nt + 8] = Dt
    assert np.array_equal(D, A @ L1[16 * G: 16 * G + 16, :])
