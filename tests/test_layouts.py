"""Host checks of the documented byte layouts (no GPU): every formula in the
public header that places an element must be a bijection onto its buffer."""
import itertools

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


# ---------------------------------------------------------------- emit mode's LR partial
def stash_block(q):
    """64-wide block of tile columns held by 64-wide block q of the emit
    stash, as gemm_nvfp4.cu states it."""
    return ((q & 1) << 1) | (q >> 1)


def test_stash_block_formula_is_the_one_in_the_kernel():
    import os
    src = open(os.path.join(os.path.dirname(__file__), "..", "rank_gemm_b200", "csrc", "gemm_nvfp4.cu")).read()
    assert "return ((q & 1u) << 1) | (q >> 1);" in src


def test_emit_partial_over_the_stash_is_the_product():
    """The next layer's LR partial of one tile, simulated step by step: the
    epilogue warps park the tile's bf16 output in the stash (warp column set
    ch, 32-column chunk c = tile columns ch 64 + 128 (c / 2) + 32 (c % 2) ..
    +31, pair j of a chunk at stash column ch 64 + 16 c + j, the even column
    in the low half); the MMA warp then takes K16 steps j = 0..15 with A =
    stash columns 8 j .. 8 j + 7 (16 bf16 in order) and B = the L1 box
    stash_block(j / 4) at k offset 16 (j % 4).  Integer data, so equality is
    exact."""
    rng = np.random.default_rng(7)
    R, r_tot = 128, 32
    Y = rng.integers(-8, 9, size=(R, 256))            # the tile: rows x its 256 columns
    L1 = rng.integers(-8, 9, size=(256, r_tot))       # the next layer's L1 rows of those columns
    stash = np.zeros((R, 256), dtype=np.int64)        # bf16 positions (two per 32-bit column)
    for ch in range(2):
        for c in range(4):
            for j in range(16):
                for e in range(2):
                    n = ch * 64 + 128 * (c >> 1) + 32 * (c & 1) + 2 * j + e
                    t = ch * 64 + 16 * c + j
                    stash[:, 2 * t + e] = Y[:, n]
    D = np.zeros((R, r_tot), dtype=np.int64)
    for j in range(16):
        blk = stash_block(j >> 2)
        D += stash[:, 16 * j: 16 * j + 16] @ L1[64 * blk + 16 * (j & 3): 64 * blk + 16 * (j & 3) + 16, :]
    assert np.array_equal(D, Y @ L1)


def test_emit_iteration_schedule_places_one_partial_per_tile():
    """Kernel 2's k-iteration order in emit mode: per tile the FP4 k-tiles
    and low-rank chunks in order, with the previous tile's partial stage
    after FP4 k-tile min(EMIT_AT, nk - 1), none in the first tile, one extra
    after the last; the producer and the MMA warp use the same order.  Checked
    for the kernel's EMIT_AT (read from its source) and other placements."""
    import os, re
    src = open(os.path.join(os.path.dirname(__file__), "..", "rank_gemm_b200", "csrc", "gemm_nvfp4.cu")).read()
    kernel_at = int(re.search(r"constexpr int EMIT_AT = (\d+);", src).group(1))

    def iter_of(it, nk, with_part, emit_at):
        if not with_part:
            return (0, it) if it < nk else (1, it - nk)
        at = min(emit_at, nk - 1) + 1
        if it < at:
            return (0, it)
        if it == at:
            return (2, 0)
        return (0, it - 1) if it - 1 < nk else (1, it - 1 - nk)
    for emit_at, nk, nl, with_part in itertools.product((kernel_at, 0, 3, 11), (1, 2, 4, 7, 12, 48), (0, 1, 2),
                                                       (False, True)):
        seq = [iter_of(it, nk, with_part, emit_at) for it in range(nk + nl + (1 if with_part else 0))]
        assert [i for k, i in seq if k == 0] == list(range(nk))
        assert [i for k, i in seq if k == 1] == list(range(nl))
        assert sum(k == 2 for k, _ in seq) == (1 if with_part else 0)


# ---------------------------------------------------------------- K splits over a cluster
def _slices(nk, S):
    """[k0, k0 + n) of each CTA of a cluster of S: nk / S each, the first nk % S
    one more (kernel 1's 256-column stages)."""
    q, r = divmod(nk, S)
    return [(c * q + min(c, r), q + (1 if c < r else 0)) for c in range(S)]


def test_k_slices_cover_every_k_tile_once_in_order():
    for nk in range(1, 60):
        for S in (1, 2, 4, 8):
            if S > nk:
                continue
            sl = _slices(nk, S)
            assert all(n >= 1 for _, n in sl)
            flat = [k for k0, n in sl for k in range(k0, k0 + n)]
            assert flat == list(range(nk))


def test_split_formulas_are_the_kernels():
    import os
    d = os.path.join(os.path.dirname(__file__), "..", "rank_gemm_b200", "csrc")
    k1 = open(os.path.join(d, "quant_down.cu")).read()
    assert "const int ns = nq + (split < nr ? 1 : 0);" in k1
    assert "const int kb0 = split * nq + min(split, nr);" in k1


def test_split_rows_cover_the_tile():
    """Each CTA of kernel 1's cluster finishes 64 / S rows of the 64-row block:
    disjoint, complete."""
    for rows in (64,):
        for S in (1, 2, 4, 8):
            per = rows // S
            got = sorted(r for c in range(S) for r in range(c * per, (c + 1) * per))
            assert got == list(range(rows))
