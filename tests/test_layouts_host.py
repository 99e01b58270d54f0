"""Host checks of the block-scale reads of the NVFP4 GEMM against the layouts include/convrot.h
states (no GPU).

The NVFP4 GEMM does not copy whole 4096-byte weight images into tensor memory: its scale warps
read the first lane quadrant (the first 1 KB) of each image and the activation atoms, and store
them with tcgen05.st so that lane L of every quadrant holds row L of each 32-row group. These
tests emulate those reads on buffers laid out by the header's formulas and check that they give
every tensor-memory lane and column the byte the 4-fold replicated image holds there (the
layout the MXFP4 GEMM's tcgen05.cp 128x256b still reads), for every row of a tile.
"""

import numpy as np

TILE_A, TILE_B_NV = 128, 192


def image_offset(lane, j):
    """Byte j (0..31) of TMEM lane `lane` (0..127) inside a 4096-byte image."""
    return 256 * (lane // 8) + 128 * (j // 16) + 16 * (lane % 8) + j % 16


def weight_image(tile_rows, rng):
    """One 64-K chunk's image of a weight tile: scale byte (r, b) of row r < tile_rows in the
    four lanes r % 32 + 32 q at byte 4 ((r % 128) / 32) + b of the half r / 128; bytes no row
    uses are random."""
    img = rng.integers(0, 256, 4096, dtype=np.uint8)
    scales = rng.integers(0, 256, (tile_rows, 4), dtype=np.uint8)
    for r in range(tile_rows):
        for b in range(4):
            for q in range(4):
                j = 16 * (r // 128) + 4 * ((r % 128) // 32) + b
                img[image_offset(r % 32 + 32 * q, j)] = scales[r, b]
    return img, scales


def scale_warp_b_columns(img):
    """What the NVFP4 GEMM's scale warps store for one B chunk: lane L of each quadrant gets 8
    columns from the image's first quadrant, half h at 256 (L / 8) + 128 h + 16 (L % 8)."""
    out = np.zeros((128, 32), dtype=np.uint8)
    for L in range(32):
        off = 256 * (L // 8) + 16 * (L % 8)
        row = np.concatenate([img[off:off + 16], img[off + 128:off + 144]])
        for q in range(4):
            out[32 * q + L] = row
    return out


def test_weight_scale_first_quadrant_gives_every_lane_its_scales():
    rng = np.random.default_rng(0)
    img, scales = weight_image(TILE_B_NV, rng)
    cols = scale_warp_b_columns(img)
    # every lane and byte that holds a row's scale equals the replicated image's byte there
    # (bytes of rows past the tile, which the MMA never reads, may differ)
    used = {(r % 32 + 32 * q, 16 * (r // 128) + 4 * ((r % 128) // 32) + b)
            for r in range(TILE_B_NV) for b in range(4) for q in range(4)}
    for lane, j in used:
        assert cols[lane, j] == img[image_offset(lane, j)]
    # and each row's four scales sit where the MMA looks for them
    for r in range(TILE_B_NV):
        for b in range(4):
            lane, j = r % 32 + 32 * (r % 4), 16 * (r // 128) + 4 * ((r % 128) // 32) + b
            assert cols[lane, j] == scales[r, b]


def test_activation_atom_rows_fill_every_quadrant():
    """A: the scale warp of quadrant q stores atom bytes 16 L .. 16 L + 15 into lane 32 q + L;
    row r's block b must land at column r / 32, byte b, in every quadrant."""
    rng = np.random.default_rng(1)
    scales = rng.integers(0, 256, (TILE_A, 4), dtype=np.uint8)
    atom = np.zeros(512, dtype=np.uint8)
    for r in range(TILE_A):
        for b in range(4):
            atom[16 * (r % 32) + 4 * ((r % 128) // 32) + b] = scales[r, b]
    for q in range(4):
        for L in range(32):
            cols = atom[16 * L:16 * L + 16].reshape(4, 4)     # 4 columns of 4 bytes
            for c in range(4):
                r = 32 * c + L
                assert (cols[c] == scales[r]).all(), (q, L, c)


def test_staged_reads_stay_inside_their_regions():
    """The scale warps' 16-byte reads: A within the stage's 4 atoms (2 KB), B within the 4
    first quadrants (4 KB), whatever the lane."""
    a_max = max(512 * k + 16 * lane + 16 for k in range(4) for lane in range(32))
    b_max = max(1024 * k + 256 * (lane // 8) + 16 * (lane % 8) + 128 + 16
                for k in range(4) for lane in range(32))
    assert a_max == 2048 and b_max <= 4096
