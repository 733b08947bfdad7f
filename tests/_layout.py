"""Tiled operand layouts of include/sharq.h, restated in numpy for the tests.

`untile_*` turn the bytes of a prepared-activation / packed-weight buffer into
logical arrays (codes per element, scale bytes per block, metadata nibbles
per 8-element chunk) so they can be compared with the oracle; `tile_*` do the
reverse so a test can hand-build GEMM operands.  Layout only: no arithmetic
of the method lives here.
"""
import numpy as np

CODES_TILE, SP_TILE, META_TILE, SF32_TILE, SF16_TILE = 16384, 8192, 2048, 1024, 2048


def _sf_index(r, atom, i):
    return atom * 512 + (r % 32) * 16 + (r // 32) * 4 + i


# --- precomputed permutations for one tile (row r, logical position) -------

def _codes_perm():
    """byte offset in a 16 KB tile of (row, byte b of the row's 128 bytes)."""
    r = np.arange(128)[:, None]
    b = np.arange(128)[None, :]
    return r * 128 + (((b // 16) ^ (r % 8)) * 16) + b % 16          # [128, 128]


def _sp_perm():
    r = np.arange(128)[:, None]
    b = np.arange(64)[None, :]
    return r * 64 + (((b // 16) ^ ((r // 2) % 4)) * 16) + b % 16     # [128, 64]


def _sf_perm(n_blocks):
    """byte offset of the scale of block b (0..n_blocks-1) of row r."""
    r = np.arange(128)[:, None]
    b = np.arange(n_blocks)[None, :]
    return _sf_index(r, b // 4, b % 4)                                # [128, n]


CODES_PERM, SP_PERM = _codes_perm(), _sp_perm()
SF8_PERM, SF16_PERM = _sf_perm(8), _sf_perm(16)


def _nibbles(byts):
    return np.stack([byts & 0xF, byts >> 4], axis=-1).reshape(*byts.shape[:-1], -1)


def _pack_nibbles(codes):
    c = codes.reshape(*codes.shape[:-1], -1, 2).astype(np.uint8)
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)


def _tiles(buf, n_rows_tiles, KS, tile_bytes):
    return np.asarray(buf, dtype=np.uint8)[: n_rows_tiles * KS * tile_bytes].reshape(n_rows_tiles, KS, tile_bytes)


# ------------------------------------------------------------- untile -------

def untile_codes(buf, rows, K):
    """16 KB code tiles -> E2M1 codes [rows_padded, K]."""
    RT, KS = (rows + 127) // 128, K // 256
    t = _tiles(buf, RT, KS, CODES_TILE)
    byts = t[:, :, CODES_PERM]                                        # [RT, KS, 128, 128]
    byts = byts.transpose(0, 2, 1, 3).reshape(RT * 128, KS * 128)
    return _nibbles(byts)


def untile_sp_codes(buf, rows, K):
    """8 KB sparse tiles -> kept-value codes [rows_padded, K/2]."""
    RT, KS = (rows + 127) // 128, K // 256
    t = _tiles(buf, RT, KS, SP_TILE)
    byts = t[:, :, SP_PERM].transpose(0, 2, 1, 3).reshape(RT * 128, KS * 64)
    return _nibbles(byts)


def untile_meta(buf, rows, K):
    """2 KB metadata tiles -> nibbles [rows_padded, K/8]."""
    RT, KS = (rows + 127) // 128, K // 256
    t = _tiles(buf, RT, KS, META_TILE).reshape(RT, KS, 128, 16)
    byts = t.transpose(0, 2, 1, 3).reshape(RT * 128, KS * 16)
    return _nibbles(byts)


def untile_sf(buf, rows, K, per):
    """scale tiles -> bytes [rows_padded, K/per] (per = 16, 32 or 64 logical
    K per scale: 4, 2 or 1 atoms of 512 bytes per tile)."""
    RT, KS = (rows + 127) // 128, K // 256
    nb = 256 // per
    size, perm = nb // 4 * 512, _sf_perm(nb)
    t = _tiles(buf, RT, KS, size)
    return t[:, :, perm].transpose(0, 2, 1, 3).reshape(RT * 128, KS * nb)

# --------------------------------------------------------------- tile -------


def tile_codes(codes):
    """E2M1 codes [rows_padded, K] -> bytes of 16 KB tiles."""
    R, K = codes.shape
    RT, KS = R // 128, K // 256
    byts = _pack_nibbles(codes).reshape(RT, 128, KS, 128).transpose(0, 2, 1, 3)
    out = np.zeros((RT, KS, CODES_TILE), dtype=np.uint8)
    out[:, :, CODES_PERM] = byts
    return out.reshape(-1)


def tile_sp_codes(codes):
    R, Kh = codes.shape
    RT, KS = R // 128, Kh // 128
    byts = _pack_nibbles(codes).reshape(RT, 128, KS, 64).transpose(0, 2, 1, 3)
    out = np.zeros((RT, KS, SP_TILE), dtype=np.uint8)
    out[:, :, SP_PERM] = byts
    return out.reshape(-1)


def tile_meta(meta):
    R, C = meta.shape
    RT, KS = R // 128, C // 32
    byts = _pack_nibbles(meta).reshape(RT, 128, KS, 16).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(byts).reshape(-1)


def tile_sf(sf, per):
    R, nbk = sf.shape
    nb = 256 // per
    RT, KS = R // 128, nbk // nb
    size, perm = nb // 4 * 512, _sf_perm(nb)
    out = np.zeros((RT, KS, size), dtype=np.uint8)
    out[:, :, perm] = sf.reshape(RT, 128, KS, nb).transpose(0, 2, 1, 3)
    return out.reshape(-1)


def pad_rows(a, rows_padded, fill=0):
    out = np.full((rows_padded, *a.shape[1:]), fill, dtype=a.dtype)
    out[: a.shape[0]] = a
    return out
