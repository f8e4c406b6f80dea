"""A second, vectorised reader and writer of the packed cache block, written
from the block format as include/kvq.h documents it (not from the oracle's
or the kernels' offset code), so that the tests can check both of those
against the documented format from outside.

Block of 16 tokens, 1536 bytes; tau = token in the block, r = tau % 8,
th = tau // 8, q = tau // 2:
  K codes [0, 512):    logical word wi (bytes 4wi..4wi+3) of token tau at
                       16*(4r + wi%4) + 4*(2th + wi//4)
  V codes [512, 1024): 16-bit piece w (logical bytes 2w, 2w+1) of tau at
                       512 + 16*(4*(w%8) + q%4) + 4*(2*(q//4) + w//8) + 2*(tau%2)
  K meta [1024, 1280), V meta [1280, 1536): group g's {s, z} (fp16, s first)
                       at base + 8*(4r + g) + 4*th
Logical packing of a token's 128 codes into 32 bytes: element j's code
sits in byte j % 32 at bits 2*(j // 32).
"""
import numpy as np

BLK_TOK, BLK_BYTES, D = 16, 1536, 128


def _k_index():
    """[16][32] byte offsets of each token's logical K bytes."""
    idx = np.zeros((BLK_TOK, 32), np.int64)
    for tau in range(BLK_TOK):
        r, th = tau % 8, tau // 8
        for wi in range(8):
            off = 16 * (4 * r + wi % 4) + 4 * (2 * th + wi // 4)
            idx[tau, 4 * wi:4 * wi + 4] = off + np.arange(4)
    return idx


def _v_index():
    idx = np.zeros((BLK_TOK, 32), np.int64)
    for tau in range(BLK_TOK):
        q = tau // 2
        for w in range(16):
            off = 512 + 16 * (4 * (w % 8) + q % 4) + 4 * (2 * (q // 4) + w // 8) + 2 * (tau % 2)
            idx[tau, 2 * w:2 * w + 2] = off + np.arange(2)
    return idx


def _meta_index(base):
    """[16][4][2][2]: token, group, (s, z), byte."""
    idx = np.zeros((BLK_TOK, 4, 2, 2), np.int64)
    for tau in range(BLK_TOK):
        r, th = tau % 8, tau // 8
        for g in range(4):
            off = base + 8 * (4 * r + g) + 4 * th
            idx[tau, g, 0] = off + np.arange(2)
            idx[tau, g, 1] = off + 2 + np.arange(2)
    return idx


K_IDX, V_IDX = _k_index(), _v_index()
KM_IDX, VM_IDX = _meta_index(1024), _meta_index(1280)


def unpack_codes(lb):
    """Logical bytes [..., 32] -> codes [..., 128]."""
    lb = lb.astype(np.uint8)
    return np.concatenate([(lb >> (2 * g)) & 3 for g in range(4)], axis=-1)


def pack_codes(codes):
    """Codes [..., 128] in 0..3 -> logical bytes [..., 32]."""
    c = codes.astype(np.uint8).reshape(codes.shape[:-1] + (4, 32))
    out = np.zeros(codes.shape[:-1] + (32,), np.uint8)
    for g in range(4):
        out |= (c[..., g, :] & 3) << (2 * g)
    return out


def _u16(b2):
    """[..., 2] little-endian bytes -> uint16."""
    return b2[..., 0].astype(np.uint16) | (b2[..., 1].astype(np.uint16) << 8)


def read_blocks(blocks):
    """blocks [..., 1536] uint8 -> dict of per-token arrays, each with a
    leading [..., 16] token axis: k, v codes [..., 16, 128]; ks, kz, vs, vz
    fp16 bit patterns [..., 16, 4]."""
    blocks = np.asarray(blocks, np.uint8)
    k = unpack_codes(blocks[..., K_IDX])
    v = unpack_codes(blocks[..., V_IDX])
    km = _u16(blocks[..., KM_IDX])          # [..., 16, 4, 2]
    vm = _u16(blocks[..., VM_IDX])
    return {"k": k, "v": v, "ks": km[..., 0], "kz": km[..., 1], "vs": vm[..., 0], "vz": vm[..., 1]}


def write_block(k, v, ks, kz, vs, vz):
    """One block from logical content (shapes as read_blocks returns for a
    single block); bytes nothing documents stay zero."""
    blk = np.zeros(BLK_BYTES, np.uint8)
    blk[K_IDX] = pack_codes(np.asarray(k))
    blk[V_IDX] = pack_codes(np.asarray(v))
    for idx, (s, z) in ((KM_IDX, (ks, kz)), (VM_IDX, (vs, vz))):
        s = np.asarray(s, np.uint16)
        z = np.asarray(z, np.uint16)
        blk[idx[..., 0, 0]] = (s & 0xff).astype(np.uint8)
        blk[idx[..., 0, 1]] = (s >> 8).astype(np.uint8)
        blk[idx[..., 1, 0]] = (z & 0xff).astype(np.uint8)
        blk[idx[..., 1, 1]] = (z >> 8).astype(np.uint8)
    return blk
