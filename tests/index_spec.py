"""The pooled-index file format of include/msa.h, restated in Python for the
tests: the msa64 hash word by word, and a header writer / reader."""
import struct

M64 = (1 << 64) - 1
HM1, HM2 = 0x9E3779B97F4A7C15, 0xD6E8FEB86659FD93


def _rotl(x, r):
    return ((x << r) | (x >> (64 - r))) & M64


def msa64_spec(data: bytes) -> int:
    """The file hash exactly as include/msa.h states it, word by word."""
    n = len(data)
    words = struct.unpack(f"<{(n + 7) // 8}Q", bytes(data) + b"\0" * (-n % 8))
    h = [HM2 * (j + 1) & M64 for j in range(4)]
    for i, w in enumerate(words):
        h[i % 4] = _rotl(h[i % 4] ^ (w * HM1 & M64), 29) * HM2 & M64
    r = n
    for j in range(4):
        r = _rotl(r ^ (h[j] * HM1 & M64), 31) * HM2 & M64
    r ^= r >> 33
    r = r * HM1 & M64
    return r ^ (r >> 29)


def spec_header(n_docs=3, n_chunks=7, max_dc=4, host=1, layout=(32, 8, 128, 128, 64, 1), theta=1e6):
    """A header written from the format (section hashes left as zeros)."""
    Hkv, d, dr, esz = layout[1], layout[2], layout[3], 2 if layout[5] == 1 else 4
    sizes = [8 * (n_docs + 1), n_chunks * Hkv * dr * esz, (2 if host else 1) * n_chunks * Hkv * d * esz,
             0 if host else n_chunks * Hkv * d * esz]
    b = bytearray(512)
    b[0:8] = b"MSAIDX01"
    struct.pack_into("<II6idqqii", b, 8, 1, 512, *layout, theta, n_docs, n_chunks, max_dc, host)
    at = 4096
    for s, n in enumerate(sizes):
        struct.pack_into("<QQQ", b, 72 + 24 * s, at, n, 0)
        at = (at + n + 4095) // 4096 * 4096
    struct.pack_into("<Q", b, 504, msa64_spec(bytes(b[:504])))
    return b


def read_sections(path):
    """[(offset, bytes, hash)] of the four sections, read by the format."""
    with open(path, "rb") as f:
        b = f.read(512)
    return [struct.unpack_from("<QQQ", b, 72 + 24 * s) for s in range(4)]
