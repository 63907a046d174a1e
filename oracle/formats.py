"""CSA2 cache-entry codecs: a plain CPU restatement used to check the CUDA path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module;
only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg use it.

What the pages fix, and the reading taken where they are silent:

* A main-KV entry is 512 four-bit numbers plus 32 bytes of scale, 288 bytes in
  all; an indexer-K entry is 128 four-bit numbers plus a 4-byte scale, 68 bytes
  ("DeepSeek-V4.1 模型结构（0）", Q&A "890 字节全局 KV 是怎么算出来的").
  The main-KV format was chosen to differ from the indexer's, and the
  sliding-window cache stays FP8 ("DeepSeek V4.1 Flash 深度解析", 本专栏篇目,
  "FP4 从权重走进 KV 缓存").
* Element format (reading): OCP MX e2m1 -- sign bit 3, magnitude index 0..7 for
  {0, .5, 1, 1.5, 2, 3, 4, 6}.  Two codes per byte, element 2i in the low nibble.
* Main-KV scale (reading): 32 bytes over 512 values = one E4M3 byte per block of
  16, s = E4M3_RNE(amax / 6) saturating at 448.
* Indexer scale (reading): 4 bytes over 128 values = one E8M0 byte per block of
  32, exponent = ceil(log2(amax / 6)) (no clipping of the block maximum).
* SWA token (reading): 512 E4M3 codes plus one fp32 scale = amax / 448.
* Every quantisation decision is taken in fp32: amax / 6 and x / s are IEEE fp32
  divisions, then exact round-to-nearest-even onto the target grid.  A block
  whose scale is zero gets all-zero codes.
"""
import numpy as np

MAIN_DIM = 512
MAIN_BLOCK = 16
MAIN_CODE_BYTES = MAIN_DIM // 2          # 256
MAIN_SCALE_BYTES = MAIN_DIM // MAIN_BLOCK  # 32
MAIN_ENTRY_BYTES = MAIN_CODE_BYTES + MAIN_SCALE_BYTES

IX_DIM = 128
IX_BLOCK = 32
IX_CODE_BYTES = IX_DIM // 2              # 64
IX_SCALE_BYTES = IX_DIM // IX_BLOCK      # 4
IX_ENTRY_BYTES = IX_CODE_BYTES + IX_SCALE_BYTES

SWA_DIM = 512
SWA_TOKEN_BYTES = SWA_DIM + 4            # E4M3 codes + fp32 scale

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0
E4M3_MAX = 448.0

F32 = np.float32


# --------------------------------------------------------------------------- e2m1
def e2m1_encode(y):
    """Round fp32 values (already divided by their scale) to e2m1 codes.

    Round to nearest, ties to the even code, saturating at +-6.  The magnitude
    index is the count of decision points passed; at a midpoint the comparison
    is strict when the lower neighbour has the even code and inclusive when the
    upper one does.  A value that rounds to zero gets code 0 whatever its sign.
    """
    y = np.asarray(y, dtype=F32)
    m = np.abs(y)
    idx = np.zeros(m.shape, dtype=np.uint8)
    for point, inclusive in ((0.25, False), (0.75, True), (1.25, False), (1.75, True),
                             (2.5, False), (3.5, True), (5.0, False)):
        idx += (m >= point) if inclusive else (m > point)
    neg = np.signbit(y) & (idx > 0)
    return (idx | (neg.astype(np.uint8) << 3)).astype(np.uint8)


def e2m1_decode(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def pack_nibbles(codes):
    """[..., 2n] codes -> [..., n] bytes, element 2i in the low nibble of byte i."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 15
    out[..., 1::2] = packed >> 4
    return out


# --------------------------------------------------------------------------- E4M3
def e4m3_decode(codes):
    """E4M3 (the 'fn' variant: bias 7, no infinities, S.1111.111 is NaN) -> float64."""
    c = np.asarray(codes, dtype=np.int64)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


def e4m3_encode(v):
    """fp32 -> E4M3 code, round to nearest even, saturating at +-448.

    |v| lies in the binade [2^e, 2^(e+1)) whose quantum is 2^(e-3); below 2^-6
    the quantum stays 2^-9 (subnormals).  Dividing by a power of two is exact,
    so rint() performs the round-half-even step exactly.
    """
    v = np.asarray(v, dtype=F32).astype(np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, -6)
    r = np.rint(a / np.exp2(e - 3.0)) * np.exp2(e - 3.0)   # rounded magnitude
    r = np.minimum(r, E4M3_MAX)
    sub = r < 2.0 ** -6
    _, rex = np.frexp(np.where(sub, 1.0, r))
    re = rex - 1
    code_norm = ((re + 7) << 3) | (np.rint(r / np.exp2(re - 3.0)).astype(np.int64) - 8)
    code_sub = np.rint(r / 2.0 ** -9).astype(np.int64)
    code = np.where(sub, code_sub, code_norm).astype(np.int64)
    code = np.where(np.signbit(v) & (code != 0), code | 0x80, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------- E8M0
def e8m0_ceil_exponent(q):
    """ceil(log2 q) for fp32 q > 0, clamped to the E8M0 range [-127, 127].

    frexp gives q = f * 2^x with f in [0.5, 1); log2 q is x - 1 exactly when
    f == 0.5 and lies strictly inside (x - 1, x) otherwise.
    """
    q = np.asarray(q, dtype=F32).astype(np.float64)
    f, x = np.frexp(q)
    e = np.where(f == 0.5, x - 1, x)
    return np.clip(e, -127, 127).astype(np.int64)


def e8m0_value(code):
    return np.exp2(np.asarray(code, dtype=np.float64) - 127.0)


# --------------------------------------------------------------------------- entries
def _safe_div(x, s):
    """IEEE fp32 x / s, broadcasting s; zero where s is zero."""
    x = np.asarray(x, dtype=F32)
    s = np.broadcast_to(np.asarray(s, dtype=F32), x.shape)
    out = np.zeros(x.shape, dtype=F32)
    np.divide(x, s, out=out, where=s != 0)
    return out


def pack_main(x):
    """Main-KV entries: [..., 512] fp32 -> (codes [..., 256] u8, scales [..., 32] u8)."""
    x = np.asarray(x, dtype=F32)
    assert x.shape[-1] == MAIN_DIM
    blk = x.reshape(x.shape[:-1] + (MAIN_SCALE_BYTES, MAIN_BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    s_code = e4m3_encode(amax / F32(E2M1_MAX))
    s_val = e4m3_decode(s_code).astype(F32)
    codes = e2m1_encode(_safe_div(blk, s_val[..., None]))
    codes = np.where(s_val[..., None] != 0, codes, 0).astype(np.uint8)
    return pack_nibbles(codes.reshape(x.shape)), s_code


def unpack_main(codes, scales):
    """Dequantise main-KV entries to float64 [..., 512] (exact)."""
    c = unpack_nibbles(codes)
    v = e2m1_decode(c).reshape(c.shape[:-1] + (MAIN_SCALE_BYTES, MAIN_BLOCK))
    s = e4m3_decode(scales)[..., None]
    return (v * s).reshape(c.shape)


def pack_indexer(x):
    """Indexer keys (and queries): [..., 128] fp32 -> (codes [..., 64] u8, E8M0 [..., 4] u8)."""
    x = np.asarray(x, dtype=F32)
    assert x.shape[-1] == IX_DIM
    blk = x.reshape(x.shape[:-1] + (IX_SCALE_BYTES, IX_BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    e = e8m0_ceil_exponent(amax / F32(E2M1_MAX))
    e = np.where(amax == 0, -127, e)
    s_val = np.exp2(e.astype(np.float64)).astype(F32)
    codes = e2m1_encode(_safe_div(blk, s_val[..., None]))
    codes = np.where(amax[..., None] != 0, codes, 0).astype(np.uint8)
    return pack_nibbles(codes.reshape(x.shape)), (e + 127).astype(np.uint8)


def unpack_indexer(codes, scales):
    c = unpack_nibbles(codes)
    v = e2m1_decode(c).reshape(c.shape[:-1] + (IX_SCALE_BYTES, IX_BLOCK))
    return (v * e8m0_value(scales)[..., None]).reshape(c.shape)


def pack_swa(x):
    """SWA tokens: [..., 512] fp32 -> (E4M3 codes [..., 512] u8, fp32 scale [...])."""
    x = np.asarray(x, dtype=F32)
    amax = np.max(np.abs(x), axis=-1)
    scale = (amax / F32(E4M3_MAX)).astype(F32)
    codes = e4m3_encode(_safe_div(x, scale[..., None]))
    codes = np.where(scale[..., None] != 0, codes, 0).astype(np.uint8)
    return codes, scale


def unpack_swa(codes, scale):
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]
