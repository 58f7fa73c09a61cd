"""Hand-built bf16 chunks that hit the NVFP4 format's special points (test data only).

Each builder returns uint16 bf16 bit patterns shaped [B, L, H, d] with head_dim d = 128,
so the same bytes can be quantised by the oracle and by the CUDA path.
"""
import numpy as np

from tests._bf16 import f32_to_bf16_bits

E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_positive_values():
    """The 126 positive finite E4M3 magnitudes from the bit layout (bias 7, 3 mantissa bits)."""
    vals = [m * 2.0 ** -9 for m in range(1, 8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append((1 + m / 8) * 2.0 ** (e - 7))
    return vals


def fixed_point_chunk(k: int, d: int = 128) -> np.ndarray:
    """Blocks [6 s, c1 s, ..., c15 s] * 2^k for every positive E4M3 scale s and every E2M1
    value c (both signs); blocks with s = 448 hold the chunk maximum 2688 * 2^k."""
    signed = [v for v in E2M1_MAG] + [-v for v in E2M1_MAG]
    others = [v for i, v in enumerate(signed) if i != 7]  # drop the leading +6
    scales = e4m3_positive_values()
    scales = scales + [448.0] * ((-len(scales)) % (d // 16))
    x = np.zeros(len(scales) * 16)
    for b, s in enumerate(scales):
        x[b * 16] = 6.0 * s
        x[b * 16 + 1:b * 16 + 16] = np.array(others) * s
    x *= 2.0 ** k
    return f32_to_bf16_bits(x.astype(np.float32)).reshape(1, -1, 1, d)


def tie_chunk(k: int, d: int = 128) -> np.ndarray:
    """One block of exact E2M1 midpoints (scale 1, g = 2^k) and an anchor row."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    row = [6.0] + mids + [-m for m in mids]
    x = np.zeros((2, d))
    x[0, :len(row)] = row
    x[0, 16:16 + len(row)] = [-v for v in row]
    x[1, 0] = 2688.0
    x *= 2.0 ** k
    return f32_to_bf16_bits(x.astype(np.float32)).reshape(1, 2, 1, d)


def underflow_chunk(d: int = 128) -> np.ndarray:
    """Block scales that round to 0 and to the smallest subnormal, an all-zero block, a
    block of negative zeros, and a chunk whose 1/(s*g) overflows."""
    x = np.zeros((6, d))
    x[0, 0] = 2688.0
    x[1, 0] = 6.0 * 2.0 ** -11          # block scale rounds to 0
    x[2, 0] = 6.0 * 1.5 * 2.0 ** -10     # block scale 2^-9
    x[2, 1] = -6.0 * 2.0 ** -11
    x[3, :16] = -0.0
    x[4, 16:32] = np.linspace(-1, 1, 16)
    bits = f32_to_bf16_bits(x.astype(np.float32))
    bits[3, :16] = 0x8000                # -0.0
    return bits.reshape(1, 6, 1, d)


def tiny_scale_chunk(d: int = 128) -> np.ndarray:
    """Chunk maximum 2^-113: blocks of 2^-131 get scale 2^-9 and 1/(s*g) overflows fp32."""
    x = np.zeros((2, d))
    x[0, 0] = 2.0 ** -113
    x[1, 0] = 2.0 ** -131
    x[1, 1] = -(2.0 ** -131)
    x[1, 20] = 2.0 ** -128
    return f32_to_bf16_bits(x.astype(np.float32)).reshape(1, 2, 1, d)


def pad_tokens(bits: np.ndarray, multiple: int = 2) -> np.ndarray:
    """Append zero tokens so the chunk length is a multiple of ``multiple``."""
    L = bits.shape[1]
    extra = (-L) % multiple
    if extra == 0:
        return bits
    z = np.zeros((bits.shape[0], extra) + bits.shape[2:], np.uint16)
    return np.concatenate([bits, z], axis=1)
