"""Counter-based uniform draws used by the sampler (jitter of stratified samples
and the u's of inverse-CDF sampling).

The NeRF page draws these with torch.rand ("Hierarchical sampling" section);
here every draw is a pure function of (seed, ray, stream, index) so that the CUDA
path and this oracle can draw the same numbers independently. The generator is
the SplitMix64 output function (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014), applied twice:

    key = mix(seed)
    h   = mix(key XOR (ray << 20 | stream << 16 | index))
    u   = (h >> 40) * 2^-24          (24 bits, exact in fp32 and fp64)

Streams: 0 = stratified jitter, 1 = inverse-CDF draws.
"""
import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def mix(x):
    """SplitMix64 output for state x: add the golden gamma, then two
    xor-shift-multiply rounds and a final xor-shift (all mod 2^64)."""
    z = np.asarray(x, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z + _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def draw_bits(seed, ray, stream, index):
    """24-bit integer m of the draw u = m * 2^-24 (numpy broadcasting)."""
    key = mix(np.uint64(seed))
    ray = np.asarray(ray, dtype=np.uint64)
    index = np.asarray(index, dtype=np.uint64)
    ctr = (ray << np.uint64(20)) | (np.uint64(stream) << np.uint64(16)) | index
    return (mix(key ^ ctr) >> np.uint64(40)).astype(np.int64)


def draw_uniform(seed, ray, stream, index):
    """u in [0, 1) as fp64 (exactly representable in fp32)."""
    return draw_bits(seed, ray, stream, index).astype(np.float64) * 2.0 ** -24
