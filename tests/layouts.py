"""Scale-factor layout conversions used by the tests.

The MMA layout is the data format documented in include/mxmoe.h (512-byte
atoms of 128 rows x 4 scale columns; atom index (r/128)*(S/4) + s/4, byte
(r%32)*16 + ((r%128)/32)*4 + s%4).  The oracle works in row-major scales; the
tests convert between the two.  No arithmetic of the method lives here.
"""
import numpy as np


def mma_offsets(R: int, S: int) -> np.ndarray:
    r = np.arange(R, dtype=np.int64)[:, None]
    s = np.arange(S, dtype=np.int64)[None, :]
    return ((r // 128) * (S // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4


def rowmajor_to_mma(sf: np.ndarray) -> np.ndarray:
    R, S = sf.shape
    out = np.zeros(R * S, dtype=np.uint8)
    out[mma_offsets(R, S).ravel()] = sf.ravel()
    return out


def mma_to_rowmajor(buf: np.ndarray, R: int, S: int) -> np.ndarray:
    return np.asarray(buf).reshape(-1)[mma_offsets(R, S)]
