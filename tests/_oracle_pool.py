"""Worker functions for a process pool that runs the oracle's quantiser on chunks of a
large matrix (test infrastructure; the pool is started with the "spawn" method so no
CUDA state is inherited)."""
import numpy as np

from oracle import mxfp8


def fake_quant_rows(a):
    """Oracle rowwise MXFP8 quantise + dequantise of a chunk of rows (E4M3, OCP rule)."""
    return mxfp8.fake_quant_rowwise(np.asarray(a, dtype=np.float64))
