"""Comparison helpers shared by the GPU parity tests."""
import numpy as np

# Tolerances (stated for this verification step): fp32 paths 1e-5 relative, bf16 paths
# 2e-2 after normalisation; both measured per output row as max|gpu - ref| / max|ref|.
TOL = {"f32": 1e-5, "bf16": 2e-2}
MARGIN = 1e-4


def row_rel_err(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(gpu - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return num / np.maximum(den, 1e-30)


def is_root_path(parents, accepted, n):
    """accepted[0:n] is a chain root -> ... with each node the child of the previous."""
    prev = 0
    for k in range(n):
        c = int(accepted[k])
        if c <= 0 or parents[c] != prev:
            return False
        prev = c
    return True


def compare_accept(gpu: dict, ref: dict, parents: np.ndarray, exact_all: bool = False):
    """Bit-exact comparison of the walk; sequences whose oracle walk met a decision inside
    the margin are only checked for validity unless ``exact_all``.  Returns the number of
    sequences compared exactly."""
    B, N = parents.shape
    exact = 0
    for b in range(B):
        g_len = int(gpu["accept_len"][b])
        if exact_all or ref["near"][b] == 0:
            assert g_len == ref["accept_len"][b], (b, g_len, ref["accept_len"][b])
            np.testing.assert_array_equal(gpu["accepted_nodes"][b], ref["accepted_nodes"][b])
            assert gpu["next_token"][b] == ref["next_token"][b], (b, gpu["next_token"][b], ref["next_token"][b])
            exact += 1
        else:
            assert 0 <= g_len < N and is_root_path(parents[b], gpu["accepted_nodes"][b], g_len)
            assert (gpu["accepted_nodes"][b, g_len:] == -1).all()
    return exact
