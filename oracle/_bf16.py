"""bf16 decoding for the oracle (its own copy; the CUDA side decodes in hardware)."""

import numpy as np


def f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32, exact: the bits are the top half."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def gather_tokens(pages: np.ndarray, table_row: np.ndarray, length: int) -> np.ndarray:
    """Logical tokens [length, H, d] of one sequence from a page pool [P, H, b_p, d].

    Logical token p lives in physical page table_row[p // b_p] at slot p % b_p
    (the PagedAttention layout the pages build on, §4.3).
    """
    b_p = pages.shape[2]
    n = (length + b_p - 1) // b_p
    ids = np.asarray(table_row[:n], dtype=np.int64)
    x = pages[ids]                       # [n, H, b_p, d]
    x = x.transpose(0, 2, 1, 3)          # [n, b_p, H, d]
    return x.reshape(n * b_p, x.shape[2], x.shape[3])[:length]
