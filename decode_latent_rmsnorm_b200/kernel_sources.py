"""Which CUDA source files each timed kernel is built from, and a digest of
them, so that a profiler figure recorded for a kernel (its DRAM traffic per
launch) is used only while that kernel's source is unchanged."""

from __future__ import annotations

import hashlib
import os

_CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")

# kernel label (as the library reports it) -> source files, relative to csrc/
KERNEL_SOURCES = {
    "tc_decode_attention": ("tc_decode.cuh", "tc_ptx.cuh", "common.cuh"),
    "tc_attention": ("tc_attention_pair.cuh", "tc_attention.cuh", "tc_gemm.cuh", "tc_ptx.cuh", "common.cuh"),
    "tc_norm_kv_b_proj": ("tc_gemm.cuh", "tc_ptx.cuh", "common.cuh"),
}


def source_digest(kernel: str) -> str | None:
    """sha256 over the kernel's source files (None for an unknown kernel)."""
    files = KERNEL_SOURCES.get(kernel)
    if files is None:
        return None
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(_CSRC, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


if __name__ == "__main__":
    for k in KERNEL_SOURCES:
        print(k, source_digest(k))
