"""CPU oracle for the fused NVFP4 + binary-sign low-rank GEMM.

TEST INFRASTRUCTURE ONLY.  A plain, slow, obviously-correct restatement of
what the GPU library computes, in NumPy and FP64 (FP32 where the format fixes
the rounding).  It shares no code with the CUDA path and imports nothing from
it.  Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import it; the library itself never does and has no CPU
fallback.

  nvfp4      E2M1 / E4M3 codecs, nibble packing, activation and weight quantisers
  biloco     sign packing, the GEMM part, z = alpha * (V^T x), the correction, y
  decompose  greedy sign peeling of W into U diag(alpha) V^T + R and the joint refit
"""

from . import nvfp4, biloco, decompose  # noqa: F401
