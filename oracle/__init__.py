"""fp64 CPU oracle for sparse-V decode attention over a block-quantized KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never imports, links or calls it, and it shares no code with the library (no
kernels, helpers, tables or constant generators).

What it follows (one web page is the authority for the method):
  tproger.ru, "Пропуск 90% работы по деквантизации ускорил декодирование LLM"
  (sparse V dequantization, Tom Turney's llama.cpp Metal kernel):
    * section "Решение — не ускорять, а пропускать" (Solution: do not speed up,
      skip): attention weights come from K before any V work, and a position
      whose weight is below the threshold 1e-6 has its V dequantization and
      accumulation skipped entirely;
    * section "FAQ": K must always be dequantized (it produces the weights);
      a skipped position contributes under a millionth of the maximum;
    * section "Почему это работает для любой квантизации" (why it works for any
      quantization): q8_0, q4_0 and a Walsh-Hadamard-rotated codebook format.
  The block formats themselves (q8_0: d = absmax/127, x = q*d; q4_0:
  d = absmax/-8 with the signed extreme, x = (q-8)*d; rotated LUT: per-vector
  norm and a 16-entry Lloyd-Max codebook for N(0, 1/D)) are the workload
  definitions this library is built for; where the pages leave an arithmetic
  step open, each module says which reading it takes.

Modules:
  quant      quantizers / dequantizers (fp32 arithmetic stated op by op; fp64 dequant)
  codebook   Lloyd-Max codebook for a Gaussian (fp64 Lloyd iteration)
  attention  dense attention, schedule-exact sparse-V attention, log-sum-exp combine

Parity pins: every function here is pinned in ``tests/test_oracle_*.py`` against
something other than itself (brute force, closed forms, a published table,
library routines for special cases, invariants).
"""
from . import quant, codebook, attention  # noqa: F401
