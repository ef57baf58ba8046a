"""CPU oracle for the QLoRA-linear hot path (NF4 quantize, double quantization,
doubleDequant, fused LoRA forward/backward).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline / reference leg may import this package.  It shares no code with
the CUDA library and never calls it.  Every function cites the web page and
section it follows; see ``codec`` (plain C through ctypes) and ``linear``
(NumPy float64).

Parity status:
  pinned   - codebook (printed table + construction), quantize (brute force,
             invariants), double quantization (closed-form bit count, exact
             mean, error bound), dequant (definition + BF16 rounding vs torch),
             forward/backward (finite differences, special cases, merged-weight
             identity, rank bound), the E4M3 codec (torch's float8_e4m3fn),
             AdamW (torch.optim.AdamW and closed forms).
  unpinned - the exact 8-bit format of the double-quantized constants (the
             pages disagree: 8-bit floats vs INT8; INT8 absmax is our reading),
             the nibble order inside a byte, and the codebook offset delta
             beyond the 4-decimal window the printed table fixes.
"""
from . import adamw, codec, linear  # noqa: F401
