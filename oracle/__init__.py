"""Float64 CPU oracle of the attention forward (test infrastructure only).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark use
it; the CUDA library neither imports nor calls anything here.
"""

from .attention import attend_rows, attention_forward, logits, softmax_with_sink, visible  # noqa: F401
