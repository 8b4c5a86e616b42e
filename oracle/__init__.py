"""CPU oracle (test infrastructure only): a plain, slow, independent restatement of the
QLoRA quantized linear layer.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg import it; the CUDA library never does."""
from . import nf4_oracle  # noqa: F401
