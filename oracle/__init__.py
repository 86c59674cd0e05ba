"""fp64 CPU oracle (test infrastructure; never on the product path).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA
library in ``exact_attention_130_b200``.
"""
from .attention import (  # noqa: F401
    attention_bwd,
    attention_fwd,
    attention_fwd_rows,
    decode,
    decode_paged,
    decode_split,
    merge_partials,
    online_attention_fwd,
    scores,
    softmax_rows,
)
from .fp8 import (  # noqa: F401
    attention_fp8,
    attention_fp8_rounded_p,
    e4m3_decode,
    e4m3_encode,
    fp8_dequantize,
    fp8_prepare,
    hadamard_rotate_f32,
    quantize_blocks,
)
from .dropout_bias import (  # noqa: F401
    attention_bwd_ex,
    attention_fwd_ex,
    dropout_keep,
    keep_threshold,
    philox4x32_10,
)
