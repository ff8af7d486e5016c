"""fp64 CPU oracle for exact softmax attention: TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the C-ABI library and
its Python binding) never imports, links or calls it, and this package imports
nothing from the product.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test against a
closed form, an invariant, brute force, a finite-difference check or an
independent library routine, except where a function's docstring says
"parity unpinned".
"""

from .attention import (  # noqa: F401
    attention_forward,
    attention_backward,
    attention_probabilities,
    attention_forward_loops,
    attention_backward_loops,
    online_softmax_forward,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    FP8_TAU,
    hadamard,
    rotate_rows,
    e4m3_round,
    e4m3_encode,
    e4m3_decode,
    block_quantize,
    per_tensor_quantize,
    fp8_attention_forward,
    naive_fp8_attention_forward,
)
from .varlen import varlen_forward, varlen_backward  # noqa: F401
from .mxfp8 import (  # noqa: F401
    mx_quantize,
    mx_dequantize,
    mx_roundtrip,
    mxfp8_attention_forward,
)
