"""fp64 CPU oracle for exact tiled attention (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline legs use this
package; the CUDA library never imports or links it.
"""
from .attention import (  # noqa: F401
    attention_ref,
    combine_partials,
    decode_ref,
    online_softmax_attention,
    probabilities,
    scores,
    unpack_decode_cache,
)
