"""Float64 CPU oracle for exact attention (test infrastructure only).

This package is the checker, not the product. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. It shares no code with the CUDA path in
``exact_attention_102_b200/`` and imports nothing from it; inputs reach it as
plain numpy arrays.

Modules
-------
attention
    The plain definitions: 3-pass safe-softmax attention forward with the
    per-row logsumexp, its analytic gradients, the paged-KV decode (gather
    through the block table, then the forward definition), the logsumexp
    merge of split partials, the packed variable-length form (sequences of
    unequal query / key lengths, grouped KV heads, bottom-right causal), and
    the FP8 e4m3 block quantiser used by the diagnostic FP8 oracle, and the
    gradients of the FP8 forward (straight through the quantisation, back
    through the rotation).
dropout
    Attention with dropout on the probabilities: the Philox4x32-10
    counter-based generator written from its published definition, the keep
    mask it defines element by element, and the dropout forward and backward.
online
    A second, independent implementation of the forward: the tiled one-pass
    online-softmax recurrence (running max m, running sum l, unnormalised O
    rescaled by exp(m_old - m_new), one final diag(l)^-1). It exists only to
    pin ``attention.attention_fwd``.

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
invariants, finite differences, a library routine (torch's e4m3 cast) or the
independent recurrence; see each docstring for its pin.
"""

from .attention import (  # noqa: F401
    attention_fwd,
    attention_bwd,
    attention_rows,
    attention_block_sparse,
    attention_varlen,
    attention_varlen_bwd,
    paged_decode,
    paged_prefill,
    combine_partials,
    round_bf16,
    quantize_e4m3,
    dequantize_blocks_e4m3,
    fp8_block_quantize,
    attention_fp8_bwd,
)
from .dropout import (  # noqa: F401
    attention_dropout,
    attention_dropout_bwd,
    drop_threshold,
    keep_mask,
    philox4x32_10,
)
from .online import tiled_online_fwd  # noqa: F401
