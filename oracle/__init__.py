"""Oracle for the Tail-Replay tail-replay hot path: plain, slow, fp64, on the CPU.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference leg import this package.  The product
(``linear_attention_state_zero_b200``) never imports it, and this package imports
nothing from the product: the two share no code.  Inputs come from the seeded
generators in ``synth``.

Sources (web pages on the Tail-Replay paper, arXiv 2608.30310):

* "Tail-Replay reading notes" -- the cc.laoqi.cc reading notes page
  (Tail-Replay：混合 LLM 前缀缓存的短尾重放机制), sections 2.1-2.5: the cache
  record, the four-step hit path (section 2.2), Eq. (1) and the error analysis
  (section 2.3), the tail-FFN skip (section 2.5), the symbol table with
  k = ceil(r*m) (section 2.1).
* "Tail-Replay technical summary" -- the gist.science page, "Key Mechanisms":
  zero start, per-group replay from the cached FA output hiddens.

Every function states the passage it follows.  Where the pages are silent (the
GDN layer internals), the reading is stated in the function and listed in the
design notes; those functions are pinned by special cases and invariants, not
by printed values ("parity pinned to the oracle, not to the pages" for the
layer internals).
"""
from .tail_replay import (  # noqa: F401
    bf16_round,
    conv_state,
    ffn_residual,
    gated_rmsnorm,
    gates,
    gdn_scan,
    in_projection,
    l2_normalize,
    out_projection_residual,
    replay_group,
    replay_layer,
    rmsnorm,
    short_conv,
    silu,
    state_error,
    tail_len,
    tail_rows,
    transition_product,
)
