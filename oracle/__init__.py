"""Plain fp64 CPU oracle for the gated delta rule (GDN and KDA token mixers).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
Python binding) may import, call or execute anything in this package; only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` use it.  It shares no code with the GPU path.

Source of the method: "Super Apriel: One Checkpoint, Many Speeds", §2A (mixer
vocabulary): Kimi Delta Attention is the delta rule recurrence with a
channel-wise gate and Gated DeltaNet the same recurrence with a scalar gate per
head and token.  The pages name the mixers but never print the update; the
update used here is the published gated delta rule,

    S_t = S_{t-1} · Diag(alpha_t) · (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t,

with S_t a d_v x d_k matrix per (sequence, head), alpha_t a scalar (GDN) or a
d_k-vector (KDA) in [0, 1], and beta_t a scalar.

Modules
-------
recurrent   the definition, token by token (the oracle proper); decode_step and
            verify_steps (K tokens with the state after each) run it from a state;
            prefill_varlen runs packed sequences from a pool of state slots
chunked     an independent fp64 chunk-wise restatement, used only to pin the
            chunk algebra against the definition
backward    the gradients of the recurrence (inputs, gates and initial state),
            token by token in reverse
chunked_backward
            the same gradients from the chunk algebra (the state gradient chained
            through the chunks in reverse), pinned against backward
prologue    L2-normalised q, k and the gate from its logit (the fused prologue)
"""

from .recurrent import gated_delta_rule, decode_step, verify_steps, prefill_varlen  # noqa: F401
from .chunked import chunked_gated_delta_rule  # noqa: F401
from .backward import gated_delta_rule_backward  # noqa: F401
from .chunked_backward import chunked_gated_delta_rule_backward  # noqa: F401
from .prologue import apply_prologue, gate_from_logit, l2_normalise  # noqa: F401
