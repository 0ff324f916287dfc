"""KDA oracle (test infrastructure only).

A plain, slow, fp64 CPU implementation of the Kimi Delta Attention recurrence
(Kimi Linear summary, section 3 "Kimi Delta Attention"):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t

and of its scalar-gate relative, Gated DeltaNet (Rationalist Deep-Dive, section 2.3):

    S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T

and of the general DPLR recurrence it specialises (Deep-Dive, section 3.2):

    S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never imports, links or calls anything here, and this
package imports nothing from the product.
"""

from .kda_oracle import (  # noqa: F401
    build_oracle,
    load_library,
    oracle_forward,
    oracle_gdn_forward,
    oracle_dplr_forward,
    oracle_decode_steps,
    oracle_threads,
)
