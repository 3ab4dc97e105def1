"""fp64 CPU oracle of the fused Transformer encoder layer (forward + backward).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``transformer_layer_pre_b200``) never imports it and
shares no code with it: the CUDA library fails loudly when it is missing
instead of falling back here.

Every function is a plain restatement, in float64 numpy, of what the source
pages define; library matmuls serve as steps, nothing is tiled, fused or
reordered.  Citations name the page and the section they follow:

* "DeepSpeed Transformer Kernel usage guide" (page 1): configuration surface,
  Step 2 (parameter tables: dropout sites, seed, fp16, pre_layer_norm,
  intermediate_size <= 0 -> 4*hidden, layer_norm_eps = 1e-12) and Step 3
  (memory switches: what is recomputed in backward).
* "Forward-pass compute-graph optimisation in the Transformer" (page 4),
  section 2 (module order of one encoder layer; post-LN ordering) and the
  attention formula softmax(Q K^T / sqrt(d_k)) V.
* "Transformer deployment" (page 2), section "matrix-operation restructuring"
  (the attention pseudo-code: scale after Q K^T, softmax over the last axis).
* "AI-infra engineers and the Transformer" (page 3), section 2.1 Steps 2-3
  (fused QKV Linear(D, 3D) split into heads), section 2.3 (GELU, erf form;
  keeping the GELU input), section 5.1 (inverted dropout x*mask/(1-p)).

* "Progressive Layer Dropping" (page 5), schedule section: the keep level
  theta(t) and per-step layer skipping in a stack (``oracle.pld``).

Readings taken where the pages are silent (the dropout counter layout, the
dropout site after softmax, both hidden-dropout sites, erf GELU, biased
variance, the depth profile and random draw of layer dropping) are stated in
the docstrings below.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
something other than itself (cuRAND's host Philox, standard-normal table values,
closed forms, finite differences, PyTorch's float64 TransformerEncoderLayer).
"""

from .layer import (  # noqa: F401
    LayerConfig,
    philox4x32_10,
    dropout_keep,
    dropout_threshold,
    round_to_storage,
    layer_norm_forward,
    layer_norm_backward,
    layer_norm_backward_from_output,
    gelu,
    gelu_grad,
    gelu_tanh,
    gelu_tanh_grad,
    softmax_rows,
    attention_forward,
    attention_backward,
    layer_forward,
    layer_backward,
    layer_forward_backward,
    WEIGHT_NAMES,
)
from .pld import pld_keep, pld_keep_prob, pld_theta, stack_forward_backward  # noqa: F401
