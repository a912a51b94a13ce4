"""Plain, slow FP64 CPU oracle of the sparse-MoE block decode (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run this package.  The
GPU library never calls it, and it calls nothing of the GPU library: the two
share no code.  Their only common input is the seeded generator in ``synth``.

Every function restates one step of the method in the order the pages give it
and cites the passage it follows.  Sources (web pages, by title and section):

* [KAIST-EN] "KAIST drops calibration from MoE decoding, speeds up blocks by up
  to 2.69x over vLLM" -- opening paragraph (decode is memory bound; the routed
  experts' weights are loaded per token), "The threshold promises a budget but
  does not keep it", "Top-k instead of a threshold", "A reader built from
  weights alone".
* [KAIST-FR] its French twin, "KAIST supprime la calibration du decodage MoE
  ..." -- "Top-k plutot que seuil", "Un lecteur construit a partir des seuls
  poids".
* [SELECTOR] "Calibration-free top-k MoE selector saves tuning" (quotes the
  paper's abstract: BF16 weights, ternary sketch, low-rank recovery map).
* [TOPK-OVR] "MoE top_k override (--moe-top-k)" -- "Ce que ca fait" (a token
  picks 8 of 128 experts; the expert MLP is a gated "SwitchGLU"); "Combinaison
  avec d'autres optimisations" (4-bit checkpoints; ``oracle.q4``).
* [TWN] Li, Zhang and Liu, "Ternary Weight Networks" (2016): the ternarisation
  threshold 0.7*mean|W| and the scale alpha = mean |W| over the kept entries.
  The pages name a "ternary sketch" without its formula; TWN is the reading
  adopted for it.

A second restatement in plain C99 (``oracle/c/msb_oracle.c``, loaded through
``oracle.c_oracle``) is held against this one by ``tests/test_oracle_c.py``.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, hand-worked examples (``tests/golden/``), brute force or
library routines -- except the exact GPU outputs at k < I, which have no worked
example on the pages (parity with the paper's own implementation is therefore
unpinned; parity of the GPU path with this oracle is what the GPU tests check).
"""
from .moe_block import (  # noqa: F401
    bf16_to_f64,
    round_to_bf16,
    route,
    ternary_sketch,
    channel_scores,
    topk_channels,
    threshold_channels,
    calibrate_threshold,
    expert_output,
    lowrank_term,
    moe_block,
    dense_moe,
    rmsnorm,
    stack_layer,
    read_bytes,
    SynthLayer,
    ArrayLayer,
)
from . import q4  # noqa: F401,E402
