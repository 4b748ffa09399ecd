"""Plain fp64 CPU oracle for Sketch Attention (SA) and STCA.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA path (``sketch_attention_flashsa_b200``) and imports
nothing from it; callers hand it numpy arrays.

Every function evaluates the plain dense definition from the pages in float64
(numpy), one (user, head) problem at a time, with no blocking, fusion or
reordering beyond the definition. Each docstring cites the passage it follows
in "SequenceO1: End-to-End Ultra-Long (100K) Sequence Modeling in
Recommendation with Low-Rank Caching" (full text, arXiv 2609.08443).

Pins (tests/test_oracle_pins.py, run with ``-m "not gpu"``) tie every function
to closed forms, conservation laws, special cases, invariances and finite
differences; none of them re-types the formulas below.
"""
from .sa import (sa_forward_proto, sa_forward_token, sa_backward_proto,
                 sa_backward_token, sa_forward, sa_backward, sa_problem)
from .stca import stca_forward, stca_backward
from .diag import token_max_weight, weight_histogram, renormalized_sketch
from .cache import SketchCache, splitmix64, key_hash
from .refine import layer_norm, swish, swiglu_ffn, refine, project_queries, stacked_sa, round_bf16

__all__ = ["sa_forward_proto", "sa_forward_token", "sa_backward_proto",
           "sa_backward_token", "sa_forward", "sa_backward", "sa_problem",
           "stca_forward", "stca_backward", "token_max_weight", "weight_histogram", "renormalized_sketch",
           "SketchCache", "splitmix64", "key_hash", "layer_norm", "swish", "swiglu_ffn", "refine", "project_queries",
           "stacked_sa", "round_bf16"]
