"""fp64 CPU oracle for the Hymba hybrid-head layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package.  See ``hymba_oracle`` for the
definitions, their sources and the readings taken where the sources are silent.
"""
from .hymba_oracle import *  # noqa: F401,F403
from .hymba_oracle import (KV_CONSUME, KV_OWN, KV_PRODUCE, attention, attention_probs,  # noqa: F401
                           branch_fusion, layer_decode_step, layer_forward, layer_prefill_state, linear, meta_prepend, rms_normalize,
                           selective_scan, silu, softplus, split_in_proj, ssm_alpha_matrix,
                           ssm_branch, ssm_decay_rate, ssm_from_alpha, stack_forward,
                           swiglu_ffn, visibility_mask, visible)
