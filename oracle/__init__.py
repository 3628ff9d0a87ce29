"""fp64 CPU oracle (test infrastructure only; see ``bifocal_ref``)."""
from .bifocal_ref import (FREQ_INTERP, MODES, POS_ALIAS, bifocal_attention, bifocal_attention_ie,  # noqa: F401
                          bifocal_decode_reference, bifocal_scores, cached_key_to_raw, dynamic_factor, kv_head_for,
                          long_branch_rope,
                          rope_causal_attention, rope_keys_for_cache, rope_omega, rope_rotate)
