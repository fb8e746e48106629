"""CPU fp64 oracle for Dynamic Bifocal RoPE attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, shares no code with it, and has no CPU fallback through it.

Source: "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
(Tang, Wang, Gu, Han, Cai), as summarised by the gist.science technical
summaries (Portuguese "Resumo Técnico: Jet-Long" and French "Résumé Technique :
Jet-Long") and the chatpaper.ai abstract.
"""
from .bifocal import (  # noqa: F401
    group_size,
    position_map,
    correction_shift,
    rope_inv_freq,
    rope_rotate,
    bifocal_attention,
    bifocal_attention_kv,
    bifocal_attention_ie_merge,
    bifocal_attention_from_raw,
    bifocal_decode,
    causal_rope_attention,
    brute_force_tiny,
)
