"""Exact causal attention with RoPE and masked sequence packing on B200.

The compute runs in liblwm_attn.so (hand-written CUDA for sm_100a); this
package is its thin Python binding.  Functions carry the names of the C entry
points declared in include/lwm_attn.h.  The shared library is loaded on first
use of any of them; if it is missing that use raises ImportError (there is no
fallback).  ``long_context_causal_attention_b200.build`` compiles it.
"""
_EXPORTS = (
    "ENTRY_POINTS", "LIB_PATH", "LwmAttnDesc", "LwmError", "alloc_workspace", "lwm_attn_bwd",
    "lwm_attn_fwd", "lwm_attn_kernel_launches", "lwm_attn_set_timing_events",
    "lwm_attn_read_status", "lwm_attn_workspace_size", "lwm_rope_apply", "lwm_status_string",
    "make_desc", "lwm_attn_selftest_wait", "lwm_rope_apply_at", "lwm_attn_merge",
    "lwm_accumulate", "lwm_convert_f32", "lwm_attn_fwd_pair", "lwm_attn_bwd_pair",
    "lwm_packed_cross_entropy", "lwm_attn_decode", "lwm_attn_decode_workspace_size", "DECODE_MAX_NEW",
    "lwm_attn_fwd_pair_f32", "lwm_attn_bwd_pair_f32",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS or name == "_lib":
        import importlib
        mod = importlib.import_module(__name__ + "._lib")
        return mod if name == "_lib" else getattr(mod, name)
    raise AttributeError(name)
