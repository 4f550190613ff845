"""Float64 CPU oracle for the masked attention JVP.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``, never by the product
package. It shares no code with the CUDA path; its mask code
(``oracle.masks``) and its arithmetic (``oracle.jvp_attention``) are written
from the Causal-rCM report, Appendix B (Eq. 42-45) and Sections 2.3 / 3.1.1;
``oracle.attention_backward`` is the gradient of the same masked attention;
``oracle.kv_cache`` is chunk attention over a key/value cache and the
rotary rotation of cached keys (Sec. 3.2.1 "KV Cache");
``oracle.layer_prologue`` is the primal-tangent prologue of an attention
layer (QK-norm and RoPE with their tangents, Sec. 3.2.2 "JVP FSDP2").
Every function here is pinned by tests in ``tests/test_oracle*.py``.
"""
from .masks import (DENSE, FRAME_CAUSAL, CHUNK_CAUSAL, TEACHER_FORCING,
                    MaskSpec, key_intervals, allowed_pairs)
from .jvp_attention import jvp_attention, jvp_attention_head
from .attention_backward import attention_backward, attention_backward_head
from .kv_cache import cache_attention, cache_attention_head, rope_rows
from .layer_prologue import qkv_prologue, rms_norm_jvp

__all__ = ["DENSE", "FRAME_CAUSAL", "CHUNK_CAUSAL", "TEACHER_FORCING",
           "MaskSpec", "key_intervals", "allowed_pairs",
           "jvp_attention", "jvp_attention_head",
           "attention_backward", "attention_backward_head",
           "cache_attention", "cache_attention_head", "rope_rows",
           "qkv_prologue", "rms_norm_jvp"]
