"""fp64 CPU oracle of the recurrent-depth block (test infrastructure only; see rdt_oracle)."""
from .rdt_oracle import *  # noqa: F401,F403
from .rdt_oracle import (rmsnorm, rope_angles, apply_rope, silu, swiglu_ffn, causal_attention,
                         gqa_attention, router_topk, moe_combine, attention_sublayer,
                         moe_sublayer, loop_forward, loop_step_rows, input_injection,
                         spectral_radius, mla_attention_explicit, mla_attention_absorbed,
                         LoopTrace, Routing, NEAR_TIE, NEAR_HALT, halting_probability,
                         loop_forward_act, ActResult, apply_rope_at, LoopKVCache,
                         attention_cached, loop_prefill, loop_decode,
                         depth_rope_angles, apply_depth_rope, depth_attention_sublayer, DepthKV)
