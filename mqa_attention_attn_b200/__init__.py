"""B200-native fused grouped-KV attention forward: causal/non-causal prefill
and single-token decode against a KV cache (GQA, MQA and MHA, plus the MLA
absorbed-latent decode), as sm_100a CUDA kernels behind a C ABI.

``mqa_attention_attn_b200.inputs`` holds the seeded workload generators.
The kernels are reached through ``mqa_attention_attn_b200.binding`` (loaded
lazily; it raises if the CUDA library has not been built).
"""
import importlib

__all__ = ["inputs", "binding", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
