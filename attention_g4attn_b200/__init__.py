"""g4attn: Gemma-4-style attention (QKNorm, p-RoPE, GQA, keys-as-values, sliding window)
as hand-written sm_100a CUDA kernels behind a C ABI.

The compute entry points live in `attention_g4attn_b200.binding` and load the in-tree
shared library `libg4attn.so`; importing them raises if that library is missing.
`synth` (seeded inputs) and `workloads` (named shapes) need no GPU and no library.
"""
_BINDING_NAMES = (
    "g4attn_qknorm_rope", "g4attn_prefill", "g4attn_decode",
    "g4attn_prefill_workspace_size", "g4attn_decode_workspace_size",
    "g4attn_status_string", "LayerCfg", "G4AttnError", "library_path",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
