"""Routed MoE expert layer (Inkling 2 Small: 384 experts, top-8, NVFP4 or
MXFP8 experts) for NVIDIA B200, as a C-ABI CUDA library with a thin Python
binding.

    from fp8_moe_expert_top_b200 import ExpertLayer, binding

`binding` mirrors the C entry points one to one; `ExpertLayer` owns the device
buffers of one layer and runs route -> permute -> expert GEMMs -> combine.
The shared library is loaded on first use and every call raises if it is
missing; there is no fallback path.
"""


def __getattr__(name):
    if name == "ExpertLayer":
        from .layer import ExpertLayer
        return ExpertLayer
    if name in ("binding", "layer", "inputs", "build"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
