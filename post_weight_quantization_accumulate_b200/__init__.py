"""GPTQ per-layer quantization on B200 (sm_100a).

The compute path is the C-ABI library ``libgptq.so`` built from ``csrc/``;
``binding`` marshals torch tensors into its calls and ``layer`` sequences them
for one linear layer.  Importing this package does not load the library; the
first call into ``binding`` does, and raises if the library is missing (there
is no CPU fallback).
"""
__all__ = ["binding", "layer", "synth", "build"]
