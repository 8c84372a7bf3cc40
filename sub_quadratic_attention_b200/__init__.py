"""SPECTRE frequency-domain token mixing on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libspectre_mix.so`` built from
``csrc/``; :mod:`sub_quadratic_attention_b200.binding` marshals arguments to
it.  :mod:`sub_quadratic_attention_b200.workloads` draws the seeded synthetic
inputs.
"""
__all__ = ["binding", "workloads"]
