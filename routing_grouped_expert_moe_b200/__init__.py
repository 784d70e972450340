"""B200-native forward pass of one Mixture-of-Experts layer.

Route (x @ W_gate, softmax, top-k, renormalise) -> permute by expert id ->
grouped expert FFN (tcgen05 / TMEM GEMMs) -> deterministic combine, all in
hand-written sm_100a kernels behind a C ABI (``include/moe_b200.h``).

The ops live in :mod:`routing_grouped_expert_moe_b200.binding`; importing them
loads ``lib/libmoe_b200.so`` and raises if it has not been built.  The
expert-parallel forward over a torch.distributed group is in
:mod:`routing_grouped_expert_moe_b200.expert_parallel`.
"""
import importlib

__all__ = ["binding", "expert_parallel", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
