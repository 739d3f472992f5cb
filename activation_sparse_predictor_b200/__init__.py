"""Predictor-gated, neuron-aware sparse FFN decode for B200 (sm_100a).

The compute path is the C-ABI library ``libpi.so`` (hand-written CUDA for
sm_100a, declared in ``include/pi.h``); ``activation_sparse_predictor_b200.pi``
is its thin Python binding (argument marshalling only).  ``synth`` prepares
seeded synthetic inputs.  There is no CPU fallback: importing the binding
without the built library raises.
"""
__all__ = ["pi", "synth", "build"]
