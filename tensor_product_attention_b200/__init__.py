"""Tensor Product Attention (TPA) hot path for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``libtpa.so`` (include/tpa.h), built in-tree by
``python -m tensor_product_attention_b200.build``.  ``binding`` wraps it with the same
call names; importing this package does not load the library.
"""
__all__ = ["binding", "inputs"]
