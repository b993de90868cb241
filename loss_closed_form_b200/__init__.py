"""B200-native exact RoPE-attention loss and closed-form gradient.

The computation lives in ``librope_attn.so`` (CUDA for sm_100a, C ABI in
``include/rope_attn.h``); ``loss_closed_form_b200.rope_attn`` is its Python binding.
Importing this package does not load the library.
"""
