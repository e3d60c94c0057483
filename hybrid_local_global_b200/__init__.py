"""B200-native interleaved local/global causal GQA attention (prefill and
batched decode) with (p-)RoPE, ring-buffer KV slots and KV sharing.

The compute path lives in ``libgemma_attn.so`` (CUDA for sm_100a, C ABI in
``include/gemma_attn.h``). ``native`` is its ctypes binding, ``stack`` runs a
multi-layer block through it, ``synth`` makes the seeded synthetic inputs.
Importing ``native`` fails loudly when the library has not been built.
"""
