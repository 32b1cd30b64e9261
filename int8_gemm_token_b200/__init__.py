"""B200-native W8A8 quantized linear layer (PDMIX + LLM.int8() decomposition).

The compute lives in ``libw8a8.so`` (hand-written sm_100a CUDA behind a C ABI
declared in ``include/w8a8.h``). ``int8_gemm_token_b200.w8a8`` is the thin
ctypes binding over it; ``int8_gemm_token_b200.synth`` makes the seeded
synthetic inputs.
"""
