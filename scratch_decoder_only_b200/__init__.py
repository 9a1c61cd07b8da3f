"""B200-native GPT training step behind a C ABI (libgpt.so).

Import ``scratch_decoder_only_b200.gpt`` for the binding; this package
initialiser stays import-light so the input generators can be used without
loading the CUDA library.
"""
