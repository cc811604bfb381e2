"""B200-native (sm_100a) GPT-2-style training step.

* `gpt_transformer_step_b200.binding` -- ctypes binding of the C ABI (libgptstep.so);
  importing it fails loudly if the CUDA library has not been built.
* `gpt_transformer_step_b200.fixtures` -- seeded synthetic inputs (no model arithmetic).
* `gpt_transformer_step_b200.build` -- nvcc build of the library for sm_100a.
"""
