"""B200-native observation-window KV-cache compression (libkvc).

The compute path lives in the CUDA library ``libkvc.so`` built from ``csrc/``;
``kvc`` is its thin ctypes binding.  ``synth`` holds the seeded input
generators.  Importing the package does not load the library; the first call
through ``kvc`` does, and fails loudly if it is missing.
"""
