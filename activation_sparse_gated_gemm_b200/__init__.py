"""TwELL sparse ReLU-gated FFN forward for B200 (sm_100a).

The compute path is the C-ABI library ``libtwell.so`` built from ``csrc/``;
``twell`` is its ctypes binding. ``synth`` draws seeded synthetic inputs.
Importing the package does not load the library; the first call does, and it
raises if the library is missing.
"""
