"""B200-native online-softmax (flash) attention forward.

The compute path is the C-ABI CUDA library ``libattn_b200.so`` (sm_100a);
:mod:`.binding` marshals torch tensors into it. :mod:`.inputs` holds the seeded
synthetic workloads. Importing the package does not load the library; the first
call does, and fails loudly if it is missing.
"""
