"""B200-native (sm_100a) DeepSeek-V4 compressed sparse attention, one layer.

The compute path is the C-ABI library ``liblcsc.so`` (hand-written CUDA);
``lib`` is its thin ctypes binding.  ``workloads`` and ``synth`` describe
and generate the seeded synthetic benchmark inputs.
"""
