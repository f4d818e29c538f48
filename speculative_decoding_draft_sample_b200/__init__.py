"""B200-native hot path of DSpark-style confidence-scheduled speculative decoding.

The compute lives in ``libdspark.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/dspark.h``); ``binding`` marshals PyTorch
tensors into those calls. ``workloads`` draws the seeded synthetic inputs.
"""
