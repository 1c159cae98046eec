"""B200-native DF-SSM decode step: 1-bit scaffold + int8 low-rank projections
feeding a fused conv1d / selective-SSM / gated-RMSNorm step.

The compute runs in ``libdfssm.so`` (hand-written sm_100a CUDA behind a C ABI);
``bit_scaffold_quantized_b200.dfssm`` is the thin ctypes binding over it and
``bit_scaffold_quantized_b200.synth`` draws the seeded synthetic inputs.
"""
