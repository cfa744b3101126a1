"""B200-native (sm_100a) Hyena long-convolution library.

``subquadratic_sequence_b200.hyena`` is the binding of the C ABI
(include/hyena.h); ``subquadratic_sequence_b200.synth`` draws the seeded
synthetic inputs; ``subquadratic_sequence_b200.build`` compiles the CUDA
library in-tree.
"""
