"""B200-native OSC (Outlier Separation in Channel dimension) W4A4 linear.

The compute path is libosc.so (hand-written sm_100a CUDA behind a C ABI, see
include/osc.h); ``w4a4_outlier_separated_b200.osc`` is its thin Python binding.
"""
