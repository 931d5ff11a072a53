"""B200-native WHALE attention-fusion forward.

The compute path is the C-ABI library libwhale_fusion.so (hand-written sm_100a CUDA).
`wukong_hstu_cross_b200.whale` is its thin ctypes binding; importing it loads the
library and raises if it is missing. `inputs` holds the seeded synthetic inputs.
"""
