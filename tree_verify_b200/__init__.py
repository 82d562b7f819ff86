"""B200 (sm_100a) draft-tree verification for EAGLE / EAGLE-2 speculative sampling.

The computation lives in the CUDA library ``libeagle_verify.so`` (C ABI:
include/eagle_verify.h); :mod:`tree_verify_b200.binding` marshals torch tensors
into it and :mod:`tree_verify_b200.step` allocates the buffers of one step.
"""
