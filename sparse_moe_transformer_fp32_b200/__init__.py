"""Forward pass of one Beam sparse-MoE layer on B200 (sm_100a).

The compute path is libbeam_moe.so (hand-written CUDA behind the C ABI in
include/beam_moe.h); :mod:`.beam_moe` is its Python binding and :mod:`.workloads`
holds the seeded synthetic inputs.  Build the library with
``python -m sparse_moe_transformer_fp32_b200.build``.
"""
