"""B200-native (sm_100a) Mixture-of-Experts feed-forward layer behind a C ABI.

``sparse_expert_moe_b200.moe`` is the Python binding of ``include/moe.h``;
``sparse_expert_moe_b200.inputs`` draws the seeded synthetic workloads;
``sparse_expert_moe_b200.build`` compiles ``libmoe_b200.so`` with nvcc.
"""
