"""B200-native forward pass of the Online Scaled DeltaNet (OSDN) token mixer.

The compute lives in ``libosdn.so`` (hand-written sm_100a CUDA kernels behind a C ABI,
declared in ``include/osdn.h``).  Import ``delta_rule_recurrent_osdn_b200.osdn`` for the thin
Python binding and ``delta_rule_recurrent_osdn_b200.inputs`` for the seeded workloads; this
package module imports neither, so the input generators work on machines without a GPU.
"""
