"""B200-native fused mixed-precision MoE layer over Any-Precision bit-plane
weights (PagedWeight's hot path).  The compute runs in the CUDA library
``libpw_b200.so`` built from ``csrc/``; ``binding`` marshals arguments to its
C ABI.  ``synth`` draws seeded synthetic layers."""
